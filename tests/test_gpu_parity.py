"""GPU parity: libhadq (through the C ABI) against the float64 oracle.

Every case runs the CUDA path on seeded inputs and compares element by
element with the oracle on the same bits (tests/parity_check.py states the
tolerances).  The sweep covers every kernel family (segment / team / per-token
row kernels), every block size 1..8192, every output format and both input
dtypes at sizes the oracle finishes in seconds, with ragged row counts and
grids that loop several times.  The five workload configurations run at full
size in the launch configuration bench.py times; for the two largest the
oracle checks a seeded row sample.
"""

import json
import os

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import build as hbuild
from hadamard_rotation_bit_b200 import hadq as H
from hadamard_rotation_bit_b200 import workloads as W
from tests import parity_check as pc

pytestmark = pytest.mark.gpu

NPROC = max(1, min(16, (os.cpu_count() or 2) // 2))


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    hbuild.build()
    H.load_library()
    # This module covers the CUDA-core kernels everywhere (the full-size bf16
    # 4096 / 8192 rotations would otherwise take the tensor-core path, which
    # tests/test_gpu_tensor_path.py covers).
    old = H.hadq_set_impl("butterfly")
    yield
    H.hadq_set_impl(old)


def _log(name, rep):
    path = os.environ.get("HADQ_PARITY_LOG")
    if path:
        with open(path, "a") as f:
            f.write(json.dumps({"case": name, **rep}) + "\n")
    print(name, rep)


def to_dev(x_np, x_dtype):
    if x_dtype == "bf16":
        return torch.from_numpy(np.ascontiguousarray(x_np).view(np.int16)).view(torch.bfloat16).cuda()
    return torch.from_numpy(np.ascontiguousarray(x_np, dtype=np.float32)).cuda()


def run_quant(x_np, x_dtype, block, fmt, group):
    codes, scales = H.hadq_rotate_quant(to_dev(x_np, x_dtype), block, fmt, group)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def run_rotate(x_np, x_dtype, block, out_dtype):
    out = H.hadq_rotate(to_dev(x_np, x_dtype), block,
                        out_dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    if out_dtype == "f32":
        return out.cpu().numpy()
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


def synth(rows, n, x_dtype, seed, outliers=True, dist="normal"):
    """Seeded test input with a few outlier channels; returns (stored bits, float64 values)."""
    rng = np.random.default_rng(seed)
    v = rng.standard_t(3, (rows, n)) if dist == "t" else rng.standard_normal((rows, n))
    if outliers and n >= 8:
        v[:, rng.choice(n, max(1, n // 64), replace=False)] *= 40.0
    v = v.astype(np.float32)
    stored = v if x_dtype == "f32" else W.f32_to_bf16_bits(v)
    return stored, W.bits_to_float64(stored, x_dtype)


# ------------------------------------------------------------------ sweep

SIZES = [  # (rows, n, block): segment kernels (b <= 128) and team kernels (b >= 256)
    (37, 8, 0), (37, 16, 0), (37, 32, 0), (37, 64, 0), (37, 128, 0),
    (29, 1024, 1), (29, 1024, 2), (29, 1024, 4), (29, 1024, 16), (29, 1024, 32), (29, 1024, 64), (29, 1024, 128),
    (13, 96, 32), (11, 200, 8), (9, 48, 16), (5, 14336, 128),
    (37, 256, 0), (37, 512, 0), (37, 1024, 0), (21, 2048, 0), (19, 4096, 0), (7, 8192, 0),
    (9, 2048, 256), (5, 4096, 512), (5, 4096, 1024), (3, 8192, 2048), (3, 12288, 4096), (3, 16384, 8192),
]


def _fmt_ok(n, fmt, group):
    if fmt == "int4":
        return n % group == 0
    if fmt == "mxfp4":
        return n % 32 == 0
    if fmt == "nvfp4":
        return n % 16 == 0
    return True


@pytest.mark.parametrize("rows,n,block", SIZES)
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_rotate_sweep(rows, n, block, x_dtype):
    stored, x64 = synth(rows, n, x_dtype, seed=n + block + rows)
    pc.check_rotation_f32(x64, run_rotate(stored, x_dtype, block, "f32"), block)
    pc.check_rotation_bf16(x64, run_rotate(stored, x_dtype, block, "bf16"), block)


@pytest.mark.parametrize("rows,n,block", SIZES)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 64), ("int4", 128), ("int8", 0), ("mxfp4", 32),
                                       ("nvfp4", 16)])
def test_quant_sweep(rows, n, block, fmt, group):
    if not _fmt_ok(n, fmt, group):
        pytest.skip("group does not divide n")
    if fmt == "int8" and n > 32768:
        pytest.skip("per-token int8 limit")
    x_dtype = "bf16" if (n + rows) % 2 else "f32"
    stored, x64 = synth(rows, n, x_dtype, seed=7 * n + block + rows, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, x_dtype, block, fmt, group)
    _log(f"sweep-{fmt}{group}-{rows}x{n}-b{block}-{x_dtype}", pc.check(fmt, x64, codes, scales, block, group))


@pytest.mark.parametrize("rows,n,block,fmt,group", [
    (2500, 4096, 0, "int4", 128),      # team kernel, grid loops several times, ragged last wave
    (20001, 256, 0, "mxfp4", 32),      # 64 teams per CTA, ragged
    (40007, 128, 0, "int4", 128),      # segment kernel grid-stride tail
    (3001, 8192, 0, "mxfp4", 32),      # two-warp teams, several iterations
    (1023, 14336, 128, "int8", 0),     # per-token rows, grid loops
    (517, 16384, 2048, "int8", 0),     # per-token team-row kernel
    (3001, 8192, 0, "nvfp4", 16),      # two-warp teams, NVFP4
    (40007, 80, 16, "nvfp4", 16),      # 16-element segments (n = 80), grid-stride tail
])
def test_multi_iteration_grids(rows, n, block, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=rows)
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    _log(f"grid-{fmt}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group))


# ---------------------------------------------------- workload configs

def _config(key, row_ids=None):
    w = W.WORKLOADS[key]
    stored = W.generate(key, workers=NPROC)
    if w.fmt is None:
        out = run_rotate(stored, w.x_dtype, w.block, w.out_dtype)
    else:
        out = run_quant(stored, w.x_dtype, w.block, w.fmt, w.group)
    if row_ids is None:
        row_ids = np.arange(w.rows)
    x64 = W.bits_to_float64(stored[row_ids], w.x_dtype)
    return w, stored, out, row_ids, x64


def test_config_c1():
    w, _, (codes, scales), _, x64 = _config("c1")
    _log("c1", pc.check_int4(x64, codes, scales, w.block, w.group))


def test_config_c2():
    w, _, (codes, scales), _, x64 = _config("c2")
    _log("c2", pc.check_int4(x64, codes, scales, w.block, w.group))


def test_config_c3():
    w, _, (codes, scales), _, x64 = _config("c3")
    _log("c3", pc.check_int8(x64, codes, scales, w.block))


def _sample_rows(rows, stored_absmax, seed, n_random=2048, edge=256, top=64):
    rng = np.random.default_rng(seed)
    ids = np.concatenate([np.arange(edge), np.arange(rows - edge, rows), rng.choice(rows, n_random, replace=False),
                          np.argsort(stored_absmax)[-top:]])
    return np.unique(ids)


def test_config_c4():
    wq = W.WORKLOADS["c4q"]
    q_stored = W.generate("c4q", workers=NPROC)
    q_out = run_rotate(q_stored, "bf16", wq.block, "bf16")
    k_stored = W.generate("c4k", workers=NPROC)
    k_codes, k_scales = run_quant(k_stored, "bf16", 128, "int4", 128)
    # oracle on heads 0 and 511 in full plus a seeded sample of rows
    rng = np.random.default_rng(4)
    ids = np.unique(np.concatenate([np.arange(4096), np.arange(wq.rows - 4096, wq.rows),
                                    rng.choice(wq.rows, 65536, replace=False)]))
    _log("c4q", pc.check_rotation_bf16(W.bits_to_float64(q_stored[ids], "bf16"), q_out[ids], 128))
    _log("c4k", pc.check_int4(W.bits_to_float64(k_stored[ids], "bf16"), k_codes[ids], k_scales[ids], 128, 128))


def test_config_c5():
    w = W.WORKLOADS["c5"]
    stored = W.generate("c5", workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, "mxfp4", 32)
    absmax = np.abs(W.bits_to_float64(stored[:, ::64], "bf16")).max(1)
    ids = _sample_rows(w.rows, absmax, seed=5)
    _log("c5", pc.check_mxfp4(W.bits_to_float64(stored[ids], "bf16"), codes[ids], scales[ids], w.block))


# ------------------------------------------------------------- edge cases

def test_zero_rows_is_a_noop():
    x = torch.empty(0, 4096, dtype=torch.bfloat16, device="cuda")
    codes, scales = H.hadq_rotate_quant(x, 0, "int4", 128)
    assert codes.numel() == 0 and scales.numel() == 0


@pytest.mark.parametrize("fmt,group", [("int4", 128), ("int8", 0), ("mxfp4", 32), ("nvfp4", 16)])
@pytest.mark.parametrize("n,block", [(4096, 0), (1024, 128)])
def test_all_zero_rows(fmt, group, n, block):
    stored = np.zeros((5, n), dtype=np.uint16)
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    assert not codes.any() and not np.asarray(scales, dtype=np.float64).any()


def test_scale_overflow_and_subnormal_scales():
    rng = np.random.default_rng(9)
    v = rng.standard_normal((6, 1024)).astype(np.float32)
    v[0] *= 3e6          # absmax/7 above fp16 range -> inf scale, zero codes
    v[1] *= 1e-6         # subnormal fp16 scales -> clamped codes
    v[2] *= 3e-7
    v[3, :] = 0.0
    v[3, 5] = 1e-30      # scale rounds to 0
    x64 = v.astype(np.float64)
    for block in (0, 64):
        codes, scales = run_quant(v, "f32", block, "int4", 32)
        rep = pc.check_int4(x64, codes, scales, block, 32)
        assert np.isinf(scales[0]).all() and not pc.unpack_nibbles(codes[0:1], True).any()
        _log(f"edge-int4-b{block}", rep)
        codes, scales = run_quant(v, "f32", block, "mxfp4", 32)
        _log(f"edge-mxfp4-b{block}", pc.check_mxfp4(x64, codes, scales, block))
        codes, scales = run_quant(v, "f32", block, "nvfp4", 16)       # saturating and zero E4M3 scales
        _log(f"edge-nvfp4-b{block}", pc.check_nvfp4(x64, codes, scales, block))
        codes, scales = run_quant(v, "f32", block, "int8", 0)
        _log(f"edge-int8-b{block}", pc.check_int8(x64, codes, scales, block))


def test_exact_ties_and_sign_of_zero():
    # rows whose rotation is exactly known: x = H/sqrt(n) applied to a chosen y
    n = 64
    y = np.zeros((4, n))
    y[0, :8] = [7.0, 2.5, 3.5, -2.5, 0.5, 1.5, -0.5, -7.0]          # int4 ties with scale 1
    y[1, :8] = [6.0, 5.0, 0.25, 0.75, -1.25, -1.75, 2.5, -0.1]      # E2M1 ties, negative zero
    y[2, 0] = 1.0
    y[3, :] = -0.01
    y[3, 0] = 4.0
    x = oracle.rotate(y, 0).astype(np.float32)   # not exact: ties become near-ties (boundary window)
    for fmt, group in (("int4", 32), ("mxfp4", 32), ("int8", 0), ("nvfp4", 16)):
        codes, scales = run_quant(x, "f32", 0, fmt, group)
        _log(f"ties-{fmt}", pc.check(fmt, x.astype(np.float64), codes, scales, 0, group))


def test_in_place_and_involution():
    for x_dtype, tdt in (("f32", torch.float32), ("bf16", torch.bfloat16)):
        stored, x64 = synth(33, 4096, x_dtype, seed=1)
        x = to_dev(stored, x_dtype)
        ref = H.hadq_rotate(x.clone(), 0)
        H.hadq_rotate(x, 0, out=x)           # in place
        torch.cuda.synchronize()
        assert torch.equal(x, ref)
    stored, x64 = synth(33, 4096, "f32", seed=2)
    x = to_dev(stored, "f32")
    back = H.hadq_rotate_inverse(H.hadq_rotate(x, 0), 0)
    torch.cuda.synchronize()
    err = (back.double() - x.double()).abs().max().item()
    assert err <= 1e-5 * x.double().abs().max().item()


def test_guard_bytes_around_outputs():
    rows, n, group = 37, 1024, 64
    stored, x64 = synth(rows, n, "bf16", seed=11)
    x = to_dev(stored, "bf16")
    pad = 4096
    cbytes, sbytes = rows * n // 2, rows * (n // group) * 2
    cbuf = torch.full((cbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((sbytes + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    codes = cbuf[pad:pad + cbytes].view(rows, n // 2)
    scales = sbuf[pad:pad + sbytes].view(torch.float16).view(rows, n // group)
    H.hadq_rotate_quant(x, 0, "int4", group, codes=codes, scales=scales)
    torch.cuda.synchronize()
    cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
    assert (cb[:pad] == 0xA5).all() and (cb[pad + cbytes:] == 0xA5).all()
    assert (sb[:pad] == 0x5A).all() and (sb[pad + sbytes:] == 0x5A).all()
    pc.check_int4(x64, codes.cpu().numpy(), scales.cpu().numpy(), 0, group)
    # rotation output guards, team kernel with fp32 output
    obuf = torch.full((rows * n + 2 * pad,), -7.0, dtype=torch.float32, device="cuda")
    out = obuf[pad:pad + rows * n].view(rows, n)
    H.hadq_rotate(x, 256, out=out)
    torch.cuda.synchronize()
    ob = obuf.cpu().numpy()
    assert (ob[:pad] == -7.0).all() and (ob[pad + rows * n:] == -7.0).all()


def test_failed_call_leaves_outputs_untouched():
    x = torch.zeros(4, 1024, dtype=torch.bfloat16, device="cuda")
    codes = torch.full((4, 512), 0x3C, dtype=torch.uint8, device="cuda")
    scales = torch.full((4, 8), 1.5, dtype=torch.float16, device="cuda")
    with pytest.raises(H.HadqError) as e:
        H.hadq_rotate_quant(x, 96, "int4", 128, codes=codes, scales=scales)   # bad block
    assert e.value.status == H.HADQ_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (codes == 0x3C).all() and (scales == 1.5).all()


def test_side_stream_and_host_entry_point():
    rows, n = 257, 4096
    stored, x64 = synth(rows, n, "bf16", seed=21)
    s = torch.cuda.Stream()
    x = to_dev(stored, "bf16")
    torch.cuda.synchronize()
    with torch.cuda.stream(s):
        c1, s1 = H.hadq_rotate_quant(x, 0, "int4", 128, stream=s)
    s.synchronize()
    pc.check_int4(x64, c1.cpu().numpy(), s1.cpu().numpy(), 0, 128)
    # host buffers through hadq_rotate_quant_host
    xh = torch.from_numpy(stored.view(np.int16)).view(torch.bfloat16).pin_memory()
    ch = torch.empty((rows, n // 2), dtype=torch.uint8).pin_memory()
    sh = torch.empty((rows, n // 128), dtype=torch.float16).pin_memory()
    xd = torch.empty_like(x)
    cd = torch.empty_like(c1)
    sd = torch.empty_like(s1)
    H.hadq_rotate_quant_host(xh, 0, "int4", 128, ch, sh, xd, cd, sd, stream=s)
    s.synchronize()
    assert torch.equal(ch, c1.cpu()) and torch.equal(sh, s1.cpu())


def test_offsets_beyond_2_31_elements():
    """Rows whose element offsets exceed 2^31 (64-bit indexing in every kernel family)."""
    n = 8192
    rows = (1 << 31) // n + 64            # 2^31 + 2^19 elements, 4.3 GB of bf16
    x = torch.zeros((rows, n), dtype=torch.bfloat16, device="cuda")
    tail, x64 = synth(64, n, "bf16", seed=31)
    x[-64:] = torch.from_numpy(tail.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales = H.hadq_rotate_quant(x, 0, "mxfp4", 32)
    torch.cuda.synchronize()
    pc.check_mxfp4(x64, codes[-64:].cpu().numpy(), scales[-64:].cpu().numpy(), 0)
    codes, scales = H.hadq_rotate_quant(x, 128, "int4", 128)
    torch.cuda.synchronize()
    pc.check_int4(x64, codes[-64:].cpu().numpy(), scales[-64:].cpu().numpy(), 128, 128)
    del x, codes, scales
    torch.cuda.empty_cache()



@pytest.mark.parametrize("rows,n,block,x_dtype", [(37, 1024, 0, "f32"), (29, 1024, 32, "bf16"), (9, 2048, 256, "bf16"),
                                                  (13, 48, 16, "f32")])
@pytest.mark.parametrize("t", [1.0, 0.25, 3.0, "amax"])
def test_nvfp4_tensor_scale(rows, n, block, x_dtype, t):
    """hadq_rotate_quant_nvfp4: blocks and codes of y / t (t = 1, a power of
    2, a non-power of 2, and the full-range choice amax(y) / (6 * 448))."""
    stored, x64 = synth(rows, n, x_dtype, seed=n + rows, dist="t")
    if t == "amax":
        t = float(np.abs(oracle.rotate(x64, block)).max() / (6 * 448))
    codes, scales = H.hadq_rotate_quant_nvfp4(to_dev(stored, x_dtype), t, block)
    torch.cuda.synchronize()
    _log(f"nvfp4-t{t:.4g}-{rows}x{n}-b{block}",
         pc.check_nvfp4(x64, codes.cpu().numpy(), scales.cpu().numpy(), block, tensor_scale=t))
