"""GPU parity of the tensor-core (tcgen05 + TMA) path against the float64 oracle.

The path serves full-size rotations of b = 4096 and 8192 and block-128
rotations (R3 heads, R4 rotation_size 128) with bf16 input and is the
default there.  Every test runs it (hadq_set_impl(tensor)), compares with
the oracle exactly as the butterfly tests do, and checks that no bounded wait
inside the kernel ran out (hadq_device_faults() == 0).
"""


import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from hadamard_rotation_bit_b200 import workloads as W
from tests import parity_check as pc
from tests.test_gpu_parity import NPROC, _log, run_quant, run_rotate, synth, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def tensor_path():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    old = H.hadq_set_impl("tensor")
    H.hadq_device_faults(clear=True)
    yield
    torch.cuda.synchronize()
    faults = H.hadq_device_faults(clear=True)
    H.hadq_set_impl(old)
    assert faults == 0, f"tensor-core kernel reported fault bits {faults}"


SIZES = [(4, 4096, 0), (19, 4096, 0), (2, 8192, 0), (7, 8192, 0), (3, 12288, 4096), (3, 16384, 8192),
         (1, 4096, 0), (1, 8192, 0)]


@pytest.mark.parametrize("rows,n,block", SIZES)
def test_tc_rotate(rows, n, block):
    stored, x64 = synth(rows, n, "bf16", seed=n + rows + 101)
    _log(f"tc-rot-f32-{rows}x{n}", pc.check_rotation_f32(x64, run_rotate(stored, "bf16", block, "f32"), block))
    _log(f"tc-rot-bf16-{rows}x{n}", pc.check_rotation_bf16(x64, run_rotate(stored, "bf16", block, "bf16"), block))


@pytest.mark.parametrize("rows,n,block", SIZES)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 64), ("int4", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_tc_quant(rows, n, block, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=3 * n + rows + group, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    _log(f"tc-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group))


@pytest.mark.parametrize("rows,n,fmt,group", [(2501, 4096, "int4", 128), (3001, 8192, "mxfp4", 32),
                                              (1037, 4096, "mxfp4", 32), (999, 8192, "int4", 64),
                                              (1501, 4096, "nvfp4", 16), (777, 8192, "nvfp4", 16)])
def test_tc_many_tiles_ragged(rows, n, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=rows + 7)
    codes, scales = run_quant(stored, "bf16", 0, fmt, group)
    _log(f"tc-grid-{fmt}-{rows}x{n}", pc.check(fmt, x64, codes, scales, 0, group))


def test_default_path_is_the_tensor_core_kernel():
    """With the default choice (auto) the full-size bf16 rotation takes the tensor-core
    kernel: same codes as the forced tensor path, bit for bit."""
    stored, x64 = synth(64, 4096, "bf16", seed=5)
    c_t, s_t = run_quant(stored, "bf16", 0, "int4", 128)
    H.hadq_set_impl("auto")
    c_d, s_d = run_quant(stored, "bf16", 0, "int4", 128)
    H.hadq_set_impl("tensor")
    np.testing.assert_array_equal(c_d, c_t)
    np.testing.assert_array_equal(s_d, s_t)


def test_tc_config_c2():
    w = W.WORKLOADS["c2"]
    stored = W.generate("c2", workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, "int4", 128)
    _log("tc-c2", pc.check_int4(W.bits_to_float64(stored, "bf16"), codes, scales, w.block, 128))


def test_tc_config_c5():
    w = W.WORKLOADS["c5"]
    stored = W.generate("c5", workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, "mxfp4", 32)
    rng = np.random.default_rng(5)
    ids = np.unique(np.concatenate([np.arange(256), np.arange(w.rows - 256, w.rows),
                                    rng.choice(w.rows, 2048, replace=False)]))
    _log("tc-c5", pc.check_mxfp4(W.bits_to_float64(stored[ids], "bf16"), codes[ids], scales[ids], w.block))


def test_tc_matches_butterfly_codes():
    """Both implementations agree with the oracle; here also with each other
    outside the oracle's boundary window (same C2 slice, same format)."""
    stored, x64 = synth(512, 4096, "bf16", seed=77)
    c_tc, s_tc = run_quant(stored, "bf16", 0, "int4", 128)
    H.hadq_set_impl("butterfly")
    c_bf, s_bf = run_quant(stored, "bf16", 0, "int4", 128)
    H.hadq_set_impl("tensor")
    pc.check_int4(x64, c_tc, s_tc, 0, 128)
    pc.check_int4(x64, c_bf, s_bf, 0, 128)
    differ = (pc.unpack_nibbles(c_tc, True) != pc.unpack_nibbles(c_bf, True)).sum()
    assert differ <= 64, f"{differ} codes differ between the two implementations"


def test_tc_guard_bytes_and_offsets():
    rows, n = 37, 8192
    stored, x64 = synth(rows, n, "bf16", seed=12)
    x = to_dev(stored, "bf16")
    pad = 4096
    cbytes, sbytes = rows * n // 2, rows * n // 32
    cbuf = torch.full((cbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((sbytes + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    codes = cbuf[pad:pad + cbytes].view(rows, n // 2)
    scales = sbuf[pad:pad + sbytes].view(rows, n // 32)
    H.hadq_rotate_quant(x, 0, "mxfp4", 32, codes=codes, scales=scales)
    torch.cuda.synchronize()
    cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
    assert (cb[:pad] == 0xA5).all() and (cb[pad + cbytes:] == 0xA5).all()
    assert (sb[:pad] == 0x5A).all() and (sb[pad + sbytes:] == 0x5A).all()
    pc.check_mxfp4(x64, codes.cpu().numpy(), scales.cpu().numpy(), 0)


def test_tc_offsets_beyond_2_31_elements():
    n = 8192
    rows = (1 << 31) // n + 64
    x = torch.zeros((rows, n), dtype=torch.bfloat16, device="cuda")
    tail, x64 = synth(64, n, "bf16", seed=31)
    x[-64:] = torch.from_numpy(tail.view(np.int16)).view(torch.bfloat16).cuda()
    codes, scales = H.hadq_rotate_quant(x, 0, "mxfp4", 32)
    torch.cuda.synchronize()
    pc.check_mxfp4(x64, codes[-64:].cpu().numpy(), scales[-64:].cpu().numpy(), 0)
    del x, codes, scales
    torch.cuda.empty_cache()


# ------------------------------------------------------- block-128 kernel

B128 = [(37, 128), (1, 128), (300, 128), (13, 1024), (5, 14336), (129, 4096)]


@pytest.mark.parametrize("rows,n", B128)
def test_tc128_rotate(rows, n):
    stored, x64 = synth(rows, n, "bf16", seed=n + rows + 5)
    _log(f"tc128-rot-f32-{rows}x{n}", pc.check_rotation_f32(x64, run_rotate(stored, "bf16", 128, "f32"), 128))
    _log(f"tc128-rot-bf16-{rows}x{n}", pc.check_rotation_bf16(x64, run_rotate(stored, "bf16", 128, "bf16"), 128))


@pytest.mark.parametrize("rows,n", B128)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 64), ("int4", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_tc128_quant(rows, n, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=5 * n + rows + group, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, "bf16", 128, fmt, group)
    _log(f"tc128-{fmt}{group}-{rows}x{n}", pc.check(fmt, x64, codes, scales, 128, group))


@pytest.mark.parametrize("rows,n", [(5, 14336), (77, 4096), (33, 16384), (3, 8192)])
def test_tc128_int8_per_token(rows, n):
    stored, x64 = synth(rows, n, "bf16", seed=rows * 3 + n)
    codes, scales = run_quant(stored, "bf16", 128, "int8", 0)
    _log(f"tc128-int8-{rows}x{n}", pc.check_int8(x64, codes, scales, 128))


def test_tc128_config_c3():
    w = W.WORKLOADS["c3"]
    stored = W.generate("c3", workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, "int8", 0)
    _log("tc128-c3", pc.check_int8(W.bits_to_float64(stored, "bf16"), codes, scales, w.block))


def test_tc128_config_c4():
    wq = W.WORKLOADS["c4q"]
    q_stored = W.generate("c4q", workers=NPROC)
    q_out = run_rotate(q_stored, "bf16", 128, "bf16")
    k_stored = W.generate("c4k", workers=NPROC)
    k_codes, k_scales = run_quant(k_stored, "bf16", 128, "int4", 128)
    rng = np.random.default_rng(4)
    ids = np.unique(np.concatenate([np.arange(4096), np.arange(wq.rows - 4096, wq.rows),
                                    rng.choice(wq.rows, 65536, replace=False)]))
    _log("tc128-c4q", pc.check_rotation_bf16(W.bits_to_float64(q_stored[ids], "bf16"), q_out[ids], 128))
    _log("tc128-c4k", pc.check_int4(W.bits_to_float64(k_stored[ids], "bf16"), k_codes[ids], k_scales[ids], 128, 128))


def test_tc128_guard_bytes_ragged_blocks():
    rows, n = 301, 128
    stored, x64 = synth(rows, n, "bf16", seed=19)
    x = to_dev(stored, "bf16")
    pad = 4096
    cbytes, sbytes = rows * n // 2, rows * n // 128 * 2
    cbuf = torch.full((cbytes + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((sbytes + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    codes = cbuf[pad:pad + cbytes].view(rows, n // 2)
    scales = sbuf[pad:pad + sbytes].view(torch.float16).view(rows, 1)
    H.hadq_rotate_quant(x, 128, "int4", 128, codes=codes, scales=scales)
    torch.cuda.synchronize()
    cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
    assert (cb[:pad] == 0xA5).all() and (cb[pad + cbytes:] == 0xA5).all()
    assert (sb[:pad] == 0x5A).all() and (sb[pad + sbytes:] == 0x5A).all()
    pc.check_int4(x64, codes.cpu().numpy(), scales.cpu().numpy(), 128, 128)



@pytest.mark.parametrize("rows,n,block", [(19, 4096, 0), (7, 8192, 0), (33, 1024, 128)])
@pytest.mark.parametrize("t", [0.25, 3.0, "amax"])
def test_tc_nvfp4_tensor_scale(rows, n, block, t):
    stored, x64 = synth(rows, n, "bf16", seed=n + rows, dist="t")
    if t == "amax":
        t = float(np.abs(oracle.rotate(x64, block)).max() / (6 * 448))
    codes, scales = H.hadq_rotate_quant_nvfp4(to_dev(stored, "bf16"), t, block)
    torch.cuda.synchronize()
    _log(f"tc-nvfp4-t{t:.4g}-{rows}x{n}-b{block}",
         pc.check_nvfp4(x64, codes.cpu().numpy(), scales.cpu().numpy(), block, tensor_scale=t))


@pytest.mark.parametrize("key", ["c2n", "c5n"])
def test_tc_nvfp4_configs(key):
    w = W.WORKLOADS[key]
    rows = w.rows if key == "c2n" else 8192
    stored = W.generate(key, slice(0, rows), workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, "nvfp4", 16)
    rng = np.random.default_rng(6)
    ids = np.unique(np.concatenate([np.arange(128), np.arange(rows - 128, rows), rng.choice(rows, 1024, replace=False)]))
    _log(f"tc-{key}", pc.check_nvfp4(W.bits_to_float64(stored[ids], "bf16"), codes[ids], scales[ids], w.block))


# ------------------------- blocks of 256 .. 2048 on the block-128 kernel

# (rows, n, block): block and full size, ragged chunk counts, tiles that loop
BLK = [(37, 256, 0), (300, 4096, 256), (13, 512, 0), (129, 8192, 512), (5, 1024, 0), (77, 4096, 1024),
       (3, 2048, 0), (65, 14336, 2048), (1000, 1024, 0)]


@pytest.mark.parametrize("rows,n,block", BLK)
def test_tc_blocks_rotate(rows, n, block):
    stored, x64 = synth(rows, n, "bf16", seed=n + rows + block)
    _log(f"tcb-rot-f32-{rows}x{n}-b{block}", pc.check_rotation_f32(x64, run_rotate(stored, "bf16", block, "f32"), block))
    pc.check_rotation_bf16(x64, run_rotate(stored, "bf16", block, "bf16"), block)


@pytest.mark.parametrize("rows,n,block", BLK)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_tc_blocks_quant(rows, n, block, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=7 * n + rows + group + block,
                        dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    _log(f"tcb-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group))


@pytest.mark.parametrize("n,block,fmt,group", [(8192, 256, "int4", 128), (1024, 0, "mxfp4", 32)])
def test_tc_blocks_match_butterfly(n, block, fmt, group):
    """The per-Linear shapes through both implementations: both pass the
    oracle and agree on all but a few boundary codes."""
    stored, x64 = synth(512, n, "bf16", seed=n + block + 1, dist="t")
    c_tc, s_tc = run_quant(stored, "bf16", block, fmt, group)
    H.hadq_set_impl("butterfly")
    c_bf, s_bf = run_quant(stored, "bf16", block, fmt, group)
    H.hadq_set_impl("tensor")
    pc.check(fmt, x64, c_tc, s_tc, block, group)
    pc.check(fmt, x64, c_bf, s_bf, block, group)
    assert (c_tc != c_bf).sum() <= 32
