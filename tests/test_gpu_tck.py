"""GPU parity of the tensor-core kernels for blocks of b = K * 2^m, 2^m >= 128.

"Rotation Transform" (AutoRound docs), section 1.5: the base Hadamard matrix
of order K combined with a Sylvester block.  These kernels rotate each
128-element chunk by H_128 on the tensor core and finish H_(2^m / 128) and the
Paley H_K in the registers of the thread that holds one output of every
chunk.  Every instantiated (K, 2^m / 128) pair is checked against the oracle
for both rotation outputs and per-token int8, with block-diagonal use, grids
that loop, zero / tiny / large rows, exact output extents and agreement with
the staged kernels that serve the same shapes under the butterfly choice.
"""

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import _log, run_quant, run_rotate, synth, to_dev

pytestmark = pytest.mark.gpu

# (K, 2^m / 128) pairs with K * 2^m / 128 <= 128 chunks: every instantiation.
PAIRS = [(12, 1), (12, 2), (12, 4), (12, 8), (20, 1), (20, 2), (20, 4), (28, 1), (28, 2), (28, 4), (36, 1),
         (36, 2), (52, 1), (52, 2), (60, 1), (60, 2), (108, 1)]


@pytest.fixture(autouse=True)
def _tensor_impl():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()
    old = H.hadq_set_impl("tensor")
    yield
    H.hadq_set_impl(old)


@pytest.mark.parametrize("k,hi", PAIRS)
def test_tck_rotate_full(k, hi):
    n = k * 128 * hi
    rows = 3 + (k + hi) % 5
    stored, x64 = synth(rows, n, "bf16", seed=k * 10 + hi)
    _log(f"tck-rot-{rows}x{n}", pc.check_rotation_f32(x64, run_rotate(stored, "bf16", 0, "f32"), 0))
    pc.check_rotation_bf16(x64, run_rotate(stored, "bf16", 0, "bf16"), 0)


@pytest.mark.parametrize("k,hi", PAIRS)
def test_tck_int8_per_token(k, hi):
    n = k * 128 * hi
    rows = 4 + (k * hi) % 7
    stored, x64 = synth(rows, n, "bf16", seed=k * 100 + hi)
    codes, scales = run_quant(stored, "bf16", 0, "int8", 0)
    _log(f"tck-int8-{rows}x{n}", pc.check_int8(x64, codes, scales, 0))


@pytest.mark.parametrize("rows,n,block", [(5, 3 * 28 * 128, 28 * 128), (3, 2 * 20 * 512, 20 * 512),
                                          (4, 5 * 12 * 128, 12 * 128), (2, 2 * 60 * 256, 60 * 256)])
def test_tck_block_diagonal(rows, n, block):
    stored, x64 = synth(rows, n, "bf16", seed=n + block)
    _log(f"tck-blk-{rows}x{n}-b{block}", pc.check_rotation_f32(x64, run_rotate(stored, "bf16", block, "f32"), block))
    pc.check_rotation_bf16(x64, run_rotate(stored, "bf16", block, "bf16"), block)


@pytest.mark.parametrize("rows,n", [(1537, 28 * 128), (301, 20 * 512), (149, 12 * 1024)])
def test_tck_grids_that_loop(rows, n):
    """More blocks than CTAs (one per SM), counts that do not divide evenly."""
    stored, x64 = synth(rows, n, "bf16", seed=rows)
    codes, scales = run_quant(stored, "bf16", 0, "int8", 0)
    _log(f"tck-grid-int8-{rows}x{n}", pc.check_int8(x64, codes, scales, 0))
    pc.check_rotation_f32(x64, run_rotate(stored, "bf16", 0, "f32"), 0)


def test_tck_special_rows():
    """Zero rows (zero scale, zero codes), rows so small that the scale is tiny
    (per-element division), and large rows near the fp32 range."""
    n = 28 * 512
    rng = np.random.default_rng(3)
    v = rng.standard_normal((6, n)).astype(np.float32)
    v[0] = 0.0
    v[1] *= 1e-37
    v[2] *= 1e-30
    v[3] *= 1e30
    v[4, :] = 0.0
    v[4, 17] = 2e-38     # bf16 normal (subnormal bf16 inputs are not exercised)
    from hadamard_rotation_bit_b200 import workloads as W
    stored = W.f32_to_bf16_bits(v)
    x64 = W.bits_to_float64(stored, "bf16")
    codes, scales = run_quant(stored, "bf16", 0, "int8", 0)
    assert not codes[0].any() and scales[0] == 0.0
    _log("tck-special-int8", pc.check_int8(x64, codes, scales, 0))
    pc.check_rotation_f32(x64, run_rotate(stored, "bf16", 0, "f32"), 0)


def test_tck_guard_bytes():
    """Codes, scales and rotation outputs are written exactly: sentinels around them survive."""
    rows, n = 7, 20 * 256
    stored, x64 = synth(rows, n, "bf16", seed=77)
    x = to_dev(stored, "bf16")
    pad = 512
    cbuf = torch.full((rows * n + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((rows * 4 + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    codes = cbuf[pad:pad + rows * n].view(torch.int8).view(rows, n)
    scales = sbuf[pad:pad + rows * 4].view(torch.float32)
    H.hadq_rotate_quant(x, 0, "int8", 0, codes=codes, scales=scales)
    obuf = torch.full((rows * n + 2 * pad,), -7.0, dtype=torch.float32, device="cuda")
    out = obuf[pad:pad + rows * n].view(rows, n)
    H.hadq_rotate(x, 0, out=out)
    torch.cuda.synchronize()
    cb, sb, ob = cbuf.cpu().numpy(), sbuf.cpu().numpy(), obuf.cpu().numpy()
    assert (cb[:pad] == 0xA5).all() and (cb[-pad:] == 0xA5).all()
    assert (sb[:pad] == 0x5A).all() and (sb[-pad:] == 0x5A).all()
    assert (ob[:pad] == -7.0).all() and (ob[-pad:] == -7.0).all()
    pc.check_int8(x64, codes.cpu().numpy(), scales.cpu().numpy(), 0)
    pc.check_rotation_f32(x64, out.cpu().numpy(), 0)


def test_tck_matches_staged_kernel():
    """Both implementations of the same shape pass the oracle and agree on all
    but a few boundary codes (they sum in different orders)."""
    stored, x64 = synth(64, 28 * 512, "bf16", seed=21)
    c_tc, s_tc = run_quant(stored, "bf16", 0, "int8", 0)
    H.hadq_set_impl("butterfly")
    c_st, s_st = run_quant(stored, "bf16", 0, "int8", 0)
    H.hadq_set_impl("tensor")
    pc.check_int8(x64, c_tc, s_tc, 0)
    pc.check_int8(x64, c_st, s_st, 0)
    differ = int((c_tc != c_st).sum())
    assert differ <= 64, f"{differ} codes differ between the two implementations"
    np.testing.assert_allclose(s_tc, s_st, rtol=1e-6)


def test_tck_involution():
    """H_K (x) H_(2^m) / sqrt(b) is its own inverse: rotating the fp32 result again
    (staged kernel, fp32 input) returns the bf16 input."""
    stored, x64 = synth(5, 52 * 256, "bf16", seed=8)
    y = H.hadq_rotate(to_dev(stored, "bf16"), 0, out_dtype=torch.float32)
    back = H.hadq_rotate(y, 0)
    torch.cuda.synchronize()
    err = np.abs(back.cpu().numpy().astype(np.float64) - x64).max(axis=1) / np.linalg.norm(x64, axis=1)
    assert err.max() < 1e-6, err.max()
    assert oracle.resolve_block(52 * 256, 0) == 52 * 256


# ------------------------------------------------ the grouped quantizers

@pytest.mark.parametrize("k,hi", PAIRS)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 64), ("int4", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_tck_grouped_quant(k, hi, fmt, group):
    n = k * 128 * hi
    rows = 3 + (k * hi + group) % 6
    stored, x64 = synth(rows, n, "bf16", seed=k * 1000 + hi * 10 + group,
                        dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, "bf16", 0, fmt, group)
    _log(f"tck-{fmt}{group}-{rows}x{n}", pc.check(fmt, x64, codes, scales, 0, group))


@pytest.mark.parametrize("rows,n,block,fmt,group", [(5, 3 * 28 * 128, 28 * 128, "int4", 128),
                                                    (3, 2 * 20 * 512, 20 * 512, "mxfp4", 32),
                                                    (4, 5 * 12 * 128, 12 * 128, "nvfp4", 16),
                                                    (301, 20 * 512, 0, "int4", 64),
                                                    (149, 12 * 1024, 0, "mxfp4", 32)])
def test_tck_grouped_blocks_and_grids(rows, n, block, fmt, group):
    stored, x64 = synth(rows, n, "bf16", seed=rows + n + block + group)
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    _log(f"tck-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group))


@pytest.mark.parametrize("fmt,group", [("int4", 128), ("mxfp4", 32), ("nvfp4", 16)])
def test_tck_grouped_matches_staged(fmt, group):
    stored, x64 = synth(64, 28 * 512, "bf16", seed=23 + group, dist="t")
    c_tc, s_tc = run_quant(stored, "bf16", 0, fmt, group)
    H.hadq_set_impl("butterfly")
    c_st, s_st = run_quant(stored, "bf16", 0, fmt, group)
    H.hadq_set_impl("tensor")
    pc.check(fmt, x64, c_tc, s_tc, 0, group)
    pc.check(fmt, x64, c_st, s_st, 0, group)
    assert (c_tc != c_st).sum() <= 32


def test_config_c3km_full_size():
    """The bench's c3km workload: 8192 x 14336 bf16, H_28 (x) H_512, MXFP4,
    every row checked."""
    from hadamard_rotation_bit_b200 import workloads as W
    w = W.WORKLOADS["c3km"]
    stored = W.generate("c3km")
    codes, scales = run_quant(stored, "bf16", w.block, w.fmt, w.group)
    _log("c3km", pc.check_mxfp4(W.bits_to_float64(stored, "bf16"), codes, scales, w.block))
