"""GPU parity of the non-power-of-2 rotations, b = K * 2^m, against the oracle.

"Rotation Transform" (AutoRound docs), section 1.5: a dimension that is not a
power of 2 is factored n = K * 2^m and rotated by a base Hadamard matrix of
order K combined with a Sylvester block.  The oracle builds H_K (Paley's
second construction, its reading of the unprinted base matrices) and the
dense Kronecker product explicitly; the kernel mixes the K sub-blocks with a
compile-time sign table and runs the 2^m butterfly.  Every covered K, both
input dtypes, every output format, block-diagonal use, random Hadamard signs
on both sides, ragged row counts, grids that loop, and the full R4 rotation
of the 8192 x 14336 down_proj input (K = 28, 2^m = 512) at full size.
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

# (rows, n, block): every covered K at its smallest and a larger 2^m, full
# rows and block-diagonal ones
SIZES = [(13, 12 * 64, 0), (9, 12 * 1024, 0), (11, 20 * 64, 0), (7, 20 * 256, 0), (10, 28 * 64, 0),
         (6, 28 * 512, 0), (5, 36 * 128, 0), (5, 52 * 64, 0), (5, 52 * 256, 0), (4, 60 * 128, 0),
         (3, 108 * 64, 0), (2, 108 * 128, 0), (4, 3 * 28 * 64, 28 * 64), (3, 2 * 20 * 128, 20 * 128)]


@pytest.fixture(autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()


@pytest.mark.parametrize("rows,n,block", SIZES)
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_ksize_rotate(rows, n, block, x_dtype):
    if x_dtype == "f32" and oracle.resolve_block(n, block) > 16384:
        pytest.skip("fp32 blocks above 16384 elements do not fit the kernel's shared memory")
    stored, x64 = synth(rows, n, x_dtype, seed=n + rows)
    _log(f"ks-rot-{x_dtype}-{rows}x{n}-b{block}", pc.check_rotation_f32(x64, run_rotate(stored, x_dtype, block, "f32"), block))
    pc.check_rotation_bf16(x64, run_rotate(stored, x_dtype, block, "bf16"), block)


@pytest.mark.parametrize("rows,n,block", SIZES)
@pytest.mark.parametrize("fmt,group", [("int4", 32), ("int4", 64), ("int4", 128), ("int8", 0), ("mxfp4", 32),
                                       ("nvfp4", 16)])
def test_ksize_quant(rows, n, block, fmt, group):
    if fmt == "int8" and block not in (0, n):
        pytest.skip("per-token int8 with a K * 2^m block needs the full row")
    stored, x64 = synth(rows, n, "bf16", seed=2 * n + rows + group, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    codes, scales = run_quant(stored, "bf16", block, fmt, group)
    _log(f"ks-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group))


@pytest.mark.parametrize("n,fmt,group", [(28 * 512, "int4", 128), (12 * 256, "int8", 0), (20 * 64, "mxfp4", 32)])
def test_ksize_fp32_input_quant(n, fmt, group):
    stored, x64 = synth(9, n, "f32", seed=n + 3)
    codes, scales = run_quant(stored, "f32", 0, fmt, group)
    pc.check(fmt, x64, codes, scales, 0, group)


@pytest.mark.parametrize("rows,n,fmt,group", [(2001, 12 * 64, "int4", 128), (1537, 28 * 128, "int8", 0),
                                              (777, 20 * 256, "mxfp4", 32)])
def test_ksize_grids_that_loop(rows, n, fmt, group):
    """More blocks than resident CTAs: every CTA runs several blocks."""
    stored, x64 = synth(rows, n, "bf16", seed=rows)
    codes, scales = run_quant(stored, "bf16", 0, fmt, group)
    pc.check(fmt, x64, codes, scales, 0, group)


@pytest.mark.parametrize("side", ["after", "before"])
@pytest.mark.parametrize("n,block,fmt,group", [(28 * 512, 0, "int4", 128), (12 * 128, 0, "int8", 0),
                                               (2 * 20 * 64, 20 * 64, "mxfp4", 32)])
def test_ksize_random_hadamard(side, n, block, fmt, group):
    b = oracle.resolve_block(n, block)
    signs = np.where(np.random.default_rng(b).random(b) < 0.5, -1, 1).astype(np.int8)
    stored, x64 = synth(7, n, "bf16", seed=b + 1)
    c, s = H.hadq_rotate_quant_signed(to_dev(stored, "bf16"), torch.from_numpy(signs).cuda(), side, block, fmt, group)
    torch.cuda.synchronize()
    y = oracle.rotate_signed(x64, block, signs, side)
    pc.check(fmt, x64, c.cpu().numpy(), s.cpu().numpy(), block, group, y=y)
    r = H.hadq_rotate_signed(to_dev(stored, "bf16"), torch.from_numpy(signs).cuda(), side, block,
                             out_dtype=torch.float32)
    torch.cuda.synchronize()
    pc.check_rotation_f32(x64, r.cpu().numpy(), block, y=y)


def test_ksize_involution_and_in_place():
    """H_K (x) H_(2^m) is symmetric: rotating twice returns x (fp32, in place)."""
    stored, x64 = synth(6, 28 * 256, "f32", seed=9)
    x = to_dev(stored, "f32")
    H.hadq_rotate(x, 0, out=x)
    H.hadq_rotate_inverse(x, 0, out=x)
    torch.cuda.synchronize()
    err = np.abs(x.cpu().numpy().astype(np.float64) - x64).max(axis=1) / np.linalg.norm(x64, axis=1)
    assert err.max() < 1e-6, err.max()


def test_ksize_guard_bytes():
    """Outputs are written exactly: sentinel bytes around codes and scales survive."""
    rows, n = 5, 20 * 128
    stored, x64 = synth(rows, n, "bf16", seed=4)
    pad = 256
    codes = torch.full((rows * n // 2 + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    scales = torch.full((rows * n // 128 * 2 + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    cv = codes[pad:pad + rows * n // 2].view(rows, n // 2)
    sv = scales[pad:pad + rows * n // 64].view(torch.float16).view(rows, n // 128)
    H.hadq_rotate_quant(to_dev(stored, "bf16"), 0, "int4", 128, codes=cv, scales=sv)
    torch.cuda.synchronize()
    c, s = codes.cpu().numpy(), scales.cpu().numpy()
    assert (c[:pad] == 0xA5).all() and (c[-pad:] == 0xA5).all()
    assert (s[:pad] == 0x5A).all() and (s[-pad:] == 0x5A).all()
    pc.check_int4(x64, cv.cpu().numpy(), sv.cpu().numpy(), 0, 128)


def test_config_c3k_full_size():
    """The R4 down_proj input rotated in full: 8192 x 14336 bf16, H_28 (x) H_512,
    int8 per token (the bench's c3k configuration), every row checked."""
    w = W.WORKLOADS["c3k"]
    stored = W.generate("c3k", workers=NPROC)
    codes, scales = run_quant(stored, "bf16", w.block, w.fmt, w.group)
    _log("c3k", pc.check_int8(W.bits_to_float64(stored, "bf16"), codes, scales, w.block))
