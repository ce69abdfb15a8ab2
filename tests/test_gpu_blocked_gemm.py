"""GPU: FP4 codes with their scales in the tiled layout of block-scaled GEMMs,
fed straight into a W4A4 product.

"Rotation Transform" (AutoRound docs), introduction and section 2.1: the
rotated activations are quantized to MXFP4 / NVFP4 for the matmuls that
consume them, and x R (W R)^T = x W^T.  The blocked formats write the same
codes and scale values as HADQ_MXFP4 / HADQ_NVFP4, with the scales laid out
as block-scaled tensor-core GEMMs read them (the "1D block scaling factors"
layout of NVIDIA's cuBLAS documentation), restated here from its definition
as an index map of its own.  Checked: codes bit-identical to the row-major
formats, scales equal after undoing the layout, padding rows zero, parity
with the oracle, and a block-scaled GEMM (torch.nn.functional.scaled_mm, a
library GEMM) on the library's outputs of both x and W equal to the float64
product of the decoded codes, within 0.2 of x W^T (relative Frobenius
error), and for MXFP4 closer to x W^T than the same product without the
rotation when x has outlier channels.
"""

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import _log, synth, to_dev

pytestmark = pytest.mark.gpu

E2M1 = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


@pytest.fixture(autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()


def tile_offsets(rows_padded: int, cols: int) -> np.ndarray:
    """Byte offset of scale (r, c): 128 x 4 tiles of 512 bytes, row-block
    major; inside a tile (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4."""
    r = np.arange(rows_padded)[:, None]
    c = np.arange(cols)[None, :]
    return ((r // 128) * (cols // 4) + c // 4) * 512 + (r % 32) * 16 + ((r // 32) % 4) * 4 + c % 4


def unblock(flat: np.ndarray, rows: int, cols: int) -> np.ndarray:
    return flat.reshape(-1)[tile_offsets((rows + 127) // 128 * 128, cols)[:rows]]


def decode_fp4(codes_packed: np.ndarray, scales: np.ndarray, fmt: str) -> np.ndarray:
    """Values of packed E2M1 codes (element 2i in the low nibble) times their
    block scales (E8M0: 2^(byte - 127); E4M3: the float8 value)."""
    lo, hi = codes_packed & 0xF, codes_packed >> 4
    q = np.empty((codes_packed.shape[0], codes_packed.shape[1] * 2), dtype=np.uint8)
    q[:, 0::2], q[:, 1::2] = lo, hi
    v = E2M1[q & 7] * np.where(q & 8, -1.0, 1.0)
    blk = 32 if fmt.startswith("mxfp4") else 16
    if blk == 32:
        s = np.ldexp(1.0, scales.astype(np.int64) - 127)
    else:
        s = torch.from_numpy(scales.copy()).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    return v * np.repeat(s, blk, axis=1)


@pytest.mark.parametrize("fmt", ["mxfp4", "nvfp4"])
@pytest.mark.parametrize("rows,n,block", [(256, 4096, 0), (300, 4096, 0), (5, 8192, 0), (129, 8192, 0),
                                          (300, 14336, 128), (129, 8192, 256), (37, 2048, 0), (130, 14336, 0),
                                          (5, 28 * 256, 0)])
def test_blocked_scales_match_row_major(fmt, rows, n, block):
    """Every tensor-core shape: full 4096 / 8192, blocks of 128 .. 2048, K * 2^m
    (14336 = 28 * 512, 7168 = 28 * 256)."""
    stored, x64 = synth(rows, n, "bf16", seed=rows + n + block, dist="t")
    x = to_dev(stored, "bf16")
    c_rm, s_rm = H.hadq_rotate_quant(x, block, fmt, 32 if fmt == "mxfp4" else 16)
    c_bl, s_bl = H.hadq_rotate_quant(x, block, fmt + "_blocked", 32 if fmt == "mxfp4" else 16)
    torch.cuda.synchronize()
    cols = n // (32 if fmt == "mxfp4" else 16)
    assert s_bl.shape == ((rows + 127) // 128 * 128, cols)
    assert torch.equal(c_rm, c_bl)
    flat = s_bl.cpu().numpy().reshape(-1)
    np.testing.assert_array_equal(unblock(flat, rows, cols), s_rm.cpu().numpy())
    pad = np.ones(flat.size, dtype=bool)
    pad[tile_offsets((rows + 127) // 128 * 128, cols)[:rows].reshape(-1)] = False
    assert not flat[pad].any(), "padding rows are zero"
    _log(f"blocked-{fmt}-{rows}x{n}-b{block}", pc.check(fmt, x64, c_bl.cpu().numpy(), unblock(flat, rows, cols), block,
                                                         32 if fmt == "mxfp4" else 16))


def _scaled_mm(a_codes, a_scales, w_codes, w_scales, fmt, k):
    F = torch.nn.functional
    blk = 32 if fmt == "mxfp4" else 16
    sdt = torch.float8_e8m0fnu if fmt == "mxfp4" else torch.float8_e4m3fn
    recipe = F.ScalingType.BlockWise1x32 if fmt == "mxfp4" else F.ScalingType.BlockWise1x16
    sw = F.SwizzleType.SWIZZLE_32_4_4
    m, nw = a_codes.shape[0], w_codes.shape[0]
    a = a_codes.view(torch.float4_e2m1fn_x2)
    b = w_codes.view(torch.float4_e2m1fn_x2).t()                 # [K/2, N], column-major
    sa = a_scales.view(sdt).reshape(m, k // blk)
    sb = w_scales.view(sdt).reshape(-1).reshape(k // blk, nw)
    return F.scaled_mm(a, b, sa, recipe, sb, recipe, sw, sw, output_dtype=torch.bfloat16)


@pytest.mark.parametrize("fmt,k,block", [("mxfp4", 4096, 0), ("nvfp4", 4096, 0), ("mxfp4", 14336, 128),
                                         ("mxfp4", 14336, 0)])
def test_w4a4_gemm_on_blocked_outputs(fmt, k, block):
    """x (256 x K bf16, outlier channels) and W (512 x K bf16) rotated and
    quantized by the library (R1 at K = 4096; the down_proj input at
    K = 14336, by blocks of 128 or in full); their codes and tiled scales go
    straight into a block-scaled GEMM."""
    m, nw = 256, 512
    blk = 32 if fmt == "mxfp4" else 16
    xs, x64 = synth(m, k, "bf16", seed=41)
    ws, w64 = synth(nw, k, "bf16", seed=42, outliers=False)
    cx, sx = H.hadq_rotate_quant(to_dev(xs, "bf16"), block, fmt + "_blocked", blk)
    cw, sw = H.hadq_rotate_quant(to_dev(ws, "bf16"), block, fmt + "_blocked", blk)
    torch.cuda.synchronize()
    try:
        y = _scaled_mm(cx, sx, cw, sw, fmt, k)
        torch.cuda.synchronize()
    except (RuntimeError, NotImplementedError, TypeError) as e:
        pytest.skip(f"block-scaled FP4 GEMM not available here: {str(e).splitlines()[0]}")
    y = y.float().cpu().numpy().astype(np.float64)
    # the GEMM's own arithmetic: the float64 product of the decoded operands
    a = decode_fp4(cx.cpu().numpy(), unblock(sx.cpu().numpy(), m, k // blk), fmt)
    w = decode_fp4(cw.cpu().numpy(), unblock(sw.cpu().numpy(), nw, k // blk), fmt)
    ref = a @ w.T
    bound = 1e-2 * np.abs(ref) + 1e-4 * (np.abs(a) @ np.abs(w).T)   # bf16 output, fp32 accumulation
    assert (np.abs(y - ref) <= bound).all(), float((np.abs(y - ref) / bound).max())
    # the library's codes are the oracle's (boundary cases aside)
    pc.check(fmt, x64, cx.cpu().numpy(), unblock(sx.cpu().numpy(), m, k // blk), block, blk)
    # the W4A4 product approximates x W^T, better with the rotation than without
    exact = x64 @ w64.T
    err_rot = np.linalg.norm(y - exact) / np.linalg.norm(exact)
    _, cxn, sxn = oracle.quantize(x64, fmt, blk)
    _, cwn, swn = oracle.quantize(w64, fmt, blk)
    err_plain = np.linalg.norm(decode_fp4(cxn, sxn, fmt) @ decode_fp4(cwn, swn, fmt).T - exact) / np.linalg.norm(exact)
    _log(f"w4a4-{fmt}-k{k}-b{block}", {"rel_err_rotated": err_rot, "rel_err_unrotated": err_plain})
    assert err_rot < 0.2, err_rot
    if fmt == "mxfp4":
        # one power-of-2 scale per 32 elements: outlier channels cost the other
        # elements of their block their precision unless the rotation spreads
        # them (NVFP4's finer blocks and E4M3 scales do not need it here:
        # measured 0.135 rotated against 0.119 unrotated on this input)
        assert err_rot < err_plain, (err_rot, err_plain)
