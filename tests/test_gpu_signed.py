"""GPU parity of the random Hadamard entry points against the float64 oracle.

hadq_rotate_signed / hadq_rotate_quant_signed multiply every block by
R = H_b diag(s) / sqrt(b) (side "after", the random_hadamard_matrix of
"Rotation Transform" section 1.5) or by its transpose diag(s) H_b / sqrt(b)
(side "before").  Each case runs through the C ABI on seeded inputs and is
compared element by element with oracle.rotate_signed under the same
tolerances as the deterministic rotation.  Both implementations are covered:
the tensor-core kernels (default for bf16 at b = 4096, 8192 and 128, either
side: signs after in the epilogue, signs before flipped in the staged tile
ahead of the MMA, and at b = 128 both folded into the H_128 operand) and the
CUDA-core butterfly kernels (everything else).
"""


import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import _log, synth, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(params=["auto", "butterfly"])
def path(request):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()
    old = H.hadq_set_impl(request.param)
    H.hadq_device_faults(clear=True)
    yield request.param
    torch.cuda.synchronize()
    faults = H.hadq_device_faults(clear=True)
    H.hadq_set_impl(old)
    assert faults == 0, f"tensor-core kernel reported fault bits {faults}"


def signs_for(b, seed, odd_values=False):
    """b int8 signs; with odd_values, negatives and non-negatives other than +/-1
    (the contract: negative = -1, anything else = +1)."""
    rng = np.random.default_rng(seed)
    s = np.where(rng.random(b) < 0.5, -1, 1).astype(np.int8)
    if odd_values:
        s = np.where(s < 0, rng.choice([-128, -77, -1], b), rng.choice([0, 1, 42, 127], b)).astype(np.int8)
    return s


def run_signed_quant(stored, x_dtype, block, signs, side, fmt, group):
    codes, scales = H.hadq_rotate_quant_signed(to_dev(stored, x_dtype), torch.from_numpy(signs).cuda(), side,
                                               block, fmt, group)
    torch.cuda.synchronize()
    return codes.cpu().numpy(), scales.cpu().numpy()


def run_signed_rotate(stored, x_dtype, block, signs, side, out_dtype):
    out = H.hadq_rotate_signed(to_dev(stored, x_dtype), torch.from_numpy(signs).cuda(), side, block,
                               out_dtype=torch.float32 if out_dtype == "f32" else torch.bfloat16)
    torch.cuda.synchronize()
    if out_dtype == "f32":
        return out.cpu().numpy()
    return out.view(torch.int16).cpu().numpy().view(np.uint16)


CASES = [  # (rows, n, block, x_dtype): which kernel serves it under "auto"
    (19, 4096, 0, "bf16"),     # tensor core, n = 4096
    (7, 8192, 0, "bf16"),      # tensor core, n = 8192
    (33, 1024, 128, "bf16"),   # tensor core, block 128
    (5, 14336, 128, "bf16"),   # tensor core, block 128, 112 blocks per row
    (37, 1024, 0, "f32"),      # team kernel
    (9, 2048, 256, "bf16"),    # team kernel, block 256
    (3, 12288, 4096, "f32"),   # team kernel, block 4096
    (29, 1024, 32, "f32"),     # segment kernel
    (13, 96, 32, "bf16"),      # segment kernel, ragged n
    (11, 200, 8, "f32"),       # segment kernel, b = 8
    (37, 64, 0, "bf16"),       # segment kernel, full 64
]


def _fmt_ok(n, fmt, group):
    return (fmt != "int4" or n % group == 0) and (fmt != "mxfp4" or n % 32 == 0) and (fmt != "nvfp4" or n % 16 == 0)


@pytest.mark.parametrize("rows,n,block,x_dtype", CASES)
@pytest.mark.parametrize("side", ["after", "before"])
def test_signed_rotate(path, rows, n, block, x_dtype, side):
    b = oracle.resolve_block(n, block)
    stored, x64 = synth(rows, n, x_dtype, seed=n + rows + 3)
    s = signs_for(b, n + block)
    y = oracle.rotate_signed(x64, block, s, side)
    _log(f"signed-{path}-{side}-rot-f32-{rows}x{n}-b{block}",
         pc.check_rotation_f32(x64, run_signed_rotate(stored, x_dtype, block, s, side, "f32"), block, y=y))
    _log(f"signed-{path}-{side}-rot-bf16-{rows}x{n}-b{block}",
         pc.check_rotation_bf16(x64, run_signed_rotate(stored, x_dtype, block, s, side, "bf16"), block, y=y))


@pytest.mark.parametrize("rows,n,block,x_dtype", CASES)
@pytest.mark.parametrize("side", ["after", "before"])
@pytest.mark.parametrize("fmt,group", [("int4", 128), ("int4", 32), ("int8", 0), ("mxfp4", 32), ("nvfp4", 16)])
def test_signed_quant(path, rows, n, block, x_dtype, side, fmt, group):
    if not _fmt_ok(n, fmt, group):
        pytest.skip("group does not divide n")
    b = oracle.resolve_block(n, block)
    stored, x64 = synth(rows, n, x_dtype, seed=2 * n + rows + group, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    s = signs_for(b, 3 * n + block + group)
    y = oracle.rotate_signed(x64, block, s, side)
    codes, scales = run_signed_quant(stored, x_dtype, block, s, side, fmt, group)
    _log(f"signed-{path}-{side}-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, codes, scales, block, group, y=y))


@pytest.mark.parametrize("rows,n,block,x_dtype", [(19, 4096, 0, "bf16"), (7, 8192, 0, "bf16"), (33, 1024, 128, "bf16"),
                                                  (37, 1024, 0, "f32"), (29, 1024, 32, "f32")])
@pytest.mark.parametrize("side", ["after", "before"])
def test_signed_any_negative_int8_is_minus_one(path, rows, n, block, x_dtype, side):
    b = oracle.resolve_block(n, block)
    stored, x64 = synth(rows, n, x_dtype, seed=rows)
    s = signs_for(b, 99, odd_values=True)
    assert set(np.unique(s)) - {-1, 1}
    y = oracle.rotate_signed(x64, block, s, side)
    codes, scales = run_signed_quant(stored, x_dtype, block, s, side, "int4", 128)
    pc.check_int4(x64, codes, scales, block, 128, y=y)


@pytest.mark.parametrize("rows,n,block,x_dtype", [(19, 4096, 0, "bf16"), (7, 8192, 0, "bf16"),
                                                  (33, 1024, 128, "bf16"), (37, 1024, 0, "f32")])
def test_signed_after_then_before_is_identity(path, rows, n, block, x_dtype):
    """R^T R = I on the device: rotate with side after, then before, in fp32."""
    b = oracle.resolve_block(n, block)
    stored, x64 = synth(rows, n, x_dtype, seed=rows + 1)
    s = torch.from_numpy(signs_for(b, 5)).cuda()
    y = H.hadq_rotate_signed(to_dev(stored, x_dtype), s, "after", block, out_dtype=torch.float32)
    back = H.hadq_rotate_signed(y, s, "before", block).cpu().numpy()
    err = np.abs(back - x64).max(axis=1) / np.linalg.norm(x64, axis=1)
    assert err.max() < 2e-5


def test_signed_all_plus_matches_deterministic(path):
    """All-plus signs reproduce hadq_rotate_quant bit for bit (same kernel family)."""
    for rows, n, block, x_dtype in [(19, 4096, 0, "bf16"), (33, 1024, 128, "bf16"), (29, 1024, 32, "f32")]:
        stored, _ = synth(rows, n, x_dtype, seed=rows + 2)
        x = to_dev(stored, x_dtype)
        ones = torch.ones(oracle.resolve_block(n, block), dtype=torch.int8, device="cuda")
        c0, s0 = H.hadq_rotate_quant(x, block, "int4", 128)
        c1, s1 = H.hadq_rotate_quant_signed(x, ones, "after", block, "int4", 128)
        torch.cuda.synchronize()
        assert torch.equal(c0, c1) and torch.equal(s0.view(torch.int16), s1.view(torch.int16))


def test_signed_exact_zero_rows_code_as_plus_zero(path):
    """A zero row rotates to exact zeros; negating them must not set MXFP4
    sign bits (the oracle codes +0 and -0 as 0)."""
    rows, n = 8, 4096
    stored, x64 = synth(rows, n, "bf16", seed=8)
    stored[::2] = 0
    x64[::2] = 0.0
    s = signs_for(n, 17)
    y = oracle.rotate_signed(x64, 0, s, "after")
    codes, scales = run_signed_quant(stored, "bf16", 0, s, "after", "mxfp4", 32)
    assert (codes[::2] == 0).all() and (scales[::2] == 0).all()
    pc.check_mxfp4(x64, codes, scales, 0, y=y)


@pytest.mark.parametrize("key", ["c2r", "c2rb", "c3rb", "c5rb"])
def test_signed_config_full_size(key):
    """The bench's random Hadamard workloads at full size in the default
    kernel choice, all on the tensor cores: c2r (4096 x 4096 bf16 -> int4
    g128, signs after, applied in the epilogue), c2rb (the same, signs before,
    flipped in each staged tile ahead of the MMA), c3rb (8192 x 14336, block
    128, int8 per token, signs folded into the H_128 operand) and c5rb
    (65536 x 8192 -> MXFP4, signs before; oracle on a seeded row sample)."""
    from hadamard_rotation_bit_b200 import workloads as W
    from tests.test_gpu_parity import NPROC
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()
    w = W.WORKLOADS[key]
    stored = W.generate(key, workers=NPROC)
    s = W.generate_signs(key)
    ids = slice(None)
    if key == "c5rb":
        rng = np.random.default_rng(7)
        ids = np.unique(np.concatenate([np.arange(256), np.arange(w.rows - 256, w.rows),
                                        rng.choice(w.rows, 2048, replace=False)]))
    x64 = W.bits_to_float64(stored[ids], "bf16")
    y = oracle.rotate_signed(x64, w.block, s, w.signs)
    H.hadq_device_faults(clear=True)
    codes, scales = run_signed_quant(stored, "bf16", w.block, s, w.signs, w.fmt, w.group)
    assert H.hadq_device_faults(clear=True) == 0
    _log(f"signed-{key}", pc.check(w.fmt, x64, codes[ids], scales[ids], w.block, w.group, y=y))
