"""Weight-side rotation with the same kernels (the offline half of R1 / R4).

A rotation R fused offline into a Linear layer's weight W [out, in] is
W' = W R, i.e. every row of W (one output feature over in_features) rotated
like an activation row.  The online half rotates the activations, and the
layer output is unchanged: (x R)(W R)^T = x R R^T W^T = x W^T ("Rotation
Transform", introduction and section 1.1 R1 / R4; section 2 for the
block-diagonal per-Linear mode; section 1.5 for the random Hadamard R).

Both halves go through the C ABI (hadq_rotate / hadq_rotate_signed, fp32
output) on seeded synthetic activations and weights.  The rotated W is first
compared element by element with the oracle's W R (1e-5 of each row's norm);
then the invariant itself is checked, in float64, against x W^T from the
stored input bits.
The fp32 rotation error is about 1e-7 of each row's norm, so the product
error is bounded by a few 1e-7 x |x_row| |w_row|; the test allows 1e-5.
"""

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import synth, to_dev

pytestmark = pytest.mark.gpu


def _fused_error(x64, w64, xr, wr):
    y_ref = x64 @ w64.T
    y = xr.astype(np.float64) @ wr.astype(np.float64).T
    scale = np.linalg.norm(x64, axis=1)[:, None] * np.linalg.norm(w64, axis=1)[None, :]
    return float(np.max(np.abs(y - y_ref) / scale))


@pytest.mark.parametrize("n,block,x_dtype", [(4096, 0, "bf16"), (8192, 0, "bf16"), (14336, 128, "bf16"),
                                             (2048, 0, "bf16"), (1024, 0, "f32"), (4096, 256, "f32")])
def test_weight_side_rotation_keeps_the_layer_output(n, block, x_dtype):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()
    xs, x64 = synth(48, n, x_dtype, seed=n + block)
    ws, w64 = synth(96, n, x_dtype, seed=n + block + 1, outliers=False)
    xr = H.hadq_rotate(to_dev(xs, x_dtype), block, out_dtype=torch.float32)
    wr = H.hadq_rotate(to_dev(ws, x_dtype), block, out_dtype=torch.float32)
    torch.cuda.synchronize()
    pc.check_rotation_f32(w64, wr.cpu().numpy(), block)          # W R against the oracle
    err = _fused_error(x64, w64, xr.cpu().numpy(), wr.cpu().numpy())
    assert err < 1e-5, err


@pytest.mark.parametrize("n,block", [(4096, 0), (1024, 128)])
def test_weight_side_random_hadamard_keeps_the_layer_output(n, block):
    """The same with R = H diag(s) / sqrt(b) (signs after) on both sides."""
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()
    b = n if block == 0 else block
    signs = torch.from_numpy(np.where(np.random.default_rng(b).random(b) < 0.5, -1, 1).astype(np.int8)).cuda()
    xs, x64 = synth(32, n, "bf16", seed=3 * n)
    ws, w64 = synth(64, n, "bf16", seed=3 * n + 1, outliers=False)
    xr = H.hadq_rotate_signed(to_dev(xs, "bf16"), signs, "after", block, out_dtype=torch.float32)
    wr = H.hadq_rotate_signed(to_dev(ws, "bf16"), signs, "after", block, out_dtype=torch.float32)
    torch.cuda.synchronize()
    pc.check_rotation_f32(w64, wr.cpu().numpy(), block, y=oracle.rotate_signed(w64, block, signs.cpu().numpy(), "after"))
    err = _fused_error(x64, w64, xr.cpu().numpy(), wr.cpu().numpy())
    assert err < 1e-5, err
