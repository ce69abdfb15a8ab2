"""GPU parity of the orbitquant path: RPBH rotation and the codebook quantizer.

"orbitquant 0.2.0", Method Conformance: RPBH is a permutation, Rademacher
signs, a block FWHT and orthonormal scaling; activations are quantized online
by a per-token norm, rotation of the normalized activation, the nearest
centroid of a fixed unit-sphere Lloyd-Max codebook per (dimension, bits), and
rescaling.  The oracle gathers, signs and rotates with explicit matrices and
builds its own codebook; the library's codebook (hadq_codebook, host code)
feeds the kernel.  Random permutations at blocks 128, 4096 and 8192, every
output format, both input dtypes, 2- and 4-bit codebooks with and without
the permutation, a non-power-of-2 row (14336 = 28 * 512), zero rows.
"""

import numpy as np
import pytest
import torch

import oracle
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import _log, synth, to_dev

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    H.load_library()


def rpbh_args(n, seed):
    rng = np.random.default_rng(seed)
    perm = rng.permutation(n).astype(np.int32)
    signs = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    return perm, signs, torch.from_numpy(perm).cuda(), torch.from_numpy(signs).cuda()


@pytest.mark.parametrize("rows,n,block", [(5, 4096, 128), (7, 4096, 4096), (3, 8192, 8192), (9, 1024, 32),
                                          (4, 14336, 128), (6, 2048, 0), (3, 8192, 1024)])
@pytest.mark.parametrize("x_dtype", ["bf16", "f32"])
def test_rpbh_rotate(rows, n, block, x_dtype):
    stored, x64 = synth(rows, n, x_dtype, seed=n + block + rows)
    perm, signs, pd, sd = rpbh_args(n, n + 1)
    y = oracle.rpbh_rotate(x64, block, perm, signs)
    out = H.hadq_rotate_rpbh(to_dev(stored, x_dtype), pd, sd, block, out_dtype=torch.float32)
    torch.cuda.synchronize()
    _log(f"rpbh-rot-{x_dtype}-{rows}x{n}-b{block}", pc.check_rotation_f32(x64, out.cpu().numpy(), block, y=y))
    ob = H.hadq_rotate_rpbh(to_dev(stored, x_dtype), pd, sd, block, out_dtype=torch.bfloat16)
    torch.cuda.synchronize()
    pc.check_rotation_bf16(x64, ob.view(torch.int16).cpu().numpy().view(np.uint16), block, y=y)


@pytest.mark.parametrize("n,block", [(4096, 128), (4096, 4096), (8192, 8192), (4096, 512)])
@pytest.mark.parametrize("fmt,group", [("int4", 128), ("int4", 32), ("int8", 0), ("mxfp4", 32), ("nvfp4", 16)])
def test_rpbh_quant(n, block, fmt, group):
    rows = 11
    stored, x64 = synth(rows, n, "bf16", seed=3 * n + block, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    perm, signs, pd, sd = rpbh_args(n, block)
    c, s = H.hadq_rotate_quant_rpbh(to_dev(stored, "bf16"), pd, sd, block, fmt, group)
    torch.cuda.synchronize()
    y = oracle.rpbh_rotate(x64, block, perm, signs)
    _log(f"rpbh-{fmt}{group}-{rows}x{n}-b{block}", pc.check(fmt, x64, c.cpu().numpy(), s.cpu().numpy(), block, group,
                                                             y=y))


def test_rpbh_identity_is_the_plain_rotation():
    """Identity permutation and all-plus signs: the same codes as hadq_rotate_quant."""
    stored, _ = synth(9, 4096, "bf16", seed=5)
    x = to_dev(stored, "bf16")
    perm = torch.arange(4096, dtype=torch.int32, device="cuda")
    ones = torch.ones(4096, dtype=torch.int8, device="cuda")
    H.hadq_set_impl("butterfly")
    try:
        c0, s0 = H.hadq_rotate_quant(x, 128, "int4", 128)
        c1, s1 = H.hadq_rotate_quant_rpbh(x, perm, ones, 128, "int4", 128)
        torch.cuda.synchronize()
    finally:
        H.hadq_set_impl("auto")
    assert torch.equal(c0, c1) and torch.equal(s0.view(torch.int16), s1.view(torch.int16))


def _codebook_dev(n, bits):
    c, t = H.hadq_codebook(n, bits)
    return torch.from_numpy(t.copy()).cuda()


@pytest.mark.parametrize("rows,n,block", [(9, 4096, 4096), (7, 4096, 128), (5, 8192, 8192), (6, 1024, 64),
                                          (4, 14336, 0), (5, 2048, 16)])
@pytest.mark.parametrize("bits", [2, 4])
@pytest.mark.parametrize("rpbh", [False, True])
def test_codebook_quantizer(rows, n, block, bits, rpbh):
    if rpbh and n == 14336 and block == 0:
        pytest.skip("RPBH's block FWHT is a power-of-2 block")
    stored, x64 = synth(rows, n, "bf16", seed=n + bits + block)
    thr = _codebook_dev(n, bits)
    if rpbh:
        perm, signs, pd, sd = rpbh_args(n, n + bits)
        y = oracle.rpbh_rotate(x64, block, perm, signs)
        codes, norms = H.hadq_rotate_quant_codebook(to_dev(stored, "bf16"), bits, thr, block, perm=pd, signs=sd)
    else:
        y = oracle.rotate(x64, block)
        codes, norms = H.hadq_rotate_quant_codebook(to_dev(stored, "bf16"), bits, thr, block)
    torch.cuda.synchronize()
    _log(f"codebook{bits}-{'rpbh-' if rpbh else ''}{rows}x{n}-b{block}",
         pc.check_codebook(x64, codes.cpu().numpy(), norms.cpu().numpy(), block, bits, y=y))


def test_codebook_fp32_input_and_zero_rows():
    rows, n, bits = 6, 4096, 4
    stored, x64 = synth(rows, n, "f32", seed=21)
    stored[1] = 0
    x64[1] = 0
    thr = _codebook_dev(n, bits)
    codes, norms = H.hadq_rotate_quant_codebook(to_dev(stored, "f32"), bits, thr, 256)
    torch.cuda.synchronize()
    assert norms[1].item() == 0.0
    pc.check_codebook(x64, codes.cpu().numpy(), norms.cpu().numpy(), 256, bits)


def test_codebook_many_rows_grid_loops():
    """More rows than resident CTAs, and the full-size R1 shape (4096 x 4096)."""
    rows, n, bits = 4096, 4096, 4
    stored, x64 = synth(rows, n, "bf16", seed=33)
    thr = _codebook_dev(n, bits)
    perm, signs, pd, sd = rpbh_args(n, 34)
    codes, norms = H.hadq_rotate_quant_codebook(to_dev(stored, "bf16"), bits, thr, 4096, perm=pd, signs=sd)
    torch.cuda.synchronize()
    _log("codebook4-rpbh-4096x4096", pc.check_codebook(x64, codes.cpu().numpy(), norms.cpu().numpy(), 4096, bits,
                                                       y=oracle.rpbh_rotate(x64, 4096, perm, signs)))


# ------------------------------------------ RPBH on the tensor cores (n = 4096)

@pytest.mark.parametrize("impl", ["tensor", "butterfly"])
@pytest.mark.parametrize("fmt,group", [("int4", 128), ("int4", 32), ("mxfp4", 32), ("nvfp4", 16), ("f32", 0),
                                       ("bf16", 0), ("codebook", 4), ("codebook", 2)])
def test_rpbh_4096_tiles_both_impls(impl, fmt, group):
    """Full-row RPBH at n = 4096: the gather-then-MMA kernel (tensor) and the
    staged kernel (butterfly) on 1001 rows (251 tiles of 4 rows, the last one
    ragged, more tiles than CTAs), every output format and the 2- and 4-bit
    codebook quantizer."""
    rows, n = 1001, 4096
    stored, x64 = synth(rows, n, "bf16", seed=rows + len(fmt) + group, dist="t" if fmt in ("mxfp4", "nvfp4") else "normal")
    perm, signs, pd, sd = rpbh_args(n, 77 + group)
    y = oracle.rpbh_rotate(x64, n, perm, signs)
    old = H.hadq_set_impl(impl)
    try:
        if fmt == "codebook":
            codes, norms = H.hadq_rotate_quant_codebook(to_dev(stored, "bf16"), group, _codebook_dev(n, group), n,
                                                        perm=pd, signs=sd)
            torch.cuda.synchronize()
            _log(f"rpbh-{impl}-codebook{group}-{rows}x{n}",
                 pc.check_codebook(x64, codes.cpu().numpy(), norms.cpu().numpy(), n, group, y=y))
        elif fmt in ("f32", "bf16"):
            out = H.hadq_rotate_rpbh(to_dev(stored, "bf16"), pd, sd, n,
                                     out_dtype=torch.float32 if fmt == "f32" else torch.bfloat16)
            torch.cuda.synchronize()
            if fmt == "f32":
                _log(f"rpbh-{impl}-rot-{rows}x{n}", pc.check_rotation_f32(x64, out.cpu().numpy(), n, y=y))
            else:
                pc.check_rotation_bf16(x64, out.view(torch.int16).cpu().numpy().view(np.uint16), n, y=y)
        else:
            c, s = H.hadq_rotate_quant_rpbh(to_dev(stored, "bf16"), pd, sd, n, fmt, group)
            torch.cuda.synchronize()
            _log(f"rpbh-{impl}-{fmt}{group}-{rows}x{n}",
                 pc.check(fmt, x64, c.cpu().numpy(), s.cpu().numpy(), n, group, y=y))
    finally:
        H.hadq_set_impl(old)


def test_rpbh_4096_identity_matches_plain_tensor_kernel():
    """Identity permutation and all-plus signs through the gather kernel: the
    same codes as the plain n = 4096 tensor-core rotation, bit for bit (the
    gather only moves data; the MMA and epilogue are the same arithmetic)."""
    stored, _ = synth(37, 4096, "bf16", seed=6)
    x = to_dev(stored, "bf16")
    perm = torch.arange(4096, dtype=torch.int32, device="cuda")
    ones = torch.ones(4096, dtype=torch.int8, device="cuda")
    c0, s0 = H.hadq_rotate_quant(x, 0, "int4", 128)
    c1, s1 = H.hadq_rotate_quant_rpbh(x, perm, ones, 4096, "int4", 128)
    torch.cuda.synchronize()
    assert torch.equal(c0, c1) and torch.equal(s0.view(torch.int16), s1.view(torch.int16))


def test_rpbh_4096_guard_bytes():
    rows, n = 9, 4096
    stored, x64 = synth(rows, n, "bf16", seed=19)
    perm, signs, pd, sd = rpbh_args(n, 19)
    pad = 1024
    cbuf = torch.full((rows * n // 2 + 2 * pad,), 0xA5, dtype=torch.uint8, device="cuda")
    sbuf = torch.full((rows * n // 64 + 2 * pad,), 0x5A, dtype=torch.uint8, device="cuda")
    codes = cbuf[pad:pad + rows * n // 2].view(rows, n // 2)
    scales = sbuf[pad:pad + rows * n // 64].view(torch.float16).view(rows, n // 128)
    H.hadq_rotate_quant_rpbh(to_dev(stored, "bf16"), pd, sd, n, "int4", 128, codes=codes, scales=scales)
    torch.cuda.synchronize()
    cb, sb = cbuf.cpu().numpy(), sbuf.cpu().numpy()
    assert (cb[:pad] == 0xA5).all() and (cb[-pad:] == 0xA5).all()
    assert (sb[:pad] == 0x5A).all() and (sb[-pad:] == 0x5A).all()
    pc.check_int4(x64, codes.cpu().numpy(), scales.cpu().numpy(), n, 128, y=oracle.rpbh_rotate(x64, n, perm, signs))


def test_config_c2p_full_size():
    """The bench's c2p workload (4096 x 4096 bf16, its seeded permutation and
    signs, int4 g128) in the launch the bench times; every row checked."""
    from hadamard_rotation_bit_b200 import workloads as W
    w = W.WORKLOADS["c2p"]
    stored = W.generate("c2p")
    perm, signs = W.generate_rpbh("c2p")
    x64 = W.bits_to_float64(stored, "bf16")
    c, s = H.hadq_rotate_quant_rpbh(to_dev(stored, "bf16"), torch.from_numpy(perm).cuda(),
                                    torch.from_numpy(signs).cuda(), w.block, w.fmt, w.group)
    torch.cuda.synchronize()
    _log("c2p", pc.check_int4(x64, c.cpu().numpy(), s.cpu().numpy(), w.block, w.group,
                              y=oracle.rpbh_rotate(x64, w.block, perm, signs)))
