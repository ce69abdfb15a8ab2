"""libhadq host-side behaviour that needs no GPU.

The library must load, export every function include/hadq.h declares, and
reject bad arguments on the host -- before any CUDA call -- with the right
status.  Only argument combinations that fail validation (or are empty) are
called here, so nothing reaches the device.
"""

import ctypes
import os
import re

import numpy as np

import pytest

from hadamard_rotation_bit_b200 import build as hbuild
from hadamard_rotation_bit_b200 import hadq as H

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

A = 0x10000          # a fake, 16-byte aligned device address (never dereferenced)
B = 0x20000000
C = 0x40000000


@pytest.fixture(scope="module")
def lib():
    hbuild.build()
    return H.load_library()


def header_functions():
    src = open(os.path.join(ROOT, "include", "hadq.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(hadq_[a-z0-9_]+)\s*\(", src)))


def test_exports_every_declared_symbol(lib):
    names = header_functions()
    assert len(names) >= 9
    for name in names:
        assert hasattr(lib, name), name
    assert sorted(names) == sorted(H.EXPORTS)


def test_status_strings_and_version(lib):
    for st in range(5):
        assert lib.hadq_status_string(st)
    assert lib.hadq_version() == 200


def _q(lib, x=A, xd=1, rows=4, n=1024, block=0, fmt=0, group=128, codes=B, scales=C):
    return lib.hadq_rotate_quant(x, xd, rows, n, block, fmt, group, codes, scales, None)


def _r(lib, x=A, xd=1, rows=4, n=1024, block=0, out=B, od=0):
    return lib.hadq_rotate(x, xd, rows, n, block, out, od, None)


def test_empty_calls_are_noops(lib):
    assert _q(lib, rows=0, x=None, codes=None, scales=None) == H.HADQ_OK
    assert _r(lib, rows=0, x=None, out=None) == H.HADQ_OK
    assert lib.hadq_rotate_inverse(None, 0, 0, 64, 0, None, 0, None) == H.HADQ_OK


@pytest.mark.parametrize("kw,status", [
    (dict(rows=-1), H.HADQ_ERR_INVALID_ARG),
    (dict(n=0), H.HADQ_ERR_INVALID_ARG),
    (dict(n=1000), H.HADQ_ERR_INVALID_ARG),              # full rotation of a non-power-of-2
    (dict(block=96), H.HADQ_ERR_INVALID_ARG),            # block not a power of 2
    (dict(n=896, block=256), H.HADQ_ERR_INVALID_ARG),    # block does not divide n
    (dict(n=16384), H.HADQ_ERR_UNSUPPORTED),             # full rotation above 8192
    (dict(block=-2), H.HADQ_ERR_INVALID_ARG),
    (dict(xd=7), H.HADQ_ERR_INVALID_ARG),
    (dict(group=48), H.HADQ_ERR_INVALID_ARG),
    (dict(group=256), H.HADQ_ERR_INVALID_ARG),
    (dict(fmt=9), H.HADQ_ERR_INVALID_ARG),
    (dict(fmt=1, group=64), H.HADQ_ERR_INVALID_ARG),     # int8 is per token
    (dict(fmt=1, group=0, n=65536, block=128), H.HADQ_ERR_UNSUPPORTED),
    (dict(fmt=2, group=16), H.HADQ_ERR_INVALID_ARG),
    (dict(x=None), H.HADQ_ERR_INVALID_ARG),
    (dict(codes=None), H.HADQ_ERR_INVALID_ARG),
    (dict(x=A + 8), H.HADQ_ERR_MISALIGNED),
    (dict(scales=C + 2), H.HADQ_ERR_MISALIGNED),
    (dict(codes=A + 16), H.HADQ_ERR_INVALID_ARG),        # codes overlap x
    (dict(scales=B + 64), H.HADQ_ERR_INVALID_ARG),       # scales overlap codes
    (dict(rows=2 ** 62), H.HADQ_ERR_INVALID_ARG),        # rows * n overflows
])
def test_rotate_quant_validation(lib, kw, status):
    assert _q(lib, **kw) == status
    assert lib.hadq_last_error().decode()


@pytest.mark.parametrize("kw,status", [
    (dict(od=5), H.HADQ_ERR_INVALID_ARG),
    (dict(out=None), H.HADQ_ERR_INVALID_ARG),
    (dict(out=A + 64), H.HADQ_ERR_INVALID_ARG),          # partial overlap
    (dict(out=A, od=0, xd=1), H.HADQ_ERR_INVALID_ARG),   # in place with different dtypes
    (dict(out=B + 4), H.HADQ_ERR_MISALIGNED),
    (dict(n=12, block=4), H.HADQ_ERR_UNSUPPORTED),       # n not a multiple of 8
])
def test_rotate_validation(lib, kw, status):
    assert _r(lib, **kw) == status


def test_host_entry_point_validation(lib):
    f = lib.hadq_rotate_quant_host
    # valid device side, bad host side
    assert f(None, 1, 4, 1024, 0, 0, 128, A, B, A, B, C, None) == H.HADQ_ERR_INVALID_ARG
    assert f(A + 4, 1, 4, 1024, 0, 0, 128, B, C, A, B, C, None) == H.HADQ_ERR_MISALIGNED
    # bad device side
    assert f(A, 1, 4, 1024, 0, 0, 128, B, C, A + 8, B, C, None) == H.HADQ_ERR_MISALIGNED
    assert f(A, 1, 0, 1024, 0, 0, 128, B, C, None, None, None, None) == H.HADQ_OK


def test_output_size_helpers(lib):
    assert lib.hadq_codes_bytes(4096, 4096, 0) == 4096 * 2048
    assert lib.hadq_scales_bytes(4096, 4096, 0, 128) == 4096 * 32 * 2
    assert lib.hadq_codes_bytes(8192, 14336, 1) == 8192 * 14336
    assert lib.hadq_scales_bytes(8192, 14336, 1, 0) == 8192 * 4
    assert lib.hadq_codes_bytes(65536, 8192, 2) == 65536 * 4096
    assert lib.hadq_scales_bytes(65536, 8192, 2, 32) == 65536 * 256
    assert lib.hadq_scales_bytes(4, 100, 0, 128) == 0
    assert lib.hadq_codes_bytes(4, 64, 7) == 0


def test_binding_raises_without_cuda_tensor(lib):
    import torch
    with pytest.raises(H.HadqError):
        H.hadq_rotate_quant(torch.zeros(4, 96, dtype=torch.float64), 0, "int4", 32)


# ------------------------------------------------- random Hadamard entry points

S = 0x60000000       # a fake device address for the signs (never dereferenced)


def _qs(lib, x=A, rows=4, n=1024, block=0, signs=S, side=0, fmt=0, group=128, codes=B, scales=C):
    return lib.hadq_rotate_quant_signed(x, 1, rows, n, block, signs, side, fmt, group, codes, scales, None)


def _rs(lib, x=A, rows=4, n=1024, block=0, signs=S, side=0, out=B, od=0):
    return lib.hadq_rotate_signed(x, 1, rows, n, block, signs, side, out, od, None)


def test_signed_empty_calls_are_noops(lib):
    assert _qs(lib, rows=0, x=None, signs=None, codes=None, scales=None) == H.HADQ_OK
    assert _rs(lib, rows=0, x=None, signs=None, out=None) == H.HADQ_OK
    assert _rs(lib, rows=0, x=None, signs=None, out=None, side=H.HADQ_SIGNS_BEFORE) == H.HADQ_OK


@pytest.mark.parametrize("call", [_qs, _rs])
def test_signed_validation(lib, call):
    assert call(lib, side=2) == H.HADQ_ERR_INVALID_ARG
    assert "side" in lib.hadq_last_error().decode()
    assert call(lib, side=-1) == H.HADQ_ERR_INVALID_ARG
    assert call(lib, rows=0, side=5) == H.HADQ_ERR_INVALID_ARG      # a bad side is rejected even when empty
    assert call(lib, signs=None) == H.HADQ_ERR_INVALID_ARG
    assert call(lib, signs=None, side=H.HADQ_SIGNS_BEFORE) == H.HADQ_ERR_INVALID_ARG
    assert call(lib, n=1000) == H.HADQ_ERR_INVALID_ARG               # shape checks still apply
    assert call(lib, x=A + 8) == H.HADQ_ERR_MISALIGNED


def test_signed_rejects_signs_overlapping_an_output(lib):
    # codes at B cover rows * n / 2 bytes; signs inside that range
    assert _qs(lib, signs=B + 16) == H.HADQ_ERR_INVALID_ARG
    assert "signs" in lib.hadq_last_error().decode()
    assert _qs(lib, signs=C + 16) == H.HADQ_ERR_INVALID_ARG           # inside the scales
    assert _rs(lib, signs=B + 96) == H.HADQ_ERR_INVALID_ARG           # inside out (fp32, 16 KB)
    assert _qs(lib, signs=S + 8) == H.HADQ_ERR_MISALIGNED             # signs must be 16-byte aligned
    assert _rs(lib, signs=S + 1, side=H.HADQ_SIGNS_BEFORE) == H.HADQ_ERR_MISALIGNED
    # block 128: the signs span only 128 bytes, so B - 128 just touches nothing
    assert _rs(lib, block=128, signs=B - 128, x=None) == H.HADQ_ERR_INVALID_ARG   # null x still caught first



def test_nvfp4_validation(lib):
    f = lib.hadq_rotate_quant_nvfp4
    assert f(None, 1, 0, 1024, 0, 1.0, None, None, None) == H.HADQ_OK
    for bad in (0.0, -1.0, float("inf"), float("nan")):
        assert f(A, 1, 4, 1024, 0, bad, B, C, None) == H.HADQ_ERR_INVALID_ARG
        assert "tensor_scale" in lib.hadq_last_error().decode()
    assert f(A, 1, 4, 1000, 0, 1.0, B, C, None) == H.HADQ_ERR_INVALID_ARG           # full non-power-of-2
    assert f(A, 1, 4, 1032, 8, 1.0, B, C, None) == H.HADQ_ERR_INVALID_ARG           # 16 does not divide n
    assert _q(lib, fmt=3, group=32) == H.HADQ_ERR_INVALID_ARG                        # NVFP4 blocks are 16
    assert lib.hadq_scales_bytes(4, 1024, 3, 16) == 4 * 64
    assert lib.hadq_scales_bytes(4, 1024, 3, 0) == 4 * 64
    assert lib.hadq_scales_bytes(4, 1024, 3, 32) == 0
    assert lib.hadq_codes_bytes(4, 1024, 3) == 2048


# ------------------------------------------------- binding-level buffer checks

def test_binding_rejects_host_tensors_for_device_arguments(lib):
    """The C ABI takes device pointers; the binding refuses host tensors
    before any call (a host address would reach the kernel otherwise)."""
    import torch
    x = torch.zeros(4, 128, dtype=torch.bfloat16)
    for call in (lambda: H.hadq_rotate(x, 0), lambda: H.hadq_rotate_quant(x, 0, "int4", 128),
                 lambda: H.hadq_rotate_quant_nvfp4(x, 1.0, 0),
                 lambda: H.hadq_rotate_signed(x, torch.ones(128, dtype=torch.int8), "after", 0),
                 lambda: H.hadq_rotate_quant_signed(x, torch.ones(128, dtype=torch.int8), "before", 0, "mxfp4", 32)):
        with pytest.raises(H.HadqError) as e:
            call()
        assert e.value.status == H.HADQ_ERR_INVALID_ARG and "CUDA tensor" in str(e.value)


def test_binding_checks_host_output_sizes(lib):
    """Caller-supplied outputs must hold what the call writes; the sizes the
    binding allocates itself (output_shapes) are exactly the library's."""
    import torch
    for rows, n, fmt, group in [(5, 4096, "int4", 128), (5, 4096, "int4", 32), (3, 14336, "int8", 0),
                                (7, 8192, "mxfp4", 32), (9, 48, "nvfp4", 16), (5, 4096, "mxfp4_blocked", 32),
                                (300, 8192, "nvfp4_blocked", 16)]:
        cs, cd, ss, sd = H.output_shapes(rows, n, fmt, group if fmt == "int4" else 32)
        codes, scales = torch.empty(cs, dtype=cd), torch.empty(ss, dtype=sd)
        assert codes.numel() * codes.element_size() == lib.hadq_codes_bytes(rows, n, H.FMTS[fmt])
        assert scales.numel() * scales.element_size() == lib.hadq_scales_bytes(rows, n, H.FMTS[fmt], group)
        H._quant_outputs(lib, rows, n, fmt, group, codes, scales, None)          # host side: accepted
        with pytest.raises(H.HadqError) as e:
            H._quant_outputs(lib, rows, n, fmt, group, codes[:-1], scales, None)
        assert "holds" in str(e.value)
    with pytest.raises(H.HadqError):
        H._holds("out", torch.empty(8, 4)[:, :2], 16)                             # not contiguous
    assert H._block_len(4096, 0) == 4096 and H._block_len(4096, -1) == 4096 and H._block_len(4096, 128) == 128


def test_impl_choice_is_explicit_and_checked(lib):
    """hadq_set_impl selects the implementation for the shapes both cover; it
    touches no device and rejects values outside the enum."""
    assert H.hadq_get_impl() == "auto"
    assert H.hadq_set_impl("butterfly") == "auto"
    assert H.hadq_get_impl() == "butterfly"
    assert H.hadq_set_impl("auto") == "butterfly"
    assert lib.hadq_set_impl(7) == H.HADQ_ERR_INVALID_ARG
    assert "HADQ_IMPL" in lib.hadq_last_error().decode()
    assert H.hadq_get_impl() == "auto"


def test_k_size_shape_rules(lib):
    """Non-power-of-2 sizes b = K * 2^m: covered K run, others are refused on
    the host before any CUDA call (fake aligned addresses, never touched)."""
    a, c, sc = 0x100000, 0x20000000, 0x40000000
    f = lib.hadq_rotate_quant
    bf, i4, i8 = H.HADQ_BF16, H.FMTS["int4"], H.FMTS["int8"]
    assert f(a, bf, 0, 28 * 512, 0, i4, 128, c, sc, None) == H.HADQ_OK            # empty call, covered size
    assert f(a, bf, 0, 44 * 64, 0, i4, 128, c, sc, None) == H.HADQ_ERR_INVALID_ARG   # K = 44 not covered
    assert "K * 2^m" in lib.hadq_last_error().decode()
    assert f(a, bf, 0, 28 * 32, 0, i4, 32, c, sc, None) == H.HADQ_ERR_UNSUPPORTED    # 2^m < 64
    assert f(a, bf, 0, 28 * 2048, 0, i4, 128, c, sc, None) == H.HADQ_ERR_UNSUPPORTED  # above 32768
    assert f(a, bf, 0, 3 * 28 * 64, 28 * 64, i8, 0, c, sc, None) == H.HADQ_ERR_UNSUPPORTED  # int8 needs full rows
    assert f(a, bf, 0, 3 * 28 * 64, 28 * 64, i4, 64, c, sc, None) == H.HADQ_OK       # block-diagonal K-size
    assert f(a, bf, 0, 28 * 64 + 8, 28 * 64, i4, 32, c, sc, None) == H.HADQ_ERR_INVALID_ARG  # block must divide n


@pytest.mark.parametrize("d,bits", [(3, 2), (16, 1), (64, 3), (4096, 4), (4096, 2), (14336, 4), (256, 6)])
def test_library_codebook_agrees_with_the_oracle(lib, d, bits):
    """The library's own Lloyd-Max codebook (C++, host) against the oracle's
    independent one.  Both stop Lloyd's iteration when no centroid moves by
    more than 1e-13 of the largest; the iteration converges linearly, slowly
    at 256 levels, so the two agree to 1e-9 of the largest centroid up to 4
    bits (1e-8 of a centroid spacing) and to 1e-6 beyond."""
    import oracle
    c, t = H.hadq_codebook(d, bits)
    oc, ot = oracle.sphere_lloyd_max(d, bits)
    tol = (1e-9 if bits <= 4 else 1e-6) * np.abs(oc).max()
    np.testing.assert_allclose(c, oc, rtol=0, atol=tol)
    np.testing.assert_allclose(t, ot, rtol=0, atol=tol)


def test_library_codebook_rejects_bad_arguments(lib):
    c = np.zeros(256)
    t = np.zeros(255)
    assert lib.hadq_codebook(1, 4, c.ctypes.data, t.ctypes.data) == H.HADQ_ERR_INVALID_ARG
    assert lib.hadq_codebook(64, 0, c.ctypes.data, t.ctypes.data) == H.HADQ_ERR_INVALID_ARG
    assert lib.hadq_codebook(64, 9, c.ctypes.data, t.ctypes.data) == H.HADQ_ERR_INVALID_ARG
    assert lib.hadq_codebook(64, 4, None, t.ctypes.data) == H.HADQ_ERR_INVALID_ARG


def test_blocked_fp4_formats_sizes_and_checks(lib):
    """The tiled-scale FP4 formats: scales padded to whole 128-row tiles, the
    group rules of their base formats, whole 4-column tiles, and the
    tensor-core shapes only (everything else HADQ_ERR_UNSUPPORTED, before any
    CUDA call)."""
    mxb, nvb = H.FMTS["mxfp4_blocked"], H.FMTS["nvfp4_blocked"]
    assert lib.hadq_scales_bytes(5, 4096, mxb, 32) == 128 * 128
    assert lib.hadq_scales_bytes(128, 4096, mxb, 0) == 128 * 128
    assert lib.hadq_scales_bytes(129, 8192, nvb, 16) == 256 * 512
    assert lib.hadq_scales_bytes(5, 4096 + 32, mxb, 32) == 0                        # 129 scale columns
    assert lib.hadq_codes_bytes(5, 4096, mxb) == 5 * 2048
    assert _q(lib, fmt=mxb, group=16) == H.HADQ_ERR_INVALID_ARG
    assert _q(lib, fmt=nvb, group=32) == H.HADQ_ERR_INVALID_ARG
    assert _q(lib, n=1056, fmt=mxb, group=32) == H.HADQ_ERR_INVALID_ARG              # 33 scale columns
    assert _q(lib, fmt=6, group=32) == H.HADQ_ERR_INVALID_ARG                         # no such format
    assert _q(lib, n=1024, block=64, fmt=mxb, group=32) == H.HADQ_ERR_UNSUPPORTED     # not a tensor-core size
    assert _q(lib, xd=0, n=4096, fmt=mxb, group=32) == H.HADQ_ERR_UNSUPPORTED         # fp32 input
    assert _q(lib, xd=0, n=4096, block=128, fmt=nvb, group=16) == H.HADQ_ERR_UNSUPPORTED   # fp32 blocks
    assert lib.hadq_set_impl(1) == H.HADQ_OK                                          # butterfly kernels
    try:
        assert _q(lib, n=4096, fmt=mxb, group=32) == H.HADQ_ERR_UNSUPPORTED
    finally:
        assert lib.hadq_set_impl(0) == H.HADQ_OK


def test_tile_layout_map_matches_the_tiled_rearrangement():
    """The GPU tests' index map of the tiled GEMM scale layout (offset
    arithmetic) agrees with the layout written as a rearrangement: pad to
    128-row x 4-column tiles, order the tiles row-block major, and inside a
    tile put the four 32-row slabs side by side (r % 32 outermost, then the
    slab, then the column)."""
    from tests.test_gpu_blocked_gemm import tile_offsets
    for rows, cols in [(128, 4), (300, 128), (5, 256), (257, 8)]:
        pr, pc_ = (rows + 127) // 128 * 128, (cols + 3) // 4 * 4
        m = np.zeros((pr, pc_), dtype=np.int64)
        m[:rows, :cols] = np.arange(rows * cols).reshape(rows, cols) + 1
        t = m.reshape(pr // 128, 128, pc_ // 4, 4).transpose(0, 2, 1, 3)          # tiles, row-block major
        t = t.reshape(-1, 4, 32, 4).transpose(0, 2, 1, 3)                          # (slab, r % 32) -> (r % 32, slab)
        ref = t.reshape(-1)
        off = tile_offsets(pr, cols)
        got = np.zeros(ref.size, dtype=np.int64)
        got[off[:rows].reshape(-1)] = m[:rows, :cols].reshape(-1)
        np.testing.assert_array_equal(got, ref)
