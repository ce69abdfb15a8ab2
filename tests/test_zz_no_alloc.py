"""hadq_rotate_quant_host_static: the entry point for callers that cannot
allocate device memory (a host-only application linking libhadq, or a plugin
inside a framework that owns every device allocation).  It stages through the
library's own static device array, so the caller passes host buffers only.

The GPU test calls it through the C ABI three times in a row: two shapes and
formats, then the first shape again with another seed, so outputs left in the
shared array by an earlier call (a kernel that did not run) cannot match.
Every output is compared with the existing host-buffer entry point, which
uses caller-owned device buffers and runs the same kernels (so the two must
be identical), and element by element with the float64 oracle under the
parity rule of the other GPU tests.  This file is collected last.
"""

import ctypes

import numpy as np
import pytest
import torch

from hadamard_rotation_bit_b200 import build as hbuild
from hadamard_rotation_bit_b200 import hadq as H
from hadamard_rotation_bit_b200 import workloads as W
from tests import parity_check as pc

CASES = [(512, 4096, 0, "int4", 128, 1), (1024, 1024, 128, "mxfp4", 32, 2), (512, 4096, 0, "int4", 128, 3)]


def _pinned_input(rows, n, seed):
    v = np.random.default_rng(seed).standard_normal((rows, n)).astype(np.float32)
    v[:, :: max(1, n // 40)] *= 30.0
    bits = W.f32_to_bf16_bits(v)
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).pin_memory(), W.bits_to_float64(bits, "bf16")


@pytest.mark.gpu
def test_static_scratch_entry_point_matches_host_entry_point():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    hbuild.build()
    lib = H.load_library()
    stream = torch.cuda.current_stream()
    for rows, n, block, fmt, group, seed in CASES:
        xh, x64 = _pinned_input(rows, n, seed)
        cs, cd, ss, sd = H.output_shapes(rows, n, fmt, group if fmt == "int4" else 32)
        c_static = torch.full(cs, 0x5A, dtype=cd).pin_memory()
        s_static = torch.zeros(ss, dtype=sd).pin_memory()
        st = lib.hadq_rotate_quant_host_static(
            ctypes.c_void_p(xh.data_ptr()), H.HADQ_BF16, rows, n, block, H.FMTS[fmt], group,
            ctypes.c_void_p(c_static.data_ptr()), ctypes.c_void_p(s_static.data_ptr()),
            ctypes.c_void_p(stream.cuda_stream))
        assert st == H.HADQ_OK, lib.hadq_last_error().decode()
        # the existing entry point, with device buffers owned by the caller
        c_ref = torch.empty(cs, dtype=cd).pin_memory()
        s_ref = torch.empty(ss, dtype=sd).pin_memory()
        xd = torch.empty(xh.shape, dtype=xh.dtype, device="cuda")
        H.hadq_rotate_quant_host(xh, block, fmt, group, c_ref, s_ref, xd,
                                 torch.empty(cs, dtype=cd, device="cuda"), torch.empty(ss, dtype=sd, device="cuda"),
                                 stream=stream)
        torch.cuda.synchronize()
        assert torch.equal(c_static, c_ref), f"codes differ for {rows}x{n} {fmt}"
        assert torch.equal(s_static.view(torch.uint8), s_ref.view(torch.uint8)), f"scales differ for {rows}x{n} {fmt}"
        pc.check(fmt, x64, c_static.numpy(), s_static.numpy(), block, group)


def test_static_scratch_entry_point_rejects_oversize_and_bad_args():
    """Checked on the host before any CUDA call, so this runs without a GPU."""
    hbuild.build()
    lib = H.load_library()
    a, b, c = 0x100000, 0x20000000, 0x40000000       # fake, aligned host addresses (never dereferenced)
    f = lib.hadq_rotate_quant_host_static
    # 4096 x 4096 bf16 (32 MiB) plus its codes does not fit in the 32 MiB array
    assert f(a, H.HADQ_BF16, 4096, 4096, 0, H.FMTS["int4"], 128, b, c, None) == H.HADQ_ERR_UNSUPPORTED
    assert "32 MiB" in lib.hadq_last_error().decode()
    assert f(None, H.HADQ_BF16, 16, 4096, 0, H.FMTS["int4"], 128, b, c, None) == H.HADQ_ERR_INVALID_ARG
    assert f(a + 8, H.HADQ_BF16, 16, 4096, 0, H.FMTS["int4"], 128, b, c, None) == H.HADQ_ERR_MISALIGNED
    assert f(a, H.HADQ_BF16, 16, 4096, 0, H.FMTS["int4"], 48, b, c, None) == H.HADQ_ERR_INVALID_ARG
    assert f(None, H.HADQ_BF16, 0, 4096, 0, H.FMTS["int4"], 128, None, None, None) == H.HADQ_OK
