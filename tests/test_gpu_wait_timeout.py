"""The bounded waits of the tensor-core kernels give up instead of hanging.

tests/c/wait_timeout.cu runs the kernels' own mbarrier wait on a barrier that
nothing arrives on (a flag that nothing sets): the wait must return after
its limit of about one second, the kernel must record the fault, free its
tensor memory and exit, and the CUDA context must stay usable -- a normal
libhadq call right after it still matches the oracle.  No fault, trap or
hang is involved.
"""

import ctypes
import os
import subprocess

import numpy as np
import pytest
import torch

from hadamard_rotation_bit_b200 import build as hbuild
from hadamard_rotation_bit_b200 import hadq as H
from tests import parity_check as pc
from tests.test_gpu_parity import synth, to_dev

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

pytestmark = pytest.mark.gpu


def test_wait_gives_up_and_context_survives(tmp_path):
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    hbuild.build()
    so = str(tmp_path / "libwait_timeout.so")
    cmd = [hbuild._nvcc()] + hbuild.ARCH_FLAGS + ["-O2", "-std=c++17", "-Xcompiler", "-fPIC", "--shared",
                                                  "-cudart", "shared", "-I", hbuild.CSRC,
                                                  os.path.join(ROOT, "tests", "c", "wait_timeout.cu"), "-o", so]
    res = subprocess.run(cmd, capture_output=True, text=True)
    assert res.returncode == 0, res.stderr
    lib = ctypes.CDLL(so)
    result, waited, fault = ctypes.c_uint(0), ctypes.c_ulonglong(0), ctypes.c_uint(0)
    rc = lib.run_wait_timeout(ctypes.byref(result), ctypes.byref(waited), ctypes.byref(fault))
    assert rc == 0, f"launch or synchronize failed ({rc})"
    assert result.value == 2, "the wait on a barrier nobody arrives on did not give up"
    assert 0.9e9 <= waited.value <= 5e9, f"waited {waited.value} ns"
    assert fault.value != 0
    # the context is intact: the library still works and is still right
    stored, x64 = synth(16, 4096, "bf16", seed=3)
    codes, scales = H.hadq_rotate_quant(to_dev(stored, "bf16"), 0, "int4", 128)
    torch.cuda.synchronize()
    pc.check_int4(x64, codes.cpu().numpy(), scales.cpu().numpy(), 0, 128)
    assert H.hadq_device_faults(clear=True) == 0     # libhadq's own fault word was not touched
