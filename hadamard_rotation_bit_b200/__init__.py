"""libhadq: B200-native online Hadamard rotation fused with RTN / MXFP4 quantization.

The compute path is the C-ABI library ``libhadq.so`` (hand-written CUDA for
sm_100a, declared in ``include/hadq.h``); ``hadamard_rotation_bit_b200.hadq``
is a thin ctypes binding with the same entry-point names.  The binding loads
the library lazily, so ``workloads`` (input recipes) can be imported on a
machine without a GPU.
"""

__version__ = "0.1.0"
