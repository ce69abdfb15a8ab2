"""ctypes binding for libhadq (include/hadq.h).  Argument marshalling only.

The entry points keep the C names.  Tensors are passed as raw device
pointers; every step of the rotation and quantization runs in libhadq's CUDA
kernels.  There is no fallback: if ``libhadq.so`` is missing or the CUDA call
fails, a ``HadqError`` is raised.

    codes, scales = hadq_rotate_quant(x, block=0, fmt="int4", group=128)

``x`` is any contiguous fp32 / bf16 CUDA tensor; its last dimension is n
(the rotated dimension), all leading dimensions are rows.
"""

from __future__ import annotations

import ctypes
import os
import threading

import torch

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libhadq.so")

HADQ_OK, HADQ_ERR_INVALID_ARG, HADQ_ERR_UNSUPPORTED, HADQ_ERR_MISALIGNED, HADQ_ERR_CUDA = range(5)
HADQ_F32, HADQ_BF16 = 0, 1
FMTS = {"int4": 0, "int8": 1, "mxfp4": 2, "nvfp4": 3, "mxfp4_blocked": 4, "nvfp4_blocked": 5}
HADQ_SIGNS_AFTER, HADQ_SIGNS_BEFORE = 0, 1
SIDES = {"after": HADQ_SIGNS_AFTER, "before": HADQ_SIGNS_BEFORE}
EXPORTS = (
    "hadq_rotate", "hadq_rotate_inverse", "hadq_rotate_quant", "hadq_rotate_quant_host",
    "hadq_codes_bytes", "hadq_scales_bytes", "hadq_status_string", "hadq_last_error", "hadq_version",
    "hadq_device_faults", "hadq_rotate_quant_host_static", "hadq_rotate_signed", "hadq_rotate_quant_signed",
    "hadq_rotate_quant_nvfp4", "hadq_set_impl", "hadq_get_impl", "hadq_codebook",
    "hadq_rotate_rpbh", "hadq_rotate_quant_rpbh", "hadq_rotate_quant_codebook",
)
IMPLS = {"auto": 0, "butterfly": 1, "tensor": 2}

_lock = threading.Lock()
_lib = None


class HadqError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"libhadq status {status}: {message}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libhadq.so once and declare the C signatures."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(path):
            raise HadqError(-1, f"{path} is not built; run `python -m hadamard_rotation_bit_b200.build`")
        lib = ctypes.CDLL(path)
        vp, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int
        lib.hadq_rotate.argtypes = [vp, i32, i64, i64, i64, vp, i32, vp]
        lib.hadq_rotate_inverse.argtypes = [vp, i32, i64, i64, i64, vp, i32, vp]
        lib.hadq_rotate_quant.argtypes = [vp, i32, i64, i64, i64, i32, i64, vp, vp, vp]
        lib.hadq_rotate_quant_host.argtypes = [vp, i32, i64, i64, i64, i32, i64, vp, vp, vp, vp, vp, vp]
        for f in ("hadq_rotate", "hadq_rotate_inverse", "hadq_rotate_quant", "hadq_rotate_quant_host"):
            getattr(lib, f).restype = i32
        lib.hadq_codes_bytes.argtypes = [i64, i64, i32]
        lib.hadq_codes_bytes.restype = i64
        lib.hadq_scales_bytes.argtypes = [i64, i64, i32, i64]
        lib.hadq_scales_bytes.restype = i64
        lib.hadq_status_string.argtypes = [i32]
        lib.hadq_status_string.restype = ctypes.c_char_p
        lib.hadq_last_error.argtypes = []
        lib.hadq_last_error.restype = ctypes.c_char_p
        lib.hadq_version.argtypes = []
        lib.hadq_version.restype = i32
        lib.hadq_device_faults.argtypes = [i32]
        lib.hadq_device_faults.restype = i32
        lib.hadq_rotate_quant_host_static.argtypes = [vp, i32, i64, i64, i64, i32, i64, vp, vp, vp]
        lib.hadq_rotate_quant_host_static.restype = i32
        lib.hadq_rotate_signed.argtypes = [vp, i32, i64, i64, i64, vp, i32, vp, i32, vp]
        lib.hadq_rotate_signed.restype = i32
        lib.hadq_rotate_quant_signed.argtypes = [vp, i32, i64, i64, i64, vp, i32, i32, i64, vp, vp, vp]
        lib.hadq_rotate_quant_signed.restype = i32
        lib.hadq_rotate_quant_nvfp4.argtypes = [vp, i32, i64, i64, i64, ctypes.c_float, vp, vp, vp]
        lib.hadq_rotate_quant_nvfp4.restype = i32
        lib.hadq_set_impl.argtypes = [i32]
        lib.hadq_set_impl.restype = i32
        lib.hadq_get_impl.argtypes = []
        lib.hadq_get_impl.restype = i32
        lib.hadq_codebook.argtypes = [i64, i32, vp, vp]
        lib.hadq_codebook.restype = i32
        lib.hadq_rotate_rpbh.argtypes = [vp, i32, i64, i64, i64, vp, vp, vp, i32, vp]
        lib.hadq_rotate_rpbh.restype = i32
        lib.hadq_rotate_quant_rpbh.argtypes = [vp, i32, i64, i64, i64, vp, vp, i32, i64, vp, vp, vp]
        lib.hadq_rotate_quant_rpbh.restype = i32
        lib.hadq_rotate_quant_codebook.argtypes = [vp, i32, i64, i64, i64, vp, vp, i32, vp, vp, vp, vp]
        lib.hadq_rotate_quant_codebook.restype = i32
        _lib = lib
        return lib


def _check(status: int) -> None:
    if status != HADQ_OK:
        lib = load_library()
        msg = lib.hadq_last_error().decode() or lib.hadq_status_string(status).decode()
        raise HadqError(status, msg)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.float32:
        return HADQ_F32
    if t == torch.bfloat16:
        return HADQ_BF16
    raise HadqError(HADQ_ERR_INVALID_ARG, f"unsupported dtype {t} (float32 or bfloat16)")


def _stream_handle(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream) if hasattr(stream, "cuda_stream") else int(stream)


def _on_device(name: str, t: torch.Tensor, dev: torch.device) -> None:
    """The C ABI takes device pointers: a host tensor here would be read or
    written by the kernel through a host address."""
    if not t.is_cuda:
        raise HadqError(HADQ_ERR_INVALID_ARG, f"{name} must be a CUDA tensor (got {t.device})")
    if t.device != dev:
        raise HadqError(HADQ_ERR_INVALID_ARG, f"{name} is on {t.device}, x on {dev}")


def _on_host(name: str, t: torch.Tensor) -> None:
    if t.is_cuda:
        raise HadqError(HADQ_ERR_INVALID_ARG, f"{name} must be a host tensor (got {t.device})")


def _holds(name: str, t: torch.Tensor, nbytes: int) -> None:
    """A caller-supplied buffer must be contiguous and at least nbytes long:
    the C ABI receives only its address."""
    if not t.is_contiguous():
        raise HadqError(HADQ_ERR_INVALID_ARG, f"{name} must be contiguous")
    if t.numel() * t.element_size() < nbytes:
        raise HadqError(HADQ_ERR_INVALID_ARG,
                        f"{name} holds {t.numel() * t.element_size()} bytes, the call writes {nbytes}")


def _quant_outputs(lib, rows: int, n: int, fmt: str, group: int, codes, scales, dev) -> None:
    if fmt not in FMTS:
        raise HadqError(HADQ_ERR_INVALID_ARG, f"unknown fmt {fmt!r}")
    for name, t, nbytes in (("codes", codes, int(lib.hadq_codes_bytes(rows, n, FMTS[fmt]))),
                            ("scales", scales, int(lib.hadq_scales_bytes(rows, n, FMTS[fmt], group)))):
        if dev is None:
            _on_host(name, t)
        else:
            _on_device(name, t, dev)
        _holds(name, t, nbytes)


def _rows_n(x: torch.Tensor):
    if not x.is_contiguous():
        raise HadqError(HADQ_ERR_INVALID_ARG, "tensors must be contiguous")
    n = x.shape[-1] if x.dim() else 1
    return (x.numel() // n if n else 0), n


def hadq_device_faults(clear: bool = True) -> int:
    """Fault bits of kernels whose bounded waits ran out (0 = none)."""
    return int(load_library().hadq_device_faults(1 if clear else 0))


def hadq_set_impl(impl: str) -> str:
    """Choose the implementation for the shapes both cover ("auto", "tensor"
    or "butterfly", see include/hadq.h); returns the previous choice."""
    lib = load_library()
    if impl not in IMPLS:
        raise HadqError(HADQ_ERR_INVALID_ARG, f"unknown impl {impl!r}")
    prev = hadq_get_impl()
    _check(lib.hadq_set_impl(IMPLS[impl]))
    return prev


def hadq_get_impl() -> str:
    code = int(load_library().hadq_get_impl())
    return {v: k for k, v in IMPLS.items()}[code]


def hadq_codebook(d: int, bits: int):
    """The library's unit-sphere Lloyd-Max codebook for rows of length d:
    (centroids, thresholds) as float64 numpy arrays (see include/hadq.h)."""
    import numpy as np
    lib = load_library()
    c = np.empty(1 << bits, dtype=np.float64)
    t = np.empty(max(1, (1 << bits) - 1), dtype=np.float64)
    _check(lib.hadq_codebook(int(d), int(bits), c.ctypes.data, t.ctypes.data))
    return c, t[: (1 << bits) - 1]


def codes_nbytes(rows: int, n: int, fmt: str) -> int:
    return int(load_library().hadq_codes_bytes(rows, n, FMTS[fmt]))


def scales_nbytes(rows: int, n: int, fmt: str, group: int) -> int:
    return int(load_library().hadq_scales_bytes(rows, n, FMTS[fmt], group))


def output_shapes(rows: int, n: int, fmt: str, group: int):
    """(codes shape, codes dtype, scales shape, scales dtype) of hadq_rotate_quant."""
    if fmt == "int4":
        return (rows, n // 2), torch.uint8, (rows, n // group), torch.float16
    if fmt == "int8":
        return (rows, n), torch.int8, (rows,), torch.float32
    if fmt == "mxfp4":
        return (rows, n // 2), torch.uint8, (rows, n // 32), torch.uint8
    if fmt == "nvfp4":
        return (rows, n // 2), torch.uint8, (rows, n // 16), torch.uint8
    if fmt in ("mxfp4_blocked", "nvfp4_blocked"):
        # the tiled GEMM scale layout: rows padded to 128, stored as 128 x 4 tiles
        blk = 32 if fmt == "mxfp4_blocked" else 16
        return (rows, n // 2), torch.uint8, ((rows + 127) // 128 * 128, n // blk), torch.uint8
    raise HadqError(HADQ_ERR_INVALID_ARG, f"unknown fmt {fmt!r}")


def hadq_rotate(x: torch.Tensor, block: int = 0, out: torch.Tensor | None = None,
                out_dtype: torch.dtype | None = None, stream=None) -> torch.Tensor:
    """out = x . diag(H_b) / sqrt(b) along the last dimension (see include/hadq.h)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _on_device("out", out, x.device)
    _holds("out", out, rows * n * out.element_size())
    _check(lib.hadq_rotate(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, out.data_ptr(),
                           _dtype_code(out.dtype), _stream_handle(stream)))
    return out


def hadq_rotate_inverse(x: torch.Tensor, block: int = 0, out: torch.Tensor | None = None,
                        out_dtype: torch.dtype | None = None, stream=None) -> torch.Tensor:
    """Inverse rotation (the same symmetric, involutory operation)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _on_device("out", out, x.device)
    _holds("out", out, rows * n * out.element_size())
    _check(lib.hadq_rotate_inverse(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, out.data_ptr(),
                                   _dtype_code(out.dtype), _stream_handle(stream)))
    return out


def hadq_rotate_quant(x: torch.Tensor, block: int = 0, fmt: str = "int4", group: int = 128,
                      codes: torch.Tensor | None = None, scales: torch.Tensor | None = None, stream=None):
    """Rotate and quantize in one pass; returns (codes, scales) (see include/hadq.h)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    cs, cd, ss, sd = output_shapes(rows, n, fmt, group if fmt == "int4" else 32)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=x.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=x.device)
    _quant_outputs(lib, rows, n, fmt, group, codes, scales, x.device)
    _check(lib.hadq_rotate_quant(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, FMTS[fmt], group,
                                 codes.data_ptr(), scales.data_ptr(), _stream_handle(stream)))
    return codes, scales


def hadq_rotate_quant_host(x_host: torch.Tensor, block: int, fmt: str, group: int,
                           codes_host: torch.Tensor, scales_host: torch.Tensor,
                           x_dev: torch.Tensor, codes_dev: torch.Tensor, scales_dev: torch.Tensor,
                           stream=None) -> None:
    """Host-buffer form: copy in, rotate+quantize, copy out, all enqueued on `stream`."""
    lib = load_library()
    rows, n = _rows_n(x_host)
    _on_host("x_host", x_host)
    _quant_outputs(lib, rows, n, fmt, group, codes_host, scales_host, None)
    _on_device("x_dev", x_dev, x_dev.device)
    _holds("x_dev", x_dev, rows * n * x_host.element_size())
    _quant_outputs(lib, rows, n, fmt, group, codes_dev, scales_dev, x_dev.device)
    _check(lib.hadq_rotate_quant_host(x_host.data_ptr(), _dtype_code(x_host.dtype), rows, n, block, FMTS[fmt], group,
                                      codes_host.data_ptr(), scales_host.data_ptr(), x_dev.data_ptr(),
                                      codes_dev.data_ptr(), scales_dev.data_ptr(), _stream_handle(stream)))


def hadq_rotate_quant_host_static(x_host: torch.Tensor, block: int, fmt: str, group: int,
                                  codes_host: torch.Tensor, scales_host: torch.Tensor, stream=None) -> None:
    """Host buffers only: the library stages through its own static device
    array (32 MiB per GPU), so this call allocates no device memory."""
    lib = load_library()
    rows, n = _rows_n(x_host)
    _on_host("x_host", x_host)
    _quant_outputs(lib, rows, n, fmt, group, codes_host, scales_host, None)
    _check(lib.hadq_rotate_quant_host_static(x_host.data_ptr(), _dtype_code(x_host.dtype), rows, n, block, FMTS[fmt],
                                             group, codes_host.data_ptr(), scales_host.data_ptr(),
                                             _stream_handle(stream)))


def _signs_ptr(signs: torch.Tensor | None, dev: torch.device, b: int) -> int | None:
    if signs is None:
        return None
    if signs.dtype != torch.int8 or not signs.is_contiguous():
        raise HadqError(HADQ_ERR_INVALID_ARG, "signs must be a contiguous int8 tensor")
    _on_device("signs", signs, dev)
    _holds("signs", signs, b)
    return signs.data_ptr()


def _block_len(n: int, block: int) -> int:
    """b of the call (block 0 or -1: the whole row)."""
    return n if block in (0, -1) or block >= n else block


def hadq_rotate_signed(x: torch.Tensor, signs: torch.Tensor, side: str = "after", block: int = 0,
                       out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None,
                       stream=None) -> torch.Tensor:
    """Random Hadamard rotation: every block times H_b diag(s) / sqrt(b)
    (side "after") or diag(s) H_b / sqrt(b) (side "before"); ``signs`` holds
    the b int8 signs on the device (see include/hadq.h)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    sp = _signs_ptr(signs, x.device, _block_len(n, block))
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _on_device("out", out, x.device)
    _holds("out", out, rows * n * out.element_size())
    _check(lib.hadq_rotate_signed(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, sp,
                                  SIDES[side], out.data_ptr(), _dtype_code(out.dtype), _stream_handle(stream)))
    return out


def hadq_rotate_quant_signed(x: torch.Tensor, signs: torch.Tensor, side: str = "after", block: int = 0,
                             fmt: str = "int4", group: int = 128, codes: torch.Tensor | None = None,
                             scales: torch.Tensor | None = None, stream=None):
    """Random Hadamard rotation and quantization in one pass; returns (codes, scales)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    sp = _signs_ptr(signs, x.device, _block_len(n, block))
    cs, cd, ss, sd = output_shapes(rows, n, fmt, group if fmt == "int4" else 32)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=x.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=x.device)
    _quant_outputs(lib, rows, n, fmt, group, codes, scales, x.device)
    _check(lib.hadq_rotate_quant_signed(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, sp,
                                        SIDES[side], FMTS[fmt], group, codes.data_ptr(), scales.data_ptr(),
                                        _stream_handle(stream)))
    return codes, scales


def hadq_rotate_quant_nvfp4(x: torch.Tensor, tensor_scale: float = 1.0, block: int = 0,
                            codes: torch.Tensor | None = None, scales: torch.Tensor | None = None, stream=None):
    """Rotate and quantize to NVFP4 with a per-tensor scale; returns (codes, E4M3 scales)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    cs, cd, ss, sd = output_shapes(rows, n, "nvfp4", 16)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=x.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=x.device)
    _quant_outputs(lib, rows, n, "nvfp4", 16, codes, scales, x.device)
    _check(lib.hadq_rotate_quant_nvfp4(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, float(tensor_scale),
                                       codes.data_ptr(), scales.data_ptr(), _stream_handle(stream)))
    return codes, scales


def _rpbh_ptrs(perm, signs, dev, n):
    if perm is None or signs is None:
        raise HadqError(HADQ_ERR_INVALID_ARG, "RPBH needs perm (int32) and signs (int8)")
    if perm.dtype != torch.int32 or signs.dtype != torch.int8:
        raise HadqError(HADQ_ERR_INVALID_ARG, "perm must be int32 and signs int8")
    for name, t, nb in (("perm", perm, 4 * n), ("signs", signs, n)):
        _on_device(name, t, dev)
        _holds(name, t, nb)
    return perm.data_ptr(), signs.data_ptr()


def hadq_rotate_rpbh(x: torch.Tensor, perm: torch.Tensor, signs: torch.Tensor, block: int = 0,
                     out: torch.Tensor | None = None, out_dtype: torch.dtype | None = None, stream=None):
    """RPBH rotation: x[..., perm] * signs, then the block rotation (see include/hadq.h)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    pp, sp = _rpbh_ptrs(perm, signs, x.device, n)
    if out is None:
        out = torch.empty(x.shape, dtype=out_dtype or x.dtype, device=x.device)
    _on_device("out", out, x.device)
    _holds("out", out, rows * n * out.element_size())
    _check(lib.hadq_rotate_rpbh(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, pp, sp, out.data_ptr(),
                                _dtype_code(out.dtype), _stream_handle(stream)))
    return out


def hadq_rotate_quant_rpbh(x: torch.Tensor, perm: torch.Tensor, signs: torch.Tensor, block: int = 0,
                           fmt: str = "int4", group: int = 128, codes: torch.Tensor | None = None,
                           scales: torch.Tensor | None = None, stream=None):
    """RPBH rotation and quantization in one pass; returns (codes, scales)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    pp, sp = _rpbh_ptrs(perm, signs, x.device, n)
    cs, cd, ss, sd = output_shapes(rows, n, fmt, group if fmt == "int4" else 32)
    if codes is None:
        codes = torch.empty(cs, dtype=cd, device=x.device)
    if scales is None:
        scales = torch.empty(ss, dtype=sd, device=x.device)
    _quant_outputs(lib, rows, n, fmt, group, codes, scales, x.device)
    _check(lib.hadq_rotate_quant_rpbh(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, pp, sp, FMTS[fmt], group,
                                      codes.data_ptr(), scales.data_ptr(), _stream_handle(stream)))
    return codes, scales


def hadq_rotate_quant_codebook(x: torch.Tensor, bits: int, thresholds: torch.Tensor, block: int = 0,
                               perm: torch.Tensor | None = None, signs: torch.Tensor | None = None,
                               codes: torch.Tensor | None = None, norms: torch.Tensor | None = None, stream=None):
    """Per-token norm + nearest-centroid codes of the (RPBH or plain) rotation;
    ``thresholds``: float64 device tensor of 2^bits - 1 decision boundaries
    (e.g. from hadq_codebook(n, bits)).  Returns (codes uint8, norms fp32)."""
    lib = load_library()
    rows, n = _rows_n(x)
    _on_device("x", x, x.device)
    pp = sp = None
    if perm is not None or signs is not None:
        pp, sp = _rpbh_ptrs(perm, signs, x.device, n)
    if thresholds.dtype != torch.float64:
        raise HadqError(HADQ_ERR_INVALID_ARG, "thresholds must be float64")
    _on_device("thresholds", thresholds, x.device)
    _holds("thresholds", thresholds, ((1 << bits) - 1) * 8)
    if codes is None:
        codes = torch.empty((rows, n * bits // 8), dtype=torch.uint8, device=x.device)
    if norms is None:
        norms = torch.empty((rows,), dtype=torch.float32, device=x.device)
    for name, t, nb in (("codes", codes, rows * n * bits // 8), ("norms", norms, rows * 4)):
        _on_device(name, t, x.device)
        _holds(name, t, nb)
    _check(lib.hadq_rotate_quant_codebook(x.data_ptr(), _dtype_code(x.dtype), rows, n, block, pp, sp, int(bits),
                                          thresholds.data_ptr(), codes.data_ptr(), norms.data_ptr(),
                                          _stream_handle(stream)))
    return codes, norms
