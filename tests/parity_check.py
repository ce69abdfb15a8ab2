"""Element-by-element comparison of libhadq outputs with the float64 oracle.

Tolerances (the statement of the problem, with the readings below):

* rotated fp32: max |gpu - oracle| <= 1e-5 * ||x_row||_2 for every row;
* rotated bf16: the round-to-nearest-even of a value within the fp32
  tolerance (between bf16(y - d) and bf16(y + d), d = 1e-5 * ||x_row||);
* int4, MXFP4 and NVFP4 codes: bit-exact, except where the oracle's
  pre-round value (y / s in code units) lies within 1e-6 of a rounding
  boundary; there either adjacent code is accepted and the case is counted;
* per-token int8 codes: the same rule with the window taken relative to the
  row absmax, W = 1e-6 * m / s (about 1.3e-4 code units).  The pre-round
  value reaches |y / s| = 127, where one fp32 ulp is 7.6e-6 code units, so
  no fp32 computation can place it within an absolute 1e-6 of a boundary;
  the literal-window counts are recorded beside it;
* scales: fp16 / E8M0 / E4M3 scales exact, except where the oracle's pre-rounding
  value lies within 1e-6 (relative) of a rounding boundary of the scale
  format, where the other neighbour is accepted (and the group's codes are
  then checked against the oracle's codes for that neighbour); fp32 int8
  scales within 1e-6 relative.

Every candidate value is computed by the oracle; a GPU output only selects
which oracle candidate it must equal.
"""

from __future__ import annotations

import numpy as np

import oracle

WINDOW = 1e-6          # code-boundary window, in code units (int4, MXFP4, NVFP4)
SCALE_WINDOW = 1e-6    # relative window of a scale-rounding boundary
INT8_WINDOW_REL = 1e-6  # per-token int8: window relative to the row absmax


def unpack_nibbles(packed: np.ndarray, signed: bool) -> np.ndarray:
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    lo, hi = p & 0xF, p >> 4
    out = np.empty(p.shape[:-1] + (p.shape[-1] * 2,), dtype=np.int64)
    out[..., 0::2], out[..., 1::2] = lo, hi
    if signed:
        out = np.where(out >= 8, out - 16, out)
    return out


def check_rotation_f32(x64: np.ndarray, y_gpu: np.ndarray, block: int, y=None) -> dict:
    y = oracle.rotate(x64, block) if y is None else y
    err = np.abs(np.asarray(y_gpu, dtype=np.float64) - y).max(axis=1)
    norm = np.linalg.norm(x64, axis=1)
    rel = err / np.where(norm > 0, norm, 1.0)
    bad = rel > 1e-5
    assert not bad.any(), f"{bad.sum()} rows exceed 1e-5 * ||x||: worst {rel.max():.3e}"
    return {"rows": len(rel), "worst_rel_err": float(rel.max())}


def _bf16_value(bits):
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_rotation_bf16(x64: np.ndarray, y_bits: np.ndarray, block: int, y=None) -> dict:
    """bf16 output = round-to-nearest-even of a value within the fp32 tolerance.

    With d = 1e-5 * ||x_row||, the output must lie between bf16(y - d) and
    bf16(y + d) (rounding is monotone).  Away from zero this is within one
    bf16 ulp of bf16(y); near zero the fp32 error bound (relative to the row
    norm) dominates the ulp of the element.
    """
    y = oracle.rotate(x64, block) if y is None else y
    d = 1e-5 * np.linalg.norm(x64, axis=1, keepdims=True)
    lo = _bf16_value(oracle.to_bf16_bits(y - d))
    hi = _bf16_value(oracle.to_bf16_bits(y + d))
    want = _bf16_value(oracle.to_bf16_bits(y))
    gv = _bf16_value(y_bits)
    bad = (gv < lo) | (gv > hi)
    assert not bad.any(), f"{bad.sum()} bf16 outputs outside bf16([y - d, y + d])"
    a = np.abs(want)
    ulp = np.ldexp(1.0, np.maximum(np.frexp(np.where(a > 0, a, 1.0))[1] - 1, -126) - 7)
    return {"elements": int(y.size), "not_bit_equal": int((gv != want).sum()),
            "max_ulps_from_rne_of_oracle": float((np.abs(gv - want) / ulp).max())}


def _check_codes(got, v, w, encode):
    """got must equal encode(v) except where encode(v - w) != encode(v + w)."""
    lo, mid, hi = encode(v - w), encode(v), encode(v + w)
    boundary = lo != hi
    ok = (got == mid) | (boundary & ((got == lo) | (got == hi)))
    return ok, boundary


def check_int4(x64, codes_packed, scales_fp16, block: int, group: int, y=None) -> dict:
    y = oracle.rotate(x64, block) if y is None else y
    rows, n = y.shape
    g = y.reshape(rows, n // group, group)
    m = np.abs(g).max(axis=-1)
    s_gpu = np.asarray(scales_fp16, dtype=np.float16).astype(np.float64).reshape(rows, n // group)
    cand_lo = oracle.to_fp16(m / 7 * (1 - SCALE_WINDOW))
    cand_mid = oracle.to_fp16(m / 7)
    cand_hi = oracle.to_fp16(m / 7 * (1 + SCALE_WINDOW))
    scale_ok = (s_gpu == cand_mid) | (s_gpu == cand_lo) | (s_gpu == cand_hi)
    assert scale_ok.all(), f"{(~scale_ok).sum()} int4 scales outside the oracle's candidates"
    s_ref = s_gpu                       # now known to be one of the oracle's candidates
    q_gpu = unpack_nibbles(codes_packed, signed=True).reshape(rows, n // group, group)
    usable = (s_ref > 0) & np.isfinite(s_ref)
    safe = np.where(usable, s_ref, 1.0)[..., None]
    v = g / safe

    def enc(t):
        return np.where(usable[..., None], np.clip(np.rint(t), -7, 7), 0)
    ok, boundary = _check_codes(q_gpu, v, WINDOW, enc)
    assert ok.all(), f"{(~ok).sum()} int4 codes differ outside the boundary window"
    return {"elements": int(y.size), "groups": int(m.size),
            "scale_boundary_groups": int((cand_lo != cand_hi).sum()),
            "scale_took_neighbour": int((s_gpu != cand_mid).sum()),
            "code_boundary_cases": int(boundary.sum()),
            "code_differs_in_window": int((q_gpu != enc(v)).sum())}


def check_int8(x64, codes, scales_fp32, block: int, y=None) -> dict:
    """Per-token int8: the window is 1e-6 of the row absmax (in code units
    1e-6 * m / s, about 1.3e-4); the literal 1e-6 code-unit window is counted
    beside it (``*_literal``) and not asserted (see the module docstring)."""
    y = oracle.rotate(x64, block) if y is None else y
    q_o, s_o = oracle.quantize_int8_per_token(y)
    s_o = s_o.astype(np.float64)
    s_gpu = np.asarray(scales_fp32, dtype=np.float32).astype(np.float64)
    rel = np.abs(s_gpu - s_o) / np.where(s_o > 0, s_o, 1.0)
    assert (rel <= 1e-6).all() and ((s_o == 0) == (s_gpu == 0)).all(), f"int8 scale rel err {rel.max():.3e}"
    m = np.abs(y).max(axis=1)
    usable = (s_o > 0) & np.isfinite(s_o)
    safe = np.where(usable, s_o, 1.0)[:, None]
    v = y / safe
    w = INT8_WINDOW_REL * m[:, None] / safe

    def enc(t):
        return np.where(usable[:, None], np.clip(np.rint(t), -127, 127), 0)
    got = np.asarray(codes, dtype=np.int8).astype(np.int64)
    ok, boundary = _check_codes(got, v, w, enc)
    assert ok.all(), f"{(~ok).sum()} int8 codes differ outside the boundary window"
    ok_lit, boundary_lit = _check_codes(got, v, WINDOW, enc)
    return {"elements": int(y.size), "rows": int(len(m)), "worst_scale_rel_err": float(rel.max()),
            "window": "1e-6 x row absmax",
            "code_boundary_cases": int(boundary.sum()), "code_differs_in_window": int((got != q_o).sum()),
            "code_boundary_cases_literal": int(boundary_lit.sum()),
            "code_differs_outside_literal_window": int((~ok_lit).sum())}


def check_mxfp4(x64, codes_packed, scales_e8m0, block: int, y=None) -> dict:
    y = oracle.rotate(x64, block) if y is None else y
    rows, n = y.shape
    g = y.reshape(rows, n // 32, 32)
    m = np.abs(g).max(axis=-1)
    e_gpu = np.asarray(scales_e8m0, dtype=np.uint8).astype(np.int64).reshape(rows, n // 32) - 127
    e_lo = oracle.e8m0_exponent(m * (1 - SCALE_WINDOW))
    e_mid = oracle.e8m0_exponent(m)
    e_hi = oracle.e8m0_exponent(m * (1 + SCALE_WINDOW))
    scale_ok = (e_gpu == e_mid) | (e_gpu == e_lo) | (e_gpu == e_hi)
    assert scale_ok.all(), f"{(~scale_ok).sum()} E8M0 exponents outside the oracle's candidates"
    v = np.ldexp(g, -e_gpu[..., None])
    got = unpack_nibbles(codes_packed, signed=False).reshape(rows, n // 32, 32)
    ok, boundary = _check_codes(got, v, WINDOW, oracle.e2m1_encode)
    assert ok.all(), f"{(~ok).sum()} E2M1 codes differ outside the boundary window"
    return {"elements": int(y.size), "groups": int(m.size),
            "scale_boundary_groups": int((e_lo != e_hi).sum()),
            "scale_took_neighbour": int((e_gpu != e_mid).sum()),
            "code_boundary_cases": int(boundary.sum()),
            "code_differs_in_window": int((got != oracle.e2m1_encode(v)).sum())}


def _e4m3_value(byte):
    """Value of E4M3 bytes (sign, exponent bias 7, 3 mantissa bits; 0x7F/0xFF unused)."""
    b = np.asarray(byte, dtype=np.uint8).astype(np.int64)
    e, m = (b >> 3) & 15, b & 7
    mag = np.where(e > 0, np.ldexp(1.0 + m / 8.0, e - 7), np.ldexp(m / 8.0, -6))
    return np.where(b & 0x80, -mag, mag)


def check_nvfp4(x64, codes_packed, scales_e4m3, block: int, y=None, tensor_scale: float = 1.0) -> dict:
    """NVFP4: E4M3 scale of max|v| / 6 per 16 elements (v = y / tensor_scale),
    E2M1 codes of v / s (code window 1e-6 in units of v / s).  The scale may take the other rounding neighbour only
    when max|v| / 6 lies within 1e-6 (relative) of an E4M3 rounding boundary;
    the codes are then checked against the oracle's codes for the GPU's scale."""
    y = oracle.rotate(x64, block) if y is None else y
    rows, n = y.shape
    g = y.reshape(rows, n // 16, 16) / tensor_scale
    m = np.abs(g).max(axis=-1)
    s_gpu = _e4m3_value(np.asarray(scales_e4m3, dtype=np.uint8).reshape(rows, n // 16))
    cand_lo = oracle.to_e4m3(m / 6 * (1 - SCALE_WINDOW))
    cand_mid = oracle.to_e4m3(m / 6)
    cand_hi = oracle.to_e4m3(m / 6 * (1 + SCALE_WINDOW))
    scale_ok = (s_gpu == cand_mid) | (s_gpu == cand_lo) | (s_gpu == cand_hi)
    assert scale_ok.all(), f"{(~scale_ok).sum()} E4M3 scales outside the oracle's candidates"
    got = unpack_nibbles(codes_packed, signed=False).reshape(rows, n // 16, 16)
    usable = s_gpu > 0
    safe = np.where(usable, s_gpu, 1.0)[..., None]
    v = g / safe

    def enc(t):
        return np.where(usable[..., None], oracle.e2m1_encode(t), 0)
    ok, boundary = _check_codes(got, v, WINDOW, enc)
    assert ok.all(), f"{(~ok).sum()} NVFP4 codes differ outside the boundary window"
    return {"elements": int(y.size), "groups": int(m.size),
            "scale_boundary_groups": int((cand_lo != cand_hi).sum()),
            "scale_took_neighbour": int((s_gpu != cand_mid).sum()),
            "code_boundary_cases": int(boundary.sum()),
            "code_differs_in_window": int((got != enc(v)).sum())}


def unpack_codes(packed, bits: int) -> np.ndarray:
    """8 // bits codes per byte, code i in bits [i * bits, (i + 1) * bits)."""
    p = np.asarray(packed, dtype=np.uint8).astype(np.int64)
    per = 8 // bits
    out = np.empty(p.shape[:-1] + (p.shape[-1] * per,), dtype=np.int64)
    for i in range(per):
        out[..., i::per] = (p >> (bits * i)) & ((1 << bits) - 1)
    return out


def check_codebook(x64, codes_packed, norms, block: int, bits: int, y=None) -> dict:
    """Codebook quantizer: norms within 1e-6 relative of ||y||; codes the
    oracle's nearest centroid of y / ||y|| (its own Lloyd-Max codebook for
    d = n), except within 1e-6 of a decision threshold in code units -- the
    distance between the two centroids that threshold separates."""
    y = oracle.rotate(x64, block) if y is None else y
    rows, n = y.shape
    c, t = oracle.sphere_lloyd_max(n, bits)
    q_o, r_o = oracle.quantize_codebook(y, c, t)
    r_gpu = np.asarray(norms, dtype=np.float32).astype(np.float64).reshape(rows)
    rel = np.abs(r_gpu - r_o) / np.where(r_o > 0, r_o, 1.0)
    assert (rel <= 1e-6).all() and ((r_o == 0) == (r_gpu == 0)).all(), f"norm rel err {rel.max():.3e}"
    u = y / np.where(r_o > 0, r_o, 1.0)[:, None]
    j = np.abs(u[..., None] - t).argmin(axis=-1)          # nearest threshold
    w = WINDOW * (c[j + 1] - c[j])
    got = unpack_codes(codes_packed, bits).reshape(rows, n)

    def enc(v):
        return np.searchsorted(t, v, side="left")
    ok, boundary = _check_codes(got, u, w, enc)
    assert ok.all(), f"{(~ok).sum()} codebook codes differ outside the boundary window"
    return {"elements": int(y.size), "rows": rows, "worst_norm_rel_err": float(rel.max()),
            "code_boundary_cases": int(boundary.sum()), "code_differs_in_window": int((got != q_o).sum())}


def check(fmt, x64, out0, out1, block, group, y=None):
    """``y``: the oracle's rotation when it is not ``oracle.rotate(x64, block)``
    (e.g. a random Hadamard rotation)."""
    if fmt == "int4":
        return check_int4(x64, out0, out1, block, group, y=y)
    if fmt == "int8":
        return check_int8(x64, out0, out1, block, y=y)
    if fmt == "mxfp4":
        return check_mxfp4(x64, out0, out1, block, y=y)
    if fmt == "nvfp4":
        return check_nvfp4(x64, out0, out1, block, y=y)
    raise ValueError(fmt)
