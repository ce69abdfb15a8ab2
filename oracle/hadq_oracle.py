"""Float64 reference for rotate / rotate+quantize.  Test infrastructure only.

Every function follows a passage of the pages (cited in its docstring) or,
where the pages are silent, a reading stated in the docstring.  The code is
deliberately plain: explicit matrices, dense products, whole-array numpy
expressions, no blocking or fusion beyond what the definitions state.

Every function is pinned, in tests/test_oracle_pins.py, to something other
than itself (hand-worked cases, closed forms, invariants, library routines).
End-to-end rotated-and-quantized values of a whole workload are parity
unpinned by the pages: none prints a worked example, so they are pinned only
through the pinned parts.
"""

from __future__ import annotations

import functools

import numpy as np

INT4_QMAX = 7      # symmetric int4 range +/-7 (scale = absmax / 7)
INT8_QMAX = 127    # symmetric int8 range +/-127 (scale = absmax / 127)
MX_GROUP = 32      # MX block size ("Rotation Transform", section 2.1: 32 for MXFP)
NV_GROUP = 16      # NVFP4 block size (same section: 16 for NVFP)
E4M3_MAX = 448.0   # largest finite FP8 E4M3 magnitude

# E2M1 magnitudes indexed by the 3-bit code (exponent 2 bits, mantissa 1 bit).
E2M1_GRID = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0], dtype=np.float64)


# ---------------------------------------------------------------------------
# Rotation
# ---------------------------------------------------------------------------

def _is_pow2(v: int) -> bool:
    return v >= 1 and (v & (v - 1)) == 0


@functools.lru_cache(maxsize=6)
def _sylvester(size: int) -> np.ndarray:
    h = np.ones((1, 1), dtype=np.float64)
    while h.shape[0] < size:
        h = np.block([[h, h], [h, -h]])
    h.setflags(write=False)
    return h


def sylvester_hadamard(size: int) -> np.ndarray:
    """Unnormalised Sylvester Hadamard matrix of order ``size`` (entries +/-1).

    "Rotation Transform" (AutoRound docs), section 1.5: the deterministic
    matrix is built by the doubling H -> [[H, H], [H, -H]]; its size must be a
    power of 2.  Starting from H_1 = [1] fixes the natural (Hadamard) row
    order.  The result is read-only and cached.
    """
    size = int(size)
    if not _is_pow2(size):
        raise ValueError(f"Sylvester Hadamard size must be a power of 2, got {size}")
    return _sylvester(size)


# ---------------------------------------------------------------------------
# Non-power-of-2 sizes: n = K * 2^m
# ---------------------------------------------------------------------------
# "Rotation Transform", section 1.5: for non-power-of-2 dimensions
# get_hadamard_K(n) factors n = K * 2^m and combines a known base Hadamard
# matrix of order K with a Sylvester block.  The pages name the orders (12,
# 20, 28, 36, 40, 52, 60, 108, 140, 156, 172) but print no base matrix.
# Reading: the base matrix of order K = 2 (q + 1) is Paley's second
# construction over the field of q elements (q = 1 mod 4 a prime power;
# R. E. A. C. Paley, "On orthogonal matrices", J. Math. Phys. 12, 1933), and
# the combination is the Kronecker product H_n = H_K (x) H_(2^m), the base
# factor outermost as the Sylvester doubling H_2k = H_2 (x) H_k puts its own.
# These K are covered: 12, 20, 28, 36, 52, 60, 108 (40 = 2 * 20 is the K = 20
# matrix with one more Sylvester factor).  The matrices are symmetric, so
# H_n / sqrt(n) stays its own inverse.

# K -> (p, k): the field GF(p^k), q = p^k = K / 2 - 1.
PALEY_FIELDS = {12: (5, 1), 20: (3, 2), 28: (13, 1), 36: (17, 1), 52: (5, 2), 60: (29, 1), 108: (53, 1)}
# GF(p^2) = GF(p)[i] / (i^2 - nu), nu a quadratic non-residue mod p.
GF2_NONRESIDUE = {3: 2, 5: 2}


def _gf_elements(p: int, k: int):
    """Field elements as coefficient pairs (a, b) meaning a + b*i; element
    index t = a + p * b (k = 1: b = 0, index = the residue)."""
    return [(t % p, t // p) for t in range(p ** k)]


def _gf_index(e, p: int) -> int:
    return e[0] + p * e[1]


def _gf_sub(e1, e2, p: int):
    return ((e1[0] - e2[0]) % p, (e1[1] - e2[1]) % p)


def _gf_mul(e1, e2, p: int, nu: int):
    a, b = e1
    c, d = e2
    return ((a * c + nu * b * d) % p, (a * d + b * c) % p)


def quadratic_character(p: int, k: int) -> np.ndarray:
    """chi over GF(p^k) by element index: 0 at 0, +1 on the nonzero squares,
    -1 on the non-squares (the squares found by squaring every element)."""
    nu = GF2_NONRESIDUE.get(p, 0) if k == 2 else 0
    els = _gf_elements(p, k)
    chi = -np.ones(len(els), dtype=np.int64)
    chi[0] = 0
    for e in els[1:]:
        chi[_gf_index(_gf_mul(e, e, p, nu), p)] = 1
    return chi


def jacobsthal(p: int, k: int) -> np.ndarray:
    """Q[a, b] = chi(a - b) over the field elements in index order."""
    els = _gf_elements(p, k)
    chi = quadratic_character(p, k)
    return np.array([[chi[_gf_index(_gf_sub(a, b, p), p)] for b in els] for a in els], dtype=np.int64)


def paley_hadamard(order: int) -> np.ndarray:
    """Paley II Hadamard matrix of order K = 2 (q + 1) (entries +/-1).

    C = [[0, 1^T], [1, Q]] is the symmetric conference matrix of order q + 1
    (index 0 the point at infinity, then the field elements in index order);
    H = C (x) [[1, 1], [1, -1]] + I (x) [[1, -1], [-1, -1]].
    """
    if order not in PALEY_FIELDS:
        raise ValueError(f"no base Hadamard matrix of order {order}; covered: {sorted(PALEY_FIELDS)}")
    p, k = PALEY_FIELDS[order]
    q = p ** k
    c = np.zeros((q + 1, q + 1), dtype=np.int64)
    c[0, 1:] = 1
    c[1:, 0] = 1
    c[1:, 1:] = jacobsthal(p, k)
    a = np.array([[1, 1], [1, -1]])
    b = np.array([[1, -1], [-1, -1]])
    return (np.kron(c, a) + np.kron(np.eye(q + 1, dtype=np.int64), b)).astype(np.float64)


def split_size(size: int):
    """(K, 2^m) with size = K * 2^m: K = 1 for a power of 2, else the covered
    base order K = 4 * (odd part of size) (a Hadamard order above 2 is a
    multiple of 4).  Raises for a size with no covered base matrix."""
    size = int(size)
    if _is_pow2(size):
        return 1, size
    odd = size
    while odd % 2 == 0:
        odd //= 2
    k = 4 * odd
    if k not in PALEY_FIELDS or size % k != 0:
        raise ValueError(f"size {size} = K * 2^m needs a base Hadamard matrix of order {k}, "
                         f"not covered ({sorted(PALEY_FIELDS)})")
    return k, size // k


@functools.lru_cache(maxsize=2)
def _kron_hadamard(size: int) -> np.ndarray:
    k, s = split_size(size)
    h = np.kron(paley_hadamard(k), sylvester_hadamard(s))
    h.setflags(write=False)
    return h


def hadamard_matrix(size: int) -> np.ndarray:
    """Unnormalised Hadamard matrix of order ``size`` used by the rotation:
    Sylvester for a power of 2, H_K (x) H_(2^m) otherwise (read-only, cached)."""
    k, _ = split_size(size)
    return sylvester_hadamard(size) if k == 1 else _kron_hadamard(int(size))


def resolve_block(n: int, block) -> int:
    """Block size actually applied to a row of length ``n``.

    ``None``, ``-1``, ``0`` and ``n`` all mean the full dimension ("Rotation
    Transform", section 2.1: block_size None/-1 means full-dimension
    Hadamard).  Otherwise the block must divide ``n`` and be a size with a
    Hadamard matrix: a power of 2 (sections 1.2 and 1.5) or K * 2^m with a
    covered base order K (section 1.5, non-power-of-2 dimensions).
    """
    n = int(n)
    if block is None or int(block) in (-1, 0, n):
        b = n
    else:
        b = int(block)
    if b < 1 or n % b != 0:
        raise ValueError(f"block {block!r} does not divide n={n}")
    split_size(b)
    return b


def rotate(x, block=0) -> np.ndarray:
    """y = x . diag(H_b, ..., H_b) / sqrt(b) for every row of ``x`` (float64).

    The online rotation of "Rotation Transform", section 1.1 (R1 on the
    residual stream, R3 per head on Q/K, R4 on the down_proj input) and the
    per-Linear block-diagonal mode of section 2: each row is cut into
    consecutive blocks of ``b`` elements and each block is multiplied by the
    normalised Hadamard matrix of section 1.5 (Sylvester for a power of 2,
    H_K (x) H_(2^m) for b = K * 2^m, see ``hadamard_matrix``).  The product is a dense
    O(b^2)-per-block float64 matmul of the exact upcast input.  H is
    symmetric, so x . H and H . x agree, and H/sqrt(b) is its own inverse.
    """
    x = np.asarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("rotate expects a 2-D (rows, n) array")
    rows, n = x.shape
    b = resolve_block(n, block)
    h = hadamard_matrix(b)
    y = (x.reshape(rows * (n // b), b) @ h) / np.sqrt(float(b))
    return y.reshape(rows, n)


def sign_vector(signs) -> np.ndarray:
    """The +/-1 diagonal of a random Hadamard rotation as float64.

    The signs are persisted as int8 ("Rotation Transform", section 1.7: a
    random rotation is stored as an int8 +/-1 matrix); reading: a negative
    entry is -1, any other entry +1.
    """
    return np.where(np.asarray(signs).reshape(-1).astype(np.int64) < 0, -1.0, 1.0)


def random_hadamard_matrix(signs, side: str = "after") -> np.ndarray:
    """Normalised random Hadamard matrix of order b = len(signs).

    "Rotation Transform", section 1.5: random_hadamard_matrix(size) is
    H @ diag(+/-1) / sqrt(N) -- side ``"after"``.  Side ``"before"`` is
    diag(+/-1) @ H / sqrt(N), its transpose and so its inverse (H and the
    diagonal are symmetric); it puts the signs on the input, ahead of the
    Hadamard transform, in the order of the Rademacher signs and block FWHT
    of orbitquant's RPBH rotation ("orbitquant 0.2.0", how it works).
    """
    s = sign_vector(signs)
    h = hadamard_matrix(s.size)
    # A product with a diagonal matrix scales columns (on the right) or rows
    # (on the left); written out that way it costs O(b^2) instead of O(b^3).
    if side == "after":
        r = h * s[None, :]          # H @ diag(s): column j times s_j
    elif side == "before":
        r = s[:, None] * h          # diag(s) @ H: row j times s_j
    else:
        raise ValueError(f"side must be 'after' or 'before', got {side!r}")
    return r / np.sqrt(float(s.size))


def rotate_signed(x, block, signs, side: str = "after") -> np.ndarray:
    """y = x . diag(R, ..., R) with R = random_hadamard_matrix(signs, side).

    The random-Hadamard variant of ``rotate`` ("Rotation Transform", section
    1.2: random_r1..random_r4 replace the deterministic matrix at a
    position): each block of b = len(signs) elements is multiplied by the same
    R, as a dense float64 product.
    """
    x = np.asarray(x, dtype=np.float64)
    if x.ndim != 2:
        raise ValueError("rotate_signed expects a 2-D (rows, n) array")
    rows, n = x.shape
    b = resolve_block(n, block)
    if sign_vector(signs).size != b:
        raise ValueError(f"need {b} signs (one per column of the {b}-point block)")
    r = random_hadamard_matrix(signs, side)
    return (x.reshape(rows * (n // b), b) @ r).reshape(rows, n)


# ---------------------------------------------------------------------------
# Rounding onto binary floating-point grids (scales and outputs)
# ---------------------------------------------------------------------------

def _floor_log2(a: np.ndarray) -> np.ndarray:
    """floor(log2(a)) for a > 0, exact (from the binary exponent)."""
    _, p = np.frexp(a)          # a = f * 2**p with f in [0.5, 1)
    return p.astype(np.int64) - 1


def round_to_binary(v, mant_bits: int, emin: int, max_finite: float) -> np.ndarray:
    """Round-half-to-even of float64 ``v`` onto a binary floating-point grid.

    The grid has ``mant_bits`` stored mantissa bits and smallest normal
    exponent ``emin`` (subnormals below it keep the spacing 2**(emin -
    mant_bits)).  Magnitudes that round above ``max_finite`` become inf, as
    IEEE rounding does.  Used for fp16 scales (10, -14), fp32 scales (23,
    -126) and bf16 outputs (7, -126).
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    nz = a > 0
    e = np.where(nz, _floor_log2(np.where(nz, a, 1.0)), emin)
    ulp = np.ldexp(1.0, np.maximum(e, emin) - mant_bits)
    r = np.rint(v / ulp) * ulp          # v/ulp is exact: ulp is a power of 2
    return np.where(np.abs(r) > max_finite, np.copysign(np.inf, v), r)


def to_fp16(v) -> np.ndarray:
    """float64 -> IEEE binary16, round half to even (returns float64 values)."""
    return round_to_binary(v, 10, -14, 65504.0)


def to_fp32(v) -> np.ndarray:
    """float64 -> IEEE binary32, round half to even (returns float64 values)."""
    return round_to_binary(v, 23, -126, float(np.finfo(np.float32).max))


def to_bf16_bits(v) -> np.ndarray:
    """float64 -> bfloat16 bit patterns (uint16), round half to even."""
    r = round_to_binary(v, 7, -126, (2.0 - 2.0 ** -7) * 2.0 ** 127)
    return (r.astype(np.float32).view(np.uint32) >> 16).astype(np.uint16)


def fp16_scale_midpoint_distance(v):
    """Relative distance of ``v`` to the nearest fp16 rounding midpoint, and
    the fp16 value the rounding would give on the other side of it.

    Used by the parity checker: a scale whose pre-rounding value lies within
    1e-6 of a midpoint is a boundary case where either neighbour is valid.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    nz = a > 0
    e = np.where(nz, _floor_log2(np.where(nz, a, 1.0)), -14)
    ulp = np.ldexp(1.0, np.maximum(e, -14) - 10)
    lo = np.floor(a / ulp) * ulp
    hi = lo + ulp
    mid = 0.5 * (lo + hi)
    rounded = np.abs(to_fp16(a))
    alt = np.where(rounded == lo, hi, lo)
    rel = np.where(nz, np.abs(a - mid) / np.where(nz, a, 1.0), np.inf)
    return rel, np.copysign(alt, v)


# ---------------------------------------------------------------------------
# Round-to-nearest quantizers
# ---------------------------------------------------------------------------

def codes_with_scale(y, s, qmax: int) -> np.ndarray:
    """q = clamp(round_half_even(y / s), -qmax, qmax); 0 where s is 0 or inf.

    Round-to-nearest with the symmetric range (the RTN proxy of "Pre-Process
    (Rotation Preprocessing)", Workflow note: wbits, groupsize, sym).
    Readings: ties round to even; the code uses the stored (rounded) scale,
    so dequantisation q * s is self-consistent; a zero scale (all-zero group)
    or an infinite one gives zero codes.
    """
    y = np.asarray(y, dtype=np.float64)
    s = np.asarray(s, dtype=np.float64)
    ok = (s > 0) & np.isfinite(s)
    safe = np.where(ok, s, 1.0)
    q = np.clip(np.rint(y / safe), -qmax, qmax)
    q = np.where(ok, q, 0.0)
    return q.astype(np.int16)


def quantize_int4_sym(y, group: int):
    """Symmetric int4 RTN per group: scale = fp16(absmax / 7), codes in [-7, 7].

    Returns ``(codes int8 (rows, n), scales float16 (rows, n // group))``.
    """
    y = np.asarray(y, dtype=np.float64)
    rows, n = y.shape
    if group <= 0 or n % group:
        raise ValueError(f"group {group} must divide n={n}")
    g = y.reshape(rows, n // group, group)
    m = np.abs(g).max(axis=-1)
    s = to_fp16(m / INT4_QMAX)
    codes = codes_with_scale(g, s[..., None], INT4_QMAX).reshape(rows, n)
    return codes.astype(np.int8), s.astype(np.float16)


def quantize_int8_per_token(y):
    """Symmetric int8 RTN per row: scale = fp32(absmax / 127), codes in [-127, 127].

    Returns ``(codes int8 (rows, n), scales float32 (rows,))``.
    """
    y = np.asarray(y, dtype=np.float64)
    m = np.abs(y).max(axis=1)
    s = to_fp32(m / INT8_QMAX)
    codes = codes_with_scale(y, s[:, None], INT8_QMAX)
    return codes.astype(np.int8), s.astype(np.float32)


def e8m0_exponent(m) -> np.ndarray:
    """Shared MX exponent e = floor(log2(m)) - 2, clamped to [-127, 127].

    OCP MX v1.0 reading (the pages name MXFP4 but not its scale rule): the
    largest E2M1 magnitude is 6 = 1.5 * 2**2, so the exponent is the group
    absmax's exponent minus 2.  An all-zero group gets -127 (stored byte 0).
    """
    m = np.asarray(m, dtype=np.float64)
    nz = m > 0
    e = np.where(nz, _floor_log2(np.where(nz, m, 1.0)) - 2, -127)
    return np.clip(e, -127, 127)


def e2m1_encode(v) -> np.ndarray:
    """E2M1 code (sign << 3 | index) of ``v``.

    The index is that of the nearest magnitude in ``E2M1_GRID``; a tie goes
    to the even index (even mantissa bit), so 0.25 -> 0, 0.75 -> 1.0,
    1.25 -> 1.0, 1.75 -> 2, 2.5 -> 2, 3.5 -> 4, 5 -> 4; magnitudes above 6
    take 6 (saturation).  The sign bit is set for negative values, including
    those whose magnitude rounds to zero.
    """
    v = np.asarray(v, dtype=np.float64)
    a = np.abs(v)
    best = np.zeros(a.shape, dtype=np.int64)
    bestd = np.abs(a - E2M1_GRID[0])
    for i in range(1, len(E2M1_GRID)):
        d = np.abs(a - E2M1_GRID[i])
        better = (d < bestd) | ((d == bestd) & (i % 2 == 0))
        best = np.where(better, i, best)
        bestd = np.where(better, d, bestd)
    sign = (v < 0).astype(np.int64)
    return (best | (sign << 3)).astype(np.uint8)


def quantize_mxfp4(y):
    """MXFP4: per 32 elements an E8M0 exponent e and E2M1 codes of y / 2**e.

    Returns ``(codes uint8 (rows, n) in [0, 15], scales uint8 (rows, n // 32))``
    where the stored scale byte is e + 127.
    """
    y = np.asarray(y, dtype=np.float64)
    rows, n = y.shape
    if n % MX_GROUP:
        raise ValueError(f"n={n} is not a multiple of {MX_GROUP}")
    g = y.reshape(rows, n // MX_GROUP, MX_GROUP)
    m = np.abs(g).max(axis=-1)
    e = e8m0_exponent(m)
    v = np.ldexp(g, -e[..., None])
    codes = e2m1_encode(v).reshape(rows, n)
    return codes, (e + 127).astype(np.uint8)


def to_e4m3(v) -> np.ndarray:
    """float64 -> FP8 E4M3 value (returns float64 values).

    Round half to even onto 3 stored mantissa bits, smallest normal 2**-6
    (subnormal spacing 2**-9); magnitudes above the largest finite value 448
    take 448 (a saturating conversion: E4M3 has no infinity).
    """
    r = round_to_binary(v, 3, -6, np.inf)
    return np.clip(r, -E4M3_MAX, E4M3_MAX)


def e4m3_encode(v) -> np.ndarray:
    """E4M3 byte of ``to_e4m3(v)``: sign << 7 | biased exponent (bias 7) << 3 |
    mantissa; subnormals (below 2**-6) have exponent field 0."""
    q = to_e4m3(v)
    a = np.abs(q)
    normal = a >= 2.0 ** -6
    e = np.where(normal, _floor_log2(np.where(normal, a, 1.0)), -6)
    mant = np.where(normal, a / np.ldexp(1.0, e) - 1.0, a / 2.0 ** -6)   # in [0, 1)
    field = np.where(normal, (e + 7) << 3, 0).astype(np.int64) | np.rint(mant * 8).astype(np.int64)
    return (field | (np.signbit(q) & (a > 0)).astype(np.int64) << 7).astype(np.uint8)


def quantize_nvfp4(y, tensor_scale: float = 1.0):
    """NVFP4: per 16 elements an E4M3 scale and E2M1 codes.

    The pages name the scheme and its block of 16 ("Rotation Transform",
    introduction and section 2.1) but not its encoding; reading: NVIDIA's
    public NVFP4 definition.  With v = y / tensor_scale (the per-tensor
    second-level scale, 1 for the single-level form): per block
    s = E4M3(max|v| / 6) and code = E2M1 rne(v / s) (saturating at +/-6, sign
    bit 3); s == 0 gives codes 0.  Dequantization is code * s * tensor_scale.
    Returns ``(codes uint8 (rows, n) in [0, 15], scale bytes uint8 (rows, n // 16))``.
    """
    y = np.asarray(y, dtype=np.float64)
    rows, n = y.shape
    if n % NV_GROUP:
        raise ValueError(f"n={n} is not a multiple of {NV_GROUP}")
    if not (np.isfinite(tensor_scale) and tensor_scale > 0):
        raise ValueError("tensor_scale must be finite and > 0")
    g = (y / tensor_scale).reshape(rows, n // NV_GROUP, NV_GROUP)
    s = to_e4m3(np.abs(g).max(axis=-1) / 6.0)
    safe = np.where(s > 0, s, 1.0)[..., None]
    codes = np.where(s[..., None] > 0, e2m1_encode(g / safe), 0).astype(np.uint8).reshape(rows, n)
    return codes, e4m3_encode(s)


def pack_nibbles(codes) -> np.ndarray:
    """Two 4-bit codes per byte, the even-indexed element in the low nibble.

    int4 codes are stored as two's-complement nibbles (q & 0xF).
    """
    c = np.asarray(codes).astype(np.int64) & 0xF
    if c.shape[-1] % 2:
        raise ValueError("row length must be even to pack nibbles")
    return (c[..., 0::2] | (c[..., 1::2] << 4)).astype(np.uint8)


def rotate_quant(x, block, fmt: str, group: int = 0, tensor_scale: float = 1.0):
    """Rotate then quantize, as the fused path does in one pass.

    ``fmt`` is ``"int4"`` (codes packed two per byte, fp16 scales per
    ``group``), ``"int8"`` (per-token; int8 codes, fp32 scale per row),
    ``"mxfp4"`` (codes packed two per byte, E8M0 bytes per 32) or ``"nvfp4"``
    (codes packed two per byte, E4M3 bytes per 16; ``tensor_scale`` is its
    per-tensor scale).  Returns ``(y, codes_stored, scales)`` where ``y`` is
    the float64 rotation.
    """
    return quantize(rotate(x, block), fmt, group, tensor_scale)


def rotate_quant_signed(x, block, signs, side: str, fmt: str, group: int = 0, tensor_scale: float = 1.0):
    """``rotate_signed`` then the quantizer of ``rotate_quant`` (same returns)."""
    return quantize(rotate_signed(x, block, signs, side), fmt, group, tensor_scale)


def quantize(y, fmt: str, group: int = 0, tensor_scale: float = 1.0):
    """The quantizer step of ``rotate_quant`` applied to a rotated ``y``."""
    y = np.asarray(y, dtype=np.float64)
    if fmt == "nvfp4":
        if group not in (0, NV_GROUP):
            raise ValueError("NVFP4 groups are 16 elements")
        q, s = quantize_nvfp4(y, tensor_scale)
        return y, pack_nibbles(q), s
    if fmt == "int4":
        q, s = quantize_int4_sym(y, group)
        return y, pack_nibbles(q), s
    if fmt == "int8":
        if group not in (0, y.shape[1]):
            raise ValueError("int8 is per-token: group must be 0 or n")
        q, s = quantize_int8_per_token(y)
        return y, q, s
    if fmt == "mxfp4":
        if group not in (0, MX_GROUP):
            raise ValueError("MXFP4 groups are 32 elements")
        q, s = quantize_mxfp4(y)
        return y, pack_nibbles(q), s
    raise ValueError(f"unknown fmt {fmt!r}")


# ---------------------------------------------------------------------------
# orbitquant: RPBH rotation and the unit-sphere Lloyd-Max codebook quantizer
# ---------------------------------------------------------------------------
# "orbitquant 0.2.0" (PyPI page), Method Conformance: the rotation is RPBH --
# a permutation, Rademacher signs, a block FWHT and orthonormal scaling -- and
# activations are quantized online by a per-token norm, rotation of the
# normalized activation, nearest-centroid quantization and rescaling, with one
# fixed codebook per (input dimension, bit width) from "exact unit-sphere
# Lloyd-Max codebooks" (Features).  The page gives no formula; readings:
#   * RPBH(x) = (x[pi] * s) . diag(H_B, ..., H_B) / sqrt(B): v_e = x_pi(e) s_e
#     for every column e of the row (pi a permutation of the n columns, s n
#     signs), then the block rotation of ``rotate``;
#   * the codebook is the Lloyd-Max (minimum mean-square error) quantizer of
#     one coordinate T of a uniformly random unit vector in R^d, whose density
#     is f_d(t) = (1 - t^2)^((d - 3) / 2) / B(1/2, (d - 1) / 2) on [-1, 1]: a
#     rotated, normalized activation is such a vector when the rotation is
#     random, which is why the codebook needs no data;
#   * code = index of the nearest centroid of y / ||y|| (a value exactly on a
#     threshold takes the lower index); the per-token scale is ||y|| = ||x||.


def rpbh_rotate(x, block, perm, signs) -> np.ndarray:
    """RPBH rotation of every row: permute the columns by ``perm``
    (v_e = x[pi(e)]), multiply by the signs (negative int8 = -1), then the
    block-diagonal normalised Hadamard rotation of ``rotate``."""
    x = np.asarray(x, dtype=np.float64)
    rows, n = x.shape
    perm = np.asarray(perm, dtype=np.int64).reshape(-1)
    if perm.size != n or not np.array_equal(np.sort(perm), np.arange(n)):
        raise ValueError("perm must be a permutation of the n columns")
    s = sign_vector(signs)
    if s.size != n:
        raise ValueError("RPBH takes one sign per column (n signs)")
    return rotate(x[:, perm] * s[None, :], block)


def rpbh_inverse(y, block, perm, signs) -> np.ndarray:
    """Inverse of ``rpbh_rotate``: rotate back (H / sqrt(B) is its own
    inverse), undo the signs, scatter the columns back to their places."""
    y = np.asarray(y, dtype=np.float64)
    v = rotate(y, block) * sign_vector(signs)[None, :]
    x = np.empty_like(v)
    x[:, np.asarray(perm, dtype=np.int64)] = v
    return x


def sphere_marginal_cdf(t, d: int) -> np.ndarray:
    """P(T <= t) for one coordinate T of a uniform unit vector in R^d (d >= 2):
    1/2 + sign(t) / 2 * I_(t^2)(1/2, (d - 1) / 2), I the regularized
    incomplete beta function (the integral of (1 - t^2)^((d-3)/2) from 0 to x
    is B(x^2; 1/2, (d - 1)/2) / 2 after t^2 = w)."""
    from scipy.special import betainc
    t = np.clip(np.asarray(t, dtype=np.float64), -1.0, 1.0)
    return 0.5 + 0.5 * np.sign(t) * betainc(0.5, (d - 1) / 2.0, t * t)


def sphere_partial_first_moment(a, b, d: int) -> np.ndarray:
    """The integral of t f_d(t) over [a, b]: with k = (d - 3) / 2 the
    antiderivative of t (1 - t^2)^k is -(1 - t^2)^(k + 1) / (2 (k + 1))."""
    from scipy.special import betaln
    a = np.clip(np.asarray(a, dtype=np.float64), -1.0, 1.0)
    b = np.clip(np.asarray(b, dtype=np.float64), -1.0, 1.0)
    e = (d - 1) / 2.0
    norm = np.exp(betaln(0.5, e))

    def g(t):                      # (1 - t^2)^e, 0 at t = +/-1
        if e == 0:
            return np.ones_like(t)
        with np.errstate(divide="ignore"):
            return np.exp(e * np.log1p(-np.minimum(t * t, 1.0)))
    return (g(a) - g(b)) / ((d - 1) * norm)


@functools.lru_cache(maxsize=16)
def sphere_lloyd_max(d: int, bits: int, tol: float = 1e-13, max_iter: int = 200000):
    """Lloyd-Max codebook of the unit-sphere marginal f_d: ``(centroids,
    thresholds)`` with 2^bits centroids (ascending) and 2^bits - 1 thresholds.

    Lloyd's iteration, in the order of its definition: thresholds are the
    midpoints of adjacent centroids; each centroid is the conditional mean of
    T over its cell, from the exact CDF and first moment above.  Starts from
    the quantiles of the cell mid-probabilities; stops when no centroid moves
    by more than ``tol`` times the largest centroid.
    """
    from scipy.special import betaincinv
    d, bits = int(d), int(bits)
    if d < 2 or bits < 1:
        raise ValueError("need d >= 2 and bits >= 1")
    levels = 1 << bits
    p = (np.arange(levels) + 0.5) / levels
    q = betaincinv(0.5, (d - 1) / 2.0, np.abs(2 * p - 1))
    c = np.sign(p - 0.5) * np.sqrt(q)
    for _ in range(max_iter):
        t = 0.5 * (c[:-1] + c[1:])
        lo = np.concatenate([[-1.0], t])
        hi = np.concatenate([t, [1.0]])
        mass = sphere_marginal_cdf(hi, d) - sphere_marginal_cdf(lo, d)
        c_new = sphere_partial_first_moment(lo, hi, d) / mass
        moved = np.abs(c_new - c).max()
        c = c_new
        if moved <= tol * np.abs(c).max():
            break
    t = 0.5 * (c[:-1] + c[1:])
    c.setflags(write=False)
    t.setflags(write=False)
    return c, t


def quantize_codebook(y, centroids, thresholds):
    """Per-token norm, normalized values, nearest centroid.

    For every row: r = ||y||_2; u = y / r; code = number of thresholds
    strictly below u (the index of the nearest centroid; thresholds are the
    midpoints); r = 0 gives codes of u = 0.  Returns ``(codes uint8 (rows, n),
    norms float64 (rows,))``; dequantization is r * centroids[code].
    """
    y = np.asarray(y, dtype=np.float64)
    r = np.sqrt((y * y).sum(axis=1))
    u = y / np.where(r > 0, r, 1.0)[:, None]
    codes = np.searchsorted(np.asarray(thresholds, dtype=np.float64), u, side="left")
    return codes.astype(np.uint8), r


def pack_codes(codes, bits: int) -> np.ndarray:
    """8 // bits codes per byte, code i of a byte in bits [i * bits, (i + 1) * bits)."""
    c = np.asarray(codes).astype(np.int64)
    per = 8 // bits
    if c.shape[-1] % per:
        raise ValueError(f"row length must be a multiple of {per}")
    c = c.reshape(*c.shape[:-1], c.shape[-1] // per, per)
    return (c << (bits * np.arange(per))).sum(axis=-1).astype(np.uint8)
