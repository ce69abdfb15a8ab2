"""Pins of the float64 oracle to facts the pages or the mathematics fix.

Each test pins one function to something other than itself: hand-worked
fixtures (tests/golden/, each citing its passage), closed forms, an
independent library routine, an independent algorithm, or an invariant the
pages state.  A dropped normalisation, a wrong sign or index, a transposed
block, a wrong tie rule or nibble order each fails at least one of them.
"""

import struct

import numpy as np
import pytest
import scipy.linalg
import torch

import oracle
from tests.conftest import load_golden

SIZES = [2 ** k for k in range(0, 14)]   # 1 .. 8192, every size the path uses


# ----------------------------------------------------------------- Hadamard

def test_sylvester_matches_handwritten():
    g = load_golden("sylvester_small.json")
    for k in ("H1", "H2", "H4", "H8"):
        want = np.array(g[k], dtype=np.float64)
        np.testing.assert_array_equal(oracle.sylvester_hadamard(want.shape[0]), want)


@pytest.mark.parametrize("size", [s for s in SIZES if s <= 4096])
def test_sylvester_matches_scipy(size):
    # scipy.linalg.hadamard is an independent Sylvester construction (natural order).
    np.testing.assert_array_equal(oracle.sylvester_hadamard(size), scipy.linalg.hadamard(size))


def _popcount(a):
    c = np.zeros_like(a)
    while np.any(a):
        c += a & 1
        a = a >> 1
    return c


@pytest.mark.parametrize("size", SIZES)
def test_sylvester_closed_form(size):
    """H[i, j] = (-1)^popcount(i & j): full check up to 1024, sampled above."""
    h = oracle.sylvester_hadamard(size)
    rng = np.random.default_rng(size)
    if size <= 1024:
        i, j = np.meshgrid(np.arange(size), np.arange(size), indexing="ij")
    else:
        i = rng.integers(0, size, 200_000)
        j = rng.integers(0, size, 200_000)
    want = np.where(_popcount(i & j) % 2 == 0, 1.0, -1.0)
    np.testing.assert_array_equal(h[i, j], want)


@pytest.mark.parametrize("size", SIZES)
def test_hadamard_orthogonal(size):
    """H . H^T = size . I (full product up to 1024; sampled row pairs above)."""
    h = oracle.sylvester_hadamard(size)
    if size <= 1024:
        np.testing.assert_array_equal(h @ h.T, size * np.eye(size))
    else:
        rng = np.random.default_rng(size + 1)
        a = rng.integers(0, size, 64)
        b = (a + rng.integers(1, size, 64)) % size
        np.testing.assert_array_equal(np.einsum("ij,ij->i", h[a], h[b]), 0.0)
        np.testing.assert_array_equal(np.einsum("ij,ij->i", h[a], h[a]), float(size))


# ----------------------------------------------------------------- rotation

def test_rotate_hand_cases():
    g = load_golden("rotation_hand_cases.json")
    for c in g["cases"]:
        x = np.array([c["x"]], dtype=np.float64)
        want = np.array([c["y_times_sqrt_b"]], dtype=np.float64) / np.sqrt(c["b"])
        np.testing.assert_allclose(oracle.rotate(x, c["block"]), want, rtol=0, atol=1e-14)


@pytest.mark.parametrize("n", [s for s in SIZES if s >= 2])
def test_rotate_basis_vectors(n):
    """e0 -> (1/sqrt n) * ones and ones -> sqrt(n) * e0 (closed forms of H_n / sqrt(n))."""
    e0 = np.zeros((1, n))
    e0[0, 0] = 1.0
    np.testing.assert_allclose(oracle.rotate(e0), np.full((1, n), 1 / np.sqrt(n)), rtol=1e-15, atol=0)
    ones = np.ones((1, n))
    want = np.zeros((1, n))
    want[0, 0] = np.sqrt(n)
    np.testing.assert_allclose(oracle.rotate(ones), want, rtol=0, atol=1e-12 * np.sqrt(n))


@pytest.mark.parametrize("n,block", [(1024, 0), (4096, 0), (8192, 0), (14336, 128), (4096, 32), (512, 16)])
def test_rotate_norm_and_involution(n, block):
    """Orthogonality: norms preserved; H/sqrt(b) is its own inverse."""
    rng = np.random.default_rng(n + block)
    x = rng.standard_normal((8, n)) * rng.uniform(0.1, 30.0, (8, 1))
    y = oracle.rotate(x, block)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oracle.rotate(y, block), x, rtol=0, atol=1e-12 * np.abs(x).max())


@pytest.mark.parametrize("n,block", [(256, 0), (1024, 0), (1024, 128), (896, 128)])
def test_rotated_activations_meet_rotated_weights(n, block):
    """x @ R @ R^T @ W^T = x @ W^T ("Rotation Transform", introduction): the
    online-rotated activation against an offline-rotated weight (W R) gives the
    unrotated layer output."""
    rng = np.random.default_rng(7 + n)
    x = rng.standard_normal((16, n))
    w = rng.standard_normal((24, n))
    xr = oracle.rotate(x, block)
    wr = oracle.rotate(w, block)
    np.testing.assert_allclose(xr @ wr.T, x @ w.T, rtol=0, atol=1e-10 * np.sqrt(n) * 10)


def test_r3_attention_logits_unchanged():
    """R3 rotates Q and K per head with the same head_dim Hadamard, so the
    logits q k^T are unchanged ("Rotation Transform" section 1.1 R3; the
    apply_spinquant docstring: rotated K enters the cache)."""
    rng = np.random.default_rng(3)
    q = rng.standard_normal((64, 128))
    k = rng.standard_normal((80, 128))
    np.testing.assert_allclose(oracle.rotate(q) @ oracle.rotate(k).T, q @ k.T, atol=1e-11)


@pytest.mark.parametrize("n,block", [(1024, 128), (14336, 128), (4096, 1024), (256, 16)])
def test_block_mode_is_per_block_full_transform(n, block):
    rng = np.random.default_rng(11)
    x = rng.standard_normal((5, n))
    y = oracle.rotate(x, block)
    for j in range(n // block):
        sl = slice(j * block, (j + 1) * block)
        np.testing.assert_allclose(y[:, sl], oracle.rotate(x[:, sl], 0), rtol=0, atol=1e-12)


def _fwht_butterflies(x):
    """Independent fast Walsh-Hadamard transform (iterative butterflies), unnormalised."""
    a = np.array(x, dtype=np.float64, copy=True)
    n = a.shape[-1]
    h = 1
    while h < n:
        a = a.reshape(*a.shape[:-1], n // (2 * h), 2, h)
        u = a[..., 0, :].copy()
        v = a[..., 1, :].copy()
        a[..., 0, :] = u + v
        a[..., 1, :] = u - v
        a = a.reshape(*a.shape[:-3], n)
        h *= 2
    return a


@pytest.mark.parametrize("n", [2, 8, 128, 1024, 4096, 8192])
def test_dense_rotation_equals_fast_transform(n):
    rng = np.random.default_rng(n)
    x = rng.standard_normal((4, n))
    want = _fwht_butterflies(x) / np.sqrt(n)
    np.testing.assert_allclose(oracle.rotate(x), want, rtol=0, atol=1e-12 * np.sqrt(n))


def test_block_argument_forms():
    x = np.arange(16, dtype=np.float64)[None]
    full = oracle.rotate(x, 16)
    for b in (0, -1, None):
        np.testing.assert_array_equal(oracle.rotate(x, b), full)
    for bad in (3, 12, 32):
        with pytest.raises(ValueError):
            oracle.rotate(x, bad)
    for n in (10, 44, 6):                     # full sizes with no Hadamard matrix here
        with pytest.raises(ValueError):
            oracle.rotate(np.zeros((1, n)), 0)
    assert oracle.rotate(np.zeros((1, 12)), 0).shape == (1, 12)   # K = 12 is covered


# -------------------------------------------- non-power-of-2 sizes K * 2^m

def test_paley_k12_matches_hand_worked_fixture(golden):
    g = golden("paley_k12.json")
    chi = oracle.quadratic_character(5, 1)
    assert sorted(np.nonzero(chi == 1)[0].tolist()) == g["squares_mod_5"]
    np.testing.assert_array_equal(oracle.jacobsthal(5, 1), np.array(g["Q5"]))
    h = oracle.paley_hadamard(12)
    np.testing.assert_array_equal(h[:4], np.array(g["H12_rows_0_to_3"], dtype=np.float64))
    # every entry from the conference matrix written out by hand
    c, a, b = np.array(g["C6"]), np.array([[1, 1], [1, -1]]), np.array([[1, -1], [-1, -1]])
    for i in range(6):
        for j in range(6):
            for u in range(2):
                for v in range(2):
                    want = c[i, j] * a[u, v] + (b[u, v] if i == j else 0)
                    assert h[2 * i + u, 2 * j + v] == want


def test_field_squares_match_hand_worked_sets(golden):
    g = golden("paley_k12.json")
    assert sorted(np.nonzero(oracle.quadratic_character(3, 2) == 1)[0].tolist()) == g["squares_GF9"]
    assert sorted(np.nonzero(oracle.quadratic_character(13, 1) == 1)[0].tolist()) == g["squares_mod_13"]
    for k, (p, e) in oracle.PALEY_FIELDS.items():
        chi = oracle.quadratic_character(p, e)
        q = p ** e
        assert chi[0] == 0 and (chi == 1).sum() == (q - 1) // 2 and (chi == -1).sum() == (q - 1) // 2
        # the squares of a prime field are exactly {t^2 mod p}
        if e == 1:
            assert set(np.nonzero(chi == 1)[0].tolist()) == {t * t % p for t in range(1, p)}


@pytest.mark.parametrize("k", sorted(oracle.PALEY_FIELDS))
def test_paley_base_matrices_are_symmetric_hadamard(k):
    h = oracle.paley_hadamard(k)
    assert h.shape == (k, k) and set(np.unique(h).tolist()) == {-1.0, 1.0}
    np.testing.assert_array_equal(h @ h.T, k * np.eye(k))
    np.testing.assert_array_equal(h, h.T)
    # the Jacobsthal matrix of q = 1 (mod 4) is symmetric with zero diagonal and Q Q^T = q I - J
    p, e = oracle.PALEY_FIELDS[k]
    q = p ** e
    jq = oracle.jacobsthal(p, e)
    np.testing.assert_array_equal(jq, jq.T)
    np.testing.assert_array_equal(jq @ jq.T, q * np.eye(q) - np.ones((q, q)))


@pytest.mark.parametrize("n", [12, 24, 48 * 8, 20 * 16, 28 * 32, 36 * 8, 52 * 4, 60 * 4, 108 * 2, 28 * 64])
def test_k_size_rotation_is_orthogonal_and_involutory(n):
    k, s = oracle.split_size(n)
    assert k * s == n and k in oracle.PALEY_FIELDS
    h = oracle.hadamard_matrix(n)
    np.testing.assert_array_equal(h @ h.T, n * np.eye(n))
    x = np.random.default_rng(n).standard_normal((5, n))
    y = oracle.rotate(x, 0)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oracle.rotate(y, 0), x, rtol=0, atol=1e-12 * np.abs(x).max())


@pytest.mark.parametrize("n", [12 * 16, 28 * 64, 20 * 8])
def test_k_size_rotation_equals_two_stage_product(n):
    """Kronecker index convention: element e = k * 2^m + j; the dense product
    equals mixing the K sub-blocks by H_K after (or before) a 2^m-point
    butterfly inside each sub-block, computed here with an independent FWHT."""
    k, s = oracle.split_size(n)
    x = np.random.default_rng(n + 1).standard_normal((3, n))
    z = _fwht_butterflies(x.reshape(3 * k, s)).reshape(3, k, s)
    want = np.einsum("rkj,kl->rlj", z, oracle.paley_hadamard(k)).reshape(3, n) / np.sqrt(n)
    np.testing.assert_allclose(oracle.rotate(x, 0), want, rtol=0, atol=1e-12 * np.sqrt(n) * np.abs(x).max())


def test_k_size_blocks_are_per_block_full_transforms():
    x = np.random.default_rng(5).standard_normal((4, 28 * 32 * 3))
    y = oracle.rotate(x, 28 * 32)
    for j in range(3):
        sl = slice(j * 896, (j + 1) * 896)
        np.testing.assert_allclose(y[:, sl], oracle.rotate(x[:, sl], 0), rtol=0, atol=1e-12)


# ----------------------------------------------------------- float formats

def _interesting_values(rng):
    base = np.concatenate([
        rng.standard_normal(4000) * np.exp(rng.uniform(-25, 12, 4000)),
        np.ldexp(1.0, np.arange(-30, 17)),
    ])
    return base


def test_fp16_rounding_matches_numpy_and_struct():
    rng = np.random.default_rng(0)
    v = _interesting_values(rng)
    v = v[np.abs(v) < 65504]
    # exact fp16 midpoints (ties) and their neighbours
    grid = np.array([1.0, 1.5, 0.142822265625, 1024.0, 2.0 ** -14, 2.0 ** -20])
    ulps = np.ldexp(1.0, np.maximum(np.frexp(grid)[1] - 1, -14) - 10)
    mids = np.concatenate([grid + ulps / 2, grid + 1.5 * ulps])
    v = np.concatenate([v, mids, -mids])
    got = oracle.to_fp16(v)
    np.testing.assert_array_equal(got, v.astype(np.float16).astype(np.float64))
    for a, b in zip(v[::37], got[::37]):
        assert struct.unpack("<e", struct.pack("<e", a))[0] == b
    assert np.isinf(oracle.to_fp16(np.array([65520.0]))[0])
    assert oracle.to_fp16(np.array([65519.0]))[0] == 65504.0


def test_fp32_rounding_matches_numpy_and_struct():
    rng = np.random.default_rng(1)
    v = _interesting_values(rng)
    got = oracle.to_fp32(v)
    np.testing.assert_array_equal(got, v.astype(np.float32).astype(np.float64))
    for a, b in zip(v[::41], got[::41]):
        assert struct.unpack("<f", struct.pack("<f", a))[0] == b


def test_bf16_bits_match_torch():
    rng = np.random.default_rng(2)
    v = _interesting_values(rng).astype(np.float32).astype(np.float64)   # fp32-exact inputs
    ties = (np.array([1.0, -3.0, 0.5]) * (1 + 2.0 ** -8)).astype(np.float64)
    v = np.concatenate([v, ties])
    want = torch.from_numpy(v.astype(np.float32)).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(oracle.to_bf16_bits(v), want)


def test_fp16_midpoint_distance():
    mid = 1.0 + 2.0 ** -11          # exact midpoint between 1 and 1 + 2^-10
    rel, alt = oracle.fp16_scale_midpoint_distance(np.array([mid * (1 + 1e-9), mid * (1 - 1e-9), 1.3]))
    assert rel[0] < 1e-8 and rel[1] < 1e-8 and rel[2] > 1e-4
    assert alt[0] == 1.0 and alt[1] == 1.0 + 2.0 ** -10     # the neighbour not taken by RNE


# -------------------------------------------------------------- quantizers

def test_int4_hand_cases():
    for c in load_golden("rtn_cases.json")["int4"]:
        y = np.array([c["y"]])
        q, s = oracle.quantize_int4_sym(y, c["group"])
        np.testing.assert_array_equal(q[0], c["codes"])
        np.testing.assert_array_equal(s[0].astype(np.float64), c["scales"])
        np.testing.assert_array_equal(oracle.pack_nibbles(q)[0], c["packed"])


def test_int8_hand_cases():
    for c in load_golden("rtn_cases.json")["int8"]:
        q, s = oracle.quantize_int8_per_token(np.array([c["y"]]))
        np.testing.assert_array_equal(q[0], c["codes"])
        assert float(s[0]) == c["scale"]


@pytest.mark.parametrize("group", [32, 64, 128])
def test_int4_rtn_properties(group):
    rng = np.random.default_rng(group)
    y = rng.standard_normal((64, 1024)) * rng.uniform(1e-3, 1e3, (64, 1))
    q, s = oracle.quantize_int4_sym(y, group)
    g = y.reshape(64, -1, group)
    qg = q.reshape(64, -1, group).astype(np.float64)
    s64 = s.astype(np.float64)[..., None]
    assert q.min() >= -7 and q.max() <= 7
    # reconstruction error at most half a step for unclipped elements
    err = np.abs(g - qg * s64)
    assert np.all(err <= s64 / 2 * (1 + 1e-12))
    # the group's absmax element maps to +/-7
    idx = np.abs(g).argmax(axis=-1)
    top = np.take_along_axis(qg, idx[..., None], -1)[..., 0]
    np.testing.assert_array_equal(np.abs(top), 7)
    # the scale is the fp16 rounding of absmax / 7 (within half an fp16 ulp)
    m = np.abs(g).max(-1)
    assert np.all(np.abs(s64[..., 0] - m / 7) <= np.ldexp(1.0, np.frexp(m / 7)[1] - 1 - 11) * (1 + 1e-12))


def test_int8_rtn_properties():
    rng = np.random.default_rng(5)
    y = rng.standard_normal((32, 14336)) * rng.uniform(1e-2, 1e2, (32, 1))
    q, s = oracle.quantize_int8_per_token(y)
    s64 = s.astype(np.float64)[:, None]
    assert q.min() >= -127 and q.max() <= 127
    assert np.all(np.abs(y - q * s64) <= s64 / 2 * (1 + 1e-9))
    np.testing.assert_array_equal(np.abs(q[np.arange(32), np.abs(y).argmax(1)]), 127)


def test_zero_and_nonfinite_scales_give_zero_codes():
    assert np.all(oracle.codes_with_scale(np.array([1.0, -2.0]), np.array([0.0]), 7) == 0)
    assert np.all(oracle.codes_with_scale(np.array([1.0, -2.0]), np.array([np.inf]), 7) == 0)
    # absmax / 7 beyond fp16 range -> infinite scale -> zero codes
    q, s = oracle.quantize_int4_sym(np.full((1, 32), 1e6), 32)
    assert np.isinf(s[0, 0]) and np.all(q == 0)
    # tiny absmax -> subnormal fp16 scale -> codes clamp to +/-7
    q, s = oracle.quantize_int4_sym(np.array([[5e-7] + [0.0] * 31]), 32)
    assert 0 < float(s[0, 0]) < 6.2e-5 and q[0, 0] == 7


def test_e2m1_table_and_ties():
    g = load_golden("mxfp4_cases.json")
    dec = np.array(g["e2m1_decode"])
    # every code decodes to a grid value that encodes back to itself (except -0 -> +0)
    for code, val in enumerate(dec):
        got = int(oracle.e2m1_encode(np.array([val]))[0])
        assert got == (0 if code == 8 else code)
    for v, want in g["encode_cases"]:
        assert int(oracle.e2m1_encode(np.array([v]))[0]) == want, v


def test_e2m1_nearest_even_property():
    """On a dense grid: the code decodes to a nearest E2M1 magnitude (6 above
    the top), and at an exact tie the chosen code index is even."""
    dec = np.array(load_golden("mxfp4_cases.json")["e2m1_decode"])
    v = np.concatenate([np.linspace(-8, 8, 64001), np.array([0.25, 0.75, 1.25, 1.75, 2.5, 3.5, 5.0])])
    c = oracle.e2m1_encode(v).astype(np.int64)
    got = np.abs(dec[c])
    dist = np.abs(np.abs(v)[:, None] - np.abs(dec[:8])[None, :])
    best = dist.min(1)
    assert np.all(np.abs(np.abs(v) - got) == best)
    tie = (dist == best[:, None]).sum(1) == 2
    assert np.all((c[tie] & 7) % 2 == 0)
    assert np.all((c >> 3)[v < 0] == 1) and np.all((c >> 3)[v >= 0] == 0)


def test_e8m0_cases_and_bracket():
    g = load_golden("mxfp4_cases.json")
    for m, byte in g["e8m0_cases"]:
        assert int(oracle.e8m0_exponent(np.array([m]))[0]) + 127 == byte, m
    rng = np.random.default_rng(9)
    m = np.exp(rng.uniform(-60, 60, 10000))
    e = oracle.e8m0_exponent(m).astype(np.float64)
    assert np.all((2.0 ** (e + 2) <= m) & (m < 2.0 ** (e + 3)))


def test_mxfp4_block_case():
    c = load_golden("mxfp4_cases.json")["block_case"]
    q, s = oracle.quantize_mxfp4(np.array([c["y"]]))
    assert int(s[0, 0]) == c["scale_byte"]
    np.testing.assert_array_equal(q[0], c["codes"])
    np.testing.assert_array_equal(oracle.pack_nibbles(q)[0], c["packed"])


def test_mxfp4_dequant_error_bound():
    """Every unsaturated element is within half an E2M1 step of its value."""
    rng = np.random.default_rng(12)
    y = rng.standard_t(3, (16, 8192))
    q, s = oracle.quantize_mxfp4(y)
    dec = np.array(load_golden("mxfp4_cases.json")["e2m1_decode"])
    e = s.astype(np.int64) - 127
    deq = dec[q.astype(np.int64)].reshape(16, -1, 32) * np.ldexp(1.0, e)[..., None]
    v = np.abs(y.reshape(16, -1, 32)) / np.ldexp(1.0, e)[..., None]
    step = np.select([v < 2, v < 4], [0.5, 1.0], 2.0) * np.ldexp(1.0, e)[..., None]
    unsat = v <= 6
    assert np.all(np.abs(deq - y.reshape(16, -1, 32))[unsat] <= (step / 2)[unsat] * (1 + 1e-12))


def test_rotate_quant_dispatch():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((3, 256))
    y, c, s = oracle.rotate_quant(x, 0, "int4", 128)
    assert c.shape == (3, 128) and c.dtype == np.uint8 and s.shape == (3, 2) and s.dtype == np.float16
    y, c, s = oracle.rotate_quant(x, 128, "int8", 0)
    assert c.shape == (3, 256) and c.dtype == np.int8 and s.shape == (3,) and s.dtype == np.float32
    y, c, s = oracle.rotate_quant(x, 64, "mxfp4", 32)
    assert c.shape == (3, 128) and s.shape == (3, 8) and s.dtype == np.uint8
    with pytest.raises(ValueError):
        oracle.rotate_quant(x, 0, "int8", 64)


# ------------------------------------------------- incoherence (diagnostic)

def test_rotation_flattens_outliers():
    """QuIP note, "Incoherence, and the rotation that manufactures it": a
    rotation takes an outlier-planted matrix's mu down towards the Gaussian
    floor sqrt(2 ln(mn)).  The deterministic Hadamard does the same to rows
    with outlier channels (the C2-like input)."""
    rng = np.random.default_rng(0)
    x = rng.standard_normal((64, 64))
    x[:, [3, 17]] *= 25.0

    def mu(a):
        return np.abs(a).max() / np.sqrt((a ** 2).mean())
    before, after = mu(x), mu(oracle.rotate(x))
    assert before > 10 and after < 0.5 * before
    assert after < 1.5 * np.sqrt(2 * np.log(64 * 64))


# ------------------------------------------------- random Hadamard (signs)

def test_random_hadamard_hand_cases():
    """Hand-summed cases of both sign sides, full and block-diagonal."""
    gold = load_golden("random_hadamard_cases.json")
    assert "section 1.5" in gold["citation"]
    for c in gold["cases"]:
        x = np.array([c["x"]], dtype=np.float64)
        y = oracle.rotate_signed(x, c["block"], np.array(c["signs"], dtype=np.int8), c["side"])
        np.testing.assert_allclose(y[0] * np.sqrt(c["b"]), c["y_times_sqrt_b"], rtol=0, atol=1e-12)


def _rademacher(b, seed):
    return np.where(np.random.default_rng(seed).random(b) < 0.5, -1, 1).astype(np.int8)


@pytest.mark.parametrize("b", [2, 16, 128, 1024])
def test_random_hadamard_matrix_definition(b):
    """H @ diag(s): column j of the Sylvester matrix times s_j; the transpose
    puts s_j on row j.  Checked entry by entry against the closed form
    (-1)^popcount(i & j) s_j, and the stored int8 matrix's first row is s."""
    s = _rademacher(b, b)
    i, j = np.meshgrid(np.arange(b), np.arange(b), indexing="ij")
    pop = np.vectorize(lambda v: bin(int(v)).count("1"))(i & j)
    closed = np.where(pop % 2 == 0, 1.0, -1.0)
    after = oracle.random_hadamard_matrix(s, "after") * np.sqrt(b)
    before = oracle.random_hadamard_matrix(s, "before") * np.sqrt(b)
    np.testing.assert_array_equal(after, closed * s[None, :])
    np.testing.assert_array_equal(before, closed * s[:, None])
    np.testing.assert_array_equal(after[0], s)          # first row of the persisted +/-1 matrix
    np.testing.assert_array_equal(before, after.T)
    if b <= 128:                                         # the literal products with diag(s)
        np.testing.assert_array_equal(after, oracle.sylvester_hadamard(b) @ np.diag(s.astype(np.float64)))
        np.testing.assert_array_equal(before, np.diag(s.astype(np.float64)) @ oracle.sylvester_hadamard(b))


@pytest.mark.parametrize("b", [2, 8, 256, 2048])
def test_random_hadamard_orthogonal_and_inverse(b):
    s = _rademacher(b, 7 + b)
    r = oracle.random_hadamard_matrix(s, "after")
    np.testing.assert_allclose(r @ r.T, np.eye(b), rtol=0, atol=1e-12)
    x = np.random.default_rng(b).standard_normal((3, 4 * b))
    y = oracle.rotate_signed(x, b, s, "after")
    np.testing.assert_allclose(oracle.rotate_signed(y, b, s, "before"), x, rtol=0, atol=1e-12 * np.sqrt(b))
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)


@pytest.mark.parametrize("n,block", [(64, 0), (256, 32), (4096, 0)])
def test_random_hadamard_all_plus_is_deterministic(n, block):
    x = np.random.default_rng(n).standard_normal((5, n))
    b = oracle.resolve_block(n, block)
    ones = np.ones(b, dtype=np.int8)
    for side in ("after", "before"):
        np.testing.assert_allclose(oracle.rotate_signed(x, block, ones, side), oracle.rotate(x, block),
                                   rtol=0, atol=1e-12 * np.sqrt(b))
    # any non-negative int8 is +1, any negative int8 is -1
    np.testing.assert_array_equal(oracle.sign_vector(np.array([0, 1, 127, -1, -128], np.int8)),
                                  [1.0, 1.0, 1.0, -1.0, -1.0])


@pytest.mark.parametrize("n,block", [(128, 0), (1024, 128), (4096, 0)])
def test_random_hadamard_equals_signs_around_fast_transform(n, block):
    """Independent route: butterflies, then the column signs (after), or the
    signs, then butterflies (before)."""
    b = oracle.resolve_block(n, block)
    s = _rademacher(b, n + 3).astype(np.float64)
    x = np.random.default_rng(n + 1).standard_normal((3, n))
    xb = x.reshape(-1, b)
    after = (_fwht_butterflies(xb) * s / np.sqrt(b)).reshape(3, n)
    before = (_fwht_butterflies(xb * s) / np.sqrt(b)).reshape(3, n)
    si = s.astype(np.int8)
    np.testing.assert_allclose(oracle.rotate_signed(x, block, si, "after"), after, rtol=0, atol=1e-12 * np.sqrt(b))
    np.testing.assert_allclose(oracle.rotate_signed(x, block, si, "before"), before, rtol=0, atol=1e-12 * np.sqrt(b))


def test_random_hadamard_quantized_codes_follow_the_signs():
    """Symmetric RTN is odd (q(-v) = -q(v)) and the absmax ignores signs, so
    the signed-after int4 / int8 codes are the deterministic codes negated in
    the negative columns, with the same scales; MXFP4 keeps the exponents
    and flips the sign bit of the code of every nonzero value there (also
    where the magnitude rounds to 0: the sign bit follows the value)."""
    n = 256
    x = np.random.default_rng(11).standard_normal((6, n))
    s = _rademacher(n, 5)
    neg = s < 0
    for fmt, group in (("int4", 128), ("int4", 32), ("int8", 0), ("mxfp4", 32)):
        y0, c0, s0 = oracle.rotate_quant(x, 0, fmt, group)
        _, c1, s1 = oracle.rotate_quant_signed(x, 0, s, "after", fmt, group)
        np.testing.assert_array_equal(s0, s1)
        if fmt == "int8":
            np.testing.assert_array_equal(c1, np.where(neg, -c0, c0))
            continue
        lo0, hi0 = (c0 & 0xF).astype(np.int64), (c0 >> 4).astype(np.int64)
        q0 = np.stack([lo0, hi0], axis=-1).reshape(6, n)
        lo1, hi1 = (c1 & 0xF).astype(np.int64), (c1 >> 4).astype(np.int64)
        q1 = np.stack([lo1, hi1], axis=-1).reshape(6, n)
        if fmt == "int4":
            v0 = np.where(q0 >= 8, q0 - 16, q0)
            v1 = np.where(q1 >= 8, q1 - 16, q1)
            np.testing.assert_array_equal(v1, np.where(neg, -v0, v0))
        else:
            flip = neg & (y0 != 0)
            np.testing.assert_array_equal(q1, np.where(flip, q0 ^ 8, q0))
    with pytest.raises(ValueError):
        oracle.rotate_signed(x, 0, s[:128], "after")
    with pytest.raises(ValueError):
        oracle.rotate_signed(x, 0, s, "sideways")


# ------------------------------------------------------------------ NVFP4

def test_nvfp4_hand_cases():
    gold = load_golden("nvfp4_cases.json")
    assert "section 2.1" in gold["citation"]
    for c in gold["cases"]:
        q, s = oracle.quantize_nvfp4(np.array([c["y"]], dtype=np.float64), c["tensor_scale"])
        np.testing.assert_array_equal(q[0], c["codes"])
        assert int(s[0, 0]) == c["scale_byte"]
        assert float(oracle.to_e4m3(np.max(np.abs(c["y"])) / c["tensor_scale"] / 6.0)) == c["scale"]
    e = gold["e4m3"]
    np.testing.assert_array_equal(oracle.e4m3_encode(np.array(e["values"])), e["bytes"])


def test_e4m3_matches_torch_float8_in_range():
    """Inside the finite range the rounding and the byte layout are torch's
    float8_e4m3fn conversion (round half to even); every grid point and every
    midpoint between neighbours is included."""
    grid = torch.arange(0, 127, dtype=torch.uint8).view(torch.float8_e4m3fn).float().double().numpy()
    mids = (grid[1:] + grid[:-1]) / 2
    rng = np.random.default_rng(3)
    vals = np.concatenate([grid, mids, rng.uniform(0, 448, 4000), np.exp(rng.uniform(-12, 6, 4000))])
    vals = vals[vals <= 448]
    vals = np.concatenate([vals, -vals])
    want = torch.tensor(vals).to(torch.float8_e4m3fn)
    np.testing.assert_array_equal(oracle.to_e4m3(vals), want.double().numpy())
    got = oracle.e4m3_encode(vals)
    nz = oracle.to_e4m3(vals) != 0
    np.testing.assert_array_equal(got[nz], want.view(torch.uint8).numpy()[nz])
    assert (got[~nz] == 0).all()                      # a zero scale is byte 0 (no negative zero)


def test_e4m3_saturates_at_448():
    v = np.array([448.0, 449.0, 464.0, 465.0, 1e6, -1e6])
    np.testing.assert_array_equal(oracle.to_e4m3(v), [448, 448, 448, 448, 448, -448])
    np.testing.assert_array_equal(oracle.e4m3_encode(v), [126, 126, 126, 126, 126, 254])


def test_nvfp4_properties():
    rng = np.random.default_rng(12)
    y = rng.standard_t(3, (32, 256)) * np.exp(rng.uniform(-4, 4, (32, 1)))
    q, sb = oracle.quantize_nvfp4(y)
    g = y.reshape(32, 16, 16)
    s = oracle.to_e4m3(np.abs(g).max(axis=-1) / 6.0)
    np.testing.assert_array_equal(sb, oracle.e4m3_encode(s))
    qv = oracle.E2M1_GRID[q.reshape(32, 16, 16) & 7] * np.where(q.reshape(32, 16, 16) & 8, -1.0, 1.0)
    v = g / s[..., None]
    # nearest grid value (or 6 when saturated)
    err = np.abs(v - qv)
    step = np.select([np.abs(v) < 2, np.abs(v) < 4], [0.5, 1.0], 2.0)
    unsat = np.abs(v) <= 6
    assert np.all(err[unsat] <= step[unsat] / 2 + 1e-12)
    assert np.all(np.abs(qv[~unsat]) == 6)
    # the per-tensor scale only rescales: quantize(y * t, t) == quantize(y, 1)
    for t in (0.5, 3.0, 2.0 ** -7):
        q2, s2 = oracle.quantize_nvfp4(y * t, t)
        np.testing.assert_array_equal(q2, q)
        np.testing.assert_array_equal(s2, sb)
    with pytest.raises(ValueError):
        oracle.quantize_nvfp4(y, 0.0)
    y0, c, sc = oracle.rotate_quant(rng.standard_normal((3, 64)), 0, "nvfp4", 16)
    assert c.shape == (3, 32) and sc.shape == (3, 4) and sc.dtype == np.uint8
    with pytest.raises(ValueError):
        oracle.rotate_quant(rng.standard_normal((3, 64)), 0, "nvfp4", 32)


# ------------------------------------------- orbitquant: RPBH and codebooks

def test_rpbh_equals_explicit_permutation_sign_and_hadamard_matrices():
    """RPBH(x) = x P D H_blk / sqrt(B) with P the permutation matrix of pi
    (column e of x P is column pi(e) of x) and D = diag(s)."""
    rng = np.random.default_rng(11)
    n, block = 64, 16
    x = rng.standard_normal((5, n))
    perm = rng.permutation(n)
    signs = np.where(rng.random(n) < 0.5, -1, 1).astype(np.int8)
    p = np.zeros((n, n))
    p[perm, np.arange(n)] = 1.0
    hb = np.kron(np.eye(n // block), oracle.sylvester_hadamard(block)) / np.sqrt(block)
    want = x @ p @ np.diag(signs.astype(np.float64)) @ hb
    np.testing.assert_allclose(oracle.rpbh_rotate(x, block, perm, signs), want, rtol=0, atol=1e-12)
    # identity permutation and all-plus signs: the plain block rotation
    np.testing.assert_allclose(oracle.rpbh_rotate(x, block, np.arange(n), np.ones(n, np.int8)),
                               oracle.rotate(x, block), rtol=0, atol=1e-13)
    y = oracle.rpbh_rotate(x, block, perm, signs)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), np.linalg.norm(x, axis=1), rtol=1e-12)
    np.testing.assert_allclose(oracle.rpbh_inverse(y, block, perm, signs), x, rtol=0, atol=1e-12)
    with pytest.raises(ValueError):
        oracle.rpbh_rotate(x, block, np.zeros(n, np.int64), signs)


def test_sphere_cdf_matches_sampled_unit_vectors():
    """Coordinates of normalized Gaussian vectors (uniform on the sphere)."""
    rng = np.random.default_rng(3)
    for d in (3, 16, 256):
        v = rng.standard_normal((200000, d))
        t = v[:, 0] / np.linalg.norm(v, axis=1)
        for q in (-0.5, -0.1, 0.0, 0.05, 0.3):
            q = q * 3 / np.sqrt(d)
            assert abs((t <= q).mean() - oracle.sphere_marginal_cdf(q, d)) < 4e-3


def test_sphere_first_moment_matches_quadrature():
    from scipy.integrate import quad
    from scipy.special import beta
    for d in (4, 17, 1024):
        f = lambda t, d=d: (1 - t * t) ** ((d - 3) / 2) / beta(0.5, (d - 1) / 2)   # noqa: E731
        for a, b in ((-1.0, -0.2), (-0.05, 0.02), (0.01, 1.0)):
            want, _ = quad(lambda t: t * f(t), a, b, epsabs=1e-14, points=[0.0] if a < 0 < b else None)
            assert abs(oracle.sphere_partial_first_moment(a, b, d) - want) < 1e-10
            mass, _ = quad(f, a, b, epsabs=1e-14)
            got = oracle.sphere_marginal_cdf(b, d) - oracle.sphere_marginal_cdf(a, d)
            assert abs(got - mass) < 1e-10


@pytest.mark.parametrize("bits", [1, 2, 3, 4])
def test_lloyd_max_of_d3_is_the_uniform_quantizer(bits):
    """d = 3: one coordinate of a uniform point on the 2-sphere is uniform on
    [-1, 1] (Archimedes), and the Lloyd-Max quantizer of a uniform density is
    the uniform one: centroids -1 + (2i + 1) / L, thresholds -1 + 2i / L."""
    c, t = oracle.sphere_lloyd_max(3, bits)
    levels = 1 << bits
    np.testing.assert_allclose(c, -1 + (2 * np.arange(levels) + 1) / levels, rtol=0, atol=1e-12)
    np.testing.assert_allclose(t, -1 + 2 * np.arange(1, levels) / levels, rtol=0, atol=1e-12)


@pytest.mark.parametrize("d", [2, 5, 64, 4096])
def test_one_bit_codebook_is_plus_minus_mean_abs(d):
    """Two levels: threshold 0 by symmetry, centroids +/- E|T| with
    E|T| = Gamma(d / 2) / (sqrt(pi) Gamma((d + 1) / 2))."""
    from scipy.special import gammaln
    c, t = oracle.sphere_lloyd_max(d, 1)
    m = np.exp(gammaln(d / 2) - gammaln((d + 1) / 2)) / np.sqrt(np.pi)
    np.testing.assert_allclose(c, [-m, m], rtol=1e-10)
    assert abs(t[0]) < 1e-15


@pytest.mark.parametrize("d,bits", [(8, 2), (128, 3), (4096, 4), (14336, 4), (4096, 2)])
def test_lloyd_max_optimality_conditions(d, bits):
    """Thresholds are the midpoints of adjacent centroids and every centroid
    is the conditional mean of its cell (cell integrals by quadrature)."""
    from scipy.integrate import quad
    from scipy.special import betaln
    c, t = oracle.sphere_lloyd_max(d, bits)
    np.testing.assert_allclose(t, 0.5 * (c[:-1] + c[1:]), rtol=0, atol=1e-15)
    np.testing.assert_allclose(c, -c[::-1], rtol=0, atol=1e-14)
    logb = betaln(0.5, (d - 1) / 2)
    f = lambda v: np.exp(((d - 3) / 2) * np.log1p(-v * v) - logb)   # noqa: E731
    edges = np.concatenate([[-1.0], t, [1.0]])
    s = 12.0 / np.sqrt(d)          # the density is negligible beyond 12 standard deviations
    for i in range(len(c)):
        a, b = max(edges[i], -min(1.0, s)), min(edges[i + 1], min(1.0, s))
        num, _ = quad(lambda v: v * f(v), a, b, epsabs=1e-16, epsrel=1e-12, limit=200)
        den, _ = quad(f, a, b, epsabs=1e-16, epsrel=1e-12, limit=200)
        assert abs(num / den - c[i]) <= 1e-9 * abs(c).max()


def test_lloyd_max_large_d_approaches_the_gaussian_quantizer():
    """sqrt(d) T tends to N(0, 1): the 4-bit codebook times sqrt(d) at
    d = 10^6 matches a Lloyd-Max quantizer of the standard normal computed
    here from the normal's own conditional means."""
    from scipy.stats import norm
    c, _ = oracle.sphere_lloyd_max(10 ** 6, 4)
    g = norm.ppf((np.arange(16) + 0.5) / 16)
    for _ in range(20000):
        t = np.concatenate([[-np.inf], 0.5 * (g[:-1] + g[1:]), [np.inf]])
        g = (norm.pdf(t[:-1]) - norm.pdf(t[1:])) / (norm.cdf(t[1:]) - norm.cdf(t[:-1]))
    np.testing.assert_allclose(c * np.sqrt(10 ** 6), g, rtol=2e-5, atol=2e-5)


def test_codebook_quantizer_hand_case_and_packing():
    """d = 3, 2 bits: centroids -0.75, -0.25, 0.25, 0.75; thresholds -0.5, 0,
    0.5.  Row (3, 0, 4, -4.5) has norm sqrt(45.25); u = (0.446, 0, 0.595,
    -0.669): codes 2 (0.446 in (0, 0.5]), 1 (0 takes the lower side), 3, 0."""
    c, t = oracle.sphere_lloyd_max(3, 2)
    codes, r = oracle.quantize_codebook(np.array([[3.0, 0.0, 4.0, -4.5]]), c, t)
    np.testing.assert_array_equal(codes, [[2, 1, 3, 0]])
    assert r[0] == np.sqrt(45.25)
    assert oracle.pack_codes(codes, 2).tolist() == [[2 | (1 << 2) | (3 << 4) | (0 << 6)]]
    assert oracle.pack_codes(np.array([[5, 12]]), 4).tolist() == [[5 | (12 << 4)]]
    z, rz = oracle.quantize_codebook(np.zeros((1, 4)), c, t)
    assert rz[0] == 0 and (z == 1).all()       # u = 0 sits on the middle threshold
