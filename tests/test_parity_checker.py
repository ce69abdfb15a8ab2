"""The parity checker accepts the oracle's own outputs and rejects planted mistakes.

Mistakes are planted in oracle-computed outputs on the CPU; no GPU involved.
"""

import numpy as np
import pytest

import oracle
from tests import parity_check as pc


def _x(rows, n, seed=0, scale=3.0):
    return np.random.default_rng(seed).standard_normal((rows, n)) * scale


def test_rotation_checks_accept_oracle_and_reject_error():
    x = _x(6, 256)
    y = oracle.rotate(x, 0).astype(np.float32)
    pc.check_rotation_f32(x, y, 0)
    bad = y.copy()
    bad[3, 7] += 1e-3
    with pytest.raises(AssertionError):
        pc.check_rotation_f32(x, bad, 0)
    bits = oracle.to_bf16_bits(oracle.rotate(x, 64))
    pc.check_rotation_bf16(x, bits, 64)
    bits2 = bits.copy()
    bits2[0, 0] += 2          # two bf16 ulps
    with pytest.raises(AssertionError):
        pc.check_rotation_bf16(x, bits2, 64)


@pytest.mark.parametrize("group", [32, 128])
def test_int4_checker(group):
    x = _x(8, 512, 1)
    y, codes, scales = oracle.rotate_quant(x, 0, "int4", group)
    rep = pc.check_int4(x, codes, scales, 0, group)
    assert rep["code_differs_in_window"] == 0
    flipped = codes.copy()
    flipped[2, 5] ^= 0x10     # one nibble off by one
    with pytest.raises(AssertionError):
        pc.check_int4(x, flipped, scales, 0, group)
    s2 = scales.copy()
    s2[1, 0] = np.float16(float(s2[1, 0]) * 1.01)
    with pytest.raises(AssertionError):
        pc.check_int4(x, codes, s2, 0, group)


def test_int4_boundary_code_is_accepted():
    # a group whose element sits exactly on a rounding boundary (k + 0.5 in code units)
    y = np.zeros((1, 32))
    y[0, 0], y[0, 1] = 7.0, 2.5         # scale fp16(1.0) = 1 -> 2.5 is a tie
    x = oracle.rotate(y, 0)              # rotate is an involution: rotate(x) == y
    _, codes, scales = oracle.rotate_quant(x, 0, "int4", 32)
    q = pc.unpack_nibbles(codes, signed=True)
    assert q[0, 1] == 2
    alt = q.copy()
    alt[0, 1] = 3                        # the other side of the tie
    packed = oracle.pack_nibbles(alt)
    rep = pc.check_int4(x, packed, scales, 0, 32)
    assert rep["code_boundary_cases"] >= 1 and rep["code_differs_in_window"] == 1
    alt[0, 1] = 4                        # two codes away: rejected
    with pytest.raises(AssertionError):
        pc.check_int4(x, oracle.pack_nibbles(alt), scales, 0, 32)


def test_int8_checker():
    x = _x(4, 1024, 2)
    y, codes, scales = oracle.rotate_quant(x, 128, "int8", 0)
    pc.check_int8(x, codes, scales, 128)
    c2 = codes.copy()
    c2[0, 9] = np.int8(int(c2[0, 9]) + 1 if c2[0, 9] < 127 else 126)
    with pytest.raises(AssertionError):
        pc.check_int8(x, c2, scales, 128)
    s2 = scales.copy()
    s2[2] *= np.float32(1 + 1e-5)
    with pytest.raises(AssertionError):
        pc.check_int8(x, codes, s2, 128)


def test_mxfp4_checker():
    x = np.random.default_rng(3).standard_t(3, (4, 1024))
    y, codes, scales = oracle.rotate_quant(x, 0, "mxfp4", 32)
    pc.check_mxfp4(x, codes, scales, 0)
    c2 = codes.copy()
    c2[1, 3] ^= 0x01
    with pytest.raises(AssertionError):
        pc.check_mxfp4(x, c2, scales, 0)
    s2 = scales.copy()
    s2[0, 0] += 1
    with pytest.raises(AssertionError):
        pc.check_mxfp4(x, codes, s2, 0)


def test_nvfp4_checker():
    x = _x(8, 512, 4)
    y, codes, scales = oracle.rotate_quant(x, 0, "nvfp4", 16)
    rep = pc.check_nvfp4(x, codes, scales, 0)
    assert rep["code_differs_in_window"] == 0 and rep["groups"] == 8 * 32
    flipped = codes.copy()
    flipped[1, 3] ^= 0x01                 # one code one grid step off
    with pytest.raises(AssertionError):
        pc.check_nvfp4(x, flipped, scales, 0)
    s2 = scales.copy()
    s2[0, 0] += 1                         # next E4M3 value: 6-12 % off
    with pytest.raises(AssertionError):
        pc.check_nvfp4(x, codes, s2, 0)
    # the E4M3 byte decoder used by the checker agrees with the oracle's encoder
    vals = np.exp(np.random.default_rng(1).uniform(-12, 6, 500))
    np.testing.assert_array_equal(pc._e4m3_value(oracle.e4m3_encode(vals)), oracle.to_e4m3(vals))
    # per-tensor scale: outputs of quantize(y, t) pass with tensor_scale=t
    _, c3, s3 = oracle.rotate_quant(x, 0, "nvfp4", 16, tensor_scale=0.25)
    pc.check_nvfp4(x, c3, s3, 0, tensor_scale=0.25)
    with pytest.raises(AssertionError):
        pc.check_nvfp4(x, c3, s3, 0, tensor_scale=1.0)
