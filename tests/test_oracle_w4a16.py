"""Pins for the W4A16 oracle (packed 4-bit layout and dequantizing product), checked against
formulations independent of the oracle's code: positional base-16 numbers, exact rational sums,
single-column probes and the quantizer's own dequantized weights."""
from fractions import Fraction

import numpy as np
import pytest

import oracle
from post_weight_quantization_12_b200 import synth


def _codes(rows, cols, seed):
    return np.random.default_rng(seed).integers(0, 16, (rows, cols), dtype=np.uint8)


def test_pack_layout_is_little_endian_base16():
    """A row of codes read as one base-16 number with column 0 least significant; word w is digits
    8w .. 8w+7 of it (the layout: column c in bits 4(c mod 8).. of word c div 8)."""
    codes = _codes(5, 48, 1)
    words = oracle.pack_codes(codes)
    assert words.dtype == np.uint32 and words.shape == (5, 6)
    for r in range(5):
        big = sum(int(codes[r, c]) * 16 ** c for c in range(48))
        for w in range(6):
            assert int(words[r, w]) == (big >> (32 * w)) & 0xFFFFFFFF


def test_pack_bytes_low_nibble_is_even_column():
    codes = _codes(3, 16, 2)
    raw = oracle.pack_codes(codes).astype("<u4").tobytes()
    b = np.frombuffer(raw, np.uint8).reshape(3, 8)
    assert np.array_equal(b & 0xF, codes[:, 0::2])
    assert np.array_equal(b >> 4, codes[:, 1::2])


def test_pack_round_trip_and_rejects():
    codes = _codes(7, 64, 3)
    assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(codes)), codes)
    with pytest.raises(ValueError):
        oracle.pack_codes(codes[:, :60])
    bad = codes.copy()
    bad[0, 0] = 16
    with pytest.raises(ValueError):
        oracle.pack_codes(bad)


def _fraction_matmul(codes, scales, zeros, group, X):
    """Brute force: y[n][r] = sum_c x[n][c] * s * (q - z) in exact rationals."""
    rows, cols = codes.shape
    out = np.zeros((X.shape[0], rows), dtype=object)
    for n in range(X.shape[0]):
        for r in range(rows):
            acc = Fraction(0)
            for c in range(cols):
                g = 0 if group <= 0 else c // group
                acc += Fraction(float(X[n, c])) * Fraction(float(scales[r, g])) * \
                    (int(codes[r, c]) - int(zeros[r, g]))
            out[n, r] = acc
    return out


@pytest.mark.parametrize("group", [-1, 8, 16])
def test_matmul_exact_rationals(group):
    rng = np.random.default_rng(4)
    rows, cols, n = 6, 32, 3
    codes = _codes(rows, cols, 5)
    G = 1 if group <= 0 else cols // group
    scales = rng.uniform(1e-3, 3e-2, (rows, G)).astype(np.float32)
    zeros = rng.integers(0, 16, (rows, G), dtype=np.uint8)
    X = synth.round_to_bf16_np(rng.standard_normal((n, cols)).astype(np.float32))
    y = oracle.w4a16_matmul(oracle.pack_codes(codes), scales, zeros, group, X)
    ref = _fraction_matmul(codes, scales, zeros, group, X)
    terms = oracle.w4a16_abs_terms(oracle.pack_codes(codes), scales, zeros, group, X)
    for i in range(n):
        for r in range(rows):
            assert abs(Fraction(float(y[i, r])) - ref[i, r]) <= Fraction(1e-15) * \
                Fraction(float(terms[i, r]))


def test_single_column_probe_fixes_group_and_orientation():
    """x = e_c picks out W_hat[:, c] = s[:, c // g] (q[:, c] - z[:, c // g]) exactly."""
    rows, cols, group = 4, 256, 128
    codes = _codes(rows, cols, 6)
    scales = (2.0 ** -np.arange(1, 1 + rows * 2)).reshape(rows, 2).astype(np.float32)
    zeros = np.array([[1, 9], [3, 4], [15, 0], [7, 8]], np.uint8)
    words = oracle.pack_codes(codes)
    for c in (0, 1, 7, 8, 127, 128, 129, 255):
        X = np.zeros((1, cols), np.float32)
        X[0, c] = 1.0
        y = oracle.w4a16_matmul(words, scales, zeros, group, X)[0]
        g = c // group
        expect = scales[:, g].astype(np.float64) * (codes[:, c].astype(np.float64) - zeros[:, g])
        assert np.array_equal(y, expect)


@pytest.mark.parametrize("group", [-1, 128])
def test_matmul_of_rtn_codes_matches_quantizer_w_hat(group):
    """The codes, scales and zeros of the round-to-nearest quantizer dequantize to its W_hat
    (up to W_hat's float32 rounding of s (q - z)), so Y = X W_hat^T."""
    rng = np.random.default_rng(7)
    W = rng.standard_normal((32, 256)) * 0.02
    out = oracle.rtn_quantize(W, 4, group)
    X = synth.round_to_bf16_np(rng.standard_normal((2, 256)).astype(np.float32))
    words = oracle.pack_codes(out["codes"])
    y = oracle.w4a16_matmul(words, out["scales"], out["zeros"], group, X)
    ref = X.astype(np.float64) @ out["W_hat"].astype(np.float64).T
    terms = np.abs(X.astype(np.float64)) @ np.abs(out["W_hat"].astype(np.float64)).T
    assert np.all(np.abs(y - ref) <= 2.0 ** -23 * terms)
    assert np.array_equal(oracle.dequantize(words, out["scales"], out["zeros"], group)
                          .astype(np.float32), out["W_hat"])


def test_matmul_linear_in_x_and_zero_point():
    """Y is linear in X, and raising every code and zero by the same amount leaves it unchanged."""
    rng = np.random.default_rng(8)
    codes = rng.integers(0, 12, (8, 64), dtype=np.uint8)
    scales = rng.uniform(0.01, 0.1, (8, 2)).astype(np.float32)
    zeros = rng.integers(0, 12, (8, 2), dtype=np.uint8)
    X1 = rng.standard_normal((1, 64))
    X2 = rng.standard_normal((1, 64))
    f = lambda c, z, X: oracle.w4a16_matmul(oracle.pack_codes(c), scales, z, 32, X)
    assert np.allclose(f(codes, zeros, X1 + 2 * X2), f(codes, zeros, X1) + 2 * f(codes, zeros, X2),
                       rtol=1e-13, atol=1e-15)
    assert np.allclose(f(codes + 3, zeros + 3, X1), f(codes, zeros, X1), rtol=1e-14, atol=1e-16)


# ---------------------------------------------------------------------------------------------
# Packed 3-bit layout (32 codes per three words)
# ---------------------------------------------------------------------------------------------

def _codes3(rows, cols, seed):
    return np.random.default_rng(seed).integers(0, 8, (rows, cols), dtype=np.uint8)


def test_pack3_layout_is_little_endian_base8():
    """Each group of 32 codes, read as an octal numeral with column 32k as its last digit (the
    least significant), is the 96-bit number held in the group's three words, word 3k lowest.
    The numeral is converted by Python's own base-8 parser, not by shifts."""
    codes = _codes3(4, 96, 11)
    words = oracle.pack_codes_3bit(codes)
    assert words.dtype == np.uint32 and words.shape == (4, 9)
    for r in range(4):
        for k in range(3):
            numeral = "".join(str(int(d)) for d in codes[r, 32 * k:32 * k + 32][::-1])
            value = int(numeral, 8)
            got = int(words[r, 3 * k]) + (int(words[r, 3 * k + 1]) << 32) + \
                (int(words[r, 3 * k + 2]) << 64)
            assert got == value


@pytest.mark.parametrize("col,expect", [
    (0, (0x7, 0, 0)),                    # bits 0..2
    (10, (0xC0000000, 0x1, 0)),          # bits 30..32: straddles words 0 and 1
    (11, (0, 0xE, 0)),                   # bits 33..35
    (21, (0, 0x80000000, 0x3)),          # bits 63..65: straddles words 1 and 2
    (31, (0, 0, 0xE0000000)),            # bits 93..95
])
def test_pack3_single_code_probe(col, expect):
    """One code of 7 (all three bits set) in an otherwise zero group: the set bits, worked out by
    hand from the bit offsets 3 col .. 3 col + 2, land exactly in the words given."""
    codes = np.zeros((1, 32), np.uint8)
    codes[0, col] = 7
    assert tuple(int(w) for w in oracle.pack_codes_3bit(codes)[0]) == expect


def test_pack3_round_trip_and_rejects():
    codes = _codes3(5, 128, 12)
    assert np.array_equal(oracle.unpack_codes_3bit(oracle.pack_codes_3bit(codes)), codes)
    with pytest.raises(ValueError):
        oracle.pack_codes_3bit(codes[:, :96 + 16])
    bad = codes.copy()
    bad[2, 5] = 8
    with pytest.raises(ValueError):
        oracle.pack_codes_3bit(bad)
    # the 3-bit form of codes that fit in 3 bits holds the same values as the 4-bit form
    assert np.array_equal(oracle.unpack_codes(oracle.pack_codes(codes)),
                          oracle.unpack_codes_3bit(oracle.pack_codes_3bit(codes)))
