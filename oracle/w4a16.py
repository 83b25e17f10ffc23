"""Plain fp64 CPU oracle for the packed 4-bit weight format and the W4A16 dequantizing product.

TEST INFRASTRUCTURE ONLY, like gptq_oracle: only the tests, the smoke check and the CPU-baseline
leg of the benchmark may import it. It shares no code with the CUDA library.

Sources (web pages, cited by title and section):
  [BLOG]    "GPTQ second-order quantization" blog (English): "What the original results
            established" -- GPTQ is weight-only; in the usual W4A16 path the activations stay in
            FP16/BF16 and the speed comes from moving fewer weight bytes through a kernel that
            unpacks and dequantizes them; "Group-wise quantization" -- one scale and zero point per
            row or per group of input channels, group size traded against scale traffic.
  [BLOG-VI] the Vietnamese version, "Group-wise quantization" (group size chosen together with the
            packed layout and the runtime kernel) and its closing section (the artifact needs a
            packed INT4 kernel for the target device).

Readings taken where the pages are silent:
  * Packed layout (the pages fix none): eight 4-bit codes per little-endian 32-bit word, row by
    row; code (r, c) sits in bits 4*(c % 8) .. 4*(c % 8) + 3 of word (r, c // 8). Equivalently
    byte c // 2 of row r holds column c in its low nibble when c is even, its high nibble when odd.
  * The dequantized weight is s * (q - z) with the scale s and integer zero z of the code's row
    and group (the same grid the quantizer defines), and the product is Y = X W_hat^T: X holds
    n activation vectors of length cols (token-major, like the calibration input), Y is n x rows.
  * Precision: the activations are BF16 values; the oracle forms s * (q - z) * x exactly in fp64
    and sums in fp64.
  * Packed 3-bit layout (for the 3-bit grids; the pages fix none either): 32 codes per three
    little-endian 32-bit words, row by row; the 32 codes of columns 32k .. 32k + 31 form the
    96-bit little-endian number sum_i q_i 8^i held in words (r, 3k), (r, 3k + 1), (r, 3k + 2), so
    code i sits in bits 3i .. 3i + 2 of that number (codes 10 and 21 straddle two words).
"""
from __future__ import annotations

import numpy as np

CODES_PER_WORD = 8
BITS = 4


def pack_codes(codes: np.ndarray) -> np.ndarray:
    """uint8 codes [rows, cols] (values < 16, cols % 8 == 0) -> uint32 words [rows, cols // 8]
    in the layout stated in the module header."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    if cols % CODES_PER_WORD:
        raise ValueError("cols must be a multiple of 8")
    if codes.size and int(codes.max()) >= 1 << BITS:
        raise ValueError("codes must fit in 4 bits")
    c = codes.astype(np.uint32).reshape(rows, cols // CODES_PER_WORD, CODES_PER_WORD)
    words = np.zeros((rows, cols // CODES_PER_WORD), np.uint32)
    for p in range(CODES_PER_WORD):
        words |= c[:, :, p] << np.uint32(BITS * p)
    return words


def unpack_codes(words: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes: uint32 [rows, cols // 8] -> uint8 [rows, cols]."""
    words = np.asarray(words, dtype=np.uint32)
    rows, nw = words.shape
    out = np.zeros((rows, nw, CODES_PER_WORD), np.uint8)
    for p in range(CODES_PER_WORD):
        out[:, :, p] = (words >> np.uint32(BITS * p)) & np.uint32(0xF)
    return out.reshape(rows, nw * CODES_PER_WORD)


def pack_codes_3bit(codes: np.ndarray) -> np.ndarray:
    """uint8 codes [rows, cols] (values < 8, cols % 32 == 0) -> uint32 words [rows, 3 cols / 32]
    in the 3-bit layout stated in the module header: each group of 32 codes is written out as the
    base-8 digits of one 96-bit number, least significant first."""
    codes = np.asarray(codes)
    rows, cols = codes.shape
    if cols % 32:
        raise ValueError("cols must be a multiple of 32")
    if codes.size and int(codes.max()) >= 8:
        raise ValueError("codes must fit in 3 bits")
    words = np.zeros((rows, 3 * cols // 32), np.uint32)
    for r in range(rows):
        for k in range(cols // 32):
            value = 0
            for i in range(32):
                value += int(codes[r, 32 * k + i]) << (3 * i)
            for j in range(3):
                words[r, 3 * k + j] = (value >> (32 * j)) & 0xFFFFFFFF
    return words


def unpack_codes_3bit(words: np.ndarray) -> np.ndarray:
    """Inverse of pack_codes_3bit: uint32 [rows, 3 cols / 32] -> uint8 [rows, cols]."""
    words = np.asarray(words, dtype=np.uint32)
    rows, nw = words.shape
    if nw % 3:
        raise ValueError("a row holds whole groups of three words")
    out = np.zeros((rows, nw // 3 * 32), np.uint8)
    for r in range(rows):
        for k in range(nw // 3):
            value = (int(words[r, 3 * k]) | (int(words[r, 3 * k + 1]) << 32) |
                     (int(words[r, 3 * k + 2]) << 64))
            for i in range(32):
                out[r, 32 * k + i] = (value >> (3 * i)) & 7
    return out


def group_of_column(cols: int, group: int) -> np.ndarray:
    """Index of the scale/zero column used by each weight column: c // group, or 0 per row."""
    c = np.arange(cols)
    return np.zeros(cols, np.int64) if group <= 0 else c // group


def dequantize(words: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int) -> np.ndarray:
    """W_hat[r, c] = s[r, g(c)] * (q[r, c] - z[r, g(c)]) in fp64 ([BLOG] "Group-wise
    quantization": the scale and zero point of the weight's row, or of its group of input
    channels)."""
    q = unpack_codes(words).astype(np.float64)
    rows, cols = q.shape
    g = group_of_column(cols, group)
    s = np.asarray(scales, dtype=np.float64).reshape(rows, -1)[:, g]
    z = np.asarray(zeros, dtype=np.float64).reshape(rows, -1)[:, g]
    return s * (q - z)


def w4a16_matmul(words: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int,
                 X: np.ndarray) -> np.ndarray:
    """Y = X W_hat^T for activations X [n, cols] (BF16 values), fp64: the product the W4A16
    path computes from the packed codes ([BLOG] "What the original results established")."""
    W_hat = dequantize(words, scales, zeros, group)
    X64 = np.asarray(X, dtype=np.float64).reshape(-1, W_hat.shape[1])
    return X64 @ W_hat.T


def w4a16_abs_terms(words: np.ndarray, scales: np.ndarray, zeros: np.ndarray, group: int,
                    X: np.ndarray) -> np.ndarray:
    """sum_c |x[n, c] * W_hat[r, c]| for every output: the scale of the rounding error any
    summation order can make, used to state floating-point tolerances."""
    W_hat = np.abs(dequantize(words, scales, zeros, group))
    X64 = np.abs(np.asarray(X, dtype=np.float64).reshape(-1, W_hat.shape[1]))
    return X64 @ W_hat.T
