"""Plain fp64 CPU oracle for the data-free Hadamard rotation applied before GPTQ.

TEST INFRASTRUCTURE ONLY, like gptq_oracle: only the tests, the smoke check and the CPU-baseline
leg of the benchmark may import it. It shares no code with the CUDA library.

Source: "OptRot: Mitigating Weight Outliers via Data-Free Rotations for Post-Training
Quantization", Abstract and Figure 1 (fusible rotations applied to weights and, transposed, to
the activations, so the layer output is unchanged; rotations spread weight outliers) and
Theorem 3.1 (the round-to-nearest error bound grows with the weight incoherence mu_W).

Readings taken where the page is silent:
  * The rotation is the data-free one of the rotation family the page compares against: a
    randomized Hadamard matrix Q = diag(signs) * (I (x) H_b) / sqrt(b), H_b the Sylvester Hadamard
    matrix of order b, with b the largest power of two that divides n and is at most 4096 (a
    block-diagonal Hadamard when n is not a power of two). `signs` (+1 / -1, length n) are drawn
    by the caller and passed in.
  * It acts on the input-channel axis: W' = W Q for weights [rows, n] and X' = X Q for token-major
    activations [tokens, n], so that W' X'^T = W X^T (Q is orthogonal).
  * Weight incoherence: mu_W = max_ij |W_ij| * sqrt(m n) / ||W||_F (the page's definition of the
    quantity in Theorem 3.1; its formula did not survive extraction, this is the usual one).
"""
from __future__ import annotations

import numpy as np
import scipy.linalg

MAX_BLOCK = 4096


def hadamard_block(n: int) -> int:
    """Order b of the Hadamard blocks used for width n (largest power of two dividing n, <= 4096)."""
    if n <= 0:
        raise ValueError("n must be positive")
    b = n & -n
    return min(b, MAX_BLOCK)


def rotation_matrix(n: int, signs=None) -> np.ndarray:
    """Q = diag(signs) (I_{n/b} (x) H_b) / sqrt(b), fp64 [n, n]."""
    b = hadamard_block(n)
    Hb = scipy.linalg.hadamard(b).astype(np.float64) / np.sqrt(b)
    Q = np.kron(np.eye(n // b), Hb)
    if signs is not None:
        Q = np.asarray(signs, dtype=np.float64).reshape(n, 1) * Q
    return Q


def rotate(X: np.ndarray, signs=None) -> np.ndarray:
    """X Q for the rows of X [rows, n] (weights or token-major activations), in fp64. Q is block
    diagonal, so each block of b columns is multiplied by its own diag(signs) H_b / sqrt(b)."""
    X64 = np.asarray(X, dtype=np.float64)
    n = X64.shape[1]
    b = hadamard_block(n)
    Hb = scipy.linalg.hadamard(b).astype(np.float64) / np.sqrt(b)
    s = np.ones(n) if signs is None else np.asarray(signs, dtype=np.float64)
    out = np.empty_like(X64)
    for k in range(n // b):
        blk = slice(k * b, (k + 1) * b)
        out[:, blk] = (X64[:, blk] * s[blk]) @ Hb
    return out


def rotate_abs_terms(X: np.ndarray) -> np.ndarray:
    """sum over the inputs of |x_i| |Q_ij| for every output: the magnitude scale of any summation
    order's rounding error (used to state tolerances). Every entry of a block of Q has magnitude
    1 / sqrt(b), so this is the block's sum of |x| over sqrt(b), repeated over the block."""
    X64 = np.abs(np.asarray(X, dtype=np.float64))
    n = X64.shape[1]
    b = hadamard_block(n)
    sums = X64.reshape(X64.shape[0], n // b, b).sum(axis=2) / np.sqrt(b)
    return np.repeat(sums, b, axis=1)


def weight_incoherence(W: np.ndarray) -> float:
    """mu_W = max |W_ij| sqrt(m n) / ||W||_F ("OptRot", Theorem 3.1's incoherence)."""
    W64 = np.asarray(W, dtype=np.float64)
    m, n = W64.shape
    return float(np.abs(W64).max() * np.sqrt(m * n) / np.linalg.norm(W64))
