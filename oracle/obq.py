"""Plain fp64 CPU oracle for OBQ: greedy-order quantization with explicit inverse-Hessian
downdates, the reference GPTQ's fixed order is compared against.

TEST INFRASTRUCTURE ONLY, like gptq_oracle: only the tests, the smoke check and the CPU-baseline
leg of the benchmark may import it. It shares no code with the CUDA library.

Source: "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)", sections "The OBS / GPTQ
Trick" (after weight p is quantized, the inverse Hessian of the remaining weights is the old one
minus the outer product of its p-th column and p-th row over its (p, p) entry), "Generalized
Weight Update" (the remaining weights move by -(w_p - q_p) H^-1[:, p] / H^-1[p, p]) and "Greedy
Search" (each step quantizes the remaining weight whose quantization raises the proxy loss
least, the loss increase being (w_p - q_p)^2 / (2 H^-1[p, p])); "Limitations of OBQ" (every row
needs its own copy of H^-1).

Readings taken where the page is silent:
  * Quantizer: the per-row grid of the GPTQ oracle (reading 6 there), fixed from the original row;
    group grids depend on the column order and are not defined for a greedy order.
  * Ties in the greedy choice go to the lowest column index.
  * Arithmetic: fp64, each operation rounded once (no fused multiply-add), in the order written
    below; the quantizer decision in float32 as in the GPTQ oracle. The rank-1 downdate uses row p
    of H^-1 for both factors (H^-1 is symmetric: its p-th column equals its p-th row):
        h = H^-1[p, :];  g = h / h[p];  H^-1 <- H^-1 - outer(h, g)
  * The weights and H^-1 entries of already-quantized columns keep being updated (their values
    are never read again), and the loss reported per row is the sum of the chosen
    (w_p - q_p)^2 / H^-1[p, p], i.e. twice the summed proxy-loss increases.
"""
from __future__ import annotations

import numpy as np

from .gptq_oracle import quant_params, quantize

F32 = np.float32


def obq_row(w: np.ndarray, Hinv: np.ndarray, s, z, bits: int, order: str = "greedy",
            trace: bool = False) -> dict:
    """OBQ on one row w [c] with its own copy of the inverse Hessian Hinv [c, c] (fp64) and the
    row's grid (s, z). order = "greedy" (OBQ) or "natural" (left to right, the GPTQ order)."""
    w = np.array(w, dtype=np.float64)
    Hinv = np.array(Hinv, dtype=np.float64)
    c = w.shape[0]
    remaining = np.ones(c, dtype=bool)
    codes = np.zeros(c, np.uint8)
    w_hat = np.zeros(c, F32)
    chosen = np.zeros(c, np.int64)
    loss = 0.0
    states = []
    for step in range(c):
        q, wh = quantize(w, s, z, bits)                     # float32 grid decision per column
        d = w - wh.astype(np.float64)
        diag = np.diagonal(Hinv).copy()
        if order == "greedy":
            score = np.full(c, np.inf)
            score[remaining] = (d[remaining] * d[remaining]) / diag[remaining]
            p = int(np.argmin(score))                       # first minimum: lowest index
        else:
            p = step
        chosen[step] = p
        codes[p], w_hat[p] = q[p], wh[p]
        loss += (d[p] * d[p]) / diag[p]
        e = d[p] / diag[p]
        h = Hinv[p, :].copy()
        w = w - e * h                                       # compensation of the other weights
        g = h / h[p]
        Hinv = Hinv - np.outer(h, g)                        # OBS downdate: p leaves the problem
        remaining[p] = False
        if trace:
            states.append(w.copy())
    out = {"codes": codes, "W_hat": w_hat, "order": chosen, "loss": loss}
    if trace:
        out["states"] = states
    return out


def obq_quantize(W: np.ndarray, Hinv: np.ndarray, bits: int, order: str = "greedy") -> dict:
    """OBQ for every row of W [r, c] with the shared starting inverse Hessian Hinv [c, c]; per-row
    grids from the original W. Returns codes [r, c] uint8, W_hat [r, c] float32, order [r, c]
    (column quantized at each step), loss [r] fp64, scales / zeros [r, 1]."""
    W = np.asarray(W, dtype=np.float64)
    r, c = W.shape
    s, z = quant_params(W, bits)
    codes = np.zeros((r, c), np.uint8)
    W_hat = np.zeros((r, c), F32)
    chosen = np.zeros((r, c), np.int64)
    loss = np.zeros(r)
    for i in range(r):
        o = obq_row(W[i], Hinv, s[i], z[i], bits, order)
        codes[i], W_hat[i], chosen[i], loss[i] = o["codes"], o["W_hat"], o["order"], o["loss"]
    return {"codes": codes, "W_hat": W_hat, "order": chosen, "loss": loss,
            "scales": s.reshape(r, 1), "zeros": z.astype(np.uint8).reshape(r, 1)}
