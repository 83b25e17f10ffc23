"""Plain fp64 CPU oracle for GPTQ layer quantization.

TEST INFRASTRUCTURE ONLY. Nothing on the product path may import or call this module: only the
tests, the smoke check and the CPU-baseline leg of the benchmark use it. It shares no code with the
CUDA library (no kernels, headers, tables or helpers); the two meet only through the seeded inputs.

Every step follows the pages in their order and notation, written as plainly as possible: NumPy
matrix products and LAPACK (via numpy / scipy) serve as library steps, with no blocking, fusion or
reordering beyond what the method itself states.

Sources (web pages, cited by title and section):
  [OBQ]   "Part 2: Adaptive Rounding: Optimal Brain Quantizer (OBQ)"
  [GPTQ]  "Part 3: Adaptive Rounding: GPTQ"
  [BLOG]  "GPTQ second-order quantization" blog (English), and its Vietnamese version [BLOG-VI]
  [OPTROT] "OptRot: Mitigating Weight Outliers via Data-Free Rotations for Post-Training
           Quantization"

Readings taken where the pages are silent, garbled or disagree (each function repeats its own):
  * H = 2 X X^T / N  (X^T X for token-major X), the scale stated in [BLOG] "The objective is layer
    output"; codes do not depend on the scale of H because the damping is relative.
  * lambda = 0.01 * mean(diag H), added once to the diagonal ([BLOG] "3. Cholesky reformulation").
  * The factor read row by row is the UPPER factor R with H_d^{-1} = R^T R ([BLOG-VI] "2. Lazy batch
    update" writes W[:,B:] -= E R[B,B:]); the lower factor named in [GPTQ] "Observation 3" is its
    transpose.
  * E[:, j] = (w_j - q_j) / R_jj and W <- W - E R (the listing's sign/scale is inconsistent; this is
    the optimum of [GPTQ] "Observation 3"'s update formula rewritten with R).
  * Quantizer: asymmetric uniform min/max grid including 0, evaluated in IEEE float32 with
    round-half-to-even ([GPTQ] design table names only "asymmetric uniform"; the exact formula is
    this library's definition -- parity unpinned against the pages, pinned by invariants).
  * Per-row parameters come from the original W; group parameters from the current (compensated) W
    when the group's first column is reached.
"""
from __future__ import annotations

import numpy as np
import scipy.linalg

F32 = np.float32


# ------------------------------------------------------------------------------------------------
# S1: proxy Hessian
# ------------------------------------------------------------------------------------------------

def hessian_accumulate(S: np.ndarray, X: np.ndarray) -> np.ndarray:
    """S += X^T X for a chunk of token-major calibration inputs X [n_tokens, cols].

    [OBQ] "Goal": the input covariance E[x x^T] is the proxy Hessian; [GPTQ] "Algorithm GPTQ":
    H = X X^T (+ lambda I) with X as cols x tokens. bf16 and fp32 inputs are exact in fp64, and
    the products are exact too; only the summation rounds.
    """
    X64 = np.asarray(X, dtype=np.float64)
    S += X64.T @ X64
    return S


def hessian_finalize(S: np.ndarray, n_total: int) -> np.ndarray:
    """H = 2 S / N  ([BLOG] "The objective is layer output": H = 2 X X^T; averaged over tokens)."""
    if n_total <= 0:
        raise ValueError("n_total must be positive")
    return (2.0 / float(n_total)) * np.asarray(S, dtype=np.float64)


def hessian(X: np.ndarray) -> np.ndarray:
    """H = 2 X^T X / N for token-major X in one call."""
    S = np.zeros((X.shape[1], X.shape[1]))
    hessian_accumulate(S, X)
    return hessian_finalize(S, X.shape[0])


# ------------------------------------------------------------------------------------------------
# S2: damping
# ------------------------------------------------------------------------------------------------

def damp(H: np.ndarray, damp_rel: float = 0.01):
    """H_d = H + lambda I with lambda = damp_rel * mean(diag H).

    [BLOG] "3. Cholesky reformulation": dampening of about one percent of the average Hessian
    diagonal; [GPTQ] "Algorithm GPTQ": H = X X^T + lambda I. Returns (H_d, lambda).
    """
    H = np.asarray(H, dtype=np.float64)
    mean_diag = float(np.mean(np.diag(H)))
    if not mean_diag > 0.0:
        raise ValueError("mean of diag(H) must be positive (all-zero calibration input?)")
    lam = damp_rel * mean_diag
    return H + lam * np.eye(H.shape[0]), lam


# ------------------------------------------------------------------------------------------------
# S3-S5: upper factor of the damped inverse Hessian
# ------------------------------------------------------------------------------------------------

def inverse_hessian_factor(H: np.ndarray, damp_rel: float = 0.01) -> dict:
    """R upper triangular with (H + lambda I)^{-1} = R^T R, by the route the pages give.

    [GPTQ] "Algorithm GPTQ" (Cholesky factorization of H^{-1}) and "Observation 3": factor H_d
    (S3: H_d = L L^T), invert the triangular factor (S4: L^{-1}), form H_d^{-1} = L^{-T} L^{-1}
    (S4), factor that (S5: H_d^{-1} = L2 L2^T) and take R = L2^T, whose row p is read at
    quantization step p.
    """
    Hd, lam = damp(H, damp_rel)
    L = np.linalg.cholesky(Hd)                                              # S3
    Linv = scipy.linalg.solve_triangular(L, np.eye(L.shape[0]), lower=True)  # S4
    Hinv = Linv.T @ Linv                                                    # S4
    L2 = np.linalg.cholesky(Hinv)                                           # S5
    R = np.triu(L2.T)
    return {"Hd": Hd, "lam": lam, "L": L, "Linv": Linv, "Hinv": Hinv, "R": R}


# ------------------------------------------------------------------------------------------------
# S6: asymmetric uniform quantizer (IEEE float32, round half to even)
# ------------------------------------------------------------------------------------------------

def quant_params(v: np.ndarray, bits: int):
    """Scale and zero point of the asymmetric min/max grid for the values ``v`` (last axis).

    [GPTQ] design table: asymmetric uniform, per row or per group; [BLOG] "Group-wise
    quantization": one scale and zero point per output row or per group of input channels.
    The grid always contains 0: lo = min(0, min v), hi = max(0, max v); an all-zero vector gets
    the range [-1, 1]. s = (hi - lo) / (2^k - 1), z = clamp(rint(-lo / s), 0, 2^k - 1), all in
    float32 with each operation rounded once. Returns (s, z) as float32 arrays (z integer-valued).
    """
    maxq = F32(2 ** bits - 1)
    v32 = np.asarray(v, dtype=np.float64).astype(F32)
    lo = np.minimum(v32.min(axis=-1), F32(0))
    hi = np.maximum(v32.max(axis=-1), F32(0))
    flat = lo == hi
    lo = np.where(flat, F32(-1), lo).astype(F32)
    hi = np.where(flat, F32(1), hi).astype(F32)
    s = ((hi - lo).astype(F32) / maxq).astype(F32)
    z = np.clip(np.rint((-lo / s).astype(F32)), F32(0), maxq).astype(F32)
    return s, z


def quantize(x: np.ndarray, s: np.ndarray, z: np.ndarray, bits: int):
    """Code and dequantized value of x on the grid (s, z): q = clamp(rint(x/s) + z, 0, 2^k-1),
    q_hat = s * (q - z), in float32 (x is first rounded to float32). Returns (q uint8, q_hat f32)."""
    maxq = F32(2 ** bits - 1)
    x32 = np.asarray(x, dtype=np.float64).astype(F32)
    q = np.clip(np.rint((x32 / s).astype(F32)) + z, F32(0), maxq).astype(F32)
    w_hat = (s * (q - z)).astype(F32)
    return q.astype(np.uint8), w_hat


# ------------------------------------------------------------------------------------------------
# S6-S8: the column loop with lazy batch updates
# ------------------------------------------------------------------------------------------------

def _n_groups(cols: int, group: int) -> int:
    return 1 if group <= 0 else cols // group


def check_shapes(cols: int, group: int, block: int):
    if block <= 0:
        raise ValueError("block must be positive")
    if group > 0:
        if cols % group != 0:
            raise ValueError("cols must be a multiple of the group size")
        if not (group % block == 0 or block % group == 0):
            raise ValueError("group and block must nest (one a multiple of the other)")


def gptq_quantize(W: np.ndarray, R: np.ndarray, bits: int, group: int = -1, block: int = 128,
                  row_grid=None) -> dict:
    """GPTQ column loop in fixed left-to-right order with lazy block updates.

    [GPTQ] "Algorithm GPTQ" and "Observation 2: Lazy Batch Updates"; [BLOG-VI] "2. Lazy batch
    update". For each block of B columns [b0, b1), for each column j in order:
      * (group start) fresh scale/zero from the current, already compensated weights of the group;
      * q_j = quantize(w_j); e_j = (w_j - q_hat_j) / R_jj; E[:, j-b0] = e_j;
      * the block's later columns: W[:, j+1:b1] -= e_j R[j, j+1:b1]   (kept "in SRAM");
    then the flush W[:, b1:] -= E R[b0:b1, b1:] (one matrix product).
    Per-row parameters (group <= 0) are taken once from the original W. ``row_grid`` = (s, z)
    supplies them instead (per-row mode only): when W holds only the leading columns of wider
    rows, the grid of each whole original row is computed by the caller with quant_params.
    Returns codes [r,c] uint8, scales/zeros [r,G] (float32 / uint8), W_hat [r,c] float32,
    err [r,c] fp64 (the e_j), err_sq [r] fp64 = sum_j e_j^2, w_in [r,c] fp64 (the compensated
    value each weight had when it was quantized).
    """
    W = np.array(W, dtype=np.float64)
    R = np.asarray(R, dtype=np.float64)
    rows, cols = W.shape
    check_shapes(cols, group, block)
    G = _n_groups(cols, group)
    codes = np.zeros((rows, cols), np.uint8)
    W_hat = np.zeros((rows, cols), F32)
    err = np.zeros((rows, cols))
    w_in = np.zeros((rows, cols))
    scales = np.zeros((rows, G), F32)
    zeros = np.zeros((rows, G), F32)
    if group <= 0:
        s, z = quant_params(W, bits) if row_grid is None else row_grid
        scales[:, 0], zeros[:, 0] = s, z
    elif row_grid is not None:
        raise ValueError("row_grid applies to per-row grids only")
    for b0 in range(0, cols, block):
        b1 = min(cols, b0 + block)
        E = np.zeros((rows, b1 - b0))
        Wb = W[:, b0:b1]                      # a view: in-block updates land in W directly
        for j in range(b0, b1):
            if group > 0 and j % group == 0:
                g = j // group
                s, z = quant_params(W[:, j:j + group], bits)
                scales[:, g], zeros[:, g] = s, z
            gi = 0 if group <= 0 else j // group
            s, z = scales[:, gi], zeros[:, gi]
            q, w_hat = quantize(W[:, j], s, z, bits)
            e = (W[:, j] - w_hat.astype(np.float64)) / R[j, j]
            w_in[:, j] = W[:, j]
            codes[:, j], W_hat[:, j], err[:, j], E[:, j - b0] = q, w_hat, e, e
            Wb[:, j - b0 + 1:] -= np.outer(e, R[j, j + 1:b1])
        if b1 < cols:
            W[:, b1:] -= E @ R[b0:b1, b1:]
    return {"codes": codes, "scales": scales, "zeros": zeros.astype(np.uint8), "W_hat": W_hat,
            "err": err, "err_sq": (err ** 2).sum(axis=1), "w_in": w_in}


def gptq_quantize_unbatched(W: np.ndarray, R: np.ndarray, bits: int, group: int = -1) -> dict:
    """The eager schedule: after every column the whole remaining row is updated at once,
    W[:, j+1:] -= e_j R[j, j+1:] ([GPTQ] "Observation 2", the naive loop before lazy batching)."""
    return gptq_quantize(W, R, bits, group, block=1)


def rtn_quantize(W: np.ndarray, bits: int, group: int = -1) -> dict:
    """Round-to-nearest on the same grid with no compensation ([BLOG]: RTN treats every weight
    error as independent)."""
    W = np.asarray(W, dtype=np.float64)
    rows, cols = W.shape
    G = _n_groups(cols, group)
    codes = np.zeros((rows, cols), np.uint8)
    W_hat = np.zeros((rows, cols), F32)
    scales = np.zeros((rows, G), F32)
    zeros = np.zeros((rows, G), F32)
    for g in range(G):
        c0, c1 = (0, cols) if group <= 0 else (g * group, (g + 1) * group)
        s, z = quant_params(W[:, c0:c1], bits)
        scales[:, g], zeros[:, g] = s, z
        q, wh = quantize(W[:, c0:c1], s[:, None], z[:, None], bits)
        codes[:, c0:c1], W_hat[:, c0:c1] = q, wh
    return {"codes": codes, "scales": scales, "zeros": zeros.astype(np.uint8), "W_hat": W_hat}


# ------------------------------------------------------------------------------------------------
# Metric
# ------------------------------------------------------------------------------------------------

def layer_error(W: np.ndarray, W_hat: np.ndarray, H: np.ndarray) -> float:
    """Relative layer output error ||WX - W_hat X||^2 / ||WX||^2 = tr(dW H dW^T) / tr(W H W^T)
    with the undamped H ([BLOG] "The objective is layer output"; the factor 2/N cancels)."""
    W = np.asarray(W, dtype=np.float64)
    dW = np.asarray(W_hat, dtype=np.float64) - W
    H = np.asarray(H, dtype=np.float64)
    num = np.einsum("ij,jk,ik->", dW, H, dW)
    den = np.einsum("ij,jk,ik->", W, H, W)
    return float(num / den)


def gptq_layer(W: np.ndarray, X: np.ndarray, bits: int, group: int, block: int,
               damp_rel: float = 0.01) -> dict:
    """The whole path S1-S8 for one layer: H from X, R from H, then the column loop."""
    H = hessian(X)
    fac = inverse_hessian_factor(H, damp_rel)
    out = gptq_quantize(W, fac["R"], bits, group, block)
    out.update(H=H, R=fac["R"], lam=fac["lam"], rel_err=layer_error(W, out["W_hat"], H))
    return out
