"""The tensor-core matrix product (3xTF32 on tcgen05) behind S3-S5 and S8, against fp64 products.

Expected accuracy: each operand is carried as tf32 big + small parts (the small*small term and
the tf32 truncation of the small parts are dropped, about 2^-21 relative per product) and sums are
folded out of the tensor core every 256 k, so errors stay within a few fp32 ulps of the result's
scale; the bound used is 2e-6 relative to sum_k |a_mk| |b_kn|.
"""
import numpy as np
import pytest
import torch

from post_weight_quantization_12_b200 import _lib

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _stored(op, mn_major):
    """Storage of an operand given its logical op matrix (rows x cols) and its major-ness."""
    return np.ascontiguousarray(op.T if mn_major else op)


def _run(opA, a_mn, opBt, b_mn, alpha=1.0, beta=0.0, C0=None, lower=False, klo_m=False,
         klo_n=False, split=False):
    """opA: M x K, opBt: N x K (so op(B) = opBt^T). Returns (C, Cbig, Csmall) as numpy."""
    M, K = opA.shape
    N = opBt.shape[0]
    A = torch.from_numpy(_stored(opA, a_mn)).to(DEV)
    # op(B)[k][n]: b_mn stores B[k][n] (K x N), else B[n][k] (N x K)
    B = torch.from_numpy(_stored(opBt, b_mn)).to(DEV)
    C = torch.from_numpy(np.ascontiguousarray(C0 if C0 is not None else
                                              np.full((M, N), np.nan, np.float32))).to(DEV)
    Cb = torch.empty_like(C) if split else None
    Cs = torch.empty_like(C) if split else None
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    _lib.selftest_gemm(A, a_mn, B, b_mn, C, M, N, K, alpha, beta, lower, klo_m, klo_n, Cb, Cs, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    return C.cpu().numpy(), (Cb.cpu().numpy() if split else None), \
        (Cs.cpu().numpy() if split else None)


def _check(got, opA, opBt, alpha=1.0, beta=0.0, C0=None, mask=None):
    A = opA.astype(np.float64)
    Bt = opBt.astype(np.float64)
    ref = alpha * (A @ Bt.T)
    if beta != 0.0:
        ref = ref + beta * C0.astype(np.float64)
    scale = np.abs(alpha) * (np.abs(A) @ np.abs(Bt).T) + np.abs(beta) * (
        np.abs(C0) if C0 is not None else 0) + 1e-30
    err = np.abs(got.astype(np.float64) - ref) / scale
    if mask is not None:
        err = err[mask]
    assert np.all(np.isfinite(err)) and err.max() < 2e-6, err.max()


@pytest.mark.parametrize("a_mn", [0, 1])
@pytest.mark.parametrize("b_mn", [0, 1])
@pytest.mark.parametrize("M,N,K", [(128, 128, 32), (256, 384, 512), (200, 136, 100),
                                   (4, 260, 36)])
def test_gemm_layouts_and_ragged_sizes(a_mn, b_mn, M, N, K):
    rng = np.random.default_rng(M + N + K + 10 * a_mn + b_mn)
    opA = rng.standard_normal((M, K)).astype(np.float32)
    opBt = rng.standard_normal((N, K)).astype(np.float32)
    C, _, _ = _run(opA, a_mn, opBt, b_mn)
    _check(C, opA, opBt)


def test_gemm_long_k_folds_sums():
    rng = np.random.default_rng(3)
    M, N, K = 256, 256, 4096
    opA = (rng.standard_normal((M, K)) + 1.0).astype(np.float32)   # positive-leaning sums
    opBt = (rng.standard_normal((N, K)) + 1.0).astype(np.float32)
    C, _, _ = _run(opA, 1, opBt, 1)
    _check(C, opA, opBt)


def test_gemm_alpha_beta_and_split_output():
    rng = np.random.default_rng(4)
    M, N, K = 300, 260, 128
    opA = rng.standard_normal((M, K)).astype(np.float32)
    opBt = rng.standard_normal((N, K)).astype(np.float32)
    C0 = rng.standard_normal((M, N)).astype(np.float32)
    C, Cb, Cs = _run(opA, 0, opBt, 1, alpha=-1.0, beta=1.0, C0=C0, split=True)
    _check(C, opA, opBt, -1.0, 1.0, C0)
    np.testing.assert_array_equal(Cb + Cs, C)
    assert np.all((Cb.view(np.uint32) & 0x1FFF) == 0)


def test_gemm_lower_tiles_and_k_ranges():
    rng = np.random.default_rng(5)
    n = 384
    # a lower-triangular operand, like the inverse factor: op(A)[m][k] = V[k][m], op(B) = V
    V = np.tril(rng.standard_normal((n, n))).astype(np.float32)
    C0 = np.full((n, n), 7.0, np.float32)
    C, _, _ = _run(V.T.copy(), 1, V.T.copy(), 1, C0=C0, lower=True, klo_m=True)
    ref = V.T.astype(np.float64) @ V.astype(np.float64)
    tile = np.arange(n) // 128
    below = tile[:, None] >= tile[None, :]
    assert np.all(C[~below] == 7.0)                    # tiles above the diagonal untouched
    scale = np.abs(V.T) @ np.abs(V) + 1e-30
    assert (np.abs(C - ref) / scale)[below].max() < 2e-6
    # k ranges from the tile's column start: entries below it must not be read (poison them)
    T = rng.standard_normal((128, n)).astype(np.float32)
    Vp = V.copy()
    Vp[np.triu_indices(n, 1)] = np.nan                 # structurally zero, stored as NaN
    for i in range(0, n, 128):
        Vp[i:i + 128, i:i + 128] = np.tril(V[i:i + 128, i:i + 128])
    C, _, _ = _run(T, 0, Vp.T.copy(), 1, klo_n=True)
    _check(C, T, V.T.copy())


@pytest.mark.parametrize("n,K", [(384, 128), (1000, 96), (4096, 128)])
def test_gemm_lower_update_k128(n, K):
    """The Cholesky trailing update: C -= P P^T on lower tiles, K <= 128 (persistent variant)."""
    rng = np.random.default_rng(n + K)
    P = rng.standard_normal((n, K)).astype(np.float32)
    C0 = rng.standard_normal((n, n)).astype(np.float32)
    C, _, _ = _run(P, 0, P, 0, alpha=-1.0, beta=1.0, C0=C0, lower=True)
    tile = np.arange(n) // 128
    below = tile[:, None] >= tile[None, :]
    assert np.all(C[~below] == C0[~below])
    _check(C, P, P, -1.0, 1.0, C0, mask=below)


@pytest.mark.parametrize("M,N,K,b_mn,beta", [
    (512, 768, 128, 1, 1.0),     # trailing-update shape: R slab MN-major, C read and written
    (512, 640, 128, 0, 1.0),     # 640 columns: five 128-wide tile columns
    (256, 256, 64, 1, 0.0),      # C written only
    (1024, 384, 100, 0, 1.0),    # K not a multiple of the 32-wide stage
    # the lazy-update shape on more tiles than SMs (a CTA's tiles then cross A-band boundaries)
    (4096, 3968, 128, 1, 1.0),   # the widest update of a 4096-column layer: 992 tiles
    (1536, 1664, 128, 1, 1.0),   # 156 tiles: a few CTAs take two, some of them in two bands
    (1000, 2560, 96, 1, 1.0),    # ragged last band and K of three 32-wide stages
])
def test_gemm_k128_shapes(M, N, K, b_mn, beta):
    """K <= 128 products on multi-tile shapes: both B layouts, beta 0 and 1, ragged K."""
    rng = np.random.default_rng(M + N + K + b_mn)
    opA = rng.standard_normal((M, K)).astype(np.float32)
    opBt = rng.standard_normal((N, K)).astype(np.float32)
    C0 = rng.standard_normal((M, N)).astype(np.float32)
    C, _, _ = _run(opA, 0, opBt, b_mn, alpha=-1.0, beta=beta, C0=C0)
    _check(C, opA, opBt, -1.0, beta, C0)
