"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix, independent of
the oracle's own code path (closed forms, textbook equivalences, brute force, exact arithmetic).

Each test names the fact it pins. A plausible mistake anywhere in the oracle (a dropped term, a
wrong sign or index, a transposed operand) fails at least one of them.
"""
from fractions import Fraction
import itertools
import os

import numpy as np
import pytest
import scipy.linalg

import oracle
from post_weight_quantization_12_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand_spd(c, seed, cond_spread=1.0):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((4 * c + 8, c)) * np.exp(rng.uniform(-cond_spread, cond_spread, c))
    return oracle.hessian(X), X


def _rand_W(r, c, seed, std=0.02):
    return np.random.default_rng(seed).standard_normal((r, c)) * std


# ---------------------------------------------------------------------------------------------
# P10: the Hessian against exact rational arithmetic; the library Cholesky against a textbook one
# ---------------------------------------------------------------------------------------------

def test_hessian_exact_rational_bf16():
    """S = sum_t x_t x_t^T for bf16 inputs is exact in fp64 at this size: compare to Fractions."""
    rng = np.random.default_rng(5)
    X = synth.round_to_bf16_np(rng.standard_normal((16, 5)).astype(np.float32))
    S = np.zeros((5, 5))
    oracle.hessian_accumulate(S, X[:7])
    oracle.hessian_accumulate(S, X[7:])           # two chunks: accumulation across calls
    for i in range(5):
        for j in range(5):
            exact = sum(Fraction(float(X[t, i])) * Fraction(float(X[t, j])) for t in range(16))
            assert Fraction(S[i, j]) == exact
    H = oracle.hessian_finalize(S, 16)
    assert Fraction(H[1, 2]) == Fraction(S[1, 2]) * 2 / 16


def _textbook_cholesky(A):
    n = A.shape[0]
    L = np.zeros_like(A)
    for j in range(n):
        L[j, j] = np.sqrt(A[j, j] - sum(L[j, k] ** 2 for k in range(j)))
        for i in range(j + 1, n):
            L[i, j] = (A[i, j] - sum(L[i, k] * L[j, k] for k in range(j))) / L[j, j]
    return L


def test_cholesky_matches_textbook_and_reconstructs():
    H, _ = _rand_spd(7, 1, 1.5)
    f = oracle.inverse_hessian_factor(H, 0.01)
    np.testing.assert_allclose(f["L"], _textbook_cholesky(f["Hd"]), rtol=1e-12, atol=1e-12)
    n = H.shape[0]
    np.testing.assert_allclose(f["Hd"], H + f["lam"] * np.eye(n), rtol=0, atol=0)
    assert f["lam"] == pytest.approx(0.01 * np.trace(H) / n, rel=1e-15)
    # R^T R = H_d^{-1}, checked through H_d R^T R = I (no inverse taken here)
    np.testing.assert_allclose(f["Hd"] @ (f["R"].T @ f["R"]), np.eye(n), atol=1e-10)
    assert np.all(np.tril(f["R"], -1) == 0) and np.all(np.diag(f["R"]) > 0)


# ---------------------------------------------------------------------------------------------
# P8 / P7: the three-step route against the reversed (UL) route; trailing-block property
# ---------------------------------------------------------------------------------------------

def test_route_equals_reversed_ul_inverse():
    """Cholesky is unique, so R = U^{-1} where H_d = U U^T with U upper; U = J chol(J H_d J) J."""
    H, _ = _rand_spd(24, 2, 2.0)
    f = oracle.inverse_hessian_factor(H, 0.01)
    J = np.eye(24)[::-1]
    U = J @ np.linalg.cholesky(J @ f["Hd"] @ J) @ J
    R2 = scipy.linalg.solve_triangular(U, np.eye(24), lower=False)
    np.testing.assert_allclose(f["R"], R2, rtol=1e-9, atol=1e-12)


def test_trailing_block_property():
    """R[k:,k:] is the factor of the trailing principal block H_d[k:,k:] alone."""
    H, _ = _rand_spd(20, 3, 1.0)
    f = oracle.inverse_hessian_factor(H, 0.01)
    for k in (1, 7, 13):
        Rk = oracle.inverse_hessian_factor(f["Hd"][k:, k:], 0.0)["R"]
        np.testing.assert_allclose(f["R"][k:, k:], Rk, rtol=1e-10, atol=1e-12)


# ---------------------------------------------------------------------------------------------
# P11: the quantizer grid (definition invariants + brute-force nearest grid point)
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("bits", [2, 3, 4, 8])
def test_quantizer_grid_invariants(bits):
    rng = np.random.default_rng(bits)
    W = (rng.standard_normal((40, 64)) * rng.uniform(0.001, 1, (40, 1))).astype(np.float32)
    W[3] = np.abs(W[3])          # all positive: lo = 0
    W[4] = -np.abs(W[4])         # all negative: hi = 0
    W[5] = 0.0                   # degenerate: range [-1, 1]
    maxq = 2 ** bits - 1
    s, z = oracle.quant_params(W, bits)
    q, wh = oracle.quantize(W, s[:, None], z[:, None], bits)
    assert q.max() <= maxq and s.dtype == np.float32
    assert np.all(z == np.round(z)) and np.all((0 <= z) & (z <= maxq))
    # dequantized value is s * (q - z) in float32, and 0 is on the grid (code z)
    np.testing.assert_array_equal(wh, (s[:, None] * (q.astype(np.float32) - z[:, None])))
    _, w0 = oracle.quantize(np.zeros((40, 1)), s[:, None], z[:, None], bits)
    assert np.all(w0 == 0)
    # every value in range is within half a step of its grid point
    assert np.all(np.abs(W - wh) <= 0.5 * s[:, None] * (1 + 1e-5))
    assert z[3] == 0 and z[4] == maxq
    s5 = np.float32(np.float32(2.0) / np.float32(maxq))
    assert s[5] == s5 and z[5] == np.rint(np.float32(np.float32(1.0) / s5))
    # brute force: the code is the nearest of the 2^k grid points (no exact ties in random data)
    grid = s[:, None] * (np.arange(maxq + 1)[None, :] - z[:, None])
    brute = np.abs(W[:, :, None] - grid[:, None, :]).argmin(axis=2)
    keep = np.ones(40, bool)
    keep[5] = False
    np.testing.assert_array_equal(q[keep], brute[keep])


def test_quantizer_rounds_half_to_even():
    s, z = np.float32(0.5), np.float32(0)
    q, _ = oracle.quantize(np.array([0.75, 0.25, 1.25]), s, z, 3)   # x/s = 1.5, 0.5, 2.5
    assert list(q) == [2, 0, 2]


# ---------------------------------------------------------------------------------------------
# P1: diagonal H -> no compensation -> GPTQ is round-to-nearest, bit for bit
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("group,block", [(-1, 32), (32, 32), (16, 64), (64, 32)])
def test_identity_hessian_is_rtn(group, block):
    W = _rand_W(16, 128, 3)
    for H in (np.eye(128), np.diag(np.random.default_rng(4).uniform(0.1, 9, 128))):
        R = oracle.inverse_hessian_factor(H)["R"]
        assert np.all(R == np.diag(np.diag(R)))
        g = oracle.gptq_quantize(W, R, 4, group, block)
        r = oracle.rtn_quantize(W, 4, group)
        for k in ("codes", "scales", "zeros", "W_hat"):
            np.testing.assert_array_equal(g[k], r[k])


# ---------------------------------------------------------------------------------------------
# P2: Cholesky-row schedule == the naive OBS explicit inverse-Hessian downdate sequence
# ---------------------------------------------------------------------------------------------

def _obs_naive(W, Hd, bits):
    """Per-row grid from the original W; for p = 0..c-1: quantize w_p, move the remaining weights by
    dw_p * Hinv[p, rem] / Hinv[p, p], then downdate Hinv -= Hinv[:, p] Hinv[p, :] / Hinv[p, p]."""
    W = np.array(W, dtype=np.float64)
    rows, c = W.shape
    s, z = oracle.quant_params(W, bits)
    codes = np.zeros((rows, c), np.uint8)
    for r in range(rows):
        Hinv = np.linalg.inv(Hd)
        w = W[r].copy()
        for p in range(c):
            q, wh = oracle.quantize(w[p:p + 1], s[r], z[r], bits)
            codes[r, p] = q[0]
            dw = float(wh[0]) - w[p]
            w[p] = float(wh[0])
            w[p + 1:] += dw * Hinv[p, p + 1:] / Hinv[p, p]
            Hinv = Hinv - np.outer(Hinv[:, p], Hinv[p, :]) / Hinv[p, p]
    return codes


@pytest.mark.parametrize("c", [2, 3, 5, 8])
def test_cholesky_rows_equal_obs_downdates(c):
    H, _ = _rand_spd(c, 10 + c, 1.0)
    W = _rand_W(12, c, 20 + c)
    f = oracle.inverse_hessian_factor(H, 0.01)
    g = oracle.gptq_quantize(W, f["R"], 3, -1, block=c)
    np.testing.assert_array_equal(g["codes"], _obs_naive(W, f["Hd"], 3))


# ---------------------------------------------------------------------------------------------
# P3: the three-weight example (hand-solved golden fixture) and the general Schur-complement form
# ---------------------------------------------------------------------------------------------

def _read_fixture(name):
    vals = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.split("#")[0].strip()
        if line:
            k, v = (t.strip() for t in line.split("="))
            vals[k] = v
    return vals


def test_three_weight_example_fixture():
    fx = _read_fixture("obq_three_weight.txt")
    H = np.array([[float(t) for t in fx[f"H_row{i}"].split()] for i in range(3)])
    w = np.array([[float(t) for t in fx["w"].split()]])
    dw1, dw2 = Fraction(fx["dw1"]), Fraction(fx["dw2"])
    R = oracle.inverse_hessian_factor(H, 0.0)["R"]
    g = oracle.gptq_quantize(w, R, int(fx["bits"]), -1, block=3)
    assert Fraction(float(g["W_hat"][0, 0])) - Fraction(w[0, 0]) == dw1
    # the second weight was quantized at its compensated value w2 + dw2
    assert g["w_in"][0, 1] == pytest.approx(float(w[0, 1] + dw2), abs=1e-14)
    # the compensation direction matches the hand solution for both remaining weights
    dw3 = Fraction(fx["dw3"])
    np.testing.assert_allclose(R[0, 1:] / R[0, 0] * float(-dw1),
                               [-float(dw2), -float(dw3)], rtol=1e-13)


def test_compensation_is_schur_optimum():
    """After fixing dw_1, the remaining weights move by -H_rr^{-1} H_r1 dw_1 (the linear system)."""
    H, _ = _rand_spd(6, 7, 1.0)
    W = _rand_W(5, 6, 8)
    f = oracle.inverse_hessian_factor(H, 0.01)
    Hd = f["Hd"]
    g = oracle.gptq_quantize(W, f["R"], 4, -1, block=6)
    dw1 = g["W_hat"][:, 0].astype(np.float64) - W[:, 0]
    want = W[:, 1] + np.linalg.solve(Hd[1:, 1:], -np.outer(Hd[1:, 0], dw1))[0]
    np.testing.assert_allclose(g["w_in"][:, 1], want, rtol=1e-12, atol=1e-15)


# ---------------------------------------------------------------------------------------------
# P4: lazy batches == eager schedule; P5: the per-row loss identity; P6: scale invariance
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("group,block", [(-1, 32), (-1, 128), (-1, 48), (32, 32), (32, 128),
                                         (128, 32), (64, 64)])
def test_lazy_equals_unbatched(group, block):
    W = _rand_W(24, 256, 30)
    H, _ = _rand_spd(256, 31, 1.5)
    R = oracle.inverse_hessian_factor(H)["R"]
    a = oracle.gptq_quantize(W, R, 4, group, block)
    b = oracle.gptq_quantize_unbatched(W, R, 4, group)
    np.testing.assert_array_equal(a["codes"], b["codes"])
    np.testing.assert_array_equal(a["W_hat"], b["W_hat"])
    np.testing.assert_allclose(a["err"], b["err"], rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("group,lead", [(-1, 64), (-1, 96), (32, 64)])
def test_leading_columns_depend_only_on_leading_block(group, lead):
    """Columns 0..k-1 of a row are quantized from R's leading k x k block alone (updates only run
    to the right), so a run on the leading columns reproduces them -- given the grid of the whole
    row in per-row mode (its parameters come from the original, full row)."""
    W = _rand_W(12, 160, 42)
    H, _ = _rand_spd(160, 43, 1.5)
    R = oracle.inverse_hessian_factor(H)["R"]
    full = oracle.gptq_quantize(W, R, 3, group, 32)
    grid = oracle.quant_params(W, 3) if group <= 0 else None
    lead_run = oracle.gptq_quantize(W[:, :lead], R[:lead, :lead], 3, group, 32, row_grid=grid)
    for k in ("codes", "W_hat"):
        np.testing.assert_array_equal(lead_run[k], full[k][:, :lead])
    np.testing.assert_allclose(lead_run["err"], full["err"][:, :lead], rtol=1e-12, atol=1e-15)
    if group <= 0:
        # without the whole row's grid, the leading columns alone give another grid
        alone = oracle.gptq_quantize(W[:, :lead], R[:lead, :lead], 3, group, 32)
        assert not np.array_equal(alone["scales"], full["scales"])
        with pytest.raises(ValueError):
            oracle.gptq_quantize(W, R, 3, 32, 32, row_grid=grid)


def test_loss_identity_sum_of_squared_errors():
    """(W_hat - W) H_d (W_hat - W)^T = sum_j e_j^2 per row, since W_hat - W = -e R and
    H_d = R^{-1} R^{-T} (the LDL view of the OptRot page, Definition 3.2)."""
    W = _rand_W(10, 96, 40)
    H, _ = _rand_spd(96, 41, 1.0)
    f = oracle.inverse_hessian_factor(H)
    g = oracle.gptq_quantize(W, f["R"], 3, 32, 32)
    dW = g["W_hat"].astype(np.float64) - W
    lhs = np.einsum("ij,jk,ik->i", dW, f["Hd"], dW)
    np.testing.assert_allclose(lhs, g["err_sq"], rtol=1e-9)


def test_codes_invariant_to_hessian_scale():
    W = _rand_W(16, 64, 50)
    H, _ = _rand_spd(64, 51, 1.0)
    a = oracle.gptq_quantize(W, oracle.inverse_hessian_factor(H)["R"], 4, -1, 32)
    b = oracle.gptq_quantize(W, oracle.inverse_hessian_factor(4.0 * H)["R"], 4, -1, 32)
    for k in ("codes", "W_hat", "scales", "zeros"):
        np.testing.assert_array_equal(a[k], b[k])
    c = oracle.gptq_quantize(W, oracle.inverse_hessian_factor(3.0 * H)["R"], 4, -1, 32)
    assert (c["codes"] == a["codes"]).mean() > 0.999


# ---------------------------------------------------------------------------------------------
# Objective: metric identity, brute-force bound, GPTQ beats RTN on the test workloads (P9)
# ---------------------------------------------------------------------------------------------

def test_layer_error_equals_output_error():
    rng = np.random.default_rng(60)
    X = rng.standard_normal((300, 12))
    W = _rand_W(4, 12, 61)
    Wh = W + rng.standard_normal(W.shape) * 1e-3
    direct = np.sum(((W - Wh) @ X.T) ** 2) / np.sum((W @ X.T) ** 2)
    assert oracle.layer_error(W, Wh, oracle.hessian(X)) == pytest.approx(direct, rel=1e-10)


def test_gptq_not_below_integer_optimum():
    """Brute force over all codes of a 3-weight row on GPTQ's grid: GPTQ cannot beat the optimum,
    and the optimum's loss is what an exhaustive search finds."""
    H, _ = _rand_spd(3, 70, 1.0)
    Hd = oracle.damp(H)[0]
    R = oracle.inverse_hessian_factor(H)["R"]
    for seed in range(20):
        w = _rand_W(1, 3, 100 + seed, std=1.0)
        g = oracle.gptq_quantize(w, R, 2, -1, 3)
        s, z = g["scales"][0, 0], g["zeros"][0, 0]
        def loss(k):
            grid = (s * (np.array(k, np.float32) - np.float32(z))).astype(np.float64)
            d = grid - w[0]
            return float(d @ Hd @ d)
        best = min(loss(k) for k in itertools.product(range(4), repeat=3))
        dw = g["W_hat"][0].astype(np.float64) - w[0]
        assert dw @ Hd @ dw >= best - 1e-12


@pytest.mark.parametrize("kind", ["tiny", "heavy"])
def test_gptq_beats_rtn_on_workloads(kind):
    spec = synth.TINY if kind == "tiny" else synth.scaled_spec(synth.ATTN, 64, 256, 2048)
    W, X = synth.weights_np(spec, 0), synth.inputs_np(spec, 0)
    out = oracle.gptq_layer(W, X, spec.bits, spec.group, spec.block, spec.damp)
    rtn = oracle.rtn_quantize(W, spec.bits, spec.group)
    e_rtn = oracle.layer_error(W, rtn["W_hat"], out["H"])
    # independent input channels make H nearly diagonal, so the gain is modest but always there
    assert out["rel_err"] < e_rtn


def test_shape_rules():
    with pytest.raises(ValueError):
        oracle.check_shapes(128, 48, 32)      # groups that do not nest with blocks
    with pytest.raises(ValueError):
        oracle.check_shapes(100, 64, 64)      # cols not a multiple of the group
    with pytest.raises(ValueError):
        oracle.damp(np.zeros((3, 3)))          # all-zero calibration input
