"""Pins for the OBQ oracle against independent formulations: the hand-solved three-weight example,
explicit solves of the reduced problem at every greedy step, the GPTQ oracle's fixed-order
Cholesky schedule, round-to-nearest for a diagonal Hessian and the proxy-loss identity."""
from fractions import Fraction
import os

import numpy as np
import pytest

import oracle
from oracle import obq

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _fixture(name):
    out = {}
    for line in open(os.path.join(GOLDEN, name)):
        line = line.strip()
        if line and not line.startswith("#"):
            k, v = line.split("=")
            out[k.strip()] = v.split()
    return out


def _problem(r, c, seed):
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((6 * c, c)) * np.exp(rng.uniform(-1, 1, c))
    H = oracle.hessian(X)
    Hd = oracle.damp(H)[0]
    W = rng.standard_normal((r, c)) * 0.02
    return W, Hd


def test_first_compensation_matches_the_three_weight_example():
    fx = _fixture("obq_three_weight.txt")
    H = np.array([[float(v) for v in fx[f"H_row{i}"]] for i in range(3)])
    w = np.array([float(v) for v in fx["w"]])
    bits = int(fx["bits"][0])
    s, z = oracle.quant_params(w[None, :], bits)
    o = obq.obq_row(w, np.linalg.inv(H), s[0], z[0], bits, order="natural", trace=True)
    after = o["states"][0]
    assert float(o["W_hat"][0]) - w[0] == float(Fraction(fx["dw1"][0]))
    assert after[1] - w[1] == pytest.approx(float(Fraction(fx["dw2"][0])), abs=1e-15)
    assert after[2] - w[2] == pytest.approx(float(Fraction(fx["dw3"][0])), abs=1e-15)


def _greedy_by_explicit_solves(w, Hd, s, z, bits):
    """OBQ's greedy search re-derived at every step from the reduced problem: for the remaining
    set R and each p in R, fixing w_p to its grid value costs d_p^2 / [inv(H_RR)]_pp and moves the
    other remaining weights by -H_{R',R'}^-1 H_{R',p} (q_p - w_p) (R' = R minus p)."""
    w = w.copy()
    R = list(range(len(w)))
    order, codes = [], np.zeros(len(w), np.uint8)
    while R:
        q, wh = oracle.quantize(w, s, z, bits)
        d = w - wh.astype(np.float64)
        inv_RR = np.linalg.inv(Hd[np.ix_(R, R)])
        costs = [d[p] ** 2 / inv_RR[k, k] for k, p in enumerate(R)]
        k = int(np.argmin(costs))
        p = R[k]
        rest = [x for x in R if x != p]
        if rest:
            delta = -np.linalg.solve(Hd[np.ix_(rest, rest)], Hd[rest, p]) * (wh[p] - w[p])
            w[rest] += delta
        order.append(p)
        codes[p] = q[p]
        R = rest
    return np.array(order), codes


@pytest.mark.parametrize("seed", [1, 2, 3])
def test_greedy_order_matches_explicit_reduced_solves(seed):
    W, Hd = _problem(4, 6, seed)
    s, z = oracle.quant_params(W, 3)
    Hinv = np.linalg.inv(Hd)
    for i in range(W.shape[0]):
        o = obq.obq_row(W[i], Hinv, s[i], z[i], 3)
        order, codes = _greedy_by_explicit_solves(W[i], Hd, s[i], z[i], 3)
        assert np.array_equal(o["order"], order)
        assert np.array_equal(o["codes"], codes)


def test_natural_order_is_gptq():
    """OBQ forced to the left-to-right order is GPTQ: the GPTQ oracle's Cholesky-row schedule
    (R = upper factor of H^-1) gives the same codes and weights."""
    W, Hd = _problem(16, 24, 4)
    Hinv = np.linalg.inv(Hd)
    o = obq.obq_quantize(W, Hinv, 4, order="natural")
    R = np.linalg.cholesky(Hinv).T
    g = oracle.gptq_quantize(W, R, 4, group=-1, block=1)
    assert np.array_equal(o["codes"], g["codes"])
    assert np.allclose(o["W_hat"], g["W_hat"], rtol=0, atol=1e-6)
    assert np.array_equal(o["order"], np.tile(np.arange(24), (16, 1)))


def test_diagonal_hessian_is_round_to_nearest():
    rng = np.random.default_rng(5)
    W = rng.standard_normal((8, 16)) * 0.02
    Hd = np.diag(rng.uniform(0.5, 2.0, 16))
    o = obq.obq_quantize(W, np.linalg.inv(Hd), 4)
    rtn = oracle.rtn_quantize(W, 4)
    assert np.array_equal(o["codes"], rtn["codes"])
    assert np.array_equal(o["W_hat"], rtn["W_hat"])


def test_loss_is_the_proxy_loss_of_the_result():
    """Summed d_p^2 / H^-1[p, p] over the steps equals (w_hat - w)^T H_d (w_hat - w)."""
    W, Hd = _problem(6, 20, 6)
    o = obq.obq_quantize(W, np.linalg.inv(Hd), 3)
    dW = o["W_hat"].astype(np.float64) - W
    direct = np.einsum("ij,jk,ik->i", dW, Hd, dW)
    assert np.allclose(o["loss"], direct, rtol=1e-9)
    assert all(sorted(row) == list(range(20)) for row in o["order"])
