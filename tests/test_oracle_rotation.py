"""Pins for the Hadamard-rotation oracle against independent formulations: the closed form of the
Sylvester matrix, a butterfly transform written out by hand, orthogonality, invariance of the
layer output, the conjugated Hessian and closed-form incoherence values."""
import numpy as np
import pytest

from oracle import rotation
import oracle


def _signs(n, seed):
    return np.where(np.random.default_rng(seed).random(n) < 0.5, -1.0, 1.0)


@pytest.mark.parametrize("n,b", [(32, 32), (96, 32), (4096, 4096), (11008, 256), (12288, 4096),
                                 (49152, 4096), (8192, 4096)])
def test_block_order(n, b):
    assert rotation.hadamard_block(n) == b


@pytest.mark.parametrize("n", [64, 96])
def test_matrix_is_the_sylvester_closed_form(n):
    """Entry (i, j) of H_b is (-1)^popcount(i & j); Q is block diagonal with H_b / sqrt(b)."""
    b = rotation.hadamard_block(n)
    Q = rotation.rotation_matrix(n)
    for i in range(n):
        for j in range(n):
            if i // b != j // b:
                assert Q[i, j] == 0.0
            else:
                sign = -1.0 if bin((i % b) & (j % b)).count("1") % 2 else 1.0
                assert Q[i, j] == pytest.approx(sign / np.sqrt(b), rel=1e-15)


def test_orthogonal_with_signs():
    Q = rotation.rotation_matrix(96, _signs(96, 1))
    assert np.allclose(Q @ Q.T, np.eye(96), atol=1e-14)


def test_blockwise_rotate_equals_the_full_matrix_product():
    rng = np.random.default_rng(9)
    X = rng.standard_normal((5, 96))
    s = _signs(96, 10)
    Q = rotation.rotation_matrix(96, s)
    assert np.allclose(rotation.rotate(X, s), X @ Q, rtol=1e-13, atol=1e-14)
    assert np.allclose(rotation.rotate_abs_terms(X), np.abs(X) @ np.abs(Q), rtol=1e-13)


def _butterfly(v):
    """Unnormalised fast Walsh-Hadamard transform, written out: stage h pairs i and i + h."""
    v = list(map(float, v))
    h = 1
    while h < len(v):
        for i in range(0, len(v), 2 * h):
            for k in range(i, i + h):
                a, c = v[k], v[k + h]
                v[k], v[k + h] = a + c, a - c
        h *= 2
    return np.array(v)


def test_rotate_equals_signed_butterfly():
    """rotate(x, s) = FWHT(s * x) / sqrt(n) for a power-of-two n (x Q with Q = diag(s) H / sqrt n)."""
    rng = np.random.default_rng(2)
    n = 64
    x = rng.standard_normal(n)
    s = _signs(n, 3)
    assert np.allclose(rotation.rotate(x[None, :], s)[0], _butterfly(s * x) / np.sqrt(n),
                       rtol=1e-13, atol=1e-14)


def test_layer_output_and_hessian_invariance():
    """(W Q)(X Q)^T = W X^T, and the rotated Hessian is Q^T H Q."""
    rng = np.random.default_rng(4)
    n = 128
    W = rng.standard_normal((16, n))
    X = rng.standard_normal((200, n))
    s = _signs(n, 5)
    assert np.allclose(rotation.rotate(W, s) @ rotation.rotate(X, s).T, W @ X.T, rtol=1e-12,
                       atol=1e-11)
    Q = rotation.rotation_matrix(n, s)
    assert np.allclose(oracle.hessian(rotation.rotate(X, s)), Q.T @ oracle.hessian(X) @ Q,
                       rtol=1e-12, atol=1e-12)


def test_incoherence_closed_forms_and_outlier_spreading():
    # A matrix of equal magnitudes has mu = 1, the minimum; one non-zero entry gives sqrt(m n).
    assert rotation.weight_incoherence(np.ones((8, 32))) == pytest.approx(1.0)
    E = np.zeros((8, 32))
    E[3, 5] = 2.0
    assert rotation.weight_incoherence(E) == pytest.approx(np.sqrt(8 * 32))
    # A planted outlier is spread by the rotation: incoherence drops.
    rng = np.random.default_rng(6)
    W = rng.standard_normal((64, 256)) * 0.02
    W[:, 17] *= 50.0
    before = rotation.weight_incoherence(W)
    after = rotation.weight_incoherence(rotation.rotate(W, _signs(256, 7)))
    assert after < 0.5 * before
