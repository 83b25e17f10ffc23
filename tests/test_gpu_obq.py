"""GPU parity of the OBQ reference (through the C ABI) against the fp64 oracle.

Both sides perform the same IEEE operations in the same order (fp64 weights and inverse Hessian,
float32 grid decisions, no fused multiply-adds, greedy ties to the lowest column), so the greedy
order, the codes, W_hat, the grid and the per-row loss must agree bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(rows, cols, seed):
    """Seeded float32 weights and the fp64 inverse of a damped 2 X^T X / N (plain NumPy)."""
    rng = np.random.default_rng(seed)
    X = rng.standard_normal((8 * cols, cols)) * np.exp(rng.uniform(-1.5, 1.5, cols))
    H = 2.0 * (X.T @ X) / X.shape[0]
    Hd = H + 0.01 * np.mean(np.diag(H)) * np.eye(cols)
    W = (rng.standard_normal((rows, cols)) * 0.02).astype(np.float32)
    return W, np.linalg.inv(Hd)


def _run_gpu(W, Hinv, bits, greedy):
    rows, cols = W.shape
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    W_hat = torch.empty(rows, cols, device=DEV)
    order = torch.empty(rows, cols, dtype=torch.int32, device=DEV)
    loss = torch.empty(rows, dtype=torch.float64, device=DEV)
    scales = torch.empty(rows, device=DEV)
    zeros = torch.empty(rows, dtype=torch.uint8, device=DEV)
    _lib.obq_quantize(torch.from_numpy(W).to(DEV), torch.from_numpy(Hinv).to(DEV), bits, codes,
                      W_hat, order, loss, scales, zeros, greedy=greedy)
    torch.cuda.synchronize()
    return {k: v.cpu().numpy() for k, v in dict(codes=codes, W_hat=W_hat, order=order, loss=loss,
                                                   scales=scales, zeros=zeros).items()}


@pytest.mark.parametrize("rows,cols,bits", [(24, 128, 4), (17, 100, 3), (9, 37, 2), (5, 1, 4),
                                            (40, 64, 8)])
@pytest.mark.parametrize("greedy", [True, False])
def test_obq_bit_exact(rows, cols, bits, greedy):
    W, Hinv = _problem(rows, cols, rows + cols)
    got = _run_gpu(W, Hinv, bits, greedy)
    ref = oracle.obq_quantize(W, Hinv, bits, order="greedy" if greedy else "natural")
    assert np.array_equal(got["order"], ref["order"])
    assert np.array_equal(got["codes"], ref["codes"])
    assert np.array_equal(got["W_hat"], ref["W_hat"])
    assert np.array_equal(got["loss"], ref["loss"])
    assert np.array_equal(got["scales"], ref["scales"][:, 0])
    assert np.array_equal(got["zeros"], ref["zeros"][:, 0])


def test_obq_optional_outputs_and_flat_row():
    W, Hinv = _problem(6, 64, 3)
    W[2] = 0.0                                              # all-zero row: grid [-1, 1]
    rows, cols = W.shape
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    W_hat = torch.empty(rows, cols, device=DEV)
    _lib.obq_quantize(torch.from_numpy(W).to(DEV), torch.from_numpy(Hinv).to(DEV), 4, codes,
                      W_hat)
    torch.cuda.synchronize()
    ref = oracle.obq_quantize(W, Hinv, 4)
    assert np.array_equal(codes.cpu().numpy(), ref["codes"])
    assert np.array_equal(W_hat.cpu().numpy(), ref["W_hat"])


def test_obq_measured_layer_sampled_rows():
    """4096 rows x 128 columns, the configuration the benchmark times; sampled rows (first and
    last included) against the oracle, bit for bit."""
    W, Hinv = _problem(4096, 128, 11)
    got = _run_gpu(W, Hinv, 4, True)
    sel = np.array([0, 1, 2047, 3000, 4095])
    ref = oracle.obq_quantize(W[sel], Hinv, 4)
    assert np.array_equal(got["order"][sel], ref["order"])
    assert np.array_equal(got["codes"][sel], ref["codes"])
    assert np.array_equal(got["W_hat"][sel], ref["W_hat"])
    assert np.array_equal(got["loss"][sel], ref["loss"])
