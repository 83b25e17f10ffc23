"""GPU parity of the randomized Hadamard rotation (through the C ABI) against the fp64 oracle.

Tolerance from the arithmetic, per output with T = sum_j |x_j| |Q_ji| (oracle): bf16 and fp32
inputs are exact in fp32 and sign flips are exact; the log2(b) butterfly stages each round once
relative to the partial sums they add (<= log2(b) * 2^-24 * T, with slack for the second-order
terms), and for odd log2(b) the rounded constant 1/sqrt(b) and the final scaling each add at most
2^-24 |y| (|y| <= T): together <= (log2(b) + 2) * 2^-24 * T. A bf16 output adds its rounding, at most 2^-8
of the value (round to nearest, 8-bit significand).
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _signs(n, seed):
    return np.where(np.random.default_rng(seed).random(n) < 0.5, -1.0, 1.0)


def _sign_bits(signs):
    """Bit j % 32 of word j // 32 set where sign j is -1 (little-endian bit order)."""
    bits = np.packbits((np.asarray(signs) < 0).astype(np.uint8), bitorder="little")
    return torch.from_numpy(bits.view("<u4").view(np.int32).copy()).to(DEV)


def _input(rows, n, seed, dtype):
    spec = synth.scaled_spec(synth.ATTN, 1, n, rows)
    x = synth.inputs_torch(spec, seed, "cpu")        # heavy-tailed, bf16 values
    return x if dtype == torch.bfloat16 else x.float() * 0.37


def _check(X, Y, signs):
    n = X.shape[1]
    b = oracle.hadamard_block(n)
    L = int(np.log2(b))
    Xf = X.float().cpu().numpy()
    ref = oracle.rotate(Xf, signs)
    terms = oracle.rotate_abs_terms(Xf)
    tol = (L + 2) * 2.0 ** -24 * terms
    if Y.dtype == torch.bfloat16:
        tol = tol * (1 + 2.0 ** -8) + 2.0 ** -8 * np.abs(ref)
    y = Y.double().cpu().numpy()
    err = np.abs(y - ref)
    assert np.all(err <= tol), float((err - tol).max())


@pytest.mark.parametrize("n", [32, 64, 96, 256, 1024, 2048, 4096, 11008, 12288])
@pytest.mark.parametrize("xd,yd", [(torch.bfloat16, torch.float32), (torch.float32, torch.float32),
                                   (torch.bfloat16, torch.bfloat16),
                                   (torch.float32, torch.bfloat16)])
def test_rotate_matches_oracle(n, xd, yd):
    rows = 37
    X = _input(rows, n, 3, xd)
    signs = _signs(n, 4)
    Y = torch.empty(rows, n, dtype=yd, device=DEV)
    _lib.hadamard_rotate(X.to(DEV), Y, _sign_bits(signs))
    torch.cuda.synchronize()
    _check(X, Y, signs)


def test_rotate_without_signs_ragged_rows_strided():
    rows, n = 5, 4096
    X = _input(rows, n, 5, torch.bfloat16)
    Xd = torch.zeros(rows, n + 64, dtype=torch.bfloat16, device=DEV)
    Xd[:, :n] = X.to(DEV)
    Yd = torch.full((rows, n + 32), float("nan"), device=DEV)
    _lib.hadamard_rotate(Xd[:, :n], Yd[:, :n])
    torch.cuda.synchronize()
    _check(X, Yd[:, :n], None)
    assert torch.isnan(Yd[:, n:]).all()


@pytest.mark.parametrize("n,rows", [(4096, 9), (256, 129), (12288, 3)])
def test_rotate_in_place(n, rows):
    X = _input(rows, n, 6, torch.bfloat16)
    signs = _signs(n, 7)
    Xd = X.to(DEV).clone()
    _lib.hadamard_rotate(Xd, Xd, _sign_bits(signs))
    torch.cuda.synchronize()
    _check(X, Xd, signs)


@pytest.mark.parametrize("xd,yd", [(torch.bfloat16, torch.bfloat16), (torch.float32, torch.float32)])
def test_rotate_persistent_loop_every_row(xd, yd):
    """2500 rows of order-4096 blocks: more segments than the persistent grid holds, so CTAs loop
    (prefetching the next segment) with a ragged last round; every row against the oracle."""
    rows, n = 2500, 4096
    X = _input(rows, n, 14, xd)
    signs = _signs(n, 15)
    Y = torch.empty(rows, n, dtype=yd, device=DEV)
    _lib.hadamard_rotate(X.to(DEV), Y, _sign_bits(signs))
    torch.cuda.synchronize()
    _check(X, Y, signs)


@pytest.mark.parametrize("n", [49152, 69632])
def test_rotate_many_blocks_per_row(n):
    """12 blocks of 4096 per row (the fc2 input width; signs of the whole row in shared memory)
    and 17 blocks (wider than the shared sign table: the three-pass kernel)."""
    rows = 3
    X = _input(rows, n, 16, torch.bfloat16)
    signs = _signs(n, 17)
    Y = torch.empty(rows, n, dtype=torch.bfloat16, device=DEV)
    _lib.hadamard_rotate(X.to(DEV), Y, _sign_bits(signs))
    torch.cuda.synchronize()
    _check(X, Y, signs)


def test_rotation_preserves_layer_products():
    """(W Q)(X Q)^T on the GPU outputs equals W X^T within the rounding of the two rotations."""
    rows, n, tokens = 16, 4096, 64
    W = torch.randn(rows, n, generator=torch.Generator().manual_seed(8)) * 0.02
    X = _input(tokens, n, 9, torch.float32)
    signs = _sign_bits(_signs(n, 10))
    Wr = torch.empty(rows, n, device=DEV)
    Xr = torch.empty(tokens, n, device=DEV)
    _lib.hadamard_rotate(W.to(DEV), Wr, signs)
    _lib.hadamard_rotate(X.to(DEV), Xr, signs)
    torch.cuda.synchronize()
    got = Wr.double().cpu() @ Xr.double().cpu().T
    ref = W.double() @ X.double().T
    scale = W.double().norm(dim=1)[:, None] * X.double().norm(dim=1)[None, :]
    assert torch.all((got - ref).abs() <= 1e-5 * scale)


def test_rotate_deterministic_and_empty():
    X = _input(64, 4096, 11, torch.bfloat16).to(DEV)
    Y1 = torch.empty(64, 4096, dtype=torch.bfloat16, device=DEV)
    Y2 = torch.empty_like(Y1)
    _lib.hadamard_rotate(X, Y1)
    _lib.hadamard_rotate(X, Y2)
    E = torch.empty(0, 4096, device=DEV)
    _lib.hadamard_rotate(E, E)
    torch.cuda.synchronize()
    assert torch.equal(Y1, Y2)


def test_rotate_fullsize_calibration_sampled():
    """The 262144 x 4096 bf16 calibration input in the launch configuration the benchmark times,
    rotated in place; sampled rows (first and last tiles included) against the oracle."""
    spec = synth.ATTN
    X = synth.inputs_torch(spec, 0, DEV)
    sel = np.unique(np.concatenate([np.arange(4), np.arange(spec.n_tokens - 4, spec.n_tokens),
                                    np.random.default_rng(1).choice(spec.n_tokens, 24,
                                                                    replace=False)]))
    sel_t = torch.from_numpy(sel).to(DEV)
    before = X[sel_t].cpu()
    signs = _signs(spec.cols, 12)
    _lib.hadamard_rotate(X, X, _sign_bits(signs))
    torch.cuda.synchronize()
    _check(before, X[sel_t], signs)


def test_rotate_medium_tokens():
    """65536 tokens x 4096 channels of bf16 calibration input (512 MB, larger than L2), rotated
    into a separate bf16 buffer; sampled rows against the oracle."""
    spec = synth.scaled_spec(synth.ATTN, 1, 4096, 65536)
    X = synth.inputs_torch(spec, 2, DEV)
    Y = torch.empty_like(X)
    signs = _signs(4096, 13)
    _lib.hadamard_rotate(X, Y, _sign_bits(signs))
    torch.cuda.synchronize()
    sel_t = torch.from_numpy(np.array([0, 1, 777, 40000, 65534, 65535])).to(DEV)
    _check(X[sel_t].cpu(), Y[sel_t], signs)

