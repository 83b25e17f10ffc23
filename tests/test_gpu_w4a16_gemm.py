"""The W4A16 product for batches of more than 16 activation rows (the tensor-core form behind
gptq_w4a16_matmul), checked per output against the fp64 oracle within the bound derived for the
decode-size product: q - z and x are exact in bf16, so every product is exact; a 128-column
chunk's sum takes eight tensor-core accumulations (at most 2 ulp each, 8 * 2^-22 T), and each
chunk's scaled sum is added in fp32 (one rounding per chunk), T = sum_c |x_c w_hat_c|. A dropped
or misplaced column, a wrong group or a transposed tile moves y by about T / cols, far beyond it.
Cases: one, two and a ragged last activation tile, per-row and grouped scales, ragged rows and
columns, strided input and output, extreme codes, determinism, and the benchmark's layers."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _bound(cols):
    nchunks = -(-cols // 128)
    return 8 * 2.0 ** -22 + (nchunks + 16) * 2.0 ** -24


def _x(n, cols, seed):
    return synth.inputs_torch(synth.scaled_spec(synth.ATTN, 1, cols, n), seed, "cpu")


def _run(codes, scales, zeros, group, X, ldx=None, ldy=None):
    rows, cols = codes.shape
    n = X.shape[0]
    packed = torch.empty(rows, cols // 8, dtype=torch.int32, device=DEV)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    _lib.pack_codes_4bit(codes.to(DEV), packed, info)
    Xd = torch.zeros(n, ldx or cols, dtype=torch.bfloat16, device=DEV)
    Xd[:, :cols] = X.to(DEV)
    Y = torch.full((n, ldy or rows), float("nan"), device=DEV)
    _lib.w4a16_matmul(packed, scales.to(DEV), zeros.to(DEV), group, Xd[:, :cols], Y[:, :rows], info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    if ldy is not None:
        assert torch.isnan(Y[:, rows:]).all()            # columns past rows untouched
    return Y[:, :rows].double().cpu().numpy(), packed


def _check(codes, scales, zeros, group, X, rows_sel=None, **kw):
    y, _ = _run(codes, scales, zeros, group, X, **kw)
    rows, cols = codes.shape
    sel = np.arange(rows) if rows_sel is None else np.asarray(rows_sel)
    words = oracle.pack_codes(codes.numpy()[sel])
    Xf = X.float().numpy()
    ref = oracle.w4a16_matmul(words, scales.numpy()[sel], zeros.numpy()[sel], group, Xf)
    terms = oracle.w4a16_abs_terms(words, scales.numpy()[sel], zeros.numpy()[sel], group, Xf)
    assert np.all(np.isfinite(y[:, sel]))
    err = np.abs(y[:, sel] - ref)
    assert np.all(err <= _bound(cols) * terms), float((err / terms).max())
    return y


@pytest.mark.parametrize("rows,cols,group,n", [
    (128, 256, 128, 17),      # smallest batch: a 32-row activation tile, rows past n unused
    (256, 1024, 128, 32),     # one full 32-row tile, two weight tiles
    (100, 4096, 128, 64),     # ragged weight tile, one 64-row activation tile
    (257, 1024, 256, 100),    # group of two chunks, ragged rows, one 128-row tile
    (48, 4000, -1, 128),      # per-row scales, ragged last chunk (4000 = 31 * 128 + 32)
    (300, 2048, 128, 256),    # two activation tiles
    (130, 1536, 128, 200),    # a ragged second activation tile
])
def test_gemm_matches_oracle(rows, cols, group, n):
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, group, 61 + rows)
    _check(codes, scales, zeros, group, _x(n, cols, 13))


def test_gemm_strided_x_and_y():
    rows, cols = 200, 768
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, 128, 71)
    _check(codes, scales, zeros, 128, _x(40, cols, 14), ldx=cols + 64, ldy=rows + 24)


def test_gemm_extreme_codes_and_zeros():
    rows, cols = 128, 512
    codes = torch.zeros(rows, cols, dtype=torch.uint8)
    codes[::2] = 15
    zeros = torch.zeros(rows, 4, dtype=torch.uint8)
    zeros[1::2] = 15
    scales = torch.full((rows, 4), 0.0078125)
    _check(codes, scales, zeros, 128, _x(48, cols, 15))


def test_gemm_deterministic_and_matches_decode_rows():
    """Two calls give identical results, and each output row equals the decode-size product of
    that activation row within the same bound."""
    rows, cols = 384, 4096
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, 128, 81)
    X = _x(64, cols, 16)
    y1, packed = _run(codes, scales, zeros, 128, X)
    y2, _ = _run(codes, scales, zeros, 128, X)
    assert np.array_equal(y1, y2)
    Yd = torch.empty(2, rows, device=DEV)
    _lib.w4a16_matmul(packed, scales.to(DEV), zeros.to(DEV), 128, X[:2].to(DEV), Yd)
    torch.cuda.synchronize()
    words = oracle.pack_codes(codes.numpy())
    terms = oracle.w4a16_abs_terms(words, scales.numpy(), zeros.numpy(), 128, X[:2].float().numpy())
    assert np.all(np.abs(y1[:2] - Yd.double().cpu().numpy()) <= 2 * _bound(cols) * terms)


@pytest.mark.parametrize("n", [64, 256])
def test_gemm_fullsize_sampled_rows(n):
    """The 12288 x 49152 g128 layer in the launch configuration the benchmark times; sampled
    rows (first and last weight tiles included) against the oracle."""
    rows, cols, group = 12288, 49152, 128
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, group, 91, DEV)
    X = _x(n, cols, 17)
    y, _ = _run(codes.cpu(), scales.cpu(), zeros.cpu(), group, X)
    sel = np.unique(np.concatenate([[0, 1, 127, 128, rows - 1],
                                    np.random.default_rng(5).choice(rows, 8, replace=False)]))
    c = codes.cpu().numpy()[sel]
    words = oracle.pack_codes(c)
    Xf = X.float().numpy()
    s, z = scales.cpu().numpy()[sel], zeros.cpu().numpy()[sel]
    ref = oracle.w4a16_matmul(words, s, z, group, Xf)
    terms = oracle.w4a16_abs_terms(words, s, z, group, Xf)
    assert np.all(np.abs(y[:, sel] - ref) <= _bound(cols) * terms)
