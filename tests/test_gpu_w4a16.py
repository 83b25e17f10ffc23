"""GPU parity of the packed 4-bit format and the W4A16 product (through the C ABI) against the fp64
oracle on the same seeded inputs.

Packing is integer work: bit-exact. The product's tolerance comes from its arithmetic, per output
y[n][r] with T = sum_c |x[n][c] W_hat[r][c]| (computed by the oracle):
  * q - z and x are exact in bf16 and their products exact in fp32;
  * a 128-column chunk is summed in 8 tensor-core steps of 16 products; each step is bounded here
    by 2 ulp (2^-22) of the magnitudes it adds, i.e. <= 8 * 2^-22 * T over the chunks;
  * each chunk is scaled and added with one fp32 fma (<= 2^-24 T each, nchunks of them), and at
    most 16 warp partials are added at the end (<= 16 * 2^-24 T);
  => |y - y_oracle| <= (8 * 2^-22 + (nchunks + 16) * 2^-24) * T.
Dropping or misplacing one column changes y by about T / cols, far above that bound at these sizes.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _info():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def _pack_gpu(codes_dev):
    rows, cols = codes_dev.shape
    packed = torch.empty(rows, cols // 8, dtype=torch.int32, device=DEV)
    info = _info()
    _lib.pack_codes_4bit(codes_dev, packed, info)
    torch.cuda.synchronize()
    return packed, int(info.item())


def _words_np(packed_dev):
    return packed_dev.cpu().numpy().view(np.uint32)


def _x(n, cols, seed):
    spec = synth.scaled_spec(synth.ATTN, 1, cols, n)
    return synth.inputs_torch(spec, seed, "cpu")          # bf16 [n, cols], heavy-tailed


def _bound(cols):
    nchunks = -(-cols // 128)
    return 8 * 2.0 ** -22 + (nchunks + 16) * 2.0 ** -24


def _check_matmul(codes, scales, zeros, group, X, rows_sel=None, ldx=None, ldy=None):
    """Run the GPU product on (codes, scales, zeros, X) (CPU tensors) and compare to the oracle."""
    rows, cols = codes.shape
    n = X.shape[0]
    packed, info = _pack_gpu(codes.to(DEV))
    assert info == 0
    Xd = torch.zeros(n, ldx or cols, dtype=torch.bfloat16, device=DEV)
    Xd[:, :cols] = X.to(DEV)
    Y = torch.full((n, ldy or rows), float("nan"), device=DEV)
    info_t = _info()
    _lib.w4a16_matmul(packed, scales.to(DEV), zeros.to(DEV), group, Xd[:, :cols], Y[:, :rows],
                      info_t)
    torch.cuda.synchronize()
    assert int(info_t.item()) == 0
    y = Y[:, :rows].double().cpu().numpy()
    if ldy is not None:
        assert torch.isnan(Y[:, rows:]).all()            # columns past rows untouched
    sel = np.arange(rows) if rows_sel is None else np.asarray(rows_sel)
    words = oracle.pack_codes(codes.numpy()[sel])
    Xf = X.float().numpy()
    ref = oracle.w4a16_matmul(words, scales.numpy()[sel], zeros.numpy()[sel], group, Xf)
    terms = oracle.w4a16_abs_terms(words, scales.numpy()[sel], zeros.numpy()[sel], group, Xf)
    err = np.abs(y[:, sel] - ref)
    assert np.all(np.isfinite(y[:, sel]))
    assert np.all(err <= _bound(cols) * terms), float((err / terms).max())
    return y


# ---------------------------------------------------------------------------------------------
# packing
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols", [(1, 8), (5, 40), (3, 64), (37, 4096), (129, 11008)])
def test_pack_bit_exact(rows, cols):
    """Widths that are multiples of 32 take the 16-byte kernel, the others (8, 40) the word one."""
    codes, _, _ = synth.w4a16_operands_torch(rows, cols, -1, 11)
    packed, info = _pack_gpu(codes.to(DEV))
    assert info == 0
    assert np.array_equal(_words_np(packed), oracle.pack_codes(codes.numpy()))


def test_pack_strided_input_and_bad_code():
    codes, _, _ = synth.w4a16_operands_torch(20, 256, -1, 12)
    big = torch.zeros(20, 320, dtype=torch.uint8)
    big[:, :256] = codes
    big[5, 17] = 0x3A                                     # out of range: low nibble 0xA kept
    dev = big.to(DEV)
    packed = torch.empty(20, 32, dtype=torch.int32, device=DEV)
    info = _info()
    _lib.pack_codes_4bit(dev[:, :256], packed, info)
    torch.cuda.synchronize()
    assert int(info.item()) == _lib.GPTQ_INFO_BAD_CODE
    expect = codes.numpy().copy()
    expect[5, 17] = 0xA
    assert np.array_equal(_words_np(packed), oracle.pack_codes(expect))


def test_pack_row_pitch_not_a_multiple_of_16():
    """A row pitch of 264 bytes (8-byte aligned only) takes the word-at-a-time kernel."""
    codes, _, _ = synth.w4a16_operands_torch(9, 256, -1, 13)
    big = torch.zeros(9, 264, dtype=torch.uint8)
    big[:, :256] = codes
    dev = big.to(DEV)
    packed = torch.empty(9, 32, dtype=torch.int32, device=DEV)
    info = _info()
    _lib.pack_codes_4bit(dev[:, :256], packed, info)
    torch.cuda.synchronize()
    assert int(info.item()) == 0
    assert np.array_equal(_words_np(packed), oracle.pack_codes(codes.numpy()))


def test_pack_of_gptq_codes():
    """Codes straight from the library's own 4-bit quantizer pack and unpack exactly."""
    rows, cols = 48, 256
    W = torch.randn(rows, cols, generator=torch.Generator().manual_seed(3)) * 0.02
    R = torch.eye(cols)
    G = cols // 128
    W_hat = torch.empty(rows, cols, device=DEV)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, G, device=DEV)
    zeros = torch.empty(rows, G, dtype=torch.uint8, device=DEV)
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, 128),
                     dtype=torch.uint8, device=DEV)
    info = _info()
    _lib.quantize_layer(W.to(DEV), R.to(DEV), 4, 128, 128, W_hat, codes, scales, zeros, None, ws,
                        info)
    packed, pinfo = _pack_gpu(codes)
    assert int(info.item()) == 0 and pinfo == 0
    assert np.array_equal(oracle.unpack_codes(_words_np(packed)), codes.cpu().numpy())
    # and the product of those codes reproduces X W_hat^T
    X = _x(2, cols, 4)
    y = _check_matmul(codes.cpu(), scales.cpu(), zeros.cpu(), 128, X)
    ref = X.double().numpy() @ W_hat.double().cpu().numpy().T
    terms = np.abs(X.double().numpy()) @ np.abs(W_hat.double().cpu().numpy()).T
    assert np.all(np.abs(y - ref) <= (_bound(cols) + 2.0 ** -23) * terms)


# ---------------------------------------------------------------------------------------------
# the product
# ---------------------------------------------------------------------------------------------

@pytest.mark.parametrize("rows,cols,group,n", [
    (64, 256, 128, 1),        # one m-tile, two chunks
    (100, 4096, 128, 1),      # ragged last m-tile (100 = 6 * 16 + 4)
    (257, 1024, 256, 3),      # group of two chunks, ragged rows, a few vectors
    (48, 4000, -1, 1),        # per-row scales, ragged last chunk (4000 = 31 * 128 + 32)
    (33, 2048, 128, 8),       # full n-tile
    (40, 1536, 128, 9),       # second n-tile, one live vector in it
    (16, 512, -1, 16),        # two full n-tiles
    (1, 32, -1, 1),           # one row, one partial chunk
    (4096, 4096, 128, 1),     # attention-sized layer, decode step
])
def test_matmul_matches_oracle(rows, cols, group, n):
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, group, 21 + rows)
    X = _x(n, cols, 7)
    _check_matmul(codes, scales, zeros, group, X)


def test_matmul_strided_x_and_y():
    rows, cols = 80, 768
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, 128, 31)
    _check_matmul(codes, scales, zeros, 128, _x(5, cols, 8), ldx=cols + 64, ldy=rows + 13)


def test_matmul_extreme_codes_and_zeros():
    """All codes 0 or 15 with zero points 15 or 0: the largest |q - z| in both signs."""
    rows, cols = 32, 512
    codes = torch.zeros(rows, cols, dtype=torch.uint8)
    codes[::2] = 15
    zeros = torch.zeros(rows, 4, dtype=torch.uint8)
    zeros[1::2] = 15
    scales = torch.full((rows, 4), 0.0078125)
    _check_matmul(codes, scales, zeros, 128, _x(2, cols, 9))


def test_matmul_deterministic():
    rows, cols = 300, 8192
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, 128, 41)
    packed, _ = _pack_gpu(codes.to(DEV))
    X = _x(1, cols, 10).to(DEV)
    Ys = []
    for _ in range(2):
        Y = torch.empty(1, rows, device=DEV)
        _lib.w4a16_matmul(packed, scales.to(DEV), zeros.to(DEV), 128, X, Y)
        Ys.append(Y)
    torch.cuda.synchronize()
    assert torch.equal(Ys[0], Ys[1])


def test_matmul_empty_is_noop():
    packed = torch.zeros(4, 32, dtype=torch.int32, device=DEV)
    Y = torch.full((1, 4), 7.0, device=DEV)
    X = torch.zeros(0, 256, dtype=torch.bfloat16, device=DEV)
    _lib.w4a16_matmul(packed, torch.ones(4, 2, device=DEV),
                      torch.zeros(4, 2, dtype=torch.uint8, device=DEV), 128, X, Y[:0])
    torch.cuda.synchronize()
    assert torch.equal(Y, torch.full((1, 4), 7.0, device=DEV))


def test_matmul_fullsize_sampled_rows():
    """The 12288 x 49152 layer (302 MB of packed codes), in the launch configuration the benchmark
    times; sampled rows (first and last m-tiles included) against the oracle."""
    rows, cols, group = 12288, 49152, 128
    codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, group, 51, DEV)
    packed, info = _pack_gpu(codes)
    assert info == 0
    X = _x(1, cols, 11)
    Y = torch.empty(1, rows, device=DEV)
    info_t = _info()
    _lib.w4a16_matmul(packed, scales, zeros, group, X.to(DEV), Y, info_t)
    torch.cuda.synchronize()
    assert int(info_t.item()) == 0
    sel = np.unique(np.concatenate([np.arange(16), np.arange(rows - 16, rows),
                                    np.random.default_rng(0).choice(rows, 32, replace=False)]))
    sel_t = torch.from_numpy(sel).to(DEV)
    words = oracle.pack_codes(codes[sel_t].cpu().numpy())
    assert np.array_equal(_words_np(packed[sel_t]), words)
    s_np, z_np = scales[sel_t].cpu().numpy(), zeros[sel_t].cpu().numpy()
    Xf = X.float().numpy()
    ref = oracle.w4a16_matmul(words, s_np, z_np, group, Xf)
    terms = oracle.w4a16_abs_terms(words, s_np, z_np, group, Xf)
    y = Y[:, sel_t].double().cpu().numpy()
    assert np.all(np.abs(y - ref) <= _bound(cols) * terms)
