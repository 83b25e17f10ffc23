"""Packed 3-bit codes on the GPU (gptq_pack_codes_3bit) against the oracle's layout: bit-exact
for random codes over ragged row counts and widths, from a strided source, with the bad-code
flag, and for codes straight from the library's own 3-bit quantizer (the MLP pair's and the
175B-class per-row grids)."""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _codes3(rows, cols, seed):
    g = torch.Generator().manual_seed(seed)
    return torch.randint(0, 8, (rows, cols), generator=g, dtype=torch.uint8)


def _pack3(codes_dev):
    rows, cols = codes_dev.shape
    packed = torch.empty(rows, 3 * cols // 32, dtype=torch.int32, device=DEV)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    _lib.pack_codes_3bit(codes_dev, packed, info)
    torch.cuda.synchronize()
    return packed.cpu().numpy().view(np.uint32), int(info.item())


@pytest.mark.parametrize("rows,cols", [(1, 32), (3, 64), (7, 96), (129, 4096), (33, 11008),
                                       (2, 49152)])
def test_pack3_bit_exact(rows, cols):
    codes = _codes3(rows, cols, rows + cols)
    words, info = _pack3(codes.to(DEV))
    assert info == 0
    assert np.array_equal(words, oracle.pack_codes_3bit(codes.numpy()))


def test_pack3_strided_input_and_bad_code():
    codes = _codes3(20, 256, 5)
    big = torch.zeros(20, 320, dtype=torch.uint8)
    big[:, :256] = codes
    big[4, 42] = 0x1D                                    # out of range: low three bits 0x5 kept
    dev = big.to(DEV)
    packed = torch.empty(20, 24, dtype=torch.int32, device=DEV)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    _lib.pack_codes_3bit(dev[:, :256], packed, info)
    torch.cuda.synchronize()
    assert int(info.item()) == _lib.GPTQ_INFO_BAD_CODE
    expect = codes.numpy().copy()
    expect[4, 42] = 0x5
    assert np.array_equal(packed.cpu().numpy().view(np.uint32), oracle.pack_codes_3bit(expect))


def test_pack3_rejects_and_empty():
    lib = _lib.load()
    codes = torch.zeros(4, 64, dtype=torch.uint8, device=DEV)
    packed = torch.zeros(4, 6, dtype=torch.int32, device=DEV)
    p, q = codes.data_ptr(), packed.data_ptr()
    assert lib.gptq_pack_codes_3bit(p, 4, 48, 64, q, None, None) == _lib.GPTQ_EINVAL  # cols % 32
    assert lib.gptq_pack_codes_3bit(p, 4, 64, 60, q, None, None) == _lib.GPTQ_EINVAL  # ldc < cols
    assert lib.gptq_pack_codes_3bit(p + 4, 4, 64, 64, q, None, None) == _lib.GPTQ_EINVAL
    assert lib.gptq_pack_codes_3bit(None, 0, 64, 64, None, None, None) == _lib.GPTQ_OK
    torch.cuda.synchronize()
    assert torch.count_nonzero(packed).item() == 0


@pytest.mark.parametrize("rows,cols", [(64, 4096), (24, 11008)])
def test_pack3_of_gptq_codes(rows, cols):
    """Codes from the library's 3-bit per-row quantizer (a GPTQ layer with a real factor) pack and
    unpack exactly, and W_hat = s (q - z) holds with the unpacked codes."""
    spec = synth.scaled_spec(synth.MLP_UP, rows, cols, 2 * cols)
    X = synth.inputs_torch(spec, 3, DEV)
    W = synth.weights_torch(spec, 3, DEV)
    S = torch.zeros(cols, cols, device=DEV)
    R = torch.empty(cols, cols, device=DEV)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    _lib.hessian_accumulate(S, X, info)
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), dtype=torch.uint8,
                     device=DEV)
    _lib.prepare_hinv(S, R, X.shape[0], spec.damp, ws, info)
    W_hat = torch.empty(rows, cols, device=DEV)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, 1, device=DEV)
    zeros = torch.empty(rows, 1, dtype=torch.uint8, device=DEV)
    wq = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, 128),
                     dtype=torch.uint8, device=DEV)
    _lib.quantize_layer(W, R, 3, -1, 128, W_hat, codes, scales, zeros, None, wq, info)
    words, pinfo = _pack3(codes)
    assert int(info.item()) == 0 and pinfo == 0
    q = oracle.unpack_codes_3bit(words)
    assert np.array_equal(q, codes.cpu().numpy())
    s = scales.cpu().numpy()
    z = zeros.cpu().numpy().astype(np.float32)
    np.testing.assert_array_equal(W_hat.cpu().numpy(), s * (q.astype(np.float32) - z))
