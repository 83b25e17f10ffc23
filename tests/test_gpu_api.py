"""The user-level wrapper (api.LayerQuantizer): host calibration inputs streamed in chunks (copies
overlapping the Hessian accumulation) must give the same Hessian and codes as device-resident
inputs, and host outputs must come back complete."""
import numpy as np
import pytest
import torch

from post_weight_quantization_12_b200 import api, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def test_host_chunks_match_device_inputs():
    spec = synth.scaled_spec(synth.ATTN, 256, 512, 5000)     # 5000 tokens: ragged last chunk
    X = synth.inputs_torch(spec, 7, "cpu")
    W = synth.weights_torch(spec, 7, "cpu")
    chunked = api.LayerQuantizer(spec.cols, device=DEV)
    chunked.add_batch(X, chunk_bytes=1 << 20)                 # 1024 tokens per chunk: 5 chunks
    whole = api.LayerQuantizer(spec.cols, device=DEV)
    whole.add_batch(X.to(DEV))
    assert chunked.n_total == whole.n_total == spec.n_tokens
    torch.cuda.synchronize()
    S1 = torch.tril(chunked.S).double().cpu().numpy()
    S2 = torch.tril(whole.S).double().cpu().numpy()
    assert np.linalg.norm(S1 - S2) <= 1e-5 * np.linalg.norm(S2)
    out_h = chunked.quantize(W, bits=4, group=128, block=128, to_host=True, host_w_hat=True)
    # without host_w_hat the largest output stays on the device (the host gets what defines it)
    out_k = chunked.quantize(W, bits=4, group=128, block=128, to_host=True)
    assert out_k.codes.device.type == "cpu" and out_k.W_hat.device.type == "cuda"
    assert np.array_equal(out_k.codes.numpy(), out_h.codes.numpy())
    out_d = whole.quantize(W.to(DEV), bits=4, group=128, block=128)
    assert out_h.info == 0 and out_d.info == 0
    assert out_h.codes.device.type == "cpu" and out_h.W_hat.device.type == "cpu"
    match = (out_h.codes.numpy() == out_d.codes.cpu().numpy()).mean()
    assert match >= 0.995, match
    # every returned host tensor is complete: W_hat = s * (q - z) row by row
    s = out_h.scales.numpy().repeat(128, axis=1)
    z = out_h.zeros.numpy().repeat(128, axis=1).astype(np.float32)
    np.testing.assert_array_equal(out_h.W_hat.numpy(), s * (out_h.codes.numpy().astype(np.float32) - z))


def test_pack_4bit_linear_reproduces_x_w_hat():
    """A 4-bit group-128 layer from LayerQuantizer, packed and applied to bf16 activations, gives
    X W_hat^T within the product's rounding bound."""
    spec = synth.scaled_spec(synth.ATTN, 96, 512, 4096)
    X = synth.inputs_torch(spec, 3, DEV)
    W = synth.weights_torch(spec, 3, DEV)
    q = api.LayerQuantizer(spec.cols, device=DEV)
    q.add_batch(X)
    out = q.quantize(W, bits=4, group=128, block=128)
    lin = api.pack_4bit(out)
    assert lin.group == 128 and lin.rows == 96 and lin.cols == 512
    A = X[:3].contiguous()
    Y = lin(A)
    torch.cuda.synchronize()
    ref = A.double() @ out.W_hat.double().T
    terms = A.double().abs() @ out.W_hat.double().abs().T
    bound = 8 * 2.0 ** -22 + (4 + 16) * 2.0 ** -24 + 2.0 ** -23
    assert torch.all((Y.double() - ref).abs() <= bound * terms)


def test_rotate_helper_keeps_layer_products():
    W = torch.randn(8, 256, generator=torch.Generator().manual_seed(5)).to(DEV)
    X = torch.randn(32, 256, generator=torch.Generator().manual_seed(6)).to(DEV)
    signs = torch.randint(-2 ** 31, 2 ** 31 - 1, (8,), generator=torch.Generator().manual_seed(7),
                          dtype=torch.int64).to(torch.int32).to(DEV)
    Wr, Xr = api.rotate(W, signs), api.rotate(X, signs)
    torch.cuda.synchronize()
    ref = W.double() @ X.double().T
    scale = W.double().norm(dim=1)[:, None] * X.double().norm(dim=1)[None, :]
    assert torch.all((Wr.double() @ Xr.double().T - ref).abs() <= 1e-5 * scale)

