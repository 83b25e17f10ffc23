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
    out_h = chunked.quantize(W, bits=4, group=128, block=128, to_host=True)
    out_d = whole.quantize(W.to(DEV), bits=4, group=128, block=128)
    assert out_h.info == 0 and out_d.info == 0
    assert out_h.codes.device.type == "cpu" and out_h.W_hat.device.type == "cpu"
    match = (out_h.codes.numpy() == out_d.codes.cpu().numpy()).mean()
    assert match >= 0.995, match
    # every returned host tensor is complete: W_hat = s * (q - z) row by row
    s = out_h.scales.numpy().repeat(128, axis=1)
    z = out_h.zeros.numpy().repeat(128, axis=1).astype(np.float32)
    np.testing.assert_array_equal(out_h.W_hat.numpy(), s * (out_h.codes.numpy().astype(np.float32) - z))
