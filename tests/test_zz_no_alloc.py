"""gptq_quantize_layer_noalloc: the column loop for callers that cannot allocate device memory
(for example code whose framework owns every device allocation through its own pool, or code that
cannot afford cudaMalloc's implicit synchronization). It keeps its error buffer in scratch built
into the library instead of a caller workspace, so its results must equal those of
gptq_quantize_layer on the same inputs -- checked here on two calls in a row, the second with
other shapes, so that whatever the first call left in the shared scratch cannot leak into it.

This file is collected last on purpose and also passes when run alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _problem(rows, cols, seed):
    spec = synth.scaled_spec(synth.ATTN, rows, cols, 4 * cols)
    W = synth.weights_np(spec, seed)
    H = oracle.hessian(synth.inputs_np(spec, seed))
    R = oracle.inverse_hessian_factor(H)["R"].astype(np.float32)
    return (torch.from_numpy(W).to(DEV).to(torch.bfloat16), torch.from_numpy(R).to(DEV))


def _outputs(rows, cols, group):
    G = 1 if group <= 0 else cols // group
    return dict(W_hat=torch.empty(rows, cols, device=DEV),
                codes=torch.empty(rows, cols, dtype=torch.uint8, device=DEV),
                scales=torch.empty(rows, G, device=DEV),
                zeros=torch.empty(rows, G, dtype=torch.uint8, device=DEV),
                err_sq=torch.empty(rows, device=DEV))


def _run(W, R, bits, group, block, noalloc):
    rows, cols = W.shape
    out = _outputs(rows, cols, group)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    if noalloc:
        _lib.quantize_layer_noalloc(W, R, bits, group, block, out["W_hat"], out["codes"],
                                    out["scales"], out["zeros"], out["err_sq"], info)
    else:
        ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, block),
                         dtype=torch.uint8, device=DEV)
        _lib.quantize_layer(W, R, bits, group, block, out["W_hat"], out["codes"], out["scales"],
                            out["zeros"], out["err_sq"], ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    return {k: v.cpu().numpy() for k, v in out.items()}


@pytest.mark.parametrize("call", [
    (1024, 1024, 4, 128, 128),   # first call: 1024 x 1024 at block 128 (2 MiB of scratch)
    (300, 640, 3, -1, 64),       # second call: other shapes, per-row grid, ragged row count
])
def test_noalloc_matches_workspace_entry_point(call):
    rows, cols, bits, group, block = call
    W, R = _problem(rows, cols, seed=rows)
    ref = _run(W, R, bits, group, block, noalloc=False)
    got = _run(W, R, bits, group, block, noalloc=True)
    # The same deterministic kernels run on the same inputs, so the results must be identical,
    # which is stricter than the parity tolerance (>= 99.5 % of codes, 1 % layer error).
    for k in ("codes", "scales", "zeros", "W_hat", "err_sq"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    """A valid call that is too large for the built-in scratch is refused before anything is
    enqueued. Real (small) buffers are passed: the call is refused on its sizes alone, and if the
    checks were ever reordered the buffers are still valid device memory."""
    lib = _lib.load()
    cols = 4096
    rows = 1
    while _lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, 128) <= \
            _lib.GPTQ_NOALLOC_SCRATCH_BYTES:
        rows *= 2
    buf = torch.zeros(4096, dtype=torch.float32, device=DEV)
    p = ctypes.c_void_p(buf.data_ptr())
    st = lib.gptq_quantize_layer_noalloc(p, _lib.GPTQ_BF16, rows, cols, cols, p, 4, -1, 128,
                                         p, p, p, p, None, p, None)
    assert st == _lib.GPTQ_EWORKSPACE
    # A call with invalid arguments is refused for them, as gptq_quantize_layer refuses it.
    st = lib.gptq_quantize_layer_noalloc(None, _lib.GPTQ_BF16, rows, cols, cols, p, 4, -1, 128,
                                         p, p, p, p, None, p, None)
    assert st == _lib.GPTQ_EINVAL
    st = lib.gptq_quantize_layer_noalloc(p, _lib.GPTQ_BF16, 64, cols, cols, p, 9, -1, 128,
                                         p, p, p, p, None, p, None)
    assert st == _lib.GPTQ_EINVAL
