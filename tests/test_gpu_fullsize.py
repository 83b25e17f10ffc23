"""Full-size parity: the configured workloads run through the C ABI exactly as the benchmark runs
them (bf16 inputs resident on the device, one Hessian call over all tokens, block 128), checked
against the fp64 oracle on outputs it can compute one by one:

* H on sampled channel pairs: exact fp64 dot products over all tokens (only those channels of X
  are copied to the host);
* R on its trailing principal block: R[k:, k:] is the factor of the trailing block of H + lambda I
  alone (the oracle pins this), so the oracle factors just that block of the GPU's H;
* codes and the per-row loss sum_j e_j^2 on sampled rows: rows are independent given R, and the
  first columns of a row depend only on the leading block of R, so for the largest layer the
  oracle runs the leading 1024 columns (group grids are local to their columns; a per-row grid
  comes from the whole original row, so the oracle computes it from the whole row and is handed
  it, and the GPU's per-row scales and zero points are compared with it bit for bit).
Tolerances as in the small-size parity tests: 1e-4 relative (H entries against the scale of their
row and column, R blocks in Frobenius norm), >= 99.5 % identical codes, loss sums within 1 %.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"

CASES = {
    # name: (spec, rows sampled, oracle columns (None = all), trailing block for R, route)
    "attn_4096x4096": (synth.ATTN, 24, None, 1024, None),
    "attn_4096x4096_three_step": (synth.ATTN, 24, None, 1024, _lib.GPTQ_ROUTE_THREE_STEP),
    "mlp_up_11008x4096": (synth.MLP_UP, 16, None, 1024, None),
    "mlp_down_4096x11008": (synth.MLP_DOWN, 12, None, 1536, None),
    "fc1_49152x12288_3bit_row": (dataclasses.replace(synth.FC1, bits=3, group=-1), 8, None, 1536,
                                 None),
    "fc1_49152x12288_4bit_g128": (synth.FC1, 8, None, 1536, None),
    "fc2_12288x49152_4bit_g128": (synth.FC2, 16, 1024, 1024, None),
    "fc2_12288x49152_3bit_row": (dataclasses.replace(synth.FC2, bits=3, group=-1), 16, 1024, 1024,
                                 None),
}


def _rel_fro(a, b):
    return float(np.linalg.norm(np.asarray(a, np.float64) - b) / np.linalg.norm(b))


@pytest.mark.parametrize("name", list(CASES))
def test_full_size_against_sampled_oracle(name):
    spec, n_rows, ocols, tb, route = CASES[name]
    seed = 0
    free = torch.cuda.mem_get_info()[0]
    need = spec.n_tokens * spec.cols * 2 + 6 * spec.cols ** 2 * 4 + 12 * spec.rows * spec.cols
    if need > 0.9 * free:
        pytest.skip(f"needs {need / 1e9:.0f} GB of device memory, {free / 1e9:.0f} GB free")
    rows, cols, n = spec.rows, spec.cols, spec.n_tokens
    rng = np.random.default_rng(123)
    X = synth.inputs_torch(spec, seed, DEV)
    info = torch.zeros(1, dtype=torch.int32, device=DEV)
    S = torch.zeros(cols, cols, device=DEV)
    _lib.hessian_accumulate(S, X, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    # sampled channels: a few random ones plus the first and last
    ch = np.unique(np.concatenate([rng.choice(cols, 12, replace=False), [0, cols - 1]]))
    Xs = X[:, torch.from_numpy(ch).to(DEV)].double().cpu().numpy()
    del X
    torch.cuda.empty_cache()
    S_ref = Xs.T @ Xs
    S_got = S[torch.from_numpy(ch).to(DEV)][:, torch.from_numpy(ch).to(DEV)].double().cpu().numpy()
    low = np.tril_indices(len(ch))
    scale = np.sqrt(np.outer(np.diag(S_ref), np.diag(S_ref)))
    assert np.max((np.abs(S_got - S_ref) / scale)[low]) < 1e-4

    R = torch.empty(cols, cols, device=DEV)
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), dtype=torch.uint8,
                     device=DEV)
    _lib.prepare_hinv(S, R, n, spec.damp, ws, info, route=route)
    torch.cuda.synchronize()
    assert info.item() == 0
    del ws
    torch.cuda.empty_cache()
    H = S  # H = 2 S / N, both triangles
    lam = spec.damp * float(torch.diagonal(H).double().mean().item())
    k = cols - tb
    Hb = H[k:, k:].double().cpu().numpy() + lam * np.eye(tb)
    Rb_ref = oracle.inverse_hessian_factor(Hb, 0.0)["R"]
    assert _rel_fro(R[k:, k:].cpu().numpy(), Rb_ref) < 1e-4

    W = synth.weights_torch(spec, seed, DEV)
    G = 1 if spec.group <= 0 else cols // spec.group
    W_hat = torch.empty(rows, cols, device=DEV)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=DEV)
    scales = torch.empty(rows, G, device=DEV)
    zeros = torch.empty(rows, G, dtype=torch.uint8, device=DEV)
    err_sq = torch.empty(rows, device=DEV)
    wq = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, spec.block),
                     dtype=torch.uint8, device=DEV)
    _lib.quantize_layer(W, R, spec.bits, spec.group, spec.block, W_hat, codes, scales, zeros,
                        err_sq, wq, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    rsel = np.sort(rng.choice(rows, n_rows, replace=False))
    ridx = torch.from_numpy(rsel).to(DEV)
    oc = cols if ocols is None else ocols
    Wfull = W[ridx].float().cpu().numpy()
    Wr = Wfull[:, :oc]
    Rr = R[:oc, :oc].double().cpu().numpy()
    grid = None
    if spec.group <= 0 and oc < cols:
        grid = oracle.quant_params(Wfull, spec.bits)
        np.testing.assert_array_equal(scales[ridx][:, 0].cpu().numpy(), grid[0])
        np.testing.assert_array_equal(zeros[ridx][:, 0].cpu().numpy(), grid[1].astype(np.uint8))
    ref = oracle.gptq_quantize(Wr, Rr, spec.bits, spec.group, spec.block, row_grid=grid)
    got_codes = codes[ridx][:, :oc].cpu().numpy()
    match = (got_codes == ref["codes"]).mean()
    assert match >= 0.995, match
    if ocols is None:
        got_err = err_sq[ridx].double().cpu().numpy()
        assert abs(got_err.sum() - ref["err_sq"].sum()) <= 0.01 * ref["err_sq"].sum()
    # every code on the grid, W_hat exactly s * (q - z), on the sampled rows
    gidx = np.zeros(cols, int) if spec.group <= 0 else np.arange(cols) // spec.group
    s_ = scales[ridx].cpu().numpy()[:, gidx]
    z_ = zeros[ridx].cpu().numpy()[:, gidx].astype(np.float32)
    q_ = codes[ridx].cpu().numpy()
    assert q_.max() <= 2 ** spec.bits - 1
    np.testing.assert_array_equal(W_hat[ridx].cpu().numpy(), s_ * (q_.astype(np.float32) - z_))
    del S, R, W, W_hat, codes, wq
    torch.cuda.empty_cache()
