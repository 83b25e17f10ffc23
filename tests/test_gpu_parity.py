"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the same seeded inputs.

Tolerances (fixed before measuring):
  * H and R: relative Frobenius error <= 1e-4 (each stage fed the GPU's own upstream result,
    converted to fp64, so errors do not compound);
  * identity Hessian: codes, scales and zero points bit-exact (GPTQ reduces to round-to-nearest);
  * general inputs: >= 99.5 % identical codes, relative layer error within 1 % of the oracle's.
The quantizer decides codes in float32 on both sides; near ties that differ in the last bit of a
compensated weight can flip a code and then the rest of that row, hence the 99.5 % bar.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import _lib, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"


def rel_fro(a, b):
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / np.linalg.norm(b))


def to_dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to(DEV).to(dtype)


def new_info():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


def gpu_hessian(X_np, x_dtype, chunks=1):
    cols = X_np.shape[1]
    S = torch.zeros(cols, cols, device=DEV)
    info = new_info()
    for part in np.array_split(X_np, chunks):
        _lib.hessian_accumulate(S, to_dev(part, x_dtype), info)
    torch.cuda.synchronize()
    assert info.item() == 0
    return S


def gpu_prepare(S, n_total, damp=0.01, route=None):
    cols = S.shape[0]
    R = torch.empty(cols, cols, device=DEV)
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), dtype=torch.uint8,
                     device=DEV)
    info = new_info()
    _lib.prepare_hinv(S, R, n_total, damp, ws, info, route=route)
    torch.cuda.synchronize()
    return R, int(info.item())


def gpu_quantize(W_t, R, bits, group, block):
    rows, cols = W_t.shape
    G = 1 if group <= 0 else cols // group
    out = dict(W_hat=torch.empty(rows, cols, device=DEV),
               codes=torch.empty(rows, cols, dtype=torch.uint8, device=DEV),
               scales=torch.empty(rows, G, device=DEV),
               zeros=torch.empty(rows, G, dtype=torch.uint8, device=DEV),
               err_sq=torch.empty(rows, device=DEV))
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, block),
                     dtype=torch.uint8, device=DEV)
    info = new_info()
    _lib.quantize_layer(W_t, R, bits, group, block, out["W_hat"], out["codes"], out["scales"],
                        out["zeros"], out["err_sq"], ws, info)
    torch.cuda.synchronize()
    assert info.item() == 0
    return {k: v.cpu().numpy() for k, v in out.items()}


# ------------------------------------------------------------------------------------------------
# S1
# ------------------------------------------------------------------------------------------------

def test_hessian_fp32_tiny():
    spec = synth.TINY
    X = synth.inputs_np(spec, 0)
    S = gpu_hessian(X, torch.float32, chunks=3).cpu().numpy()
    ref = X.astype(np.float64).T @ X.astype(np.float64)
    low = np.tril_indices(spec.cols)
    assert rel_fro(S[low], ref[low]) < 1e-6


@pytest.mark.parametrize("cols,n_tokens,chunks", [(256, 4096, 1), (384, 1000, 2), (136, 4133, 3),
                                                  (1024, 8192, 1), (8, 40, 1)])
def test_hessian_bf16_tensor_cores(cols, n_tokens, chunks):
    spec = synth.scaled_spec(synth.ATTN, 8, cols, n_tokens)
    X = synth.inputs_np(spec, 1)
    S = gpu_hessian(X, torch.bfloat16, chunks).cpu().numpy()
    ref = X.astype(np.float64).T @ X.astype(np.float64)
    low = np.tril_indices(cols)
    # The tensor core's fp32 accumulation rounds toward zero (about 6e-8 relative per MMA folded
    # into a sum); TMEM sums are flushed into S every 2048 tokens, which bounds this below 1e-5.
    assert rel_fro(S[low], ref[low]) < 1e-5
    # every lower entry individually, relative to the scale of its row and column
    scale = np.sqrt(np.outer(np.diag(ref), np.diag(ref)))
    assert np.max(np.abs(S - ref)[low] / scale[low]) < 1e-4


# ------------------------------------------------------------------------------------------------
# S2-S5
# ------------------------------------------------------------------------------------------------

ROUTES = [None, _lib.GPTQ_ROUTE_THREE_STEP, _lib.GPTQ_ROUTE_REVERSED]


@pytest.mark.parametrize("route", ROUTES, ids=["default", "three_step", "reversed"])
@pytest.mark.parametrize("cols,n_tokens", [(128, 1024), (300, 2048), (1024, 8192), (644, 4096)])
def test_prepare_hinv_stagewise(cols, n_tokens, route):
    spec = synth.scaled_spec(synth.ATTN, 8, cols, n_tokens, x_dtype="fp32")
    X = synth.inputs_np(spec, 2)
    S = gpu_hessian(X, torch.float32)
    S_in = S.cpu().numpy().astype(np.float64)
    R, info = gpu_prepare(S, n_tokens, route=route)
    assert info == 0
    H_gpu = S.cpu().numpy()
    H_ref = oracle.hessian_finalize(np.tril(S_in) + np.tril(S_in, -1).T, n_tokens)
    assert rel_fro(H_gpu, H_ref) < 1e-6
    assert np.array_equal(H_gpu, H_gpu.T)
    R_ref = oracle.inverse_hessian_factor(H_gpu.astype(np.float64), 0.01)["R"]
    R_gpu = R.cpu().numpy()
    assert np.all(np.tril(R_gpu, -1) == 0)
    assert rel_fro(R_gpu, R_ref) < 1e-4


@pytest.mark.parametrize("route", ROUTES, ids=["default", "three_step", "reversed"])
def test_prepare_reports_non_pd_pivot(route):
    cols = 256
    S = torch.eye(cols, device=DEV) * 50.0
    S[37, 37] = -1.0e4          # after damping this pivot stays negative
    _, info = gpu_prepare(S, 100, route=route)
    assert info == 38           # the original column, whichever order the factorization runs in
    assert _lib.info_status(info) == _lib.GPTQ_ENOTPD


def test_prepare_reports_bad_hessian():
    S = torch.zeros(64, 64, device=DEV)
    _, info = gpu_prepare(S, 10)
    assert info == _lib.GPTQ_INFO_BAD_HESSIAN


# ------------------------------------------------------------------------------------------------
# S6-S8
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("group,block", [(-1, 32), (-1, 128), (128, 128), (32, 128), (256, 128),
                                         (64, 64), (16, 32), (8, 128), (4, 64), (2, 32),
                                         (1, 32)])
def test_identity_hessian_bit_exact_rtn(group, block):
    rows, cols, n = 96, 512, 1024
    W = synth.weights_np(synth.scaled_spec(synth.ATTN, rows, cols, 1), 3)
    S = torch.eye(cols, device=DEV) * (n / 2.0)     # H = 2S/N = I exactly (N a power of two)
    R, info = gpu_prepare(S, n)
    assert info == 0
    Rn = R.cpu().numpy()
    assert np.all(Rn == np.diag(np.diag(Rn)))
    got = gpu_quantize(to_dev(W, torch.bfloat16), R, 4, group, block)
    ref = oracle.rtn_quantize(W, 4, group)
    for k in ("codes", "scales", "zeros", "W_hat"):
        np.testing.assert_array_equal(got[k], ref[k], err_msg=k)


@pytest.mark.parametrize("rows,cols,bits,group,block", [
    (64, 128, 4, -1, 32), (200, 512, 4, 128, 128), (130, 512, 3, -1, 128),
    (64, 384, 4, 32, 64), (48, 1024, 4, 256, 128), (40, 200, 4, -1, 64), (64, 512, 2, 64, 32),
    (33, 640, 8, 128, 128), (48, 256, 4, 8, 64), (40, 128, 4, 2, 32),
])
def test_quantize_stagewise_against_oracle(rows, cols, bits, group, block):
    spec = synth.scaled_spec(synth.ATTN, rows, cols, 4 * cols)
    W = synth.weights_np(spec, 4)
    X = synth.inputs_np(spec, 4)
    H = oracle.hessian(X)
    R64 = oracle.inverse_hessian_factor(H)["R"]
    R32 = R64.astype(np.float32)
    got = gpu_quantize(to_dev(W, torch.bfloat16), to_dev(R32), bits, group, block)
    ref = oracle.gptq_quantize(W, R32.astype(np.float64), bits, group, block)
    match = (got["codes"] == ref["codes"]).mean()
    assert match >= 0.995, match
    e_gpu = oracle.layer_error(W, got["W_hat"], H)
    e_ref = oracle.layer_error(W, ref["W_hat"], H)
    assert abs(e_gpu - e_ref) <= 0.01 * e_ref
    # the dequantized weights are exactly s * (q - z) of the GPU's own codes and grids
    G = got["scales"].shape[1]
    gidx = np.zeros(cols, int) if group <= 0 else np.arange(cols) // group
    s = got["scales"][:, gidx]
    z = got["zeros"][:, gidx].astype(np.float32)
    np.testing.assert_array_equal(got["W_hat"], (s * (got["codes"].astype(np.float32) - z)))
    assert got["codes"].max() <= 2 ** bits - 1
    # the per-row loss sum_j e_j^2 agrees wherever the row's codes agree, and in total
    same = np.all(got["codes"] == ref["codes"], axis=1)
    np.testing.assert_allclose(got["err_sq"][same], ref["err_sq"][same], rtol=1e-3, atol=1e-9)
    assert abs(got["err_sq"].sum() - ref["err_sq"].sum()) <= 0.01 * ref["err_sq"].sum()


def test_zero_rows_and_degenerate_grids():
    rows, cols = 16, 256
    W = synth.weights_np(synth.scaled_spec(synth.ATTN, rows, cols, 1), 5)
    W[3] = 0.0
    W[7, :128] = 0.0
    H = oracle.hessian(synth.inputs_np(synth.scaled_spec(synth.ATTN, rows, cols, 1024), 5))
    R32 = oracle.inverse_hessian_factor(H)["R"].astype(np.float32)
    got = gpu_quantize(to_dev(W, torch.float32), to_dev(R32), 4, 128, 128)
    ref = oracle.gptq_quantize(W, R32.astype(np.float64), 4, 128, 128)
    np.testing.assert_array_equal(got["codes"][3], ref["codes"][3])
    np.testing.assert_array_equal(got["scales"][3], ref["scales"][3])
    assert np.all(got["W_hat"][3] == 0)


# ------------------------------------------------------------------------------------------------
# End to end (S1-S8) on the oracle's sizes
# ------------------------------------------------------------------------------------------------

@pytest.mark.parametrize("which", ["tiny", "heavy"])
def test_end_to_end(which):
    spec = synth.TINY if which == "tiny" else synth.scaled_spec(synth.ATTN, 256, 1024, 16384)
    W = synth.weights_np(spec, 0)
    X = synth.inputs_np(spec, 0)
    xdt = torch.float32 if spec.x_dtype == "fp32" else torch.bfloat16
    wdt = torch.float32 if spec.w_dtype == "fp32" else torch.bfloat16
    S = gpu_hessian(X, xdt, chunks=2)
    R, info = gpu_prepare(S, X.shape[0], spec.damp)
    assert info == 0
    got = gpu_quantize(to_dev(W, wdt), R, spec.bits, spec.group, spec.block)
    ref = oracle.gptq_layer(W, X, spec.bits, spec.group, spec.block, spec.damp)
    match = (got["codes"] == ref["codes"]).mean()
    assert match >= 0.995, match
    e_gpu = oracle.layer_error(W, got["W_hat"], ref["H"])
    assert abs(e_gpu - ref["rel_err"]) <= 0.01 * ref["rel_err"]
    assert rel_fro(S.cpu().numpy(), ref["H"]) < 1e-4
    assert rel_fro(R.cpu().numpy(), ref["R"]) < 1e-4


def test_bounded_wait_reports_timeout():
    info = new_info()
    _lib.selftest_wait_timeout(info, 50)
    torch.cuda.synchronize()
    assert info.item() == _lib.GPTQ_INFO_TIMEOUT
    # the context is still usable afterwards
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum().item()) == 8.0


def test_flag_wait_reports_timeout():
    """The bounded wait on a global-memory flag (the fused factorization step's panel flags)."""
    flag = torch.zeros(1, dtype=torch.int32, device=DEV)
    info = new_info()
    _lib.selftest_flag_timeout(flag, info, 50)
    torch.cuda.synchronize()
    assert info.item() == _lib.GPTQ_INFO_TIMEOUT
    flag.fill_(1)
    info = new_info()
    _lib.selftest_flag_timeout(flag, info, 50)
    torch.cuda.synchronize()
    assert info.item() == 0
    x = torch.ones(4, device=DEV)
    assert float((x * 2).sum().item()) == 8.0


def test_deterministic_repeat():
    spec = synth.scaled_spec(synth.ATTN, 128, 512, 4096)
    X = synth.inputs_np(spec, 9)
    W = synth.weights_np(spec, 9)
    outs = []
    for _ in range(2):
        S = gpu_hessian(X, torch.bfloat16)
        R, _ = gpu_prepare(S, X.shape[0])
        outs.append((S.cpu().numpy(), R.cpu().numpy(),
                     gpu_quantize(to_dev(W, torch.bfloat16), R, 4, 128, 128)))
    np.testing.assert_array_equal(outs[0][0], outs[1][0])
    np.testing.assert_array_equal(outs[0][1], outs[1][1])
    for k in outs[0][2]:
        np.testing.assert_array_equal(outs[0][2][k], outs[1][2][k])
