"""The 7B-class decoder block quantized layer by layer, in execution order, through the public API
(`api.LayerQuantizer`), as "Part 3: Adaptive Rounding: GPTQ" ("Algorithm GPTQ") runs the method:
one layer after another, each from the calibration inputs that reach it.

Seven layers and four Hessians: q, k and v read the same input and share one H (one quantizer,
three `quantize` calls); o has its own; gate and up share one; down has its own (11008 input
channels). Each H comes from 128 sequences x 2048 tokens of its own seeded heavy-tailed input,
4-bit asymmetric grids with group 128, block 128.

Every layer is checked against the fp64 oracle as the full-size tests check one layer: H on
sampled channel pairs, R on its trailing principal block (the factor of the trailing block of
H + lambda I alone), and on sampled rows >= 99.5 % identical codes, loss sums within 1 % and
W_hat = s (q - z) exactly.
"""
import numpy as np
import pytest
import torch

import oracle
from post_weight_quantization_12_b200 import api, synth

pytestmark = pytest.mark.gpu
DEV = "cuda"
SEED = 0
ROWS_SAMPLED = 8
TRAILING = 1024


def _check_hessian_and_factor(q, X, rng):
    cols = q.cols
    ch = np.unique(np.concatenate([rng.choice(cols, 10, replace=False), [0, cols - 1]]))
    idx = torch.from_numpy(ch).to(DEV)
    Xs = X[:, idx].double().cpu().numpy()
    H_ref = 2.0 * (Xs.T @ Xs) / X.shape[0]
    H_got = q.H[idx][:, idx].double().cpu().numpy()
    scale = np.sqrt(np.outer(np.diag(H_ref), np.diag(H_ref)))
    assert np.max(np.abs(H_got - H_ref) / scale) < 1e-4
    lam = q.damp_rel * float(torch.diagonal(q.H).double().mean().item())
    k = cols - TRAILING
    Hb = q.H[k:, k:].double().cpu().numpy() + lam * np.eye(TRAILING)
    Rb_ref = oracle.inverse_hessian_factor(Hb, 0.0)["R"]
    Rb = q.R[k:, k:].double().cpu().numpy()
    assert np.linalg.norm(Rb - Rb_ref) / np.linalg.norm(Rb_ref) < 1e-4


def _check_layer(name, spec, W, out, R, rng):
    rows, cols = W.shape
    assert out.info == 0, (name, out.info)
    rsel = np.sort(rng.choice(rows, ROWS_SAMPLED, replace=False))
    ridx = torch.from_numpy(rsel).to(DEV)
    ref = oracle.gptq_quantize(W[ridx].float().cpu().numpy(), R.double().cpu().numpy(), spec.bits,
                               spec.group, spec.block)
    got = out.codes[ridx].cpu().numpy()
    match = float((got == ref["codes"]).mean())
    assert match >= 0.995, (name, match)
    e_got = float(out.err_sq[ridx].double().sum().item())
    e_ref = float(ref["err_sq"].sum())
    assert abs(e_got - e_ref) <= 0.01 * e_ref, (name, e_got, e_ref)
    gidx = np.arange(cols) // spec.group
    s_ = out.scales[ridx].cpu().numpy()[:, gidx]
    z_ = out.zeros[ridx].cpu().numpy()[:, gidx].astype(np.float32)
    q_ = out.codes[ridx].cpu().numpy()
    assert q_.max() <= 2 ** spec.bits - 1
    np.testing.assert_array_equal(out.W_hat[ridx].cpu().numpy(), s_ * (q_.astype(np.float32) - z_))
    return match


def test_decoder_block_in_execution_order():
    layers = synth.block_layers(SEED)
    need = 262144 * 11008 * 2 + 8 * 11008 ** 2 * 4 + 16 * 11008 * 4096
    free = torch.cuda.mem_get_info()[0]
    if need > 0.9 * free:
        pytest.skip(f"needs {need / 1e9:.0f} GB of device memory, {free / 1e9:.0f} GB free")
    rng = np.random.default_rng(7)
    quantizer, current = None, None
    done = []
    for i, (spec, hid) in enumerate(layers):
        if hid != current:
            # a new input: its own seeded calibration tokens and a fresh quantizer
            current = hid
            quantizer = None
            torch.cuda.empty_cache()
            X = synth.inputs_torch(spec, SEED + 10 * i, DEV)
            quantizer = api.LayerQuantizer(spec.cols, device=DEV, damp_rel=spec.damp)
            quantizer.add_batch(X)
            quantizer.prepare()
            torch.cuda.synchronize()
            assert int(quantizer.info.item()) == 0, hid
            _check_hessian_and_factor(quantizer, X, rng)
            del X
        W = synth.weights_torch(spec, SEED + 10 * i, DEV)
        out = quantizer.quantize(W, spec.bits, spec.group, spec.block)
        torch.cuda.synchronize()
        done.append((spec.name, _check_layer(spec.name, spec, W, out, quantizer.R, rng)))
        del W, out
    assert [n for n, _ in done] == ["q_proj", "k_proj", "v_proj", "o_proj", "gate_proj",
                                    "up_proj", "down_proj"]
