"""Seeded synthetic inputs for GPTQ layer quantization.

This module only draws random numbers with fixed shapes, distributions and seeds. It holds none of
the quantization arithmetic, so both the CUDA path and the CPU oracle can be fed from it without
sharing any of the method's code.

Workloads (the pages quantize OPT-175B / BLOOM-176B with real calibration text; none of that is
available, so these seeded stand-ins keep the shapes and value structure):

* weights ``W`` [rows, cols]: i.i.d. N(0, std^2), std 0.02 (0.01 for the 175B-class shapes);
* calibration inputs ``X`` token-major [n_tokens, cols]:
  - "tiny": N(0,1) times a per-channel scale s_c = exp(U[ln 0.1, ln 10]);
  - "heavy": Student-t with 3 degrees of freedom, Z / sqrt(chi2_3 / 3), with a seeded set of
    outlier channels (the first ceil(frac * cols) entries of a seeded permutation) multiplied by a
    constant factor (x20 at 1 %, x30 at 0.5 %).

Seeds: W uses seed+0, the per-channel scales / outlier permutation seed+1, X seed+2.
CPU draws use ``numpy.random.default_rng``; device draws use ``torch.Generator`` on the device.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field

import numpy as np


@dataclass(frozen=True)
class LayerSpec:
    """One linear layer to quantize: W is rows x cols, X is n_tokens x cols."""
    name: str
    rows: int
    cols: int
    n_tokens: int
    bits: int
    group: int            # -1 = one scale per row, else group size along cols
    block: int            # lazy-batch block width B
    w_std: float = 0.02
    x_kind: str = "heavy"  # "tiny" or "heavy"
    outlier_frac: float = 0.01
    outlier_mult: float = 20.0
    x_dtype: str = "bf16"  # "bf16" or "fp32"
    w_dtype: str = "bf16"
    damp: float = 0.01


# The five workloads. "tiny" is small enough for the fp64 oracle to finish in seconds.
TINY = LayerSpec("tiny", 64, 128, 1024, 4, -1, 32, x_kind="tiny", x_dtype="fp32", w_dtype="fp32")
ATTN = LayerSpec("attn_4096x4096", 4096, 4096, 262144, 4, 128, 128)
MLP_UP = LayerSpec("mlp_up_11008x4096", 11008, 4096, 131072, 3, -1, 128)
MLP_DOWN = LayerSpec("mlp_down_4096x11008", 4096, 11008, 131072, 3, -1, 128)
FC1 = LayerSpec("fc1_49152x12288", 49152, 12288, 262144, 4, 128, 128, w_std=0.01,
                outlier_frac=0.005, outlier_mult=30.0)
FC2 = LayerSpec("fc2_12288x49152", 12288, 49152, 262144, 4, 128, 128, w_std=0.01,
                outlier_frac=0.005, outlier_mult=30.0)


def block_layers(seed: int = 0):
    """The 7B-class decoder block: (layer spec, hessian id) in execution order.

    q, k, v share one H (same input); gate and up share one H; o and down have their own.
    """
    n = 128 * 2048
    mk = lambda nm, r, c: LayerSpec(nm, r, c, n, 4, 128, 128)
    return [
        (mk("q_proj", 4096, 4096), "qkv"), (mk("k_proj", 4096, 4096), "qkv"),
        (mk("v_proj", 4096, 4096), "qkv"), (mk("o_proj", 4096, 4096), "o"),
        (mk("gate_proj", 11008, 4096), "gate_up"), (mk("up_proj", 11008, 4096), "gate_up"),
        (mk("down_proj", 4096, 11008), "down"),
    ]


def scaled_spec(spec: LayerSpec, rows: int, cols: int, n_tokens: int, **kw) -> LayerSpec:
    """Same value recipe at other sizes (for small parity cases)."""
    d = dict(spec.__dict__)
    d.update(rows=rows, cols=cols, n_tokens=n_tokens, name=f"{spec.name}@{rows}x{cols}x{n_tokens}")
    d.update(kw)
    return LayerSpec(**d)


# ----------------------------------------------------------------------------------------------
# CPU (numpy) draws
# ----------------------------------------------------------------------------------------------

def outlier_channels_np(cols: int, frac: float, seed: int) -> np.ndarray:
    rng = np.random.default_rng(seed + 1)
    k = int(math.ceil(frac * cols)) if frac > 0 else 0
    return rng.permutation(cols)[:k]


def weights_np(spec: LayerSpec, seed: int) -> np.ndarray:
    """W as float32 [rows, cols]; rounded through bf16 when the spec's W is bf16."""
    rng = np.random.default_rng(seed + 0)
    w = (rng.standard_normal((spec.rows, spec.cols)) * spec.w_std).astype(np.float32)
    if spec.w_dtype == "bf16":
        w = round_to_bf16_np(w)
    return w


def inputs_np(spec: LayerSpec, seed: int) -> np.ndarray:
    """X as float32 [n_tokens, cols]; values exactly representable in bf16 when X is bf16."""
    if spec.x_kind == "tiny":
        rs = np.random.default_rng(seed + 1)
        scale = np.exp(rs.uniform(math.log(0.1), math.log(10.0), size=spec.cols))
        rx = np.random.default_rng(seed + 2)
        x = rx.standard_normal((spec.n_tokens, spec.cols)) * scale[None, :]
    else:
        rx = np.random.default_rng(seed + 2)
        z = rx.standard_normal((spec.n_tokens, spec.cols))
        chi = (rx.standard_normal((spec.n_tokens, spec.cols, 3)) ** 2).sum(axis=2)
        x = z / np.sqrt(chi / 3.0)
        idx = outlier_channels_np(spec.cols, spec.outlier_frac, seed)
        x[:, idx] *= spec.outlier_mult
    x = x.astype(np.float32)
    if spec.x_dtype == "bf16":
        x = round_to_bf16_np(x)
    return x


def round_to_bf16_np(a: np.ndarray) -> np.ndarray:
    """Round float32 values to the nearest bf16 (ties to even); returns float32 holding them."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    rounded = ((u + 0x7FFF + ((u >> 16) & 1)) >> 16) << 16
    return rounded.astype(np.uint32).view(np.float32)


def bf16_bits_np(a: np.ndarray) -> np.ndarray:
    """Upper 16 bits of float32 values that are already bf16-representable (uint16 array)."""
    return (np.ascontiguousarray(a, dtype=np.float32).view(np.uint32) >> 16).astype(np.uint16)


# ----------------------------------------------------------------------------------------------
# Device (torch) draws, for the full-size workloads
# ----------------------------------------------------------------------------------------------

def weights_torch(spec: LayerSpec, seed: int, device):
    import torch
    g = torch.Generator(device=device).manual_seed(seed + 0)
    dt = torch.bfloat16 if spec.w_dtype == "bf16" else torch.float32
    w = torch.empty(spec.rows, spec.cols, device=device, dtype=dt)
    chunk = max(1, (1 << 26) // spec.cols)
    for r0 in range(0, spec.rows, chunk):
        r1 = min(spec.rows, r0 + chunk)
        w[r0:r1] = (torch.randn(r1 - r0, spec.cols, generator=g, device=device) * spec.w_std).to(dt)
    return w


def inputs_torch(spec: LayerSpec, seed: int, device, n_tokens: int | None = None, out=None):
    """Token-major X [n_tokens, cols] drawn on ``device`` in chunks (bf16 or fp32)."""
    import torch
    n = spec.n_tokens if n_tokens is None else n_tokens
    dt = torch.bfloat16 if spec.x_dtype == "bf16" else torch.float32
    x = out if out is not None else torch.empty(n, spec.cols, device=device, dtype=dt)
    gs = torch.Generator(device=device).manual_seed(seed + 1)
    gx = torch.Generator(device=device).manual_seed(seed + 2)
    if spec.x_kind == "tiny":
        scale = torch.exp(torch.empty(spec.cols, device=device).uniform_(
            math.log(0.1), math.log(10.0), generator=gs))
    else:
        k = int(math.ceil(spec.outlier_frac * spec.cols)) if spec.outlier_frac > 0 else 0
        perm = torch.randperm(spec.cols, generator=gs, device=device)[:k]
        scale = torch.ones(spec.cols, device=device)
        scale[perm] = spec.outlier_mult
    chunk = max(1, (1 << 25) // spec.cols)
    for t0 in range(0, n, chunk):
        t1 = min(n, t0 + chunk)
        z = torch.randn(t1 - t0, spec.cols, generator=gx, device=device)
        if spec.x_kind == "tiny":
            v = z * scale
        else:
            c = torch.randn(t1 - t0, spec.cols, 3, generator=gx, device=device).square_().sum(-1)
            v = z * torch.rsqrt(c / 3.0) * scale
        x[t0:t1] = v.to(dt)
    return x


# ----------------------------------------------------------------------------------------------
# Quantized-weight operands for the W4A16 product
# ----------------------------------------------------------------------------------------------

def w4a16_operands_torch(rows: int, cols: int, group: int, seed: int, device="cpu"):
    """Stand-in quantized layer for timing and parity of the W4A16 product, drawn on ``device``:
    codes uint8 [rows, cols] uniform in 0..15 (seed+0); scales float32 [rows, G] log-uniform in
    [1e-3, 1e-2] (the step of a 4-bit grid over weights of std 0.01-0.02) and zero points uint8
    [rows, G] uniform in 0..15 (seed+1); G = 1 for group <= 0, else cols // group."""
    import torch
    G = 1 if group <= 0 else cols // group
    gc = torch.Generator(device=device).manual_seed(seed + 0)
    gm = torch.Generator(device=device).manual_seed(seed + 1)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=device)
    chunk = max(1, (1 << 26) // max(cols, 1))
    for r0 in range(0, rows, chunk):
        r1 = min(rows, r0 + chunk)
        codes[r0:r1] = torch.randint(0, 16, (r1 - r0, cols), generator=gc, device=device,
                                     dtype=torch.uint8)
    scales = torch.exp(torch.empty(rows, G, device=device).uniform_(
        math.log(1e-3), math.log(1e-2), generator=gm))
    zeros = torch.randint(0, 16, (rows, G), generator=gm, device=device, dtype=torch.uint8)
    return codes, scales, zeros
