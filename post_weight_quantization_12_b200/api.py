"""User-facing layer quantizer: allocates device buffers with PyTorch and calls the C ABI.

    q = LayerQuantizer(cols, device="cuda")
    for chunk in calibration_chunks:          # token-major [n, cols] bf16/fp32, host or device
        q.add_batch(chunk)
    out = q.quantize(W, bits=4, group=128, block=128)   # W [rows, cols] host or device

Host tensors are copied to the device (pinned-memory, non-blocking) before the call; outputs stay
on the device unless `to_host=True` (W_hat, which s (q - z) of the returned codes gives, only with
`host_w_hat=True`). PyTorch only provides memory and streams here; every step of the method runs in
the library's kernels.

A 4-bit result can be packed for the W4A16 product, and weights and calibration inputs can be
rotated before quantization:

    lin = pack_4bit(out)                      # PackedLinear4: packed codes, scales, zeros
    Y = lin(X)                                # fp32 [n, rows] = X W_hat^T for bf16 X [n, cols]
    Wr, Xr = rotate(W, signs), rotate(X, signs)   # data-free randomized Hadamard rotation
"""
from __future__ import annotations

from dataclasses import dataclass

import torch

from . import _lib


@dataclass
class QuantizedLayer:
    codes: torch.Tensor      # uint8 [rows, cols]
    scales: torch.Tensor     # fp32 [rows, G]
    zeros: torch.Tensor      # uint8 [rows, G]
    W_hat: torch.Tensor      # fp32 [rows, cols] dequantized weights
    err_sq: torch.Tensor     # fp32 [rows] sum of squared scaled errors
    info: int                # device status word after the call


class LayerQuantizer:
    """Streams calibration chunks into S, then factors and quantizes one layer (or several layers
    that share the same inputs, e.g. q/k/v projections)."""

    def __init__(self, cols: int, device="cuda", damp_rel: float = 0.01, stream=None):
        self.cols = int(cols)
        self.device = torch.device(device)
        self.damp_rel = float(damp_rel)
        self.stream = stream
        self.S = torch.zeros(self.cols, self.cols, device=self.device, dtype=torch.float32)
        self.info = torch.zeros(1, device=self.device, dtype=torch.int32)
        self.n_total = 0
        self.R = None

    def reset(self):
        """Start a new layer: S = 0, no tokens, no factor."""
        self.S.zero_()
        self.info.zero_()
        self.n_total = 0
        self.R = None

    def _on_device(self, t: torch.Tensor) -> torch.Tensor:
        if t.device == self.device:
            return t
        if t.device.type == "cpu":
            if not t.is_pinned():
                t = t.pin_memory()
            return t.to(self.device, non_blocking=True)
        return t.to(self.device)

    def add_batch(self, X: torch.Tensor, chunk_bytes: int = 256 << 20):
        """S += X^T X for token-major calibration inputs X [n_tokens, cols] (bf16 or fp32).

        A host tensor is copied in chunks of about `chunk_bytes` on a side stream into two device
        buffers, so each chunk's copy overlaps the accumulation of the previous one."""
        if X.device.type != "cpu":
            X = self._on_device(X)
            _lib.hessian_accumulate(self.S, X, self.info, self.stream)
            self.n_total += X.shape[0]
            return
        if not X.is_pinned():
            X = X.pin_memory()
        n, cols = X.shape
        rows_per = max(128, (chunk_bytes // max(1, cols * X.element_size())) // 128 * 128)
        if n <= rows_per:
            Xd = X.to(self.device, non_blocking=True)
            _lib.hessian_accumulate(self.S, Xd, self.info, self.stream)
            self.n_total += n
            return
        compute = self.stream if self.stream is not None else torch.cuda.current_stream(self.device)
        copy = torch.cuda.Stream(self.device)
        bufs = [torch.empty(rows_per, cols, dtype=X.dtype, device=self.device) for _ in range(2)]
        free = [torch.cuda.Event(), torch.cuda.Event()]   # buffer b no longer read by S1
        for b in range(2):
            free[b].record(compute)
        for i, r0 in enumerate(range(0, n, rows_per)):
            b = i & 1
            rows = min(rows_per, n - r0)
            copy.wait_event(free[b])
            with torch.cuda.stream(copy):
                bufs[b][:rows].copy_(X[r0:r0 + rows], non_blocking=True)
                landed = torch.cuda.Event()
                landed.record(copy)
            compute.wait_event(landed)
            _lib.hessian_accumulate(self.S, bufs[b][:rows], self.info, compute)
            free[b].record(compute)
        self.n_total += n
        for t in bufs:                     # keep the buffers alive until S1 has read them
            t.record_stream(compute)

    def prepare(self):
        """H = 2S/N (kept in self.S) and R, the upper factor of (H + lambda I)^-1."""
        ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, self.cols, 0),
                         device=self.device, dtype=torch.uint8)
        self.R = torch.empty(self.cols, self.cols, device=self.device, dtype=torch.float32)
        _lib.prepare_hinv(self.S, self.R, self.n_total, self.damp_rel, ws, self.info, self.stream)
        return self.R

    @property
    def H(self):
        return self.S

    def quantize(self, W: torch.Tensor, bits: int = 4, group: int = 128, block: int = 128,
                 to_host: bool = False, host_w_hat: bool = False) -> QuantizedLayer:
        """Quantize W [rows, cols] against the prepared factor. Outputs stay on the device unless
        `to_host`; then codes, scales, zeros and err_sq come back in pinned host memory, and W_hat
        (fp32, the largest output, equal to s (q - z) of the returned codes) only with
        `host_w_hat` -- otherwise it stays on the device."""
        if self.R is None:
            self.prepare()
        W = self._on_device(W)
        rows, cols = W.shape
        G = 1 if group <= 0 else cols // group
        dev = self.device
        W_hat = torch.empty(rows, cols, device=dev, dtype=torch.float32)
        codes = torch.empty(rows, cols, device=dev, dtype=torch.uint8)
        scales = torch.empty(rows, G, device=dev, dtype=torch.float32)
        zeros = torch.empty(rows, G, device=dev, dtype=torch.uint8)
        err_sq = torch.empty(rows, device=dev, dtype=torch.float32)
        ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, block),
                         device=dev, dtype=torch.uint8)
        _lib.quantize_layer(W, self.R, bits, group, block, W_hat, codes, scales, zeros, err_sq, ws,
                            self.info, self.stream)
        if to_host:
            # pinned host outputs, copied asynchronously on the same stream, one synchronization
            stream = self.stream if self.stream is not None else torch.cuda.current_stream(dev)
            outs = []
            with torch.cuda.stream(stream):
                for t in (codes, scales, zeros, W_hat if host_w_hat else None, err_sq):
                    if t is None:
                        outs.append(W_hat)
                        continue
                    h = torch.empty(t.shape, dtype=t.dtype, pin_memory=True)
                    h.copy_(t, non_blocking=True)
                    outs.append(h)
                info_h = torch.empty(1, dtype=torch.int32, pin_memory=True)
                info_h.copy_(self.info, non_blocking=True)
            stream.synchronize()
            codes, scales, zeros, W_hat, err_sq = outs
            info = int(info_h.item())
        else:
            info = int(self.info.item())
        return QuantizedLayer(codes, scales, zeros, W_hat, err_sq, info)


@dataclass
class PackedLinear4:
    """A 4-bit quantized linear layer in the packed layout the W4A16 product reads."""
    packed: torch.Tensor     # int32 [rows, cols // 8]: eight 4-bit codes per word
    scales: torch.Tensor     # fp32 [rows, G]
    zeros: torch.Tensor      # uint8 [rows, G]
    group: int               # -1 (per row) or the group size

    @property
    def rows(self) -> int:
        return self.packed.shape[0]

    @property
    def cols(self) -> int:
        return 8 * self.packed.shape[1]

    def __call__(self, X: torch.Tensor, out=None, stream=None) -> torch.Tensor:
        """fp32 [n, rows] = X W_hat^T for bf16 activations X [n, cols] (n > 16 on the tensor-core
        kernel)."""
        if out is None:
            out = torch.empty(X.shape[0], self.rows, device=X.device, dtype=torch.float32)
        _lib.w4a16_matmul(self.packed, self.scales, self.zeros, self.group, X, out, stream=stream)
        return out


def pack_4bit(layer: QuantizedLayer, stream=None) -> PackedLinear4:
    """Packs the codes of a 4-bit QuantizedLayer (device tensors) for the W4A16 product."""
    rows, cols = layer.codes.shape
    G = layer.scales.shape[1]
    packed = torch.empty(rows, cols // 8, device=layer.codes.device, dtype=torch.int32)
    _lib.pack_codes_4bit(layer.codes, packed, stream=stream)
    return PackedLinear4(packed, layer.scales, layer.zeros, -1 if G == 1 else cols // G)


def rotate(X: torch.Tensor, sign_bits=None, out=None, stream=None) -> torch.Tensor:
    """X Q with Q = diag(signs) (I (x) H_b) / sqrt(b), the randomized Hadamard rotation of the last
    axis (see gptq_hadamard_rotate); `sign_bits` int32 [cols // 32] (bit j % 32 of word j // 32 set
    negates column j) or None. Returns a new tensor of X's dtype unless `out` is given (which may
    be X itself)."""
    if out is None:
        out = torch.empty_like(X)
    _lib.hadamard_rotate(X, out, sign_bits, stream)
    return out

