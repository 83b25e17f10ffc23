"""Benchmark: GPTQ layer quantization of one 4096 x 4096 attention projection on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = the whole path for one layer on inputs already resident in HBM: S += X^T X over all
262144 calibration tokens (S1), the damped inverse-Hessian factor (S2-S5) and the blocked column
loop with lazy trailing updates (S6-S8), 4-bit, group 128, block 128. The metric is weights/s
(rows * cols / step time), whole job over all ranks; `ms_per_step` is ms per layer.

Multi-GPU: the layers are independent problems, so each rank quantizes its own layer (its own
seeded inputs) with no collective on the data path ("scaling": "weak"); the timed region is
bracketed by a barrier and device synchronizations and the max over ranks is reported.

Extra keys: `roofline` for the dominant kernel (the tensor-core Hessian SYRK, timed live with CUDA
events on its stream), `e2e` (the same work through the public API from pinned host buffers,
copies included), `cpu_baseline` (the fp64 oracle on a bounded sample of the same workload,
extrapolated; rank 0 at N=1 only), `clocks` (nvidia-smi sampled during the timed region) and
`gpu_launches` (kernels the library enqueued inside the timed region), and `w4a16`: the packed
4-bit product that consumes the quantizer's codes (decode GEMV, 1 and 8 activation vectors, and the
packing kernel), timed alone against the HBM roofline (skip it with --no-w4a16), and `rotation`:
the data-free Hadamard rotation of the layer's calibration input and weights that can precede
GPTQ, likewise (skip it with --no-rotation), and `obq`: the OBQ greedy-order reference against
GPTQ's fixed order on a 4096 x 128 layer, timed, with both proxy losses (skip it with --no-obq).
Each of these three also carries a `cpu_baseline`: the oracle on a bounded sample of its workload
(rank 0 at N=1, like the headline's).
`--impl reference` times the fp64 CPU oracle on the same workload instead (bounded samples).
"""
from __future__ import annotations

import argparse
import datetime
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "GPTQ layer quantize: weights/sec & ms per layer (4-bit g128); % of roofline"
UNIT = "weights/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
# Nominal dense tf32 / bf16 throughput ratio (1.1 / 2.25 PFLOP/s): used only if the tf32 probe
# below cannot run.
TF32_PER_BF16 = 1.1 / 2.25
CONFIGS = ("mlp_up", "mlp_down", "block", "fc1", "fc2")
# DRAM traffic of the S1 kernel from one ncu capture of 16384 tokens x 4096 channels (reads scale
# with tokens -- X is streamed once per round of tiles; writes are S, once per launch).
SYRK_CAPTURE = {"tokens": 16384, "cols": 4096, "dram_read": 269.611e6, "dram_write": 23.566e6}


def parse():
    p = argparse.ArgumentParser()
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=10)
    p.add_argument("--warmup", type=int, default=3)
    p.add_argument("--impl", default="ours", choices=["ours", "reference"])
    p.add_argument("--seed", type=int, default=0)
    p.add_argument("--tokens", type=int, default=0,
                   help="override the calibration token count (profiling runs only; the line is "
                        "then marked as not the configured workload)")
    p.add_argument("--no-e2e", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--no-w4a16", action="store_true")
    p.add_argument("--no-rotation", action="store_true")
    p.add_argument("--no-obq", action="store_true")
    p.add_argument("--cpu-sample-s", type=float, default=20.0)
    p.add_argument("--configs", default="all",
                   help="per-config leg (1 GPU only): 'all', 'none' or a comma list of "
                        + ", ".join(CONFIGS))
    return p.parse_args()


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return d, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def workload(tokens_override: int):
    from post_weight_quantization_12_b200 import synth
    spec = synth.ATTN
    if tokens_override:
        spec = synth.scaled_spec(spec, spec.rows, spec.cols, tokens_override)
    return spec


def config_dict(spec):
    return {
        "workload": f"attention projection: W {spec.rows}x{spec.cols} bf16 ~N(0,0.02^2); "
                    f"X {spec.n_tokens} tokens x {spec.cols} bf16 Student-t(3), 1% channels x20; "
                    f"{spec.bits}-bit asymmetric group {spec.group}, block {spec.block}, damp 1%",
        "rows": spec.rows, "cols": spec.cols, "n_tokens": spec.n_tokens, "bits": spec.bits,
        "group": spec.group, "block": spec.block,
        "l2": f"inputs larger than L2: X is {spec.n_tokens * spec.cols * 2 / 1e9:.2f} GB, "
              "read in full every step",
    }


# ------------------------------------------------------------------------------------------------
# clocks
# ------------------------------------------------------------------------------------------------

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.25)
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        for line in open(self.path):
            parts = [p.strip() for p in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]), parts[5:9]))
            except ValueError:
                continue
        os.unlink(self.path)
        if not rows:
            return None
        max_mhz = max(r[1] for r in rows)
        pmax = max(r[2] for r in rows)
        loaded = [r for r in rows if r[2] >= 0.5 * pmax] or rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in loaded for i, v in enumerate(r[3])
                          if v.lower().startswith("active")})
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max_mhz,
                "reasons": reasons, "samples": len(rows), "samples_under_load": len(loaded),
                "power_w_max": pmax}


# ------------------------------------------------------------------------------------------------
# CPU oracle on a bounded sample
# ------------------------------------------------------------------------------------------------

def oracle_sample(W_np, X_np, spec, budget_s: float):
    """Time the fp64 oracle stage by stage on a sample of the workload and extrapolate to the full
    layer: S1 on a token subsample (time ~ tokens), S2-S5 in full, S6-S8 on a row subsample (rows
    are independent given R; time ~ rows). Returns (seconds for the full layer, description)."""
    import numpy as np
    import oracle
    cols = spec.cols
    n_tok = X_np.shape[0]
    t0 = time.perf_counter()
    S = np.zeros((cols, cols))
    oracle.hessian_accumulate(S, X_np)
    t_s1 = time.perf_counter() - t0
    H = oracle.hessian_finalize(S, n_tok)
    t0 = time.perf_counter()
    fac = oracle.inverse_hessian_factor(H, spec.damp)
    t_s25 = time.perf_counter() - t0
    r_sub = W_np.shape[0]
    t0 = time.perf_counter()
    oracle.gptq_quantize(W_np, fac["R"], spec.bits, spec.group, spec.block)
    t_s68 = time.perf_counter() - t0
    full = t_s1 * (spec.n_tokens / n_tok) + t_s25 + t_s68 * (spec.rows / r_sub)
    desc = (f"S1 on {n_tok} of {spec.n_tokens} tokens ({t_s1:.2f} s, x{spec.n_tokens / n_tok:g}); "
            f"S2-S5 in full at {cols}x{cols} ({t_s25:.2f} s); S6-S8 on {r_sub} of {spec.rows} rows "
            f"({t_s68:.2f} s, x{spec.rows / r_sub:g}); extrapolated {full:.1f} s per layer")
    return full, desc, t_s1 + t_s25 + t_s68


def oracle_extras(rows_w4: int = 256, tokens_rot: int = 4096, rows_obq: int = 64):
    """The fp64 oracle on bounded samples of the extra legs' workloads, extrapolated to the full
    ones (time ~ rows, tokens or rows): the W4A16 product of the 12288 x 49152 g128 layer on
    `rows_w4` rows, the rotation of 262144 x 4096 calibration tokens on `tokens_rot` tokens, OBQ
    of the 4096 x 128 layer on `rows_obq` rows. Inputs are seeded CPU draws of the same shapes.
    Returns {"w4a16": {...}, "rotation": {...}, "obq": {...}}, each with the extrapolated value in
    the leg's own unit."""
    import numpy as np
    import oracle
    from post_weight_quantization_12_b200 import synth

    out = {}
    cols = 49152
    codes, scales, zeros = synth.w4a16_operands_torch(rows_w4, cols, 128, 5, "cpu")
    x = synth.inputs_torch(synth.scaled_spec(synth.ATTN, 1, cols, 1), 7, "cpu").float().numpy()
    words = oracle.pack_codes(codes.numpy())
    t0 = time.perf_counter()
    oracle.w4a16_matmul(words, scales.numpy(), zeros.numpy(), 128, x)
    dt = time.perf_counter() - t0
    full = dt * 12288 / rows_w4
    out["w4a16"] = {"value": full * 1e6, "unit": "us per product (n = 1)", "kind": "oracle",
                    "cores": cpu_threads(),
                    "sample": f"{rows_w4} of 12288 rows ({dt:.3f} s, x{12288 / rows_w4:g})"}
    xr = synth.inputs_torch(synth.scaled_spec(synth.ATTN, 1, 4096, tokens_rot), 9, "cpu")
    xr = xr.float().numpy()
    signs = np.where(np.random.default_rng(3).random(4096) < 0.5, -1.0, 1.0)
    t0 = time.perf_counter()
    oracle.rotate(xr, signs)
    dt = time.perf_counter() - t0
    full = dt * 262144 / tokens_rot
    out["rotation"] = {"value": full * 1e6, "unit": "us per 262144 x 4096 rotation",
                       "kind": "oracle", "cores": cpu_threads(),
                       "sample": f"{tokens_rot} of 262144 tokens ({dt:.3f} s, "
                                 f"x{262144 / tokens_rot:g})"}
    rng = np.random.default_rng(11)
    Xo = rng.standard_normal((1024, 128))
    Hd = oracle.damp(oracle.hessian(Xo))[0]
    Wo = (rng.standard_normal((rows_obq, 128)) * 0.02).astype(np.float32)
    t0 = time.perf_counter()
    oracle.obq_quantize(Wo, np.linalg.inv(Hd), 4)
    dt = time.perf_counter() - t0
    full = dt * 4096 / rows_obq
    out["obq"] = {"value": full * 1e3, "unit": "ms per 4096 x 128 layer (greedy)", "kind": "oracle",
                  "cores": cpu_threads(),
                  "sample": f"{rows_obq} of 4096 rows ({dt:.3f} s, x{4096 / rows_obq:g})"}
    return out


def cpu_threads():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def sample_sizes(spec, budget_s: float):
    # chosen so the three stages take roughly budget_s together on a many-core host
    n_tok = 8192 if budget_s >= 10 else 2048
    r_sub = 64 if budget_s >= 10 else 16
    return n_tok, r_sub


# ------------------------------------------------------------------------------------------------
# reference arm: the oracle itself
# ------------------------------------------------------------------------------------------------

def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import numpy as np
    from post_weight_quantization_12_b200 import synth
    spec = workload(args.tokens)
    n_tok, r_sub = sample_sizes(spec, args.cpu_sample_s)
    sub = synth.scaled_spec(spec, r_sub, spec.cols, n_tok)
    W = synth.weights_np(sub, args.seed)
    X = synth.inputs_np(sub, args.seed)
    times = []
    for i in range(args.warmup + args.steps):
        full, desc, spent = oracle_sample(W, X, spec, args.cpu_sample_s)
        if i >= args.warmup:
            times.append(full)
    t = statistics.mean(times)
    value = spec.rows * spec.cols / t
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": t * 1e3,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded; numpy draws of the same recipe)", "config": config_dict(spec),
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": cpu_threads(), "kind": "oracle",
                         "sample": desc},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "extrapolated": True,
        "note": "value and ms_per_step are extrapolated to the whole layer from bounded samples "
                "(stated in cpu_baseline.sample); each step times one sample, not one layer",
    }
    print(json.dumps(line), flush=True)
    return 0


# ------------------------------------------------------------------------------------------------
# our arm
# ------------------------------------------------------------------------------------------------

def rank_seed(seed: int, rank: int) -> int:
    """Each rank quantizes its own independent layer: seeds 1000 apart."""
    return seed + 1000 * rank


def aggregate(elapsed_ms: float, launches: int, world: int, device):
    """Job time = max over ranks (every rank's work must finish); kernel launches = sum."""
    if world <= 1:
        return elapsed_ms, launches
    import torch
    import torch.distributed as dist
    t = torch.tensor([elapsed_ms], device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    c = torch.tensor([launches], device=device, dtype=torch.int64)
    dist.all_reduce(c, op=dist.ReduceOp.SUM)
    return float(t.item()), int(c.item())


def bench_w4a16(dev, stream, peaks, peaks_src, iters=50):
    """The W4A16 product on packed 4-bit codes (decode: one activation vector; and a batch of 8),
    timed with CUDA events on the launching stream. Algorithmic bytes per launch: the packed codes
    (rows * cols / 2), scales and zero points (5 bytes per row and group), the activations
    (2 n cols) and the output (4 n rows). Inputs are larger than L2 (126 MB): the 12288 x 49152
    layer holds 326 MB of weights, and the 4096 x 4096 case cycles through 24 separate layers."""
    import torch
    from post_weight_quantization_12_b200 import _lib, synth

    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    info = torch.zeros(1, device=dev, dtype=torch.int32)

    def make(rows, cols, group, seed):
        codes, scales, zeros = synth.w4a16_operands_torch(rows, cols, group, seed, dev)
        packed = torch.empty(rows, cols // 8, device=dev, dtype=torch.int32)
        _lib.pack_codes_4bit(codes, packed, info, stream)
        return codes, packed, scales, zeros

    def timed(fn, reps):
        for _ in range(3):
            fn(0)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for k in range(reps):
            fn(k)
        b.record(stream)
        torch.cuda.synchronize(dev)
        return a.elapsed_time(b) / reps * 1e3          # us per launch

    out = {"kernel": "w4a16_gemv_kernel", "bound": "hbm", "peak_gbs": hbm,
           "peak_source": f"{peaks_src} HBM copy (kernel timed alone)", "cases": []}
    cases = [("fc2_12288x49152_g128", 12288, 49152, 128, 1, 1),
             ("fc2_12288x49152_g128", 12288, 49152, 128, 8, 1),
             ("attn_4096x4096_g128 x24 layers", 4096, 4096, 128, 1, 24)]
    made = {}
    for name, rows, cols, group, n, layers in cases:
        key = (rows, cols, group, layers)
        if key not in made:
            made.clear()
            torch.cuda.empty_cache()
            made[key] = [make(rows, cols, group, 100 + i) for i in range(layers)]
        mats = made[key]
        X = synth.inputs_torch(synth.scaled_spec(synth.ATTN, 1, cols, n), 7, dev)
        Y = torch.empty(n, rows, device=dev)
        G = cols // group

        def fn(k, mats=mats, X=X, Y=Y, group=group):
            _, packed, scales, zeros = mats[k % len(mats)]
            _lib.w4a16_matmul(packed, scales, zeros, group, X, Y, info, stream)

        us = timed(fn, max(iters, 2 * layers))
        nbytes = rows * cols / 2 + 5.0 * rows * G + 2.0 * n * cols + 4.0 * n * rows
        gbs = nbytes / (us * 1e-6) / 1e9
        case = {"layer": name, "n": n, "us": us, "bytes": nbytes, "achieved_gbs": gbs,
                "frac": gbs / hbm, "weights_per_s": rows * cols / (us * 1e-6)}
        if layers > 1:
            # the same calls replayed from a CUDA graph (as a decoder issues them): the device
            # time per product without the host's per-call work (argument checks, two tensor-map
            # encodes). The eager timing above stays the case's number.
            try:
                g = torch.cuda.CUDAGraph()
                with torch.cuda.graph(g):
                    cs = torch.cuda.current_stream(dev)
                    for k in range(layers):
                        _, packed, scales, zeros = mats[k]
                        _lib.w4a16_matmul(packed, scales, zeros, group, X, Y, info, cs)
                for _ in range(3):
                    g.replay()
                a = torch.cuda.Event(enable_timing=True)
                b = torch.cuda.Event(enable_timing=True)
                torch.cuda.synchronize(dev)
                reps = 20
                a.record()
                for _ in range(reps):
                    g.replay()
                b.record()
                torch.cuda.synchronize(dev)
                ug = a.elapsed_time(b) / (reps * layers) * 1e3
                gg = nbytes / (ug * 1e-6) / 1e9
                case["graph"] = {"us": ug, "achieved_gbs": gg, "frac": gg / hbm,
                                 "note": f"{layers} products captured in one CUDA graph, replayed"}
                del g
            except Exception as exc:  # context only: the eager number stands
                case["graph"] = {"unavailable": str(exc)[:200]}
        out["cases"].append(case)
    # batches of activation rows (n > 16): the tensor-core form of the same product; algorithmic
    # work 2 n rows cols flop (bf16 tensor peak) and the same weight bytes (HBM peak)
    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    key = (12288, 49152, 128, 1)
    if key not in made:
        made.clear()
        torch.cuda.empty_cache()
        made[key] = [make(12288, 49152, 128, 100)]
    out["gemm"] = {"kernel": "w4a16_gemm_kernel", "peak_tflops": bf16,
                   "peak_source": f"{peaks_src} bf16 burst (kernel timed alone)", "cases": []}
    for n in (64, 256):
        rows, cols, group = key[:3]
        _, packed, scales, zeros = made[key][0]
        X = synth.inputs_torch(synth.scaled_spec(synth.ATTN, 1, cols, n), 7, dev)
        Y = torch.empty(n, rows, device=dev)

        def fg(k, packed=packed, scales=scales, zeros=zeros, X=X, Y=Y):
            _lib.w4a16_matmul(packed, scales, zeros, group, X, Y, info, stream)

        us = timed(fg, 20)
        G = cols // group
        nbytes = rows * cols / 2 + 5.0 * rows * G + 2.0 * n * cols + 4.0 * n * rows
        flops = 2.0 * n * rows * cols
        out["gemm"]["cases"].append({
            "layer": "fc2_12288x49152_g128", "n": n, "us": us, "bytes": nbytes,
            "achieved_gbs": nbytes / (us * 1e-6) / 1e9, "frac_hbm": nbytes / (us * 1e-6) / 1e9 / hbm,
            "achieved_tflops": flops / (us * 1e-6) / 1e12,
            "frac_tensor": flops / (us * 1e-6) / 1e12 / bf16,
            "weights_per_s": rows * cols / (us * 1e-6)})
    # packing the quantizer's uint8 codes: reads rows * cols bytes, writes half of that
    made.clear()
    codes, packed, _, _ = make(12288, 49152, 128, 99)

    def fp(k):
        _lib.pack_codes_4bit(codes, packed, info, stream)

    us = timed(fp, 20)
    nbytes = 1.5 * codes.numel()
    out["pack"] = {"kernel": "pack_codes_4bit_vec_kernel", "layer": "12288x49152", "us": us,
                   "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9,
                   "frac": nbytes / (us * 1e-6) / 1e9 / hbm}
    # the 3-bit layout of the same layer's codes (values < 8): reads one byte per code, writes 3/8
    codes.bitwise_and_(7)
    packed3 = torch.empty(codes.shape[0], 3 * codes.shape[1] // 32, device=dev, dtype=torch.int32)

    def fp3(k):
        _lib.pack_codes_3bit(codes, packed3, info, stream)

    us = timed(fp3, 20)
    nbytes = 1.375 * codes.numel()
    out["pack3"] = {"kernel": "pack_codes_3bit_kernel", "layer": "12288x49152", "us": us,
                    "bytes": nbytes, "achieved_gbs": nbytes / (us * 1e-6) / 1e9,
                    "frac": nbytes / (us * 1e-6) / 1e9 / hbm}
    del packed3
    torch.cuda.synchronize(dev)
    if int(info.item()) != 0:
        raise RuntimeError(f"device status {int(info.item())} in the W4A16 leg")
    del codes, packed
    torch.cuda.empty_cache()
    return out


def bench_rotation(dev, stream, peaks, peaks_src, spec, X, iters=10):
    """The data-free Hadamard rotation applied before GPTQ, timed alone with CUDA events on the
    launching stream: the layer's whole calibration input (token-major bf16, rotated into a second
    buffer of the same size, both far larger than L2) and its fp32 weights. Algorithmic bytes per
    launch: one read and one write of every element."""
    import numpy as np
    import torch
    from post_weight_quantization_12_b200 import _lib, synth

    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    rng = np.random.default_rng(123)
    bits = np.packbits(rng.random(spec.cols) < 0.5, bitorder="little").view("<u4")
    sign_bits = torch.from_numpy(bits.view(np.int32).copy()).to(dev)
    W = synth.weights_torch(spec, 1, dev).float()
    cases = [("calibration X %dx%d bf16 -> bf16" % tuple(X.shape), X, torch.empty_like(X)),
             ("weights W %dx%d fp32 -> fp32" % tuple(W.shape), W, torch.empty_like(W))]
    block = _lib.hadamard_block(spec.cols)
    out = {"kernel": "hadamard4096_kernel" if block == 4096 else "hadamard_rotate_kernel",
           "bound": "hbm", "peak_gbs": hbm,
           "block": block,
           "peak_source": f"{peaks_src} HBM copy (kernel timed alone)", "cases": []}
    for name, src, dst in cases:
        for _ in range(3):
            _lib.hadamard_rotate(src, dst, sign_bits, stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(iters):
            _lib.hadamard_rotate(src, dst, sign_bits, stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        us = a.elapsed_time(b) / iters * 1e3
        nbytes = float(src.numel() * src.element_size() + dst.numel() * dst.element_size())
        gbs = nbytes / (us * 1e-6) / 1e9
        out["cases"].append({"case": name, "us": us, "bytes": nbytes, "achieved_gbs": gbs,
                             "frac": gbs / hbm})
    del cases, W
    torch.cuda.empty_cache()
    return out


def bench_obq(dev, stream, rows=4096, cols=128, tokens=32768, iters=3):
    """OBQ's greedy order against GPTQ's fixed order on a 4096 x 128 layer, 4-bit per row: the
    proxy Hessian and its damped inverse factor R come from this library's S1-S5 calls on
    token-major bf16 inputs, H^-1 = R^T R in fp64. Times the OBQ kernel (greedy, and the natural
    order through the same downdates), and reports the proxy loss sum_r (w_hat - w)^T H_d
    (w_hat - w) of OBQ, of OBQ in natural order and of the library's GPTQ column loop, plus the
    relative layer error with the undamped H. fp64 work per row ~ 2 cols^3 instructions (the
    downdates; their multiply and subtract are separate instructions). The peak is measured in
    the same run: a cuBLAS fp64 GEMM's flop rate halved (one fused multiply-add per two flop) is
    the fp64 instruction rate the GPU sustains; the nominal 148 SMs x 64 fp64 lanes x 1965 MHz =
    18.6e12 instructions/s is kept beside it for context."""
    import torch
    from post_weight_quantization_12_b200 import _lib, synth

    spec = synth.scaled_spec(synth.ATTN, rows, cols, tokens, group=-1)
    X = synth.inputs_torch(spec, 21, dev)
    W = synth.weights_torch(spec, 21, dev).float()
    S = torch.zeros(cols, cols, device=dev)
    R = torch.empty(cols, cols, device=dev)
    info = torch.zeros(1, device=dev, dtype=torch.int32)
    _lib.hessian_accumulate(S, X, info, stream)
    ws = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), device=dev,
                     dtype=torch.uint8)
    _lib.prepare_hinv(S, R, tokens, spec.damp, ws, info, stream)
    torch.cuda.synchronize(dev)
    if int(info.item()) != 0:
        raise RuntimeError(f"device status {int(info.item())} preparing the OBQ layer")
    H = S.double()                                     # undamped H = 2 X^T X / N (both triangles)
    Hinv = (R.double().T @ R.double()).contiguous()
    Hd = torch.linalg.inv(Hinv)

    outs = {}
    for name, greedy in (("obq_greedy", True), ("obq_natural", False)):
        codes = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
        W_hat = torch.empty(rows, cols, device=dev)
        _lib.obq_quantize(W, Hinv, 4, codes, W_hat, greedy=greedy, stream=stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize(dev)
        a.record(stream)
        for _ in range(iters):
            _lib.obq_quantize(W, Hinv, 4, codes, W_hat, greedy=greedy, stream=stream)
        b.record(stream)
        torch.cuda.synchronize(dev)
        outs[name] = (a.elapsed_time(b) / iters, W_hat)
    W_g = torch.empty(rows, cols, device=dev)
    codes = torch.empty(rows, cols, dtype=torch.uint8, device=dev)
    sc = torch.empty(rows, 1, device=dev)
    zz = torch.empty(rows, 1, dtype=torch.uint8, device=dev)
    wsq = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, 128), device=dev,
                      dtype=torch.uint8)
    _lib.quantize_layer(W, R, 4, -1, 128, W_g, codes, sc, zz, None, wsq, info, stream)
    torch.cuda.synchronize(dev)

    Wd = W.double()

    def proxy(Wh):
        dW = Wh.double() - Wd
        return float(((dW @ Hd) * dW).sum())

    def rel_err(Wh):
        dW = Wh.double() - Wd
        return float(((dW @ H) * dW).sum() / ((Wd @ H) * Wd).sum())

    fp64_ops = 2.0 * rows * cols ** 3
    dgemm_tflops = measure_fp64_peak(dev)
    peak = dgemm_tflops * 1e12 / 2.0
    out = {"layer": f"{rows}x{cols}, 4-bit per row, {tokens} bf16 tokens", "kernel": "obq_rows_kernel",
           "bound": "alu", "peak": peak,
           "peak_unit": "fp64 instructions/s (measured: cuBLAS fp64 GEMM 4096^3, best of 5, "
                        "flop rate / 2)",
           "dgemm_tflops": dgemm_tflops, "nominal_peak": 18.6e12}
    for name, (ms, Wh) in outs.items():
        out[name] = {"ms": ms, "weights_per_s": rows * cols / (ms / 1e3),
                     "fp64_ops_per_s": fp64_ops / (ms / 1e3),
                     "frac": fp64_ops / (ms / 1e3) / peak,
                     "proxy_loss": proxy(Wh), "rel_layer_error": rel_err(Wh)}
    out["gptq_column_loop"] = {"proxy_loss": proxy(W_g), "rel_layer_error": rel_err(W_g)}
    out["gptq_over_obq_proxy_loss"] = out["gptq_column_loop"]["proxy_loss"] / \
        out["obq_greedy"]["proxy_loss"]
    del X, S
    torch.cuda.empty_cache()
    return out


def measure_fp64_peak(dev, n=4096, reps=5):
    """Dense fp64 throughput on this GPU: torch.matmul of fp64 matrices (cuBLAS), n^3, best of
    `reps` with CUDA events; 2 n^3 flop per product. Returns TFLOP/s."""
    import torch
    g = torch.Generator(device=dev).manual_seed(6)
    a = torch.randn(n, n, device=dev, generator=g, dtype=torch.float64)
    b = torch.randn(n, n, device=dev, generator=g, dtype=torch.float64)
    c = torch.empty(n, n, device=dev, dtype=torch.float64)
    for _ in range(2):
        torch.matmul(a, b, out=c)
    best = float("inf")
    for _ in range(reps):
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        e0.record()
        torch.matmul(a, b, out=c)
        e1.record()
        torch.cuda.synchronize(dev)
        best = min(best, e0.elapsed_time(e1))
    del a, b, c
    torch.cuda.empty_cache()
    return 2.0 * n ** 3 / (best / 1e3) / 1e12


def measure_tf32_peak(dev, n=8192, reps=10):
    """Dense tf32 tensor throughput on this GPU: fp32 torch.matmul with tf32 allowed (cuBLAS),
    n^3, best of `reps` with CUDA events; 2 n^3 flop per product. The 3xTF32 products of S2-S5
    and S8 issue three tf32 products per fp32-accurate one, so their peak is a third of this."""
    import torch
    prev = torch.backends.cuda.matmul.allow_tf32
    torch.backends.cuda.matmul.allow_tf32 = True
    try:
        g = torch.Generator(device=dev).manual_seed(5)
        a = torch.randn(n, n, device=dev, generator=g)
        b = torch.randn(n, n, device=dev, generator=g)
        c = torch.empty(n, n, device=dev)
        for _ in range(3):
            torch.matmul(a, b, out=c)
        best = float("inf")
        for _ in range(reps):
            e0 = torch.cuda.Event(enable_timing=True)
            e1 = torch.cuda.Event(enable_timing=True)
            e0.record()
            torch.matmul(a, b, out=c)
            e1.record()
            torch.cuda.synchronize(dev)
            best = min(best, e0.elapsed_time(e1))
        del a, b, c
        torch.cuda.empty_cache()
        return 2.0 * n ** 3 / (best / 1e3) / 1e12
    finally:
        torch.backends.cuda.matmul.allow_tf32 = prev


def stage_ideals(rows, cols, n_tokens, block, bf16_peak_tf, tf32_peak_tf, hbm_gbs, hessian=True,
                 factor=True):
    """Roofline time (s) of each stage from its algorithmic work:
      S1: cols*(cols+1)*n_tokens flop (symmetric half) at the bf16 tensor peak;
      S2-S5: 2/3 cols^3 fp32 flop (one Cholesky and one triangular inverse, the default route),
             each as three tf32 products, at a third of the tf32 peak;
      S6-S8: 9 B per weight (fp32 read and write, one code byte) plus 8 B per trailing element
             per block (fp32 read and write of the lazy update) at the HBM copy peak."""
    out = {}
    if hessian:
        out["S1_hessian"] = cols * (cols + 1) * n_tokens / (bf16_peak_tf * 1e12)
    if factor:
        out["S2_S5_factor"] = 2.0 / 3.0 * cols ** 3 / (tf32_peak_tf * 1e12 / 3.0)
    b_trail = sum(8.0 * rows * (cols - min(cols, b0 + block)) for b0 in range(0, cols, block))
    out["S6_S8_quantize"] = (9.0 * rows * cols + b_trail) / (hbm_gbs * 1e9)
    return out


_ORACLE_FACTOR_CACHE = {}


def oracle_config_sample(spec, rows_sub=8, tok_sub=1024):
    """The fp64 oracle on a bounded sample of one layer config, extrapolated to the whole layer:
    S1 on `tok_sub` tokens at min(cols, 12288) channels (time ~ tokens x cols^2); S2-S5 in full at
    min(cols, 4096) (time ~ cols^3); S6-S8 on `rows_sub` rows at min(cols, 4096) columns (time ~
    rows x cols^2, the lazy flush's share). Returns (seconds per layer, description, the three
    extrapolated stage times)."""
    import numpy as np
    import oracle
    from post_weight_quantization_12_b200 import synth
    c1 = min(spec.cols, 12288)
    c2 = min(spec.cols, 4096)
    X = synth.inputs_np(synth.scaled_spec(spec, 1, c1, tok_sub), 31)
    t0 = time.perf_counter()
    S = np.zeros((c1, c1))
    oracle.hessian_accumulate(S, X)
    t1 = time.perf_counter() - t0
    f1 = (spec.n_tokens / tok_sub) * (spec.cols / c1) ** 2
    if c2 not in _ORACLE_FACTOR_CACHE:      # the factorization's time depends on c2 alone
        H = oracle.hessian_finalize(S[:c2, :c2], tok_sub)
        t0 = time.perf_counter()
        fac = oracle.inverse_hessian_factor(H, spec.damp)
        _ORACLE_FACTOR_CACHE[c2] = (fac, time.perf_counter() - t0)
    fac, t2 = _ORACLE_FACTOR_CACHE[c2]
    f2 = (spec.cols / c2) ** 3
    W = synth.weights_np(synth.scaled_spec(spec, rows_sub, c2, 1), 31)
    group = spec.group if spec.group <= 0 or c2 % spec.group == 0 else -1
    t0 = time.perf_counter()
    oracle.gptq_quantize(W, fac["R"], spec.bits, group, spec.block)
    t3 = time.perf_counter() - t0
    f3 = (spec.rows / rows_sub) * (spec.cols / c2) ** 2
    full = t1 * f1 + t2 * f2 + t3 * f3
    desc = (f"extrapolated: S1 on {tok_sub} tokens x {c1} channels ({t1:.2f} s, x{f1:.4g}); "
            f"S2-S5 at {c2} ({t2:.2f} s, x{f2:.4g}); S6-S8 on {rows_sub} rows x {c2} columns "
            f"({t3:.2f} s, x{f3:.4g}); {full:.1f} s per layer")
    return full, desc, (t1 * f1, t2 * f2, t3 * f3)


def bench_configs(names, dev, stream, peaks, tf32_peak, world, rank, steps=2, warmup=1,
                  cpu=True):
    """The other configured workloads, each timed like the headline step (inputs resident in HBM,
    CUDA events on the launching stream, `warmup` untimed steps, then `steps` timed ones), with the
    same stage rooflines and, on rank 0 at N = 1, its own oracle baseline on a bounded sample:
      mlp_up / mlp_down: the MLP pair at 3-bit per-row, 131072 tokens each;
      block: the 7B-class decoder block, 7 layers in execution order, 4 Hessians (q/k/v share one,
             gate/up share one), 262144 tokens each, 4-bit g128 -- weights/s over the 7 layers;
      fc1 / fc2: the 175B-class pair at 4-bit g128, 262144 tokens, plus S6-S8 at 3-bit per-row
             (the same R), reported beside it.
    Inputs larger than L2 in every case (X >= 1 GB)."""
    import dataclasses
    import torch
    from post_weight_quantization_12_b200 import _lib, synth

    bf16 = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    bf16_s = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    info = torch.zeros(1, device=dev, dtype=torch.int32)
    singles = {"mlp_up": synth.MLP_UP, "mlp_down": synth.MLP_DOWN, "fc1": synth.FC1,
               "fc2": synth.FC2}

    def ev():
        return torch.cuda.Event(enable_timing=True)

    def run_group(specs, X, seed):
        """S1 and S2-S5 once for the shared input X, then S6-S8 for each layer spec."""
        cols = specs[0].cols
        S = torch.empty(cols, cols, device=dev)
        R = torch.empty(cols, cols, device=dev)
        ws_p = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), device=dev,
                           dtype=torch.uint8)
        Ws, outs = [], []
        for i, sp in enumerate(specs):
            Ws.append(synth.weights_torch(sp, seed + 10 * i, dev))
            G = 1 if sp.group <= 0 else cols // sp.group
            outs.append(dict(W_hat=torch.empty(sp.rows, cols, device=dev),
                             codes=torch.empty(sp.rows, cols, device=dev, dtype=torch.uint8),
                             scales=torch.empty(sp.rows, G, device=dev),
                             zeros=torch.empty(sp.rows, G, device=dev, dtype=torch.uint8),
                             err_sq=torch.empty(sp.rows, device=dev),
                             ws=torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, sp.rows,
                                                                cols, sp.block),
                                            device=dev, dtype=torch.uint8)))

        def step(e=None):
            S.zero_()
            if e:
                e[0].record(stream)
            _lib.hessian_accumulate(S, X, info, stream)
            if e:
                e[1].record(stream)
            _lib.prepare_hinv(S, R, X.shape[0], specs[0].damp, ws_p, info, stream)
            if e:
                e[2].record(stream)
            for sp, W, o in zip(specs, Ws, outs):
                _lib.quantize_layer(W, R, sp.bits, sp.group, sp.block, o["W_hat"], o["codes"],
                                    o["scales"], o["zeros"], o["err_sq"], o["ws"], info, stream)
            if e:
                e[3].record(stream)

        return step, (S, R, ws_p, Ws, outs)

    def timed(step):
        for _ in range(warmup):
            step()
        torch.cuda.synchronize(dev)
        evs = [[ev() for _ in range(4)] for _ in range(steps)]
        for k in range(steps):
            step(evs[k])
        torch.cuda.synchronize(dev)
        if int(info.item()) != 0:
            raise RuntimeError(f"device status {int(info.item())} in the configs leg")
        st = [[e[i].elapsed_time(e[i + 1]) for e in evs] for i in range(3)]
        return [statistics.mean(x) for x in st]

    def fractions(ideal, got_ms):
        return {k: {"ideal_ms": ideal[k] * 1e3, "ms": got_ms[k], "frac": ideal[k] * 1e3 / got_ms[k]}
                for k in ideal}

    results = {}
    for name in names:
        torch.cuda.empty_cache()
        seed = 100
        if name in singles:
            spec = singles[name]
            X = synth.inputs_torch(spec, seed, dev)
            step, keep = run_group([spec], X, seed)
            s1, s25, s68 = timed(step)
            ms = s1 + s25 + s68
            got = {"S1_hessian": s1, "S2_S5_factor": s25, "S6_S8_quantize": s68}
            ideal = stage_ideals(spec.rows, spec.cols, spec.n_tokens, spec.block, bf16, tf32_peak,
                                 hbm)
            ideal_s = stage_ideals(spec.rows, spec.cols, spec.n_tokens, spec.block, bf16_s,
                                   tf32_peak, hbm)
            r = {"workload": f"W {spec.rows}x{spec.cols} bf16, X {spec.n_tokens} x {spec.cols} "
                             f"bf16 heavy-tailed ({spec.outlier_frac:g} of channels x"
                             f"{spec.outlier_mult:g}), {spec.bits}-bit "
                             f"{'per-row' if spec.group <= 0 else 'g%d' % spec.group}, block "
                             f"{spec.block}",
                 "ms_per_layer": ms, "weights_per_s": spec.rows * spec.cols / (ms / 1e3),
                 "stages_ms": got, "stage_roofline": fractions(ideal, got),
                 "layer_roofline": {"ideal_ms": sum(ideal.values()) * 1e3,
                                    "frac": sum(ideal.values()) * 1e3 / ms,
                                    "frac_vs_sustained_bf16": sum(ideal_s.values()) * 1e3 / ms}}
            if name in ("fc1", "fc2"):
                # the same layer at 3-bit per-row: S6-S8 only (S1-S5 do not depend on the grid)
                S, R, ws_p, Ws, outs = keep
                sp3 = dataclasses.replace(spec, bits=3, group=-1)
                o = outs[0]
                sc = torch.empty(spec.rows, 1, device=dev)
                zz = torch.empty(spec.rows, 1, device=dev, dtype=torch.uint8)

                def q3():
                    _lib.quantize_layer(Ws[0], R, 3, -1, spec.block, o["W_hat"], o["codes"], sc,
                                        zz, o["err_sq"], o["ws"], info, stream)
                q3()
                a, b = ev(), ev()
                a.record(stream)
                for _ in range(steps):
                    q3()
                b.record(stream)
                torch.cuda.synchronize(dev)
                t3 = a.elapsed_time(b) / steps
                i3 = stage_ideals(spec.rows, spec.cols, spec.n_tokens, spec.block, bf16, tf32_peak,
                                  hbm, hessian=False, factor=False)["S6_S8_quantize"]
                r["S6_S8_3bit_per_row"] = {"ms": t3, "ideal_ms": i3 * 1e3, "frac": i3 * 1e3 / t3}
                del sc, zz
            del keep, step, X
            if cpu and rank == 0 and world == 1:
                full, desc, _ = oracle_config_sample(spec)
                r["cpu_baseline"] = {"value": spec.rows * spec.cols / full, "unit": UNIT,
                                     "cores": cpu_threads(), "kind": "oracle", "sample": desc}
            results[name] = r
        elif name == "block":
            layers = synth.block_layers(seed)
            groups = []
            for spec, hid in layers:
                if not groups or groups[-1][0] != hid:
                    groups.append((hid, []))
                groups[-1][1].append(spec)
            tot = {"S1_hessian": 0.0, "S2_S5_factor": 0.0, "S6_S8_quantize": 0.0}
            ideal = {"S1_hessian": 0.0, "S2_S5_factor": 0.0, "S6_S8_quantize": 0.0}
            weights = 0
            cpu_s, cpu_desc = 0.0, []
            for gi, (hid, specs) in enumerate(groups):
                torch.cuda.empty_cache()
                X = synth.inputs_torch(specs[0], seed + 10 * gi, dev)
                step, keep = run_group(specs, X, seed + 10 * gi)
                s1, s25, s68 = timed(step)
                tot["S1_hessian"] += s1
                tot["S2_S5_factor"] += s25
                tot["S6_S8_quantize"] += s68
                for i, sp in enumerate(specs):
                    d = stage_ideals(sp.rows, sp.cols, sp.n_tokens, sp.block, bf16, tf32_peak, hbm,
                                     hessian=(i == 0), factor=(i == 0))
                    for k, v in d.items():
                        ideal[k] += v
                    weights += sp.rows * sp.cols
                    if cpu and rank == 0 and world == 1:
                        # the shared S1-S5 once per group, S6-S8 once per layer
                        if i == 0:
                            full, desc, parts = oracle_config_sample(sp)
                            cpu_s += full
                            cpu_desc.append(f"{hid} ({len(specs)} layer(s)): {desc}")
                        else:
                            cpu_s += parts[2]
                del keep, step, X
            ms = sum(tot.values())
            results[name] = {
                "workload": "7B-class decoder block: q,k,v,o 4096x4096 (q,k,v share one H), "
                            "gate,up 11008x4096 (share one H), down 4096x11008; 4 inputs of "
                            "128 seqs x 2048 tokens bf16 heavy-tailed; 4-bit g128, block 128, "
                            "run in execution order",
                "ms_per_block": ms, "weights_per_s": weights / (ms / 1e3), "weights": weights,
                "stages_ms": tot, "stage_roofline": fractions(ideal, tot),
                "layer_roofline": {"ideal_ms": sum(ideal.values()) * 1e3,
                                   "frac": sum(ideal.values()) * 1e3 / ms}}
            if cpu and rank == 0 and world == 1:
                results[name]["cpu_baseline"] = {
                    "value": weights / cpu_s, "unit": UNIT, "cores": cpu_threads(),
                    "kind": "oracle",
                    "sample": "; ".join(cpu_desc) + "; layers that share an H add their own "
                              "S6-S8 only"}
        else:
            raise ValueError(f"unknown config {name}")
    torch.cuda.empty_cache()
    return {"peaks": {"bf16_tflops_burst": bf16, "bf16_tflops_sustained": bf16_s,
                      "tf32_tflops_measured": tf32_peak, "hbm_gbs": hbm},
            "timing": f"{warmup} untimed + {steps} timed steps per config, CUDA events", **results}


def run_ours(args):
    import torch
    import torch.distributed as dist
    from post_weight_quantization_12_b200 import _lib, api, synth

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=dev)
    peaks, peaks_src = load_peaks()
    spec = workload(args.tokens)
    seed = rank_seed(args.seed, rank)
    rows, cols, n = spec.rows, spec.cols, spec.n_tokens

    X = synth.inputs_torch(spec, seed, dev)
    W = synth.weights_torch(spec, seed, dev)
    S = torch.empty(cols, cols, device=dev)
    R = torch.empty(cols, cols, device=dev)
    G = 1 if spec.group <= 0 else cols // spec.group
    W_hat = torch.empty(rows, cols, device=dev)
    codes = torch.empty(rows, cols, device=dev, dtype=torch.uint8)
    scales = torch.empty(rows, G, device=dev)
    zeros = torch.empty(rows, G, device=dev, dtype=torch.uint8)
    err_sq = torch.empty(rows, device=dev)
    ws_p = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_PREPARE, 0, cols, 0), device=dev,
                       dtype=torch.uint8)
    ws_q = torch.empty(_lib.workspace_size(_lib.GPTQ_WS_QUANTIZE, rows, cols, spec.block),
                       device=dev, dtype=torch.uint8)
    info = torch.zeros(1, device=dev, dtype=torch.int32)
    stream = torch.cuda.current_stream(dev)

    def step(ev=None):
        S.zero_()
        if ev is not None:
            ev[0].record(stream)
        _lib.hessian_accumulate(S, X, info, stream)
        if ev is not None:
            ev[1].record(stream)
        _lib.prepare_hinv(S, R, n, spec.damp, ws_p, info, stream)
        if ev is not None:
            ev[2].record(stream)
        _lib.quantize_layer(W, R, spec.bits, spec.group, spec.block, W_hat, codes, scales, zeros,
                            err_sq, ws_q, info, stream)
        if ev is not None:
            ev[3].record(stream)

    try:
        tf32_peak, tf32_src = measure_tf32_peak(dev), "measured: cuBLAS fp32 8192^3 with tf32, best of 10"
    except Exception as exc:  # the probe is context for the fractions, not part of the path
        tf32_peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"])) * TF32_PER_BF16
        tf32_src = f"bf16 x nominal ratio (probe failed: {exc})"

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize(dev)
    if int(info.item()) != 0:
        raise RuntimeError(f"device status {int(info.item())} after warm-up")

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    clocks = ClockSampler(local) if rank == 0 else None
    if clocks:
        clocks.start()
        time.sleep(0.3)
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize(dev)
    launches0 = _lib.kernel_launches()
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    torch.cuda.synchronize(dev)
    launches = _lib.kernel_launches() - launches0
    if world > 1:
        dist.barrier()
    clock_rec = clocks.stop() if clocks else None
    elapsed_ms = t_start.elapsed_time(t_end)
    s1 = [e[0].elapsed_time(e[1]) for e in evs]
    s25 = [e[1].elapsed_time(e[2]) for e in evs]
    s68 = [e[2].elapsed_time(e[3]) for e in evs]
    if int(info.item()) != 0:
        raise RuntimeError(f"device status {int(info.item())} in the timed region")

    elapsed_ms, launches = aggregate(elapsed_ms, launches, world, dev)

    ms_per_step = elapsed_ms / args.steps
    value = world * rows * cols * args.steps / (elapsed_ms / 1e3)

    # roofline of the dominant kernel: the SYRK (S1 is exactly one kernel launch). The step is
    # short and the GPU holds its maximum clock through it (the sampled clocks are in the line),
    # so the peak is the burst bf16 figure; the sustained figure was measured at a lower clock.
    t_syrk = statistics.mean(s1) / 1e3
    flops = cols * (cols + 1) * n            # symmetric half of X^T X, 2 flops per multiply-add
    achieved = flops / t_syrk / 1e12
    peak = float(peaks.get("bf16_tflops", FALLBACK_PEAKS["bf16_tflops"]))
    peak_s = float(peaks.get("bf16_tflops_sustained", FALLBACK_PEAKS["bf16_tflops_sustained"]))
    clock_note = (f"SM clock during the timed region: median {clock_rec['sm_mhz']:.0f} of "
                  f"{clock_rec['sm_max_mhz']:.0f} MHz" if clock_rec else "SM clock not sampled")
    traffic = None
    if SYRK_CAPTURE and cols == SYRK_CAPTURE["cols"]:
        traffic = SYRK_CAPTURE["dram_read"] * n / SYRK_CAPTURE["tokens"] + SYRK_CAPTURE["dram_write"]
    roofline = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": traffic,
                "kernel": "hessian_syrk_bf16_tc",
                "peak_source": f"{peaks_src} bf16 burst (cuBLAS 8192^3, best of 10); "
                               f"{clock_note}",
                "frac_vs_sustained": achieved / peak_s,
                "work": f"{flops:.4g} flop per launch = cols*(cols+1)*n_tokens",
                "traffic_source": "ncu dram bytes at 16384 tokens, reads scaled by tokens"}

    # Per-stage and whole-layer rooflines from the algorithmic work of each stage (stage_ideals):
    # S1 at the bf16 burst peak, S2-S5 at a third of the tf32 peak measured above, S6-S8 at HBM.
    hbm = float(peaks.get("hbm_gbs", FALLBACK_PEAKS["hbm_gbs"]))
    ideal = stage_ideals(rows, cols, n, spec.block, peak, tf32_peak, hbm)
    got = {"S1_hessian": statistics.mean(s1) / 1e3, "S2_S5_factor": statistics.mean(s25) / 1e3,
           "S6_S8_quantize": statistics.mean(s68) / 1e3}
    stage_roofline = {k: {"ideal_ms": ideal[k] * 1e3, "ms": got[k] * 1e3,
                          "frac": ideal[k] / got[k]} for k in ideal}
    fl_25 = 2.0 / 3.0 * cols ** 3
    b_68 = ideal["S6_S8_quantize"] * hbm * 1e9
    stage_roofline["S2_S5_factor"]["achieved_tflops_fp32_equiv"] = fl_25 / got["S2_S5_factor"] / 1e12
    stage_roofline["S6_S8_quantize"]["achieved_gbs"] = b_68 / got["S6_S8_quantize"] / 1e9
    layer_roofline = {"ideal_ms": sum(ideal.values()) * 1e3, "ms": ms_per_step,
                      "frac": sum(ideal.values()) * 1e3 / ms_per_step,
                      "basis": f"{peaks_src} peaks: bf16 burst {peak} TFLOP/s; tf32 "
                               f"{tf32_peak:.1f} TFLOP/s ({tf32_src}), 3xTF32 at a third of it; "
                               f"HBM {hbm:.0f} GB/s"}

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16/f32",
        "data": "synthetic (seeded device draws; no model weights or calibration text)",
        "config": config_dict(spec),
        "stages_ms": {"S1_hessian": statistics.mean(s1), "S2_S5_factor": statistics.mean(s25),
                      "S6_S8_quantize": statistics.mean(s68)},
        "roofline": roofline, "stage_roofline": stage_roofline, "layer_roofline": layer_roofline,
        "tf32_tflops": {"value": tf32_peak, "source": tf32_src},
        "gpu_launches": launches, "clocks": clock_rec,
    }
    if args.tokens:
        line["note"] = "token count overridden for profiling: not the configured workload"

    # S2-S5 by the pages' three-step route (two Cholesky factorizations, triangular inverse and
    # product: 4/3 cols^3 flop), timed the same way outside the headline step, for comparison
    t3 = []
    for _ in range(3):
        S.zero_()
        _lib.hessian_accumulate(S, X, info, stream)
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        _lib.prepare_hinv(S, R, n, spec.damp, ws_p, info, stream, route=_lib.GPTQ_ROUTE_THREE_STEP)
        b.record(stream)
        torch.cuda.synchronize(dev)
        t3.append(a.elapsed_time(b))
    if int(info.item()) != 0:
        raise RuntimeError(f"device status {int(info.item())} on the three-step route")
    line["S2_S5_routes_ms"] = {"reversed (default; the step above)": statistics.mean(s25),
                               "three_step": statistics.median(t3)}

    names = [] if world > 1 or args.configs == "none" else \
        (list(CONFIGS) if args.configs == "all" else [c for c in args.configs.split(",") if c])
    if names:
        del X
        torch.cuda.empty_cache()
        line["configs"] = bench_configs(names, dev, stream, peaks, tf32_peak, world, rank,
                                        cpu=not args.no_cpu_baseline)
        X = synth.inputs_torch(spec, seed, dev)

    if not args.no_w4a16:
        line["w4a16"] = bench_w4a16(dev, stream, peaks, peaks_src)
    if not args.no_rotation:
        line["rotation"] = bench_rotation(dev, stream, peaks, peaks_src, spec, X)
    if not args.no_obq:
        line["obq"] = bench_obq(dev, stream)

    # end to end through the public API from pinned host buffers
    if not args.no_e2e:
        Xh = X.cpu().pin_memory()
        Wh = W.cpu().pin_memory()
        q = api.LayerQuantizer(cols, device=dev, damp_rel=spec.damp)

        def e2e_step():
            q.reset()
            q.add_batch(Xh)
            q.prepare()
            return q.quantize(Wh, spec.bits, spec.group, spec.block, to_host=True)

        for _ in range(min(2, args.warmup)):
            e2e_step()
        torch.cuda.synchronize(dev)
        k_e2e = max(1, min(3, args.steps))
        if world > 1:
            dist.barrier()
        a = torch.cuda.Event(enable_timing=True)
        b = torch.cuda.Event(enable_timing=True)
        a.record(stream)
        for _ in range(k_e2e):
            out = e2e_step()
        b.record(stream)
        torch.cuda.synchronize(dev)
        e_ms, _ = aggregate(a.elapsed_time(b), 0, world, dev)
        h2d = Xh.numel() * Xh.element_size() + Wh.numel() * Wh.element_size()
        # the host receives codes, scales, zeros and err_sq (W_hat = s (q - z) stays on the device)
        d2h = sum(t.numel() * t.element_size() for t in (out.codes, out.scales, out.zeros,
                                                         out.err_sq))
        line["e2e"] = {"value": world * rows * cols * k_e2e / (e_ms / 1e3), "unit": UNIT,
                       "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                       "steps": k_e2e, "ms_per_step": e_ms / k_e2e}
        del Xh, Wh

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        n_tok, r_sub = sample_sizes(spec, args.cpu_sample_s)
        Xs = X[:n_tok].float().cpu().numpy()
        Ws = W[:r_sub].float().cpu().numpy()
        full, desc, spent = oracle_sample(Ws, Xs, spec, args.cpu_sample_s)
        line["cpu_baseline"] = {"value": rows * cols / full, "unit": UNIT,
                                "cores": cpu_threads(), "kind": "oracle", "sample": desc,
                                "sample_wall_s": spent}

    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        for key, val in oracle_extras().items():
            if key in line:
                line[key]["cpu_baseline"] = val

    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    return 0


def main():
    args = parse()
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
