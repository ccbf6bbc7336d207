#!/usr/bin/env python
"""Benchmark of the p4 Flash EQ-Linear hot path on B200 (one JSON line).

A step is one pass of the whole path on one batch: weight transform
(feql_weight_fft), forward (feql_forward), input gradient (feql_backward_dx)
and weight gradient (feql_backward_dw), all through the C ABI, fp16 data with
fp32 accumulation, on the Swin stage-1-like forward+backward workload
N = 128 x 3136 tokens, C = 24, D = 96 (96 -> 384 unrolled).  Inputs are
resident in HBM; each pass reads/writes ~385 MB, more than the 126 MB L2, so
no flush is needed between steps.  The same line carries "per_config": every
layer configuration (1: fp32 256x16x16, 2: ViT fc1 12608x48x192, 3: square
65536x192x192 in fp16 and fp32, 4: backward 32768x256x256, 5: the Swin stream)
and the widened workloads (C_8, p4m, C_6, the two MLP blocks) at full size,
each pass timed over 50 reps with the L2 flushed before each, median and min,
with its roofline fractions.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

--workload selects another shape (workloads.py); workload 6 is the same stream
for the cyclic group C_8 (feql_ct_* entry points, dX and dW as two passes), and
workload 7 the Swin stage-1 MLP block (fc1 -> GELU -> fc2, one fused kernel,
feql_mlp_forward; its "unfused" line times the same block as fc1 forward, a
torch GELU and fc2 forward, for context); workload 8 is the Swin stream for
p4m (rotations and reflections, feql_p4m_* entry points).

Multi-GPU (torchrun, one rank per GPU): every rank runs the full workload on
its own tokens (weak scaling); the data-parallel weight gradient is summed
with one NCCL all-reduce per step.  --impl reference times the float64 CPU
oracle (the unrolled dense method) on the host cores, on a bounded sample.
"""

from __future__ import annotations

import argparse
import csv
import io
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "p4 EQ-Linear fwd/bwd tokens/s, effective TFLOP/s and % of roofline (fp16)"
WORKLOAD_ID = 5


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", type=int, default=WORKLOAD_ID,
                    help="workload id 1-10 (group_dft_structured_b200/workloads.py; 6 is the "
                         "cyclic group C_8, 7 and 9 MLP blocks, 8 p4m, 10 C_6)")
    ap.add_argument("--dtype", choices=["fp16", "fp32"], default=None,
                    help="override the workload's dtype (e.g. the fp32 run of the square layer)")
    ap.add_argument("--e2e-steps", type=int, default=5)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--separate-backward", action="store_true",
                    help="run dX and dW as two passes instead of the fused backward")
    ap.add_argument("--no-per-config", action="store_true",
                    help="skip the per-configuration table (configurations 1-5, L2 flushed)")
    ap.add_argument("--config-reps", type=int, default=50,
                    help="timed reps per pass in the per-configuration table")
    ap.add_argument("--tokens", type=int, default=None,
                    help="override the workload's token count (smaller cases for profiling)")
    return ap.parse_args()


def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed_id(wid: int, rank: int) -> int:
    """Seed block of a rank's own tokens (weak scaling: every rank has a full batch)."""
    return wid + 1000 * rank


def dp_allreduce_grads(dW, db):
    """Data-parallel weight gradient: every rank holds dW/db of its own tokens;
    the layer's gradient is their sum (the path's one exchange step)."""
    import torch.distributed as dist
    dist.all_reduce(dW)
    if db is not None:
        dist.all_reduce(db)


def max_over_ranks(value: float, device) -> float:
    """The slowest rank's time (all ranks take part)."""
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def workload_bytes(w, elt):
    """Algorithmic HBM bytes per launch of each pass (inputs read once, outputs
    written once; Fourier weights counted as their T*D*C real values)."""
    N, C, D, T = w.N, w.C, w.D, w.T
    x, y, what, b = T * N * C * elt, T * N * D * elt, T * D * C * elt, D * elt
    return {
        "wfft": T * D * C * elt + what,
        "fwd": x + what + b + y,
        "dx": y + what + x,
        "dw": x + y + T * D * C * elt + b,
        "bwd": x + y + what + x + T * D * C * elt + b,  # x, dy, What in; dx, dW, db out
    }


def mlp_bytes(w, elt):
    """Algorithmic HBM bytes of the fused MLP block: x in, y out, both layers'
    weights (as real values) and biases; the hidden activation stays on chip."""
    N, C, H = w.N, w.C, w.D
    wts = 4 * H * C * elt * 2 + (H + C) * elt
    return {"wfft": 2 * wts, "mlp": 4 * N * C * elt * 2 + wts}


def layer_macs(w):
    """Real MACs of one contraction pass with the Fourier method: (2T-2) NCD for
    the cyclic group of even order T (bins 0 and T/2 real, the others complex),
    12 NCD for p4m (four 1-dim irreps and one 2 x 2 block); and of the unrolled
    dense method: T^2 NCD."""
    fourier = 12 if w.group == "p4m" else 2 * w.T - 2
    return fourier * w.N * w.C * w.D, w.T * w.T * w.N * w.C * w.D


def strip_comments(src: str) -> str:
    """C/CUDA source without // and /* */ comments, trailing blanks and empty lines
    (the sources contain no string literal with a comment marker)."""
    import re
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(line.rstrip() for line in src.splitlines() if line.strip())


def kernel_source_hash():
    """Hash of the CUDA sources' code (comments excluded); DRAM counters in
    profiles/traffic.json are only reported while it matches the hash they were
    taken with."""
    import hashlib
    d = os.path.join(ROOT, "group_dft_structured_b200", "csrc")
    h = hashlib.sha256()
    for f in sorted(os.listdir(d)):
        if f.endswith((".cu", ".cuh")):
            h.update(f.encode())
            with open(os.path.join(d, f), encoding="utf-8") as fh:
                h.update(strip_comments(fh.read()).encode())
    return h.hexdigest()[:16]


def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return 6650.0, "fallback"


# ----------------------------------------------------------------- clocks
class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "50"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        out, _ = self.proc.communicate(timeout=10)
        rows = [r for r in csv.reader(io.StringIO(out)) if len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        mx = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        reasons = set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for r in rows:
            for name, v in zip(names, r[5:9]):
                if v.strip().lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(sm) if sm else None,
                "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(rows)}


# --------------------------------------------------------------- baseline
def oracle_cores():
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return os.cpu_count()


def time_oracle(w, n_sample):
    """Float64 oracle (unrolled dense method) for all passes on n_sample tokens."""
    import numpy as np

    from group_dft_structured_b200.workloads import make_inputs, make_mlp_inputs
    if "mlp" in w.passes:
        from oracle import feql_mlp_oracle as M
        inp = make_mlp_inputs(w.wid, n_sample, w.C, w.D, w.C, w.dtype)
        f = {k: v.astype(np.float64) for k, v in inp.items()}
        t0 = time.perf_counter()
        M.forward(f["x"], f["W1"], f["b1"], f["W2"], f["b2"])
        return time.perf_counter() - t0
    if w.group == "p4m":
        from oracle import feql_p4m_oracle as O
    elif w.T == 4:
        from oracle import feql_oracle as O
    else:
        from oracle import feql_ct_oracle as O
    inp = make_inputs(w.wid, n_sample, w.C, w.D, w.dtype, T=w.T)
    f = {k: v.astype(np.float64) for k, v in inp.items()}
    t0 = time.perf_counter()
    if "fwd" in w.passes:
        O.forward(f["x"], f["W"], f["b"])
    if "dx" in w.passes:
        O.backward_dx(f["dy"], f["W"])
    if "dw" in w.passes:
        O.backward_dw(f["x"], f["dy"])
    return time.perf_counter() - t0


def cpu_baseline(w, target_s=3.0):
    n = min(w.N, 8192)
    t = min(time_oracle(w, n), time_oracle(w, n))
    while t < target_s and n < w.N:
        n = min(w.N, n * 2)
        t = time_oracle(w, n)
    return {"value": n / t, "unit": "tokens/s", "cores": oracle_cores(), "kind": "oracle",
            "sample": f"{n} of {w.N} tokens, passes {'+'.join(w.passes)}, float64 numpy "
                      f"(unrolled circulant{', exact GELU' if 'mlp' in w.passes else ''}), "
                      f"one timed run of {t:.2f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    from group_dft_structured_b200.workloads import WORKLOADS
    w = WORKLOADS[args.workload]
    # size one step so that the whole run stays within about two minutes
    target = min(1.5, 120.0 / max(1, args.steps + args.warmup))
    n = min(w.N, 1024)
    t = min(time_oracle(w, n), time_oracle(w, n))
    while t < target and n < w.N:
        n = min(w.N, n * 2)
        t = time_oracle(w, n)
    for _ in range(args.warmup):
        time_oracle(w, n)
    times = [time_oracle(w, n) for _ in range(args.steps)]
    total = sum(times)
    value = n * args.steps / total
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * total / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "N": w.N, "C": w.C, "D": w.D,
                   "passes": list(w.passes), "sample_tokens_per_step": n},
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": oracle_cores(),
                         "kind": "oracle",
                         "sample": f"{n} of {w.N} tokens per step, float64 numpy"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------------- ours
def setup_layer(args, w, rank, s, F, torch):
    """Buffers and calls of the EQ-Linear layer workloads (p4, C_8, p4m)."""
    from group_dft_structured_b200.workloads import make_inputs
    mode = F.FEQL_FP16 if w.dtype == "fp16" else F.FEQL_FP32
    N, C, D, T = w.N, w.C, w.D, w.T
    elt = 2 if w.dtype == "fp16" else 4
    inp = make_inputs(rank_seed_id(w.wid, rank), N, C, D, w.dtype, T=T)
    p4m = w.group == "p4m"
    wbytes = (F.feql_p4m_weight_fft_bytes(C, D, mode) if p4m
              else F.feql_ct_weight_fft_bytes(T, C, D, mode))
    wsb = (F.feql_p4m_backward_dw_workspace_bytes(N, C, D, mode) if p4m
           else F.feql_ct_backward_dw_workspace_bytes(T, N, C, D, mode))

    def buffers(first=None):
        """One set of device buffers: inputs (copied from the host arrays for the
        first set, left uninitialised for the e2e run's second set), outputs,
        the Fourier weights and the dW workspace."""
        if first is None:
            B = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
        else:
            B = {k: torch.empty_like(first[k]) for k in inp}
        dt = B["x"].dtype
        B["What"] = torch.empty(wbytes, dtype=torch.uint8, device="cuda")
        B["y"] = torch.empty((N, D, T), dtype=dt, device="cuda")
        B["dx"] = torch.empty((N, C, T), dtype=dt, device="cuda")
        B["dW"] = torch.empty((D, C, T), dtype=dt, device="cuda")
        B["db"] = torch.empty((D,), dtype=dt, device="cuda")
        B["ws"] = torch.empty(max(wsb, 16), dtype=torch.uint8, device="cuda")
        return B

    def calls_for(B, st):
        """The passes of one step on buffer set B, enqueued on stream handle st.
        One step = every row of the path: weight rDFT, forward, and the backward
        (dX and dW/db, fused into one pass over dy for p4 unless
        --separate-backward)."""
        x, W, b, dy, What, ws = B["x"], B["W"], B["b"], B["dy"], B["What"], B["ws"]
        y, dx, dW, db = B["y"], B["dx"], B["dW"], B["db"]
        if p4m:
            return {
                "wfft": lambda: F.feql_p4m_weight_fft(W, What, C, D, mode, st),
                "fwd": lambda: F.feql_p4m_forward(x, What, b, y, N, C, D, mode, st),
                "dx": lambda: F.feql_p4m_backward_dx(dy, What, dx, N, C, D, mode, st),
                "dw": lambda: F.feql_p4m_backward_dw(x, dy, dW, db, ws, ws.numel(), N, C, D,
                                                     mode, st),
            }
        return {
            "wfft": lambda: F.feql_ct_weight_fft(T, W, What, C, D, mode, st),
            "fwd": lambda: F.feql_ct_forward(T, x, What, b, y, N, C, D, mode, st),
            "dx": lambda: F.feql_ct_backward_dx(T, dy, What, dx, N, C, D, mode, st),
            "dw": lambda: F.feql_ct_backward_dw(T, x, dy, dW, db, ws, ws.numel(), N, C, D, mode,
                                                st),
            "bwd": lambda: F.feql_backward(x, dy, What, dx, dW, db, ws, ws.numel(), N, C, D,
                                           mode, st),
        }

    B0 = buffers()
    passes = ["wfft"] + (["fwd"] if "fwd" in w.passes else [])
    if "dx" in w.passes and "dw" in w.passes and not args.separate_backward and T == 4 and not p4m:
        passes.append("bwd")
    else:
        passes += [p for p in ("dx", "dw") if p in w.passes]
    macs, dense_macs = layer_macs(w)
    gemms = {"wfft": 0, "fwd": 1, "dx": 1, "dw": 1, "bwd": 2}  # layer contractions per pass
    has_bwd = any(p in passes for p in ("dx", "dw", "bwd"))
    ins = ["x", "W", "b"] + (["dy"] if has_bwd else [])
    outs = [k for k in ("y", "dx", "dW", "db")
            if (k == "y" and "fwd" in passes)
            or (k == "dx" and ("dx" in passes or "bwd" in passes))
            or (k in ("dW", "db") and ("dw" in passes or "bwd" in passes))]
    return {
        "calls": calls_for(B0, s), "calls_for": calls_for, "buffers": buffers, "B0": B0,
        "passes": passes, "tokens": N, "elt": elt,
        "launches": {"wfft": 1, "fwd": 1, "dx": 1, "dw": 2, "bwd": 2},
        "bytes": workload_bytes(w, elt),
        "flops": {p: (2 * macs * gemms[p], 2 * dense_macs * gemms[p]) for p in passes},
        "host": {k: inp[k] for k in ins}, "ins": ins, "outs": outs,
        "allreduce": (lambda B: dp_allreduce_grads(B["dW"], B["db"])) if has_bwd else None,
        "config": {"N": N, "C": C, "D": D, "T": T, "group": "p4m (D4)" if p4m else f"C_{T}"},
        "extra": {},
    }


def setup_mlp(args, w, rank, s, F, torch):
    """Buffers and calls of the fused MLP block (fc1 C -> H, GELU, fc2 H -> C)."""
    import torch.nn.functional as TF

    from group_dft_structured_b200.workloads import make_mlp_inputs
    mode = F.FEQL_FP16
    N, C, H, Co = w.N, w.C, w.D, w.C
    inp = make_mlp_inputs(rank_seed_id(w.wid, rank), N, C, H, Co, w.dtype)
    wbytes = F.feql_mlp_weight_fft_bytes(C, H, Co, mode)

    def buffers(first=None):
        if first is None:
            B = {k: torch.from_numpy(v).cuda() for k, v in inp.items()}
        else:
            B = {k: torch.empty_like(first[k]) for k in inp}
        B["What"] = torch.empty(wbytes, dtype=torch.uint8, device="cuda")
        B["y"] = torch.empty((N, Co, 4), dtype=B["x"].dtype, device="cuda")
        return B

    def calls_for(B, st):
        return {
            "wfft": lambda: F.feql_mlp_weight_fft(B["W1"], B["W2"], B["What"], C, H, Co, mode,
                                                  st),
            "mlp": lambda: F.feql_mlp_forward(B["x"], B["What"], B["b1"], B["b2"], B["y"], N, C,
                                              H, Co, mode, st),
        }

    B0 = buffers()
    x, W1, b1, W2, b2, y = (B0[k] for k in ("x", "W1", "b1", "W2", "b2", "y"))
    macs = 6 * N * H * (C + Co)
    # context: the same block as three launches with the hidden activation in HBM
    W1hat = torch.empty(F.feql_weight_fft_bytes(C, H, mode), dtype=torch.uint8, device="cuda")
    W2hat = torch.empty(F.feql_weight_fft_bytes(H, Co, mode), dtype=torch.uint8, device="cuda")
    F.feql_weight_fft(W1, W1hat, C, H, mode, s)
    F.feql_weight_fft(W2, W2hat, H, Co, mode, s)
    h = torch.empty((N, H, 4), dtype=x.dtype, device="cuda")
    y2 = torch.empty_like(y)
    stream = torch.cuda.current_stream()

    def unfused():
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        for _ in range(3):
            F.feql_forward(x, W1hat, b1, h, N, C, H, mode, s)
            g = TF.gelu(h)
            F.feql_forward(g, W2hat, b2, y2, N, H, Co, mode, s)
        a.record(stream)
        reps = 20
        for _ in range(reps):
            F.feql_forward(x, W1hat, b1, h, N, C, H, mode, s)
            g = TF.gelu(h)
            F.feql_forward(g, W2hat, b2, y2, N, H, Co, mode, s)
        z.record(stream)
        torch.cuda.synchronize()
        return a.elapsed_time(z) / reps

    ins = ["x", "W1", "b1", "W2", "b2"]
    return {
        "calls": calls_for(B0, s), "calls_for": calls_for, "buffers": buffers, "B0": B0,
        "passes": ["wfft", "mlp"], "tokens": N, "elt": 2,
        "launches": {"wfft": 1, "mlp": 1},
        "bytes": mlp_bytes(w, 2),
        "flops": {"wfft": (0, 0), "mlp": (2 * macs, 2 * 16 * N * H * (C + Co))},
        "host": {k: inp[k] for k in ins}, "ins": ins, "outs": ["y"],
        "allreduce": None,
        "config": {"N": N, "C": C, "H": H, "Co": Co, "T": 4, "gelu": "tanh form, fp16"},
        "extra": {"unfused": unfused},
    }


# ------------------------------------------------------------- per config
# Peaks for the per-config rooflines.  Nominal B200 figures (dense): HBM3e
# 8.0 TB/s, fp16 tensor 2.25 PFLOP/s, fp32 FMA on CUDA cores 148 SMs x 128 lanes
# x 2 FLOP x 1.965 GHz = 74.4 TFLOP/s.  The measured HBM and tensor figures come
# from MEASURED_PEAKS.json (copy bandwidth; cuBLAS bf16, the same tensor rate as
# fp16); the CUDA-core fp32 peak has no measurement and uses the nominal count.
NOMINAL = {"hbm_gbs": 8000.0, "tensor_tflops": 2250.0, "fp32_fma_tflops": 74.4,
           "tf32_tflops": 1125.0}

# The five layer configurations, each with the passes its throughput is quoted
# on (forward for 1-3, dX and dW for 4, forward and both gradients for 5; 3
# also in fp32).
# fp32 runs in both fp32 modes: CUDA cores ("fp32") and split TF32 on the tensor
# cores ("fp32_3xtf32", three tf32 products per product).
CONFIG_RUNS = [(1, "fp32", ("fwd",)), (1, "fp32_3xtf32", ("fwd",)), (2, "fp16", ("fwd",)),
               (3, "fp16", ("fwd",)), (3, "fp32", ("fwd",)), (3, "fp32_3xtf32", ("fwd",)),
               (4, "fp16", ("dx", "dw")), (5, "fp16", ("fwd", "dx", "dw", "bwd"))]


def peak_table():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    meas = None
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        meas = {"hbm_gbs": float(d["hbm_gbs"]), "tensor_tflops": float(d["bf16_tflops"]),
                "fp32_fma_tflops": NOMINAL["fp32_fma_tflops"],
                # tf32 runs at half the bf16 rate per FLOP (the nominal 1.125 vs 2.25 PF)
                "tf32_tflops": float(d["bf16_tflops"]) / 2}
    return meas, NOMINAL


def roofline_us(nbytes, flops, dtype, peaks):
    """Roofline time (us) and its bound: the slower of the algorithmic bytes at
    HBM bandwidth and the algorithmic FLOPs at the mode's arithmetic peak (split
    TF32 issues three tf32 products per product)."""
    t_mem = nbytes / (peaks["hbm_gbs"] * 1e9) * 1e6
    if dtype == "fp16":
        t_cmp, bound = flops / (peaks["tensor_tflops"] * 1e12) * 1e6, "tensor"
    elif dtype == "fp32_3xtf32":
        t_cmp, bound = 3 * flops / (peaks["tf32_tflops"] * 1e12) * 1e6, "tensor"
    else:
        t_cmp, bound = flops / (peaks["fp32_fma_tflops"] * 1e12) * 1e6, "alu"
    return (t_mem, "hbm") if t_mem >= t_cmp else (t_cmp, bound)


def hold_gpu(torch, ms=20.0):
    """Keeps the current stream busy for about `ms` milliseconds (a spin kernel),
    so that the host enqueues the launches that follow before the GPU reaches
    them: the CUDA-event times then hold no host-side launch gaps."""
    torch.cuda._sleep(int(ms * 1e-3 * 1.965e9))


def per_config_report(F, torch, stream, reps):
    """Every layer configuration at full size: median and min over `reps` CUDA-event
    timings of each pass, the L2 flushed before every rep by reading a buffer of
    twice its size (that leaves the L2 holding clean lines of the flush buffer,
    so neither the pass's inputs nor dirty lines of earlier writes remain)."""
    import numpy as np

    from group_dft_structured_b200 import layer as Lyr
    from group_dft_structured_b200.workloads import WORKLOADS, workload_inputs
    meas, nom = peak_table()
    s = stream.cuda_stream
    traffic = {}
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tj = json.load(f)
        if tj.get("source_hash") == kernel_source_hash():
            traffic = tj
    l2 = torch.cuda.get_device_properties(torch.cuda.current_device()).L2_cache_size
    flush = torch.ones(2 * l2 // 4, dtype=torch.float32, device="cuda")
    out = {}
    for wid, dtype, passes in CONFIG_RUNS:
        w = WORKLOADS[wid]
        N, C, D = w.N, w.C, w.D
        mode = {"fp16": F.FEQL_FP16, "fp32": F.FEQL_FP32_SIMT,
                "fp32_3xtf32": F.FEQL_FP32_3XTF32}[dtype]
        elt = 2 if dtype == "fp16" else 4
        inp = workload_inputs(wid, dtype="fp16" if dtype == "fp16" else "fp32")
        B = {k: torch.from_numpy(v).cuda() for k, v in inp.items()
             if k in (("x", "W", "b") + (("dy",) if set(passes) - {"fwd"} else ()))}
        What = torch.empty(F.feql_weight_fft_bytes(C, D, mode), dtype=torch.uint8, device="cuda")
        dt = B["x"].dtype
        y = torch.empty((N, D, 4), dtype=dt, device="cuda")
        dx = torch.empty((N, C, 4), dtype=dt, device="cuda")
        dW = torch.empty((D, C, 4), dtype=dt, device="cuda")
        db = torch.empty((D,), dtype=dt, device="cuda")
        ws = Lyr.dw_workspace(N, C, D, mode, "cuda")
        x, W, b, dy = B["x"], B["W"], B["b"], B.get("dy")
        calls = {
            "wfft": lambda: F.feql_weight_fft(W, What, C, D, mode, s),
            "fwd": lambda: F.feql_forward(x, What, b, y, N, C, D, mode, s),
            "dx": lambda: F.feql_backward_dx(dy, What, dx, N, C, D, mode, s),
            "dw": lambda: F.feql_backward_dw(x, dy, dW, db, ws, ws.numel(), N, C, D, mode, s),
            "bwd": lambda: F.feql_backward(x, dy, What, dx, dW, db, ws, ws.numel(), N, C, D,
                                           mode, s),
        }
        nbytes = workload_bytes(w, elt)
        macs = 6 * N * C * D
        flops = {"wfft": 0, "fwd": 2 * macs, "dx": 2 * macs, "dw": 2 * macs, "bwd": 4 * macs}
        calls["wfft"]()
        res = {}
        for p in ("wfft",) + tuple(passes):
            for _ in range(3):
                calls[p]()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(reps)]
            hold_gpu(torch)  # the reps queue up behind it: no host gaps between them
            for a, z in ev:
                flush.sum()
                a.record(stream)
                calls[p]()
                z.record(stream)
            torch.cuda.synchronize()
            us = sorted(a.elapsed_time(z) * 1e3 for a, z in ev)
            med, mn = float(np.median(us)), us[0]
            r = {"median_us": round(med, 3), "min_us": round(mn, 3), "reps": reps,
                 "algorithmic_bytes": nbytes[p],
                 "GB_s": round(nbytes[p] / (med * 1e-6) / 1e9, 1),
                 "traffic": traffic.get(w.name, {}).get(p)}
            if flops[p]:
                r["tokens_per_s"] = round(N / (med * 1e-6), 1)
                r["alg_TFLOP_s"] = round(flops[p] / (med * 1e-6) / 1e12, 3)
                r["dense_equiv_TFLOP_s"] = round(flops[p] * 16 / 6 / (med * 1e-6) / 1e12, 3)
                for tag, pk in (("measured", meas), ("nominal", nom)):
                    if pk is None:
                        continue
                    t_roof, bound = roofline_us(nbytes[p], flops[p], dtype, pk)
                    r[f"roofline_us_{tag}"] = round(t_roof, 3)
                    r[f"pct_roofline_{tag}"] = round(100 * t_roof / med, 2)
                    r["bound"] = bound
            res[p] = r
        if F.feql_device_status(s) != F.FEQL_OK:
            raise RuntimeError(f"device-side timeout in workload {wid}")
        key = f"{wid}_{dtype}"
        entry = {"workload": w.name, "N": N, "C": C, "D": D, "dtype": dtype,
                 "l2": f"flushed before every rep (read of a {2 * l2 >> 20} MiB buffer)",
                 "passes": res}
        t = {p: res[p]["median_us"] for p in res}
        if passes == ("fwd",):
            entry["tokens_per_s"] = round(N / (t["fwd"] * 1e-6), 1)
        elif passes == ("dx", "dw"):
            entry["tokens_per_s"] = round(N / ((t["dx"] + t["dw"]) * 1e-6), 1)
        else:
            entry["tokens_per_s"] = round(N / ((t["fwd"] + t["dx"] + t["dw"]) * 1e-6), 1)
            entry["tokens_per_s_fused_backward"] = round(N / ((t["fwd"] + t["bwd"]) * 1e-6), 1)
        out[key] = entry
        del B, x, W, b, dy, y, dx, dW, db, ws, What, calls
        torch.cuda.empty_cache()
    out.update(widening_report(F, torch, stream, reps, meas, nom, flush))
    return out


# The widened rows at full size: the C_8, C_6 and p4m layers and the two MLP
# blocks, all on the tensor cores.
WIDENING_RUNS = (6, 8, 10, 7, 9)
# Nominal special-function throughput: 16 MUFU operations per SM per clock
# (four per SM sub-partition), one tanh.approx.f16x2 (two values) per
# operation, at the maximum SM clock.
MUFU_OPS_PER_SM_CLK = 16
SM_CLOCK_GHZ = 1.965


def widening_report(F, torch, stream, reps, meas, nom, flush):
    """The per-config measurement of the widened workloads: each pass over `reps`
    CUDA-event timings with the L2 flushed before each, median and min, against
    the slower of its algorithmic bytes at HBM bandwidth and its Fourier-route
    FLOPs at the arithmetic peak of the units it runs on (tensor cores, or the
    fp32 FMA pipes for a shape the CUDA-core kernels serve).  The MLP block
    also gets a special-function floor: its GELU takes one tanh per two hidden
    values."""
    import numpy as np

    from group_dft_structured_b200.workloads import WORKLOADS
    s = stream.cuda_stream
    args = argparse.Namespace(separate_backward=True)
    out = {}
    for wid in WIDENING_RUNS:
        w = WORKLOADS[wid]
        mlp = "mlp" in w.passes
        st = (setup_mlp if mlp else setup_layer)(args, w, 0, s, F, torch)
        calls, res = st["calls"], {}
        calls["wfft"]()
        # the tensor-core kernels serve T = 4, 8, and 6 when C and D are multiples of 4
        simt = not (w.T in (4, 8) or (w.T == 6 and w.C % 4 == 0 and w.D % 4 == 0))
        for p in st["passes"]:
            for _ in range(3):
                calls[p]()
            ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                  for _ in range(reps)]
            hold_gpu(torch)
            for a, z in ev:
                flush.sum()
                a.record(stream)
                calls[p]()
                z.record(stream)
            torch.cuda.synchronize()
            us = sorted(a.elapsed_time(z) * 1e3 for a, z in ev)
            med, mn = float(np.median(us)), us[0]
            nbytes, (fl, dense_fl) = st["bytes"][p], st["flops"][p]
            r = {"median_us": round(med, 3), "min_us": round(mn, 3), "reps": reps,
                 "algorithmic_bytes": nbytes, "GB_s": round(nbytes / (med * 1e-6) / 1e9, 1)}
            if fl:
                r["tokens_per_s"] = round(w.N / (med * 1e-6), 1)
                r["alg_TFLOP_s"] = round(fl / (med * 1e-6) / 1e12, 3)
                r["dense_equiv_TFLOP_s"] = round(dense_fl / (med * 1e-6) / 1e12, 3)
                for tag, pk in (("measured", meas), ("nominal", nom)):
                    if pk is None:
                        continue
                    t_roof, bound = roofline_us(nbytes, fl, "fp32" if simt else "fp16", pk)
                    r[f"roofline_us_{tag}"] = round(t_roof, 3)
                    r[f"pct_roofline_{tag}"] = round(100 * t_roof / med, 2)
                    r["bound"] = bound
                if p == "mlp":
                    mufu = w.N * 4 * w.D / 2  # tanh.approx.f16x2 per two hidden values
                    t_xu = mufu / (MUFU_OPS_PER_SM_CLK * torch.cuda.get_device_properties(
                        0).multi_processor_count * SM_CLOCK_GHZ * 1e9) * 1e6
                    r["xu_floor_us_nominal"] = round(t_xu, 3)
                    r["pct_xu_floor"] = round(100 * t_xu / med, 2)
            res[p] = r
        if F.feql_device_status(s) != F.FEQL_OK:
            raise RuntimeError(f"device-side timeout in workload {wid}")
        out[f"{wid}_{w.dtype}"] = {
            "workload": w.name, "N": w.N, "C": w.C, "D": w.D, "T": w.T, "group": w.group,
            "dtype": w.dtype, "units": "CUDA cores (fp32 arithmetic)" if simt else "tensor cores",
            "l2": f"flushed before every rep (read of a {flush.numel() * 4 >> 20} MiB buffer)",
            "passes": res}
        del st, calls
        torch.cuda.empty_cache()
    return out


def main():
    args = parse()
    rank, world, local_rank = dist_env()
    if args.impl == "reference":
        return run_reference(args, rank, world)

    import numpy as np
    import torch
    import torch.distributed as dist

    import group_dft_structured_b200 as F
    from group_dft_structured_b200.workloads import WORKLOADS

    w = WORKLOADS[args.workload]
    if args.dtype is not None or args.tokens is not None:
        import dataclasses
        w = dataclasses.replace(w, dtype=args.dtype or w.dtype, N=args.tokens or w.N)
    torch.cuda.set_device(local_rank)
    if world > 1:
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    F.load()
    stream = torch.cuda.current_stream()
    s = stream.cuda_stream
    job = (setup_mlp if "mlp" in w.passes else setup_layer)(args, w, rank, s, F, torch)
    calls, passes, N = job["calls"], job["passes"], job["tokens"]
    B0 = job["B0"]

    def step(ev=None):
        if ev is not None:
            ev[0].record(stream)
        for i, p in enumerate(passes):
            calls[p]()
            if ev is not None:
                ev[i + 1].record(stream)
        if world > 1 and job["allreduce"] is not None:
            job["allreduce"](B0)

    def barrier():
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize()

    for _ in range(args.warmup):
        step()
    barrier()
    if F.feql_device_status(s) != F.FEQL_OK:
        raise RuntimeError("device-side timeout during warm-up")

    clocks = ClockSampler(local_rank)
    if rank == 0 or world == 1:
        clocks.start()
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(len(passes) + 1)]
           for _ in range(args.steps)]
    t_start = torch.cuda.Event(enable_timing=True)
    t_end = torch.cuda.Event(enable_timing=True)
    barrier()
    hold_gpu(torch)  # before the timed region: the host runs ahead of the GPU
    t_start.record(stream)
    for k in range(args.steps):
        step(evs[k])
    t_end.record(stream)
    barrier()
    clk = clocks.stop() if (rank == 0 or world == 1) else None
    ms = t_start.elapsed_time(t_end)
    if world > 1:
        ms = max_over_ranks(ms, "cuda")
    per_pass = {p: [evs[k][i].elapsed_time(evs[k][i + 1]) for k in range(args.steps)]
                for i, p in enumerate(passes)}
    if F.feql_device_status(s) != F.FEQL_OK:
        raise RuntimeError("device-side timeout during timing")

    # ---------------------------------------------------------- e2e (host buffers)
    # Every step copies its inputs from pinned host memory and its results back.
    # Two device buffer sets alternate between steps, and the copies run on their
    # own streams, so that step k+1's host-to-device copy overlaps step k's compute
    # and device-to-host copy (PCIe moves both directions at once).
    e2e = None
    if not args.no_e2e:
        hin = {k: torch.from_numpy(v).pin_memory() for k, v in job["host"].items()}
        sets = [B0, job["buffers"](B0)]
        hout = {k: torch.empty_like(B0[k], device="cpu").pin_memory() for k in job["outs"]}
        h2d = sum(t.numel() * t.element_size() for t in hin.values())
        d2h = sum(t.numel() * t.element_size() for t in hout.values())
        s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()
        set_calls = [job["calls_for"](B, s) for B in sets]
        in_done = [torch.cuda.Event() for _ in sets]
        comp_done = [torch.cuda.Event() for _ in sets]
        out_done = [torch.cuda.Event() for _ in sets]

        def e2e_run(nsteps):
            for k in range(nsteps):
                i = k % 2
                B = sets[i]
                if k >= 2:
                    s_in.wait_event(comp_done[i])  # step k-2 has read this set's inputs
                with torch.cuda.stream(s_in):
                    for name, t in hin.items():
                        B[name].copy_(t, non_blocking=True)
                in_done[i].record(s_in)
                stream.wait_event(in_done[i])
                if k >= 2:
                    stream.wait_event(out_done[i])  # step k-2's results are on the host
                for p in passes:
                    set_calls[i][p]()
                if world > 1 and job["allreduce"] is not None:
                    job["allreduce"](B)
                comp_done[i].record(stream)
                s_out.wait_event(comp_done[i])
                with torch.cuda.stream(s_out):
                    for name, t in hout.items():
                        t.copy_(B[name], non_blocking=True)
                out_done[i].record(s_out)

        e2e_run(2)
        barrier()
        a, z = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record(stream)
        s_in.wait_stream(stream)
        e2e_run(args.e2e_steps)
        stream.wait_stream(s_out)
        z.record(stream)
        barrier()
        e_ms = a.elapsed_time(z)
        if world > 1:
            e_ms = max_over_ranks(e_ms, "cuda")
        e2e = {"value": N * world * args.e2e_steps / (e_ms * 1e-3), "unit": "tokens/s",
               "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h),
               "steps": args.e2e_steps,
               "copies": "pinned host buffers; H2D, compute and D2H on three streams, two "
                         "device buffer sets alternating between steps"}
        del sets, set_calls
    extra = {}
    if rank == 0 and "unfused" in job["extra"]:
        extra["unfused_ms"] = round(job["extra"]["unfused"](), 5)

    if world > 1:
        dist.barrier()
        dist.destroy_process_group()
    if rank != 0:
        return 0

    # ------------------------------------------------------------- report
    value = N * world * args.steps / (ms * 1e-3)
    peak, peak_src = measured_peaks()
    nbytes = job["bytes"]
    med_ms = {p: float(np.median(v)) for p, v in per_pass.items()}
    pass_report = {}
    for p in passes:
        gbs = nbytes[p] / (med_ms[p] * 1e-3) / 1e9
        pass_report[p] = {"median_ms": round(med_ms[p], 5), "min_ms": round(min(per_pass[p]), 5),
                          "mean_ms": round(float(np.mean(per_pass[p])), 5),
                          "GB_s": round(gbs, 1), "frac_hbm": round(gbs / peak, 4),
                          "algorithmic_bytes": nbytes[p]}
        alg, dense = job["flops"][p]
        if alg:
            pass_report[p]["alg_TFLOP_s"] = round(alg / (med_ms[p] * 1e-3) / 1e12, 2)
            pass_report[p]["dense_equiv_TFLOP_s"] = round(dense / (med_ms[p] * 1e-3) / 1e12, 2)
    dom = max((p for p in passes if p != "wfft"), key=lambda p: med_ms[p])
    achieved = nbytes[dom] / (med_ms[dom] * 1e-3) / 1e9
    traffic = None
    tpath = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tpath):
        with open(tpath) as f:
            tj = json.load(f)
        if tj.get("source_hash") == kernel_source_hash():
            traffic = tj.get(w.name, {}).get(dom)
    nkern = sum(job["launches"][p] for p in passes)
    step_ms = ms / args.steps
    line = {
        "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_ms,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "f16" if w.dtype == "fp16" else "f32",
        "data": "synthetic",
        "config": dict({"workload": w.name}, **job["config"],
                       passes=passes, accumulate="f32",
                       l2="no flush: every pass streams more than twice the 126 MB L2"
                       if sum(nbytes[p] for p in passes if p != "wfft") > 2 * 126e6
                       else "no flush (inputs smaller than L2: warm)",
                       global_tokens=N * world,
                       parallelism=f"dp{world}" if world > 1 else "single"),
        "effective_TFLOP_s": round(sum(job["flops"][p][1] for p in passes) * world
                                   / (step_ms * 1e-3) / 1e12, 2),
        "roofline_pct_step": round(100 * sum(nbytes[p] for p in passes) / (step_ms * 1e-3) / 1e9
                                   / peak, 2),
        "roofline": {"bound": "hbm", "kernel": dom, "achieved": round(achieved, 1),
                     "peak": peak, "unit": "GB/s", "frac": round(achieved / peak, 4),
                     "traffic": traffic, "peak_source": peak_src,
                     "duration": "median of the pass's CUDA-event times in the timed loop"},
        "passes": pass_report,
        "gpu_launches": nkern * args.steps,
        "clocks": clk,
        "e2e": e2e,
    }
    line.update(extra)
    if (not args.no_per_config and args.workload == WORKLOAD_ID and args.dtype is None
            and args.tokens is None):
        line["per_config"] = per_config_report(F, torch, stream, args.config_reps)
    if not args.no_cpu_baseline:
        line["cpu_baseline"] = cpu_baseline(w)
    print(json.dumps(line))
    return 0

if __name__ == "__main__":
    sys.exit(main())
