#!/usr/bin/env python
"""Benchmark of the B200 fused MoE layer.

Headline workload (N=1): the decode layer E=128 experts, top-8, H=2048, I=768,
bf16 weights (1.2 GB), at the four decode batch sizes M = 1, 4, 16, 64. One
step = one forward at each of the four M (85 tokens). No forward finds its
weights in the L2 cache (126 MB): consecutive forwards use different weight
sets (identically shaped layers with their own seeded weights, as the MoE layers
of successive transformer blocks), enough of them that at least 252 MB of other
weights stream through L2 between two forwards on one set (`--l2 flush` instead
writes a 252 MB buffer before every forward, outside the timed events; the
dirty lines it leaves are written back during the timed forward). Each forward
is replayed from a CUDA graph captured once per (M, weight set) (the forward is
a fixed launch chain with no host synchronisation).

The same line carries, under "workloads", the other shapes the metric names,
each measured the same way: decode FP8 e4m3 (M = 1, 8, 32, 64, from the same
decode weights), the Zipf-skewed large decode layer (E=256, H=7168, I=2048,
bf16, M = 1, 32, 64, 128) and prefill (the same layer, M = 4096, bf16 and e4m3
from one bf16 weight set).

Reported (one JSON line, rank 0):
  value      tokens/s over all ranks = N * 85 / (device time of one step)
  roofline   gate_up GEMM (the kernel with the largest share): active-expert
             W_gate+W_up bytes per launch / its CUDA-event duration, against
             the measured HBM copy bandwidth
  per_M      per batch size: device time (mean, p50, p95), tokens/s and the
             layer's roofline fraction, against the measured peaks and against
             the nominal 8 TB/s HBM / datasheet tensor peaks
  e2e        the same metric through moe_forward_host: host->device copies of
             x and logits and the device->host copy of out inside the timing
  cpu_baseline  the CPU oracle timed on the same decode sweep on the host cores

--impl reference times the CPU oracle itself on the same workload (the
reference arm); --gpus N runs N independent replicas (the layer needs no
collective), max over ranks.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fused-MoE tokens/s and HBM GB/s vs roofline (decode M=1-64, prefill), 1 B200"
FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
NOMINAL_HBM_GBS = 8000.0          # the "~8 TB/s" the layer's target is stated against
NOMINAL_BF16_TFLOPS = 2250.0      # B200 datasheet dense bf16 (FP8: twice)
DECODE_TARGET = 0.70              # decode shapes: fraction of the HBM roofline
L2_FLUSH_BYTES = 252 << 20
L2_BYTES = 126 << 20
MAX_WEIGHT_SETS = 16


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="b200", choices=["b200", "reference"])
    ap.add_argument("--workload", default="decode",
                    choices=["tiny", "decode", "decode_fp8", "decode_e5m2", "large_decode", "prefill",
                             "prefill_fp8", "prefill_m16384", "prefill_e48", "prefill_e48_fp8", "inv_rope"],
                    help="inv_rope: the inverse-RoPE + per-head FP8 kernel alone (--only-M picks one token count)")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of replaying graphs")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-workloads", action="store_true",
                    help="measure the headline workload only (skip decode FP8, large decode and prefill)")
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--only-M", type=int, default=None,
                    help="run a single batch size of the workload (inv_rope: a single token count)")
    ap.add_argument("--fused-decode", action="store_true", help="single-launch decode path (bf16, M <= 64)")
    ap.add_argument("--l2", default="rotate", choices=["rotate", "flush", "warm"],
                    help="rotate: consecutive forwards on different weight sets (inputs larger than L2); "
                         "flush: a 252 MB write before every forward; warm: one set, no flush")
    ap.add_argument("--warm-l2", action="store_true",
                    help="same as --l2 warm (a labelled warm-cache figure, not the headline)")
    a = ap.parse_args()
    if a.warm_l2:
        a.l2 = "warm"
    return a


def workload_spec(name):
    from mixture_experts_layer_sort_b200 import synth
    if name in synth.WORKLOADS:
        wl = synth.WORKLOADS[name]
        return wl, wl.dtypes[0]
    if name.endswith("_fp8") and name[:-4] in synth.WORKLOADS:
        return synth.WORKLOADS[name[:-4]], "fp8"
    raise KeyError(name)


def read_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), float(d["bf16_tflops"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, "fallback"


def is_fp8(dtype):
    return dtype in ("fp8", "fp8_e5m2")


def fp8_format(dtype):
    return "e5m2" if dtype == "fp8_e5m2" else "e4m3"


def dtype_name(dtype):
    return "bf16" if dtype == "bf16" else fp8_format(dtype)


def weight_bytes(dtype):
    return 1 if is_fp8(dtype) else 2


def alg_bytes_layer(wl, dtype, M, A):
    """Algorithmic bytes of one forward: active-expert weights, FP8 scales, x, out, logits."""
    b = A * 3 * wl.H * wl.I * weight_bytes(dtype) + M * wl.H * 2 * 2 + M * wl.E * 4
    if is_fp8(dtype):
        b += 3 * wl.E * 4
    return b


def alg_flops_layer(wl, M):
    return 6 * M * wl.k * wl.H * wl.I


def l2_plan(wl, dtype, mode):
    """How the forwards of a workload are kept from finding their weights in L2:
    ("rotate", R, text): consecutive forwards use R different weight sets, R chosen so
    that at least 2 x L2 of other weights stream through between two forwards on one set
    (a forward streams at least the weights of k experts); ("flush", 1, text) when that
    needs more than MAX_WEIGHT_SETS sets or is not asked for; ("warm", 1, text)."""
    if mode == "warm":
        return "warm", 1, "warm: one weight set, not flushed between forwards"
    per_expert = 3 * wl.H * wl.I * weight_bytes(dtype)
    fewest = min(wl.k, wl.E) * per_expert
    R = -(-2 * L2_BYTES // fewest) + 1
    if mode == "rotate" and R <= MAX_WEIGHT_SETS:
        return "rotate", R, (f"inputs larger than L2: consecutive forwards on different weight sets ({R} sets, "
                             f"{R * wl.E * per_expert / 1e9:.1f} GB in all; at least {(R - 1) * fewest / 2**20:.0f} "
                             f"MB of other weights stream through the 126 MB L2 between two forwards on one set), "
                             f"no flush")
    return "flush", 1, "flushed (252 MB write) before every forward, outside the timed events"


def set_seed(seed, r):
    """Weight seed of set r (set 0 is the workload's own seed)."""
    return seed if r == 0 else seed + 7919 * r


def bench_config(wl, Ms, ws, l2_text):
    """The workload description both arms print (the reference arm prints the same dict)."""
    return {"workload": wl.description + f", one step = one forward at each M in {list(Ms)}",
            "E": wl.E, "topk": wl.k, "H": wl.H, "I": wl.I, "Ms": list(Ms), "global_batch": sum(Ms) * ws,
            "parallelism": f"replicas x{ws}" if ws > 1 else "single GPU",
            "l2": l2_text}


def cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except Exception:
        pass
    return None


# ----------------------------------------------------------------------------- clocks
class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while the timed regions run."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index):
        self.index = index
        self.proc = None
        self.path = None

    def start(self):
        try:
            fd, self.path = tempfile.mkstemp(suffix=".csv")
            os.close(fd)
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100", "-f", self.path], stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except Exception:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) >= 9:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}

        def num(v):
            try:
                return float(v)
            except ValueError:
                return None

        sm = [num(r[1]) for r in rows if num(r[1]) is not None]
        smax = max((num(r[2]) for r in rows if num(r[2]) is not None), default=None)
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].lower() == "active"})
        under_load = [v for v in sm if smax and v >= 0.5 * smax] or sm
        return {"sm_mhz": statistics.median(under_load) if under_load else None, "sm_max_mhz": smax,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------- distributed
def dist_setup(args):
    import torch
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return ws, rank, local


def barrier(ws):
    if ws > 1:
        import torch.distributed as dist
        dist.barrier()


def max_over_ranks(v, ws):
    if ws == 1:
        return v
    import torch
    import torch.distributed as dist
    on_gpu = dist.get_backend() == "nccl"
    t = torch.tensor([v], dtype=torch.float64, device="cuda" if on_gpu else "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def blas_threads():
    try:
        import threadpoolctl
        info = threadpoolctl.threadpool_info()
        n = [i["num_threads"] for i in info if i.get("user_api") == "blas"]
        return max(n) if n else os.cpu_count()
    except Exception:
        return os.cpu_count()


# ----------------------------------------------------------------------------- oracle timing
def time_oracle_sweep(wl, dtype, host_weights, tokens_per_M, budget_s=30.0, max_reps=50, one_thread=False):
    """Seconds per sweep of the CPU oracle over tokens_per_M (bounded: at least one sweep)."""
    import contextlib
    from oracle import moe_oracle as O
    ctx = contextlib.nullcontext()
    if one_thread:
        import threadpoolctl
        ctx = threadpoolctl.threadpool_limits(limits=1)
    cache = {}
    times = []
    with ctx:
        if is_fp8(dtype):   # fill the FP8 weight cache outside the timing, as the GPU loads once
            for M, (x, l) in tokens_per_M.items():
                O.moe_forward(x, l, wl.k, *host_weights, fp8=True, fp8_format=fp8_format(dtype),
                              weight_cache=cache, threads=1 if one_thread else None)
        t_start = time.time()
        for _ in range(max_reps):
            t0 = time.time()
            for M, (x, l) in tokens_per_M.items():
                O.moe_forward(x, l, wl.k, *host_weights, fp8=is_fp8(dtype), fp8_format=fp8_format(dtype),
                              weight_cache=cache, threads=1 if one_thread else None)
            times.append(time.time() - t0)
            if time.time() - t_start > budget_s:
                break
    return statistics.median(times), len(times)


def cpu_baseline_entry(wl, dtype, host_w, toks_np, budget_s, one_thread_Ms=(1, 4)):
    """The oracle on the host cores: the full sweep on all threads, and a smaller
    sample on one thread (both bounded), as tokens/s."""
    Ms = list(toks_np)
    tokens = sum(Ms)
    sec, reps = time_oracle_sweep(wl, dtype, host_w, toks_np, budget_s=budget_s)
    sub = {M: toks_np[M] for M in one_thread_Ms if M in toks_np}
    sec1, reps1 = time_oracle_sweep(wl, dtype, host_w, sub, budget_s=budget_s / 3, max_reps=5, one_thread=True)
    return {"value": tokens / sec, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
            "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
            "sample": f"{reps} full sweep(s) M={Ms} ({tokens} tokens) on all host threads, median",
            "one_thread": {"value": sum(sub) / sec1, "unit": "tokens/s", "cores": 1,
                           "sample": f"{reps1} sweep(s) M={list(sub)} ({sum(sub)} tokens), median"}}


def reference_arm(args, ws, rank):
    """The CPU oracle as the reference arm: rank 0 times it, the others exit."""
    if rank != 0:
        return 0
    if args.workload == "inv_rope":
        print(json.dumps({"impl": "reference", "unavailable": "the reference arm times the MoE layer; the "
                          "inverse-RoPE kernel's CPU oracle is timed inside the default bench line"}))
        return 0
    from mixture_experts_layer_sort_b200 import synth
    wl, dtype = workload_spec(args.workload)
    only_M = getattr(args, "only_M", None)
    Ms = [only_M] if only_M else list(wl.Ms)
    if args.workload in ("prefill", "prefill_fp8", "prefill_m16384", "large_decode"):
        print(json.dumps({"impl": "reference", "unavailable": "the CPU oracle needs the 22.5 GB weight set "
                          "on the host; the reference arm runs on the decode workloads"}))
        return 0
    wg, wu, wd = synth.make_weights(wl.E, wl.H, wl.I, wl.w_std, seed=args.seed, device="cpu")
    host = [w.float().numpy() for w in (wg, wu, wd)]
    toks = {}
    for M in Ms:
        x, l = synth.make_tokens(wl.E, wl.H, M, seed=args.seed, zipf_s=wl.zipf_s)
        toks[M] = (x.float().numpy(), l.numpy())
    tokens = sum(Ms)
    from oracle import moe_oracle as O
    cache = {}
    for M, (x, l) in toks.items():   # one warm-up sweep (fills the FP8 weight cache)
        O.moe_forward(x, l, wl.k, *host, fp8=is_fp8(dtype), fp8_format=fp8_format(dtype), weight_cache=cache)
    times = []
    for _ in range(args.steps):
        t0 = time.time()
        for M, (x, l) in toks.items():
            O.moe_forward(x, l, wl.k, *host, fp8=is_fp8(dtype), fp8_format=fp8_format(dtype), weight_cache=cache)
        times.append(time.time() - t0)
    sec = statistics.mean(times)
    value = tokens / sec
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "tokens/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": sec * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": bench_config(wl, Ms, args.gpus, l2_plan(wl, dtype, getattr(args, "l2", "rotate"))[2]),
        "cpu_baseline": {"value": value, "unit": "tokens/s", "cores": blas_threads(), "kind": "oracle",
                         "cpu_model": cpu_model(), "host_cpus": os.cpu_count(),
                         "sample": f"full sweep M={Ms} ({tokens} tokens) per step"},
        "e2e": {"value": value, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line))
    return 0


# ----------------------------------------------------------------------------- main arm
def traffic_from_profile(kernel_src_hash):
    """Per-launch DRAM bytes of the gate_up kernel at each M of the decode sweep from the
    committed ncu summary, or None when the kernel sources changed since the counters
    were taken."""
    p = os.path.join(ROOT, "profiles", "gate_up_gemm_decode_traffic.txt")
    try:
        d = {}
        with open(p) as f:
            for line in f:
                if "=" in line and not line.startswith("#"):
                    k, v = line.split("=", 1)
                    d[k.strip()] = v.strip()
        if d.get("kernel_source_sha256") != kernel_src_hash:
            return None
        return {int(k.split("_")[-1]): float(v) for k, v in d.items() if k.startswith("dram_bytes_per_launch_M_")}
    except Exception:
        return None


def kernel_source_hash():
    h = hashlib.sha256()
    for name in ("kernels_gemm.cu", "kernels_gemv.cu", "gemm_pipeline.cuh", "sm100.cuh", "moe_internal.h"):
        with open(os.path.join(ROOT, "mixture_experts_layer_sort_b200", "csrc", name), "rb") as f:
            h.update(f.read())
    return h.hexdigest()


class Runner:
    """Times one workload on one or more identically shaped layers (weight sets): graph
    replay per (M, set), consecutive forwards on consecutive sets (or, with a flush buffer,
    a 252 MB write before every forward, outside the events), then an eager pass, then a
    pass with the library's per-kernel CUDA events (on the forward's stream)."""

    def __init__(self, layers, wl, dtype, Ms, toks, stream, flush, use_graph):
        import torch
        self.torch = torch
        self.layers, self.wl, self.dtype, self.Ms, self.toks = list(layers), wl, dtype, list(Ms), toks
        self.stream, self.flush = stream, flush
        self.fi = 0   # forwards issued so far: forward i runs on set i % R
        dev = toks[self.Ms[0]][0].device
        self.outs = {M: torch.empty((M, wl.H), dtype=torch.bfloat16, device=dev) for M in self.Ms}
        for lay in self.layers:
            lay.reserve(max(self.Ms))
        self.A, self.launches = {}, {}
        layer = self.layers[0]
        with torch.cuda.stream(stream):
            for M in self.Ms:
                # the routing depends on the logits only: every set activates the same experts
                layer.forward(*toks[M], out=self.outs[M])
                self.A[M] = int(torch.count_nonzero(layer.debug_routing(M)["counts"]).item())
                layer.forward(*toks[M], out=self.outs[M])
                self.launches[M] = layer.last_launch_count
                for lay in self.layers[1:]:
                    lay.forward(*toks[M], out=self.outs[M])
        torch.cuda.synchronize()
        self.graphs = {}
        if use_graph:
            for M in self.Ms:
                for r, lay in enumerate(self.layers):
                    g = torch.cuda.CUDAGraph()
                    with torch.cuda.graph(g, stream=stream):
                        lay.forward(*toks[M], out=self.outs[M])
                    self.graphs[(M, r)] = g
            torch.cuda.synchronize()

    def _next(self):
        """Set of the next forward; flushes L2 first in flush mode."""
        r = self.fi % len(self.layers)
        self.fi += 1
        if self.flush is not None:
            self.flush.zero_()
        return r

    def forward(self, M, r):
        if self.graphs:
            self.graphs[(M, r)].replay()
        else:
            self.layers[r].forward(*self.toks[M], out=self.outs[M])

    def step(self, events=None):
        for i, M in enumerate(self.Ms):
            r = self._next()
            if events is not None:
                events[i][0].record(self.stream)
            self.forward(M, r)
            if events is not None:
                events[i][1].record(self.stream)

    def warm(self, n):
        with self.torch.cuda.stream(self.stream):
            for _ in range(max(n, len(self.layers))):
                self.step()
        self.torch.cuda.synchronize()

    def timed(self, steps):
        """Per-M lists of CUDA-event ms over `steps` steps, and the wall time."""
        torch = self.torch
        ev = [[[torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)] for _ in self.Ms]
              for _ in range(steps)]
        torch.cuda.synchronize()
        t0 = time.time()
        with torch.cuda.stream(self.stream):
            for s in range(steps):
                self.step(ev[s])
        torch.cuda.synchronize()
        wall = time.time() - t0
        per_M = {M: [ev[s][i][0].elapsed_time(ev[s][i][1]) for s in range(steps)] for i, M in enumerate(self.Ms)}
        return per_M, wall

    def eager_ms(self, reps=3):
        torch = self.torch
        got = {M: [] for M in self.Ms}
        with torch.cuda.stream(self.stream):
            for _ in range(reps):
                for M in self.Ms:
                    r = self._next()
                    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                    e0.record(self.stream)
                    self.layers[r].forward(*self.toks[M], out=self.outs[M])
                    e1.record(self.stream)
                    got[M].append((e0, e1))
        torch.cuda.synchronize()
        return {M: statistics.median(a.elapsed_time(b) for a, b in v) for M, v in got.items()}

    def kernel_profile(self, reps):
        """{kernel: (ms, launches)} over `reps` eager steps (summed over the sets), and the
        gate_up / down algorithmic weight bytes those launches moved."""
        wl, bw = self.wl, weight_bytes(self.dtype)
        for lay in self.layers:
            lay.profile_enable(True)
        gate_bytes = down_bytes = 0.0
        with self.torch.cuda.stream(self.stream):
            for _ in range(reps):
                for M in self.Ms:
                    r = self._next()
                    self.layers[r].forward(*self.toks[M], out=self.outs[M])
                    gate_bytes += self.A[M] * 2 * wl.H * wl.I * bw
                    down_bytes += self.A[M] * wl.H * wl.I * bw
        prof = {}
        for lay in self.layers:
            for k, (ms, n) in lay.profile_read().items():
                a, b = prof.get(k, (0.0, 0))
                prof[k] = (a + ms, b + n)
            lay.profile_enable(False)
        return prof, gate_bytes, down_bytes

    def close(self):
        self.graphs.clear()


def per_M_summary(wl, dtype, Ms, per_M_ms, eager, A, launches, hbm_gbs, bf16_tf):
    tensor_tf = bf16_tf * (2.0 if is_fp8(dtype) else 1.0)
    tensor_nom = NOMINAL_BF16_TFLOPS * (2.0 if is_fp8(dtype) else 1.0)
    out = {}
    for M in Ms:
        v = per_M_ms[M]
        t = statistics.mean(v)
        srt = sorted(v)
        b = alg_bytes_layer(wl, dtype, M, A[M])
        f = alg_flops_layer(wl, M)
        t_roof = max(b / (hbm_gbs * 1e9), f / (tensor_tf * 1e12))
        t_nom = max(b / (NOMINAL_HBM_GBS * 1e9), f / (tensor_nom * 1e12))
        out[str(M)] = {"ms": t, "ms_p50": statistics.median(srt),
                       "ms_p95": srt[min(len(srt) - 1, int(round(0.95 * (len(srt) - 1))))],
                       "ms_eager": eager.get(M), "tokens_per_s": M / (t / 1e3), "active_experts": A[M],
                       "alg_GB": b / 1e9, "alg_GBps": b / (t / 1e3) / 1e9,
                       "tflops": f / (t / 1e3) / 1e12, "tensor_frac": f / (t / 1e3) / (tensor_tf * 1e12),
                       "roofline_bound": "hbm" if b / (hbm_gbs * 1e9) >= f / (tensor_tf * 1e12) else "tensor",
                       "roofline_frac": t_roof / (t / 1e3), "roofline_frac_nominal": t_nom / (t / 1e3),
                       "launches": launches[M]}
    return out


def make_layer_sets(wl, dtypes, R, seed, dev, first=None, keep_first=False, fused_decode=False):
    """R weight sets of a workload's shape: for each set r, one layer per dtype in `dtypes`,
    all loaded from set r's bf16 weights (drawn with set_seed(seed, r); set 0's tensors may
    be passed in as `first`). Returns {dtype: [layer of set 0, ...]} and, with keep_first,
    set 0's bf16 tensors."""
    import torch
    from mixture_experts_layer_sort_b200 import MoELayer, synth
    out = {d: [] for d in dtypes}
    w0 = None
    for r in range(R):
        w = first if (r == 0 and first is not None) else \
            synth.make_weights(wl.E, wl.H, wl.I, wl.w_std, seed=set_seed(seed, r), device=dev)
        for d in dtypes:
            lay = MoELayer(wl.E, wl.k, wl.H, wl.I, d)
            lay.load_weights(*w)
            if fused_decode:
                lay.set_fused_decode(True)
            out[d].append(lay)
        if r == 0 and keep_first:
            w0 = w
        del w
    torch.cuda.empty_cache()
    return out, w0


def measure_workload(name, layers, wl, dtype, Ms, toks, stream, args, hbm_gbs, bf16_tf, flush_buf):
    """One workload entry of the bench line (an extra workload next to the headline), on
    `layers` (one per weight set; in flush mode the first alone, with flush_buf)."""
    mode, R, l2_text = l2_plan(wl, dtype, args.l2)
    flush = flush_buf if mode == "flush" else None
    r = Runner(layers[:R], wl, dtype, Ms, toks, stream, flush, use_graph=not args.no_graph)
    r.warm(max(3, args.warmup))
    steps = max(5, min(args.steps, 20))
    per_M_ms, _ = r.timed(steps)
    eager = r.eager_ms()
    prof, gate_bytes, down_bytes = r.kernel_profile(max(3, min(steps, 10)))
    r.close()
    step_ms = [sum(per_M_ms[M][s] for M in Ms) for s in range(steps)]
    ms = statistics.mean(step_ms)
    g_ms, _ = prof["gate_up"]
    d_ms, _ = prof["down"]
    tot = sum(v[0] for v in prof.values())
    gemm = {"gate_up": {"GBps": gate_bytes / (g_ms / 1e3) / 1e9 if g_ms > 0 else None},
            "down": {"GBps": down_bytes / (d_ms / 1e3) / 1e9 if d_ms > 0 else None}}
    for v in gemm.values():
        v["frac"] = v["GBps"] / hbm_gbs if v["GBps"] else None
    dom = max(("gate_up", "down"), key=lambda k: prof[k][0])
    summary = per_M_summary(wl, dtype, Ms, per_M_ms, eager, r.A, r.launches, hbm_gbs, bf16_tf)
    entry = {"workload": wl.description + f", one step = one forward at each M in {list(Ms)}",
             "l2": l2_text,
             "dtype": dtype_name(dtype), "Ms": list(Ms), "steps": steps, "ms_per_step": ms,
             "tokens_per_s": sum(Ms) / (ms / 1e3), "per_M": summary,
             "dominant_gemm": dict(kernel=dom, **gemm[dom]), "gemm_event_GBps": gemm,
             "kernel_share": {k: round(v[0] / tot, 4) for k, v in prof.items() if v[1] > 0} if tot else {},
             "launches_per_step": sum(r.launches[M] for M in Ms)}
    if name.startswith("decode"):
        entry["meets_decode_target"] = {M: summary[str(M)]["roofline_frac"] >= DECODE_TARGET for M in summary}
    return entry


ROPE_SHAPE = {"NH": 16, "D": 128, "max_pos": 32768, "Ts": (1, 64, 4096, 16384)}


def measure_inv_rope(args, dev, stream, flush, seed, hbm_gbs, cpu_on, Ts=None):
    """The inverse-RoPE + per-head FP8 quantisation kernel at several token counts (one
    kernel for all of them): device time per call with L2 flushed before each, and the
    achieved HBM bandwidth over its algorithmic bytes (2D bytes in, D codes + a 4-byte
    scale out per vector, a 4-byte position per token)."""
    import numpy as np
    import torch
    from mixture_experts_layer_sort_b200 import inv_rope_fp8_quant
    NH, D, max_pos = ROPE_SHAPE["NH"], ROPE_SHAPE["D"], ROPE_SHAPE["max_pos"]
    i = torch.arange(D // 2, dtype=torch.float64)
    ang = torch.arange(max_pos, dtype=torch.float64)[:, None] * (10000.0 ** (-2.0 * i / D))[None, :]
    table = torch.cat([torch.cos(ang), torch.sin(ang)], dim=1).float().to(dev)
    g = torch.Generator(device=dev).manual_seed(seed)
    steps = max(5, min(args.steps, 20))
    per_T = {}
    Ts = list(Ts or ROPE_SHAPE["Ts"])
    for T in Ts:
        x = torch.randn((T, NH, D), generator=g, device=dev).to(torch.bfloat16)
        pos = torch.randint(0, max_pos, (T,), generator=g, device=dev, dtype=torch.int32)
        codes = torch.empty((T, NH, D), dtype=torch.uint8, device=dev)
        scales = torch.empty((T, NH), dtype=torch.float32, device=dev)
        with torch.cuda.stream(stream):
            for _ in range(3):
                inv_rope_fp8_quant(x, pos, table, codes=codes, scales=scales, stream=stream)
        torch.cuda.synchronize()
        # replayed from a CUDA graph like the layer, so that no host launch gap is timed
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph, stream=stream):
            inv_rope_fp8_quant(x, pos, table, codes=codes, scales=scales, stream=stream)
        torch.cuda.synchronize()
        with torch.cuda.stream(stream):
            ev = []
            for _ in range(steps):
                flush.zero_()
                e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                e0.record(stream)
                graph.replay()
                e1.record(stream)
                ev.append((e0, e1))
        torch.cuda.synchronize()
        del graph
        ms = sorted(a.elapsed_time(b) for a, b in ev)
        mean = statistics.mean(ms)
        alg = T * NH * (2 * D + D + 4) + T * 4
        per_T[str(T)] = {"us": mean * 1e3, "us_p50": statistics.median(ms) * 1e3, "alg_MB": alg / 1e6,
                         "GBps": alg / (mean / 1e3) / 1e9, "frac_hbm": alg / (mean / 1e3) / 1e9 / hbm_gbs}
    entry = {"workload": f"inverse RoPE + per-head e4m3 quantisation, [T, {NH} heads, {D}] bf16, half-split "
                         f"pairs, one launch per T in {Ts}",
             "per_T": per_T, "bound": "hbm", "peak_GBps": hbm_gbs}
    if cpu_on:
        from oracle import rope_oracle as R
        T = 4096
        x = torch.randn((T, NH, D), generator=g, device=dev).to(torch.bfloat16).float().cpu().numpy()
        pos = torch.randint(0, max_pos, (T,), generator=g, device=dev, dtype=torch.int32).cpu().numpy()
        tab = table.cpu().numpy()
        t0 = time.time()
        reps = 0
        while reps < 3 or time.time() - t0 < 2.0:
            R.inv_rope_fp8_quant(x, pos, tab)
            reps += 1
            if time.time() - t0 > 10.0:
                break
        entry["cpu_baseline"] = {"value": T * reps / (time.time() - t0), "unit": "tokens/s", "kind": "oracle",
                                 "cores": 1, "sample": f"{reps} calls at T={T}"}
    return entry


def extra_workloads(args, dev, stream, flush, dec_weights, seed, hbm_gbs, bf16_tf, cpu_on):
    """Decode FP8 (from the decode weight sets), large decode and prefill bf16 + FP8 (from
    the E=256 bf16 weight sets), each measured like the headline."""
    import torch
    from mixture_experts_layer_sort_b200 import synth
    res = {}
    wl = synth.WORKLOADS["decode_fp8"]
    R = l2_plan(wl, "fp8", args.l2)[1]
    sets, _ = make_layer_sets(wl, ("fp8",), R, args.seed, dev, first=dec_weights)
    toks = {M: synth.make_tokens(wl.E, wl.H, M, seed=seed, device=dev) for M in wl.Ms}
    res["decode_fp8"] = measure_workload("decode_fp8", sets["fp8"], wl, "fp8", wl.Ms, toks, stream, args,
                                         hbm_gbs, bf16_tf, flush)
    for lay in sets["fp8"]:
        lay.close()
    if cpu_on:
        host_w = [synth.bf16_to_f32_numpy(w) for w in dec_weights]
        tnp = {M: (toks[M][0].float().cpu().numpy(), toks[M][1].cpu().numpy()) for M in wl.Ms}
        res["decode_fp8"]["cpu_baseline"] = cpu_baseline_entry(wl, "fp8", host_w, tnp, budget_s=10.0,
                                                               one_thread_Ms=(1, 8))
    del toks

    wl4, wl5 = synth.WORKLOADS["large_decode"], synth.WORKLOADS["prefill"]
    R = max(l2_plan(wl4, "bf16", args.l2)[1], l2_plan(wl5, "bf16", args.l2)[1], l2_plan(wl5, "fp8", args.l2)[1])
    sets, _ = make_layer_sets(wl4, ("bf16", "fp8"), R, args.seed, dev)
    toks = {M: synth.make_tokens(wl4.E, wl4.H, M, seed=seed, device=dev, zipf_s=wl4.zipf_s) for M in wl4.Ms}
    res["large_decode"] = measure_workload("large_decode", sets["bf16"], wl4, "bf16", wl4.Ms, toks, stream, args,
                                           hbm_gbs, bf16_tf, flush)
    del toks
    toks = {M: synth.make_tokens(wl5.E, wl5.H, M, seed=seed, device=dev) for M in wl5.Ms}
    res["prefill"] = measure_workload("prefill", sets["bf16"], wl5, "bf16", wl5.Ms, toks, stream, args,
                                      hbm_gbs, bf16_tf, flush)
    for lay in sets["bf16"]:
        lay.close()
    res["prefill_fp8"] = measure_workload("prefill_fp8", sets["fp8"], wl5, "fp8", wl5.Ms, toks, stream, args,
                                          hbm_gbs, bf16_tf, flush)
    for lay in sets["fp8"]:
        lay.close()
    del sets, toks
    torch.cuda.empty_cache()
    res["inv_rope_fp8"] = measure_inv_rope(args, dev, stream, flush, seed, hbm_gbs, cpu_on)
    return res


def rope_only(args, ws, rank, local):
    """The inverse-RoPE kernel on its own (every rank its own tokens; rank 0 prints)."""
    import torch
    dev = torch.device("cuda", local)
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    hbm_gbs, _, peak_src = read_peaks()
    res = measure_inv_rope(args, dev, stream, flush, args.seed + 1000 * rank, hbm_gbs, False,
                           Ts=[args.only_M] if args.only_M else None)
    barrier(ws)
    if rank == 0:
        print(json.dumps({"workload": "inv_rope", "n_gpus": ws, "peak_source": peak_src, **res}))
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def main():
    args = parse_args()
    ws, rank, local = dist_setup(args)
    if args.impl == "reference":
        rc = reference_arm(args, ws, rank)
        if ws > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
        return rc

    import torch

    from mixture_experts_layer_sort_b200 import synth

    if args.workload == "inv_rope":
        return rope_only(args, ws, rank, local)
    wl, dtype = workload_spec(args.workload)
    Ms = [args.only_M] if args.only_M else list(wl.Ms)
    dev = torch.device("cuda", local)
    seed = args.seed + 1000 * rank
    l2_mode, n_sets, l2_text = l2_plan(wl, dtype, args.l2)
    sets, w0 = make_layer_sets(wl, (dtype,), n_sets, args.seed, dev, keep_first=True,
                               fused_decode=args.fused_decode)
    layers = sets[dtype]
    wg, wu, wd = w0
    toks = {M: synth.make_tokens(wl.E, wl.H, M, seed=seed, device=dev, zipf_s=wl.zipf_s) for M in Ms}
    # the flush buffer: the flush mode's 252 MB write, and the inverse-RoPE measurement
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=dev)
    stream = torch.cuda.Stream(device=dev)
    tokens_per_step = sum(Ms)
    hbm_gbs, bf16_tf, peak_src = read_peaks()

    run = Runner(layers, wl, dtype, Ms, toks, stream, flush if l2_mode == "flush" else None,
                 use_graph=not args.no_graph)
    run.warm(args.warmup)

    # ---------------------------------------------------------------- timed region
    clocks = ClockSampler(torch.cuda.current_device())
    clocks.start()
    time.sleep(0.3)
    barrier(ws)
    per_M_ms, wall = run.timed(args.steps)
    barrier(ws)
    step_ms = [sum(per_M_ms[M][s] for M in Ms) for s in range(args.steps)]
    ms_per_step = max_over_ranks(statistics.mean(step_ms), ws)

    eager_ms = run.eager_ms()
    prof_steps = max(3, min(args.steps, 20))
    prof, gate_bytes, _ = run.kernel_profile(prof_steps)
    g_ms, g_n = prof["gate_up"]
    achieved = gate_bytes / (g_ms / 1e3) / 1e9 if g_ms > 0 else None
    traffic_tbl = traffic_from_profile(kernel_source_hash())
    traffic = None
    if traffic_tbl and all(M in traffic_tbl for M in Ms):
        traffic = statistics.mean(traffic_tbl[M] for M in Ms)
    total_prof = sum(v[0] for v in prof.values())

    # ---------------------------------------------------------------- other workloads of the metric
    workloads = None
    cpu_on = rank == 0 and ws == 1 and not args.no_cpu_baseline
    if ws == 1 and not args.no_workloads and args.workload == "decode" and not args.only_M:
        workloads = extra_workloads(args, dev, stream, flush, (wg, wu, wd), seed, hbm_gbs, bf16_tf, cpu_on)
    clk = clocks.stop()

    # ---------------------------------------------------------------- e2e through host buffers
    e2e = None
    if not args.no_e2e:
        host = {M: (toks[M][0].cpu().pin_memory(), toks[M][1].cpu().pin_memory(),
                    torch.empty((M, wl.H), dtype=torch.bfloat16).pin_memory()) for M in Ms}
        h2d = sum(M * wl.H * 2 + M * wl.E * 4 for M in Ms)
        d2h = sum(M * wl.H * 2 for M in Ms)
        for lay in layers:
            for M in Ms:
                lay.forward_host(*host[M], stream=stream)
        e_times = []
        fi = 0
        for s in range(args.steps):
            tot = 0.0
            for M in Ms:
                lay = layers[fi % len(layers)]   # the same rotation over the weight sets
                fi += 1
                if l2_mode == "flush":
                    flush.zero_()
                torch.cuda.synchronize()
                a = time.perf_counter()
                lay.forward_host(*host[M], stream=stream)
                tot += time.perf_counter() - a
            e_times.append(tot)
        e_sec = max_over_ranks(statistics.mean(e_times), ws)
        e2e = {"value": ws * tokens_per_step / e_sec, "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_sec * 1e3}

    # ---------------------------------------------------------------- CPU oracle on the same sweep
    cpu = None
    if cpu_on and args.workload in ("tiny", "decode", "decode_fp8", "decode_e5m2"):
        host_w = [synth.bf16_to_f32_numpy(w) for w in (wg, wu, wd)]
        tpm = {M: (toks[M][0].float().cpu().numpy(), toks[M][1].cpu().numpy()) for M in Ms}
        cpu = cpu_baseline_entry(wl, dtype, host_w, tpm, budget_s=30.0)

    per_M = per_M_summary(wl, dtype, Ms, per_M_ms, eager_ms, run.A, run.launches, hbm_gbs, bf16_tf)
    line = {
        "metric": METRIC,
        "value": ws * tokens_per_step / (ms_per_step / 1e3),
        "unit": "tokens/s",
        "n_gpus": ws,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": dtype_name(dtype),
        "data": "synthetic",
        "config": bench_config(wl, Ms, ws, l2_text),
        "launch": "CUDA graph replay per M" if run.graphs else "eager",
        "roofline": {"bound": "hbm",
                     "kernel": "gate_up (the thin-batch tensor-core GEMV up to 8 tokens, the tcgen05 grouped GEMM above)", "achieved": achieved, "peak": hbm_gbs,
                     "unit": "GB/s", "frac": (achieved / hbm_gbs) if achieved else None, "traffic": traffic,
                     "peak_source": f"{peak_src} HBM copy bandwidth",
                     "alg_bytes_per_launch": gate_bytes / max(g_n, 1),
                     "avg_launch_ms": g_ms / max(g_n, 1)},
        "layer_roofline": {
            "note": "whole-forward fractions per M (slower of algorithmic bytes at HBM bandwidth and FLOPs at "
                    "tensor peak); the decode target is >= 0.70 of the HBM roofline",
            "frac_measured_peaks": {M: round(per_M[M]["roofline_frac"], 4) for M in per_M},
            "frac_nominal_8TBps": {M: round(per_M[M]["roofline_frac_nominal"], 4) for M in per_M},
            "worst_frac_measured": min(per_M[M]["roofline_frac"] for M in per_M),
            "meets_decode_target": {M: per_M[M]["roofline_frac"] >= DECODE_TARGET for M in per_M}},
        "kernel_share": {k: round(v[0] / total_prof, 4) for k, v in prof.items() if v[1] > 0} if total_prof else {},
        "kernel_us_per_step": {k: round(v[0] * 1e3 / prof_steps, 2) for k, v in prof.items() if v[1] > 0},
        "per_M": per_M,
        "workloads": workloads,
        "e2e": e2e,
        "gpu_launches": sum(run.launches[M] for M in Ms) * args.steps,
        "cpu_baseline": cpu,
        "clocks": clk,
        "wall_s_timed": wall,
    }
    if rank == 0:
        print(json.dumps(line))
    run.close()
    for lay in layers:
        lay.close()
    if ws > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
