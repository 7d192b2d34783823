#!/usr/bin/env python
"""Throughput of the multi-LoRA delta on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload decode_bgmv|prefill_sgmv|mixed_rank_layer|diffusion_multi|tiny_sgmv]

One step = one pass of the whole path (grouping, shrink, expand; the stacked
sum for multi-adapter requests) over one batch of the workload, through the
library's C ABI.  Inputs are resident in HBM when the timed region starts;
steps rotate over independent input sets (adapter pools, activations, ids)
whose total exceeds the 126 MB L2, so no step finds its adapters in L2.  The
K timed steps run as CUDA-graph replays on one stream, bracketed by a barrier
and a device synchronise, and are timed with CUDA events on that stream; with
N > 1 every rank runs its own batches (weak scaling, no collective on the
data path) and the reported time is the max over ranks.

`e2e` repeats the measurement through the public Python call a user makes,
with the step's inputs copied from pinned host memory and its result read
back inside the timed region.  `cpu_baseline` and `--impl reference` time the
CPU oracle (test infrastructure, fp64) on a bounded sample of the same
workload on the host cores.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import threading
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "LoRA-delta tokens/s; HBM GB/s (decode) and TFLOP/s (prefill) vs B200 peak"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}

WORKLOAD_DESC = {
    "tiny_sgmv": "tiny SGMV: 64 tokens, d_in=d_out=256, rank 8, 4 adapters, 4 contiguous segments",
    "decode_bgmv": "decode BGMV: 256 requests x 1 token, d_in=d_out=4096 (Llama-3-8B q_proj), rank 16, "
                   "128 resident adapters, Zipf(1.1) ids unsorted, scale 2.0",
    "prefill_sgmv": "prefill SGMV: 32 prompts, lengths U[128,1024], MLP up-proj 4096->14336, rank 64, "
                    "64 adapters, Zipf(1.1) per request, tokens sorted into per-adapter segments",
    "mixed_rank_layer": "mixed-rank decode over one Llama-3-8B layer: 512 tokens, 1000 resident adapters, "
                        "ranks U{8,16,32,64,128}, Zipf(1.0) ids, q/k/v/o/gate/up/down",
    "diffusion_multi": "diffusion multi-adapter: 16 images x 4096 tokens, 1280->1280 x Q,K,V,O, rank 32, "
                       "200 adapters, 1-3 co-occurring adapters per image, scales U[0.5,1]",
    "merge_mlp_up": "merge: fold one rank-64 adapter of a 64-adapter pool into the Llama-3-8B MLP up-proj "
                    "weight W [14336, 4096] in place (W += s B A)",
    "prefill_qkv": "prefill SGMV over shared-input projections: 32 prompts, lengths U[128,1024], Llama-3-8B "
                   "q/k/v 4096->4096/1024/1024, rank 64, 64 adapters, Zipf(1.1) per request; one shrink "
                   "reads X once for all three, then one expand per projection",
    "prefill_linear_up": "prefill projection with its LoRA fused: 32 prompts, lengths U[128,1024], Llama-3-8B MLP "
                         "up-proj y = x W^T + s x A^T B^T, W [14336, 4096], rank 64, 64 adapters, Zipf(1.1) per "
                         "request; the delta as extra k-blocks of the tcgen05 projection",
}


def unit_of(workload: str) -> str:
    """The merge streams weight rows; every other workload, token rows."""
    return "weight rows/s" if workload == "merge_mlp_up" else "tokens/s"


# ----------------------------------------------------------------------------
# process / rank plumbing
# ----------------------------------------------------------------------------
def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", str(rank)))
    return ws, rank, local


def init_dist(world, local, backend):
    import torch
    import torch.distributed as dist
    if world <= 1:
        return None
    if backend == "nccl":
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", device_id=torch.device("cuda", local),
                                timeout=__import__("datetime").timedelta(seconds=120))
    else:
        dist.init_process_group("gloo", timeout=__import__("datetime").timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, dist, device=None) -> float:
    """Max of a per-rank float over all ranks (device tensor for NCCL, CPU for gloo)."""
    if dist is None:
        return float(x)
    import torch
    t = torch.tensor([float(x)], dtype=torch.float64, device=device or "cpu")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def rank_seed(workload_index: int, rank: int, set_index: int) -> int:
    """Independent batch per (rank, input set): weak scaling without overlap."""
    return workload_index + 1000 * rank + 100000 * set_index


def job_time_and_throughput(ms_local: float, steps: int, tokens_per_step_per_rank: int, world: int,
                            dist, device=None):
    """Whole-job numbers of a weak-scaling run: the step time is the slowest rank's
    (max over ranks of its device-timed total / steps); the throughput counts the
    tokens every rank processed in that time."""
    ms = max_over_ranks(ms_local, dist, device)
    ms_per_step = ms / steps
    return ms_per_step, world * tokens_per_step_per_rank / (ms_per_step * 1e-3)


# ----------------------------------------------------------------------------
# clocks
# ----------------------------------------------------------------------------
class ClockSampler:
    """nvidia-smi sampled every `ms` while running; summary() -> the JSON 'clocks' object."""

    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, ms: int = 50):
        self.gpu = gpu_index
        self.ms = ms
        self.rows = []
        self.proc = None
        self.thread = None
        self.marks = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.Q}", "--format=csv,noheader,nounits",
                 f"-lms", str(self.ms)], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, ValueError):
            self.proc = None
            return self
        self.thread = threading.Thread(target=self._read, daemon=True)
        self.thread.start()
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.rows.append((time.time(), line.strip()))

    def mark(self, name):
        self.marks.append((name, time.time()))

    def stop(self):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        if self.thread is not None:
            self.thread.join(timeout=5)

    def summary(self, t0, t1):
        def parse(rows):
            out = []
            for _, line in rows:
                f = [x.strip() for x in line.split(",")]
                if len(f) < 9:
                    continue
                try:
                    out.append({"sm": float(f[1]), "max": float(f[2]), "power": float(f[3]),
                                "hw": f[5], "hwt": f[6], "swt": f[7], "cap": f[8]})
                except ValueError:
                    continue
            return out
        inside = parse([r for r in self.rows if t0 <= r[0] <= t1])
        window = "timed"
        if len(inside) < 3:
            inside = parse(self.rows)
            window = "warmup+timed (timed region shorter than the sampling interval)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        reasons = set()
        for s in inside:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("cap", "sw_power_cap")):
                if s[key].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(s["sm"] for s in inside),
                "sm_max_mhz": max(s["max"] for s in inside), "reasons": sorted(reasons),
                "samples": len(inside), "window": window,
                "power_w_max": max(s["power"] for s in inside)}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return FALLBACK_PEAKS, "fallback"


# ----------------------------------------------------------------------------
# workload steps
# ----------------------------------------------------------------------------
# workload overrides for profiling one part of a workload (set by --only-proj)
OVERRIDES = {}


def build_sets(name, device, rank, n_sets):
    return build_sets_from(name, device, rank, 0, n_sets)


def _is_linear(call) -> bool:
    """The fused projection call (a base weight and token rows); a merge has W but no X."""
    return hasattr(call, "W") and hasattr(call, "X")


def launches_per_call(call) -> int:
    """Kernels one step of this call launches, as the library reports them."""
    import adapter_gemv_sgmv_b200 as L
    p = call.pool
    if _is_linear(call):
        return L.lora_kernel_launches(L.OP_LINEAR, call.n_tokens, p.n_adapters, p.d_in, len(call.seg_ad_h))
    if hasattr(call, "W"):
        return L.lora_kernel_launches(L.OP_MERGE, p.d_out, p.n_adapters, p.d_in)
    if hasattr(call, "ids_h"):
        return L.lora_kernel_launches(L.OP_BGMV, call.n_tokens, p.n_adapters, p.d_in)
    if hasattr(call, "seg_off_h"):
        n = len(call.seg_ad_h)
        return (L.lora_kernel_launches(L.OP_SGMV_SHRINK, call.n_tokens, p.n_adapters, p.d_in, n) +
                L.lora_kernel_launches(L.OP_SGMV_EXPAND, call.n_tokens, p.n_adapters, p.d_in, n))
    return L.lora_kernel_launches(L.OP_APPLY_MULTI, call.n_tokens, p.n_adapters, p.d_in,
                                  len(call.req_off_h) - 1)


def shrink_proj_passes(max_ranks, limit=256) -> int:
    """Tensor-core launches of lora_sgmv_shrink_proj: runs of consecutive projections
    whose max ranks sum to at most 256 (the header's rule)."""
    n, k = 0, limit + 1
    for r in max_ranks:
        if k + r > limit:
            n, k = n + 1, 0
        k += r
    return n


def launches_per_step(wl) -> int:
    import adapter_gemv_sgmv_b200 as L
    if wl.desc.get("op") == "sgmv_proj":
        # lora_sgmv_apply_proj on long segments: one plan, the stacked shrinks, one expand
        # launch for all the projections
        return 1 + shrink_proj_passes([c.pool.max_rank for c in wl.calls]) + 1
    return sum(launches_per_call(c) for c in wl.calls)


def make_step(wl, ws_map, stream):
    """Closure running one full pass of the path over workload `wl` on `stream`."""
    import torch
    import adapter_gemv_sgmv_b200 as L
    fns = []
    if wl.desc.get("op") == "sgmv_proj":
        # projections sharing X: one call -- one plan, one stacked shrink over all of them
        # (x read once), then each projection's expand; V stays in the workspace
        c0 = wl.calls[0]
        pools = [c.pool for c in wl.calls]
        need = L.lora_workspace_size(L.OP_APPLY_PROJ, c0.n_tokens, c0.pool.n_adapters, c0.pool.d_in, 0,
                                     sum(p.max_rank for p in pools), len(c0.seg_ad_h))
        ws = ws_map.setdefault(("apply_proj", id(wl)), L.Workspace(need, device=c0.X.device))
        Ys = [c.Y for c in wl.calls]
        scales = [c.scale for c in wl.calls]

        def proj_step():
            L.lora_sgmv_apply_proj(c0.X, Ys, pools, c0.seg_off, c0.seg_ad, scales, ws=ws, stream=stream)
        return proj_step
    for c in wl.calls:
        ws = ws_map[id(c)]
        if _is_linear(c):
            fns.append(lambda c=c, ws=ws: L.lora_linear_sgmv(c.X, c.W, c.Y, c.pool, c.seg_off, c.seg_ad, c.scale,
                                                             ws=ws, stream=stream))
        elif hasattr(c, "W"):
            # one merge of the adapter into the weight (W drifts by s B A per step; timing only)
            fns.append(lambda c=c, ws=ws: L.lora_merge(c.W, c.pool, c.adapter, c.scale, ws=ws, stream=stream))
        elif hasattr(c, "ids_h"):
            fns.append(lambda c=c, ws=ws: L.lora_bgmv(c.X, c.Y, c.pool, c.ids, c.scale, ws=ws, stream=stream))
        elif hasattr(c, "seg_off_h"):
            V = torch.empty(c.X.shape[0], c.pool.max_rank, dtype=torch.float32, device=c.X.device)
            c._V = V

            def f(c=c, ws=ws, V=V):
                L.lora_sgmv_shrink(c.X, V, c.pool, c.seg_off, c.seg_ad, ws=ws, stream=stream)
                L.lora_sgmv_expand(V, c.Y, c.pool, c.seg_off, c.seg_ad, c.scale, ws=ws, stream=stream)
            fns.append(f)
        else:
            fns.append(lambda c=c, ws=ws: L.lora_apply_multi(c.X, c.Y, c.pool, c.req_off, c.ad_off, c.ad_id,
                                                             c.ad_scale, max_ads_per_req=3, ws=ws,
                                                             stream=stream))

    def step():
        for f in fns:
            f()
    return step


def workspace_for(call):
    import adapter_gemv_sgmv_b200 as L
    p = call.pool
    if _is_linear(call):
        n = L.lora_workspace_size(L.OP_LINEAR, call.n_tokens, p.n_adapters, p.d_in, p.d_out, p.max_rank,
                                  len(call.seg_ad_h))
    elif hasattr(call, "W"):
        n = L.lora_workspace_size(L.OP_MERGE, p.d_out, p.n_adapters, p.d_in, p.d_out, p.max_rank)
    elif hasattr(call, "ids_h"):
        n = L.lora_workspace_size(L.OP_BGMV, call.n_tokens, p.n_adapters, p.d_in, p.d_out, p.max_rank)
    elif hasattr(call, "seg_off_h"):
        n = max(L.lora_workspace_size(op, call.n_tokens, p.n_adapters, p.d_in, p.d_out, p.max_rank,
                                      len(call.seg_ad_h)) for op in (L.OP_SGMV_SHRINK, L.OP_SGMV_EXPAND))
    else:
        n = L.lora_workspace_size(L.OP_APPLY_MULTI, call.n_tokens, p.n_adapters, p.d_in, p.d_out, p.max_rank,
                                  len(call.req_off_h) - 1, 3)
    return L.Workspace(n, device=(call.X if hasattr(call, "X") else call.W).device)


# ----------------------------------------------------------------------------
# traffic of a step's dominant kernel, from a committed ncu summary
# ----------------------------------------------------------------------------
def profile_traffic(workload: str):
    """DRAM bytes (read + write) per launch of the workload's dominant kernel, from
    the committed ncu summary that records it -- only while the kernel's source
    file is byte-identical to the one profiled (its sha256 is in the summary's
    record line), else None."""
    import glob
    import hashlib
    import re
    pat = re.compile(r"^traffic-record: workload=(\S+) kernel=(\S+) bytes_per_launch=(\d+) "
                     r"source=(\S+) sha256=([0-9a-f]{16})\s*$")
    for f in sorted(glob.glob(os.path.join(ROOT, "profiles", "*.md"))):
        for line in open(f):
            m = pat.match(line.strip())
            if not m or m.group(1) != workload:
                continue
            src = os.path.join(ROOT, m.group(4))
            if not os.path.exists(src):
                return None
            h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
            if h != m.group(5):
                return None
            return {"bytes": int(m.group(3)), "kernel": m.group(2), "profile": os.path.relpath(f, ROOT)}
    return None


def config_of(workload: str, tokens: int, world: int) -> dict:
    """The line's `config`: the workload itself, the same in both arms."""
    desc = WORKLOAD_DESC[workload]
    if workload in OVERRIDES:
        desc += f" -- restricted for profiling: {OVERRIDES[workload]}"
    return {"workload": desc, "tokens_per_step_per_gpu": int(tokens),
            "parallelism": f"dp{world} (independent batches per GPU, no collective)"}


# ----------------------------------------------------------------------------
# our arm
# ----------------------------------------------------------------------------
L2_BYTES = 126 * 2 ** 20


class Bench:
    """One workload's input sets on the device, one CUDA graph per set (a step =
    one graph replay), and the accounting of a step."""

    def __init__(self, name, dev, rank, stream, max_sets=16, min_set_total=4 * L2_BYTES):
        import torch
        from adapter_gemv_sgmv_b200 import accounting
        self.name = name
        self.stream = stream
        self.sets = build_sets(name, dev, rank, 1)
        self.set_bytes = self._bytes(self.sets[0])
        # enough independent sets that a step never finds the previous steps' inputs in L2
        n_sets = int(min(max_sets, max(2, -(-min_set_total // max(self.set_bytes, 1)))))
        if n_sets > 1:
            self.sets += build_sets_from(name, dev, rank, 1, n_sets)
        self.ws_map = {}
        for wl in self.sets:
            for c in wl.calls:
                self.ws_map[id(c)] = workspace_for(c)
        self.steps = [make_step(wl, self.ws_map, stream) for wl in self.sets]
        self.cost = accounting.workload_cost(self.sets[0])
        self.tokens = self.sets[0].n_tokens
        self.launches = launches_per_step(self.sets[0])
        self.graphs = []
        torch.cuda.synchronize()

    @staticmethod
    def _bytes(wl):
        n, seen_x = 0, set()
        for c in wl.calls:
            if _is_linear(c):
                io = (c.X.numel() + c.W.numel() + c.Y.numel()) * 2
            elif hasattr(c, "W"):
                io = c.W.numel() * 2
            else:
                io = c.Y.numel() * 2 + (0 if c.X.data_ptr() in seen_x else c.X.numel() * 2)
                seen_x.add(c.X.data_ptr())
            n += c.pool.A.numel() * 2 + c.pool.B.numel() * 2 + io
        return n

    def warm(self, warmup):
        import torch
        import adapter_gemv_sgmv_b200 as L
        # eager warm-up (also sets per-device function attributes before capture)
        with torch.cuda.stream(self.stream):
            for i in range(max(warmup, 3)):
                self.steps[i % len(self.steps)]()
        self.stream.synchronize()
        for ws in self.ws_map.values():
            err = L.lora_get_error(ws, stream=self.stream)
            if err:
                raise SystemExit(f"{self.name}: device error {err} during warm-up")

    def capture(self, steps):
        """One CUDA graph of `steps` consecutive steps rotating over the input sets
        (consecutive kernels overlap their prologues as they would in a model's
        graph), replayed once untimed."""
        import torch
        self.graphs.clear()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=self.stream):
            for i in range(steps):
                self.steps[i % len(self.steps)]()
        self.graphs.append(g)
        self.graph_steps = steps
        with torch.cuda.stream(self.stream):
            g.replay()
        torch.cuda.synchronize()

    def timed(self, replays=1):
        """Device time (ms) of `replays` replays of the captured graph (each
        `graph_steps` steps), CUDA events on the launching stream."""
        import torch
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        with torch.cuda.stream(self.stream):
            e0.record(self.stream)
            for _ in range(replays):
                self.graphs[0].replay()
            e1.record(self.stream)
        torch.cuda.synchronize()
        return e0.elapsed_time(e1)

    def check_errors(self):
        import adapter_gemv_sgmv_b200 as L
        for ws in self.ws_map.values():
            err = L.lora_get_error(ws, stream=self.stream)
            if err:
                raise SystemExit(f"{self.name}: device error {err} in the timed steps")

    def release(self):
        import torch
        self.graphs.clear()
        self.steps.clear()
        self.ws_map.clear()
        self.sets.clear()
        torch.cuda.synchronize()
        torch.cuda.empty_cache()


def build_sets_from(name, device, rank, start, stop):
    from workloads import make_workload, WORKLOAD_NAMES
    idx = WORKLOAD_NAMES.index(name)
    ov = OVERRIDES.get(name, {})
    return [make_workload(idx, device=device, seed=rank_seed(idx, rank, s), **ov) for s in range(start, stop)]


def roofline_of(name, cost, ms_per_step, clk, peaks, peak_src):
    """Algorithmic bytes (FLOPs for the fused projection) per step over the measured
    step time, against the measured peak."""
    t = ms_per_step * 1e-3
    gbs = cost.bytes / t / 1e9
    tflops = cost.flops / t / 1e12
    tr = profile_traffic(name)
    traffic = None
    if tr is not None:
        traffic = tr["bytes"]
    if name == "prefill_linear_up":
        # a dense projection: tensor-bound.  The burst cuBLAS peak while the SM clock
        # stayed near its maximum, the sustained (power-capped) one once it fell below 85 %
        capped = (clk.get("sm_mhz") or 0) < 0.85 * (clk.get("sm_max_mhz") or 1)
        key = "bf16_tflops_sustained" if capped else "bf16_tflops"
        pk = peaks.get(key, peaks["bf16_tflops"])
        return {"bound": "tensor", "achieved": round(tflops, 1), "peak": pk, "unit": "TFLOP/s",
                "frac": round(tflops / pk, 4), "traffic": traffic,
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json {key})" if peak_src == "measured" else "fallback",
                "algorithmic_flops_per_step": cost.flops, "algorithmic_bytes_per_step": cost.bytes}
    return {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
            "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": traffic,
            "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback",
            "algorithmic_bytes_per_step": cost.bytes}


ALL_WORKLOADS = ["tiny_sgmv", "decode_bgmv", "prefill_sgmv", "mixed_rank_layer", "diffusion_multi",
                 "prefill_qkv", "merge_mlp_up", "prefill_linear_up"]


def run_ours(args):
    import torch
    import adapter_gemv_sgmv_b200 as L

    world, rank, local = dist_env()
    if world != args.gpus:
        if args.gpus > 1:
            raise SystemExit(f"--gpus {args.gpus} needs torchrun with {args.gpus} ranks (WORLD_SIZE={world})")
    dist = init_dist(world, local, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L.load()
    stream = torch.cuda.Stream(device=dev)
    peaks, peak_src = load_peaks()

    bench = Bench(args.workload, dev, rank, stream, max_sets=args.sets)
    bench.warm(args.warmup)
    K = args.steps
    bench.capture(K)
    clocks = ClockSampler(local).start()
    time.sleep(0.25)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t_wall0 = time.time()
    ms_local = bench.timed(1)
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    clocks.stop()
    bench.check_errors()
    ms_per_step, job_tokens_s = job_time_and_throughput(ms_local, K, bench.tokens, world, dist, dev)
    clk = clocks.summary(t_wall0, t_wall1)

    # end to end through the public call, host buffers, copies inside the timed region
    e2e = run_e2e(args, bench.sets, bench.ws_map, stream, dist, dev, world)

    roof = roofline_of(args.workload, bench.cost, ms_per_step, clk, peaks, peak_src)
    roof["scope"] = "whole step (one pass of the path), algorithmic bytes per step / step time"
    t_step = ms_per_step * 1e-3
    out = {
        "metric": METRIC, "value": round(job_tokens_s, 1), "unit": unit_of(args.workload),
        "n_gpus": world, "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init adapters of the stated shapes)",
        "config": config_of(args.workload, bench.tokens, world),
        "timing": {"l2": f"inputs larger than L2: {len(bench.sets)} independent input sets rotated "
                         f"({len(bench.sets) * bench.set_bytes / 1e6:.0f} MB in total > 126 MB L2)",
                   "method": "one CUDA graph holding the K steps (input sets rotated), replayed once; "
                             "CUDA events on the launching stream, max over ranks"},
        "hbm_gbs": round(bench.cost.bytes / t_step / 1e9, 1), "tflops": round(bench.cost.flops / t_step / 1e12, 3),
        "roofline": roof,
        "gpu_launches": K * bench.launches,
        "clocks": clk,
        "e2e": e2e,
    }
    bench.release()
    del bench
    if args.workloads != "none":
        names = ALL_WORKLOADS if args.workloads == "all" else args.workloads.split(",")
        out["workloads"] = {n: time_one_workload(n, dev, rank, stream, args, peaks, peak_src, dist, world)
                            for n in names}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import gc
        gc.collect()
        wl0 = build_sets(args.workload, dev, rank, 1)[0]
        out["cpu_baseline"] = cpu_baseline(args, wl0, budget_s=args.cpu_seconds)
        del wl0
    if rank == 0:
        print(json.dumps(out), flush=True)
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


def time_one_workload(name, dev, rank, stream, args, peaks, peak_src, dist, world):
    """One workload of the table, timed in this run: its own input sets, warm-up,
    enough graph replays for a timed region of about 0.2 s (at least --steps),
    clocks sampled over that region."""
    import torch
    b = Bench(name, dev, rank, stream, max_sets=args.sets)
    b.warm(args.warmup)
    b.capture(len(b.sets))
    est = b.timed(1) / b.graph_steps
    # a graph of up to 2000 steps, replayed for a timed region of about 0.2 s
    per_graph = int(max(len(b.sets), min(2000, args.steps)))
    replays = int(max(1, min(200, 200.0 / max(est * per_graph, 1e-4))))
    b.capture(per_graph)
    steps = per_graph * replays
    clocks = ClockSampler(dev.index if dev.index is not None else 0).start()
    time.sleep(0.25)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    t0 = time.time()
    ms = b.timed(replays)
    t1 = time.time()
    if dist is not None:
        dist.barrier()
    clocks.stop()
    b.check_errors()
    ms_per_step, tok_s = job_time_and_throughput(ms, steps, b.tokens, world, dist, dev)
    clk = clocks.summary(t0, t1)
    roof = roofline_of(name, b.cost, ms_per_step, clk, peaks, peak_src)
    res = {"desc": WORKLOAD_DESC[name], "ms_per_step": round(ms_per_step, 6),
           "value": round(tok_s, 1), "unit": unit_of(name), "steps": steps,
           "tokens_per_step_per_gpu": b.tokens,
           "algorithmic_bytes_per_step": b.cost.bytes, "algorithmic_flops_per_step": b.cost.flops,
           "hbm_gbs": round(b.cost.bytes / (ms_per_step * 1e-3) / 1e9, 1),
           "tflops": round(b.cost.flops / (ms_per_step * 1e-3) / 1e12, 3),
           "roofline": roof, "gpu_launches_per_step": b.launches, "clocks": clk,
           "input_sets": len(b.sets), "input_bytes": len(b.sets) * b.set_bytes}
    b.release()
    del b
    return res


def run_e2e(args, sets, ws_map, stream, dist, dev, world):
    """Per step: pinned host -> device copy of the step's inputs, the public call, device ->
    host copy of the result; timed with CUDA events, max over ranks.  Steps are pipelined
    the way a serving loop would run them: copies in on one stream, the call on the compute
    stream, copies out on a third, rotating over up to three input sets (their own device
    buffers and pinned host buffers), so step k+1's inputs travel while step k computes and
    step k-1's result comes back.  Every step still moves all of its bytes."""
    import torch
    m = max(1, min(3, len(sets)))
    rings = []
    h2d = d2h = 0
    for si in range(m):
        wl = sets[si]
        hosts = []
        for c in wl.calls:
            # the step's inputs: x (and y, which the delta updates in place); a merge's weight;
            # the fused projection reads x and overwrites y, its weight staying resident like the pools
            ins = {"X": c.X} if _is_linear(c) else ({"W": c.W} if hasattr(c, "W") else {"X": c.X, "Y": c.Y})
            for k in ("ids", "seg_off", "seg_ad", "req_off", "ad_off", "ad_id", "ad_scale"):
                if hasattr(c, k):
                    ins[k] = getattr(c, k)
            pin = {k: torch.empty(v.shape, dtype=v.dtype, device="cpu", pin_memory=True) for k, v in ins.items()}
            for k, v in ins.items():
                pin[k].copy_(v)
            res = c.Y if hasattr(c, "Y") else c.W
            out_pin = torch.empty(res.shape, dtype=res.dtype, device="cpu", pin_memory=True)
            hosts.append((c, pin, out_pin))
        if si == 0:
            shared_x = set()
            for c, pin, out_pin in hosts:
                for k, v in pin.items():
                    if k == "X":
                        if c.X.data_ptr() in shared_x:
                            continue
                        shared_x.add(c.X.data_ptr())
                    h2d += v.numel() * v.element_size()
                d2h += out_pin.numel() * out_pin.element_size()
        ev = {name: torch.cuda.Event() for name in ("in", "cmp", "out")}
        rings.append((hosts, make_step(wl, ws_map, stream), ev))
    s_in = torch.cuda.Stream(device=dev)
    s_out = torch.cuda.Stream(device=dev)
    n = max(3, min(args.e2e_steps, args.steps))
    used = [False] * m

    def one(i):
        hosts, step, ev = rings[i % m]
        if used[i % m]:
            s_in.wait_event(ev["out"])          # this set's previous result has left the device
        used[i % m] = True
        with torch.cuda.stream(s_in):
            copied = set()
            for c, pin, out_pin in hosts:
                for k, v in pin.items():
                    dst = getattr(c, k)
                    if dst.data_ptr() in copied:
                        continue
                    copied.add(dst.data_ptr())
                    dst.copy_(v, non_blocking=True)
            ev["in"].record(s_in)
        stream.wait_event(ev["in"])
        with torch.cuda.stream(stream):
            step()
            ev["cmp"].record(stream)
        s_out.wait_event(ev["cmp"])
        with torch.cuda.stream(s_out):
            for c, pin, out_pin in hosts:
                out_pin.copy_(c.Y if hasattr(c, "Y") else c.W, non_blocking=True)
            ev["out"].record(s_out)
    for i in range(3):
        one(i)
    torch.cuda.synchronize()
    if dist is not None:
        dist.barrier()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(n):
        one(i)
    e1.record(s_out)                            # after the last result's copy, which follows everything
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1), dist, dev) / n
    return {"value": round(world * sets[0].n_tokens / (ms * 1e-3), 1), "unit": unit_of(args.workload),
            "h2d_bytes_per_step": int(h2d), "d2h_bytes_per_step": int(d2h), "steps": n,
            "ms_per_step": round(ms, 6),
            "path": f"pinned host -> device copies on a copy stream, the public Python call (eager launches) "
                    f"on the compute stream, device -> host on a third stream; steps pipelined over {m} "
                    f"input set(s)"}


# ----------------------------------------------------------------------------
# the CPU oracle (test infrastructure), timed on the host cores
# ----------------------------------------------------------------------------
def _host_calls(wl):
    """Host copies of a workload's calls for the oracle (pools compacted to used adapters)."""
    from oracle import host_pool_subset as compact_from_device_pool
    from workloads import to_host
    out = []
    for c in wl.calls:
        if _is_linear(c):
            lens = np.diff(c.seg_off_h)
            hp, remap = compact_from_device_pool(c.pool, c.seg_ad_h[(lens > 0) & (c.seg_ad_h >= 0)])
            sa = np.where((lens > 0) & (c.seg_ad_h >= 0), remap[np.maximum(c.seg_ad_h, 0)], -1).astype(np.int32)
            out.append(("linear", to_host(c.X), hp, (to_host(c.W), c.seg_off_h, sa), c))
        elif hasattr(c, "W"):
            hp, remap = compact_from_device_pool(c.pool, [c.adapter])
            out.append(("merge", to_host(c.W), hp, int(remap[c.adapter]), c))
        elif hasattr(c, "ids_h"):
            used = np.unique(c.ids_h[c.ids_h >= 0])
            hp, remap = compact_from_device_pool(c.pool, used)
            ids = np.where(c.ids_h >= 0, remap[np.maximum(c.ids_h, 0)], -1).astype(np.int32)
            out.append(("bgmv", to_host(c.X), hp, ids, c))
        elif hasattr(c, "seg_off_h"):
            lens = np.diff(c.seg_off_h)
            hp, remap = compact_from_device_pool(c.pool, c.seg_ad_h[lens > 0])
            sa = np.where(lens > 0, remap[c.seg_ad_h], 0).astype(np.int32)
            out.append(("sgmv", to_host(c.X), hp, (c.seg_off_h, sa), c))
        else:
            hp, remap = compact_from_device_pool(c.pool, c.ad_id_h)
            out.append(("multi", to_host(c.X), hp, (c.req_off_h, c.ad_off_h, remap[c.ad_id_h].astype(np.int32),
                                                    c.ad_scale_h), c))
    return out


def _oracle_pass(oracle, hc, rows_per_call):
    """Run the oracle on the given rows of every call; returns tokens processed."""
    done = 0
    for (kind, X, hp, meta, c), rows in zip(hc, rows_per_call):
        if kind == "linear":
            oracle.linear_sgmv(X, meta[0], hp, meta[1], meta[2], c.scale, rows=rows)
        elif kind == "merge":
            oracle.merge(X, hp, meta, c.scale, rows=rows)
        elif kind == "bgmv":
            oracle.bgmv_delta(X, hp, meta, c.scale, rows=rows)
        elif kind == "sgmv":
            oracle.sgmv_delta(X, hp, meta[0], meta[1], c.scale, rows=rows)
        else:
            oracle.apply_multi_delta(X, hp, *meta, rows=rows)
    return len(rows_per_call[0])


def _rows_sample(hc, n, seed):
    rng = np.random.default_rng(seed)
    N = hc[0][1].shape[0]
    return [np.sort(rng.choice(N, size=min(n, N), replace=False)).astype(np.int32) for _ in hc]


def cpu_baseline(args, wl, budget_s=12.0):
    import oracle
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    hc = _host_calls(wl)
    # calibrate on a small row sample (after one untimed pass: the first call starts the
    # thread pool), size a pass to about a tenth of the budget, then run passes until the
    # budget is spent
    probe = _rows_sample(hc, min(16, wl.n_tokens), 0)
    _oracle_pass(oracle, hc, probe)
    t0 = time.perf_counter()
    _oracle_pass(oracle, hc, probe)
    t_probe = max(time.perf_counter() - t0, 1e-4)
    per_tok = t_probe / len(probe[0])
    n_tok = int(max(1, min(wl.n_tokens, 0.1 * budget_s / per_tok)))
    tokens = 0
    passes = 0
    t0 = time.perf_counter()
    while time.perf_counter() - t0 < budget_s and passes < 100000:
        tokens += _oracle_pass(oracle, hc, _rows_sample(hc, n_tok, passes + 1))
        passes += 1
    dt = time.perf_counter() - t0
    out = {"value": round(tokens / dt, 2), "unit": unit_of(args.workload), "cores": oracle.threads(),
           "kind": "oracle",
           "sample": f"{tokens} tokens ({n_tok} sampled rows x {passes} passes) of one "
                     f"{args.workload} batch, all projections, fp64 C loops, OpenMP over rows",
           "seconds": round(dt, 2)}
    # one host thread on the tiny and decode workloads (the whole batch per pass)
    one = {}
    oracle.set_threads(1)
    try:
        from workloads import make_workload, WORKLOAD_NAMES
        for name in ("tiny_sgmv", "decode_bgmv"):
            idx = WORKLOAD_NAMES.index(name)
            w = make_workload(idx, device=wl.calls[0].pool.A.device, seed=rank_seed(idx, 0, 0))
            h = _host_calls(w)
            rows = [np.arange(w.n_tokens, dtype=np.int32) for _ in h]
            _oracle_pass(oracle, h, rows)
            n, t0 = 0, time.perf_counter()
            while time.perf_counter() - t0 < args.one_thread_seconds:
                n += _oracle_pass(oracle, h, rows)
            one[name] = {"value": round(n / (time.perf_counter() - t0), 2), "unit": "tokens/s", "cores": 1,
                         "sample": f"whole {name} batch ({w.n_tokens} tokens) per pass"}
    finally:
        oracle.set_threads(os.cpu_count() or 1)
    out["one_thread"] = one
    return out


def run_reference(args):
    """The reference arm: the CPU oracle, on our arm's workload, metric and unit."""
    world, rank, local = dist_env()
    if rank != 0:
        return
    import torch
    import oracle
    from workloads import make_workload, WORKLOAD_NAMES
    idx = WORKLOAD_NAMES.index(args.workload)
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = make_workload(idx, device=dev, seed=rank_seed(idx, 0, 0))
    cores = os.cpu_count() or 1
    oracle.set_threads(cores)
    hc = _host_calls(wl)
    probe = _rows_sample(hc, min(8, wl.n_tokens), 0)
    _oracle_pass(oracle, hc, probe)             # untimed: the first call starts the thread pool
    t0 = time.perf_counter()
    _oracle_pass(oracle, hc, probe)
    per_tok = max(time.perf_counter() - t0, 1e-5) / len(probe[0])
    total_budget = args.reference_seconds
    n_tok = int(max(1, min(wl.n_tokens, total_budget / max(args.steps + args.warmup, 1) / per_tok)))
    for w in range(args.warmup):
        _oracle_pass(oracle, hc, _rows_sample(hc, n_tok, 10_000 + w))
    tokens = 0
    t0 = time.perf_counter()
    for k in range(args.steps):
        tokens += _oracle_pass(oracle, hc, _rows_sample(hc, n_tok, k))
    dt = time.perf_counter() - t0
    v = tokens / dt
    sample = (f"each step: {n_tok} sampled token rows of one {args.workload} batch (all projections), "
              f"fp64 C loops, OpenMP over rows")
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(v, 3), "unit": unit_of(args.workload),
        "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / max(args.steps, 1) * 1e3, 3),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (seeded)",
        "config": config_of(args.workload, wl.n_tokens, args.gpus),
        "sample": f"{n_tok} token rows per step",
        "cpu_baseline": {"value": round(v, 3), "unit": unit_of(args.workload), "cores": oracle.threads(),
                         "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(v, 3), "unit": unit_of(args.workload), "h2d_bytes_per_step": 0,
                "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20000)
    ap.add_argument("--warmup", type=int, default=50)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="decode_bgmv", choices=list(WORKLOAD_DESC))
    ap.add_argument("--sets", type=int, default=16, help="rotating independent input sets (> L2 in total)")
    ap.add_argument("--e2e-steps", type=int, default=200)
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--reference-seconds", type=float, default=60.0)
    ap.add_argument("--one-thread-seconds", type=float, default=3.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--workloads", default="all",
                    help="'all', 'none' or a comma list: workloads timed in the same run next to the headline")
    ap.add_argument("--only-proj", default=None,
                    help="mixed_rank_layer only: keep just these projections (comma list, e.g. 'gate'); "
                         "for profiling one kernel on a smaller device footprint")
    args = ap.parse_args(argv)
    if args.only_proj:
        from workloads.configs import LLAMA3_8B_PROJ
        keep = args.only_proj.split(",")
        OVERRIDES["mixed_rank_layer"] = {"projections": [p for p in LLAMA3_8B_PROJ if p[0] in keep]}
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
