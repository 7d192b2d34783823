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


# DRAM traffic of the step's only kernel, from one ncu capture of the current kernel
# (dram__bytes_read.sum + dram__bytes_write.sum of one launch); None where the step has
# several kernels or no capture of the current kernel exists.
NCU_TRAFFIC = {"decode_bgmv": 21_570_560}


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
def build_sets(name, device, rank, n_sets):
    from workloads import make_workload, WORKLOAD_NAMES
    idx = WORKLOAD_NAMES.index(name)
    return [make_workload(idx, device=device, seed=rank_seed(idx, rank, s)) for s in range(n_sets)]


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
        # lora_sgmv_apply_proj on long segments: one plan, the stacked shrinks, one expand each
        return 1 + shrink_proj_passes([c.pool.max_rank for c in wl.calls]) + len(wl.calls)
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
# our arm
# ----------------------------------------------------------------------------
def run_ours(args):
    import torch
    import adapter_gemv_sgmv_b200 as L
    from adapter_gemv_sgmv_b200 import accounting

    world, rank, local = dist_env()
    if world != args.gpus:
        if args.gpus > 1:
            raise SystemExit(f"--gpus {args.gpus} needs torchrun with {args.gpus} ranks (WORLD_SIZE={world})")
    dist = init_dist(world, local, "nccl")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    L.load()

    n_sets = args.sets
    sets = build_sets(args.workload, dev, rank, n_sets)
    stream = torch.cuda.Stream(device=dev)
    ws_map = {}
    for wl in sets:
        for c in wl.calls:
            ws_map[id(c)] = workspace_for(c)
    steps = [make_step(wl, ws_map, stream) for wl in sets]
    torch.cuda.synchronize()

    cost = accounting.workload_cost(sets[0])
    tokens_per_step = sets[0].n_tokens
    set_bytes = 0
    for wl in sets:
        seen_x = set()
        for c in wl.calls:
            if _is_linear(c):
                io = (c.X.numel() + c.W.numel() + c.Y.numel()) * 2
            elif hasattr(c, "W"):
                io = c.W.numel() * 2
            else:
                io = c.Y.numel() * 2 + (0 if c.X.data_ptr() in seen_x else c.X.numel() * 2)
                seen_x.add(c.X.data_ptr())
            set_bytes += c.pool.A.numel() * 2 + c.pool.B.numel() * 2 + io
    launches_step = launches_per_step(sets[0])

    # eager warm-up (also sets per-device function attributes before capture)
    with torch.cuda.stream(stream):
        for i in range(max(args.warmup, 3)):
            steps[i % n_sets]()
    stream.synchronize()
    for ws in ws_map.values():
        err = L.lora_get_error(ws, stream=stream)
        if err:
            raise SystemExit(f"device error {err} during warm-up")

    # one graph = one pass over every input set
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=stream):
        for s in steps:
            s()
    reps = max(1, (args.steps + n_sets - 1) // n_sets)
    K = reps * n_sets
    # CUDAGraph.replay() launches on the current stream: make it the timed stream
    with torch.cuda.stream(stream):
        for _ in range(2):
            g.replay()
    torch.cuda.synchronize()

    clocks = ClockSampler(local).start()
    time.sleep(0.25)
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    t_wall0 = time.time()
    with torch.cuda.stream(stream):
        e0.record(stream)
        for _ in range(reps):
            g.replay()
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall1 = time.time()
    if dist is not None:
        dist.barrier()
    clocks.stop()
    ms_local = e0.elapsed_time(e1)
    ms_per_step, job_tokens_s = job_time_and_throughput(ms_local, K, tokens_per_step, world, dist, dev)

    # end to end through the public call, host buffers, copies inside the timed region
    e2e = run_e2e(args, sets, ws_map, stream, dist, dev, world)

    peaks, peak_src = load_peaks()
    t_step = ms_per_step * 1e-3
    gbs = cost.bytes / t_step / 1e9
    tflops = cost.flops / t_step / 1e12
    clk = clocks.summary(t_wall0, t_wall1)
    if any(_is_linear(c) for c in sets[0].calls):
        # a dense projection: tensor-bound.  Peak: the burst cuBLAS figure while the SM clock
        # stayed near its maximum over the timed region, the sustained (power-capped) one
        # once it fell below 85 % of it
        capped = (clk.get("sm_mhz") or 0) < 0.85 * (clk.get("sm_max_mhz") or 1)
        key = "bf16_tflops_sustained" if capped else "bf16_tflops"
        pk = peaks.get(key, peaks["bf16_tflops"])
        roof = {"bound": "tensor", "achieved": round(tflops, 1), "peak": pk, "unit": "TFLOP/s",
                "frac": round(tflops / pk, 4), "traffic": NCU_TRAFFIC.get(args.workload),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json {key})" if peak_src == "measured" else "fallback",
                "scope": "whole step, algorithmic FLOPs per step / step time",
                "algorithmic_flops_per_step": cost.flops, "algorithmic_bytes_per_step": cost.bytes}
    else:
        roof = {"bound": "hbm", "achieved": round(gbs, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": round(gbs / peaks["hbm_gbs"], 4), "traffic": NCU_TRAFFIC.get(args.workload),
                "peak_source": f"{peak_src} (MEASURED_PEAKS.json hbm_gbs)" if peak_src == "measured" else "fallback",
                "scope": "whole step, algorithmic bytes per step / step time",
                "algorithmic_bytes_per_step": cost.bytes}
    out = {
        "metric": METRIC, "value": round(job_tokens_s, 1), "unit": unit_of(args.workload),
        "n_gpus": world, "steps": K, "warmup": max(args.warmup, 3), "ms_per_step": round(ms_per_step, 6),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded; random-init adapters of the stated shapes)",
        "config": {"workload": WORKLOAD_DESC[args.workload], "tokens_per_step_per_gpu": tokens_per_step,
                   "parallelism": f"dp{world} (independent batches per GPU, no collective)",
                   "l2": f"rotating {n_sets} independent input sets ({set_bytes / 1e6:.0f} MB > 126 MB L2)",
                   "timing": "CUDA-graph replays of all input sets, CUDA events on the launching stream"},
        "hbm_gbs": round(gbs, 1), "tflops": round(tflops, 3),
        "roofline": roof,
        "gpu_launches": K * launches_step,
        "clocks": clk,
        "e2e": e2e,
    }
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        out["cpu_baseline"] = cpu_baseline(args, sets[0], budget_s=args.cpu_seconds)
    if rank == 0:
        print(json.dumps(out), flush=True)
    del g
    if dist is not None:
        dist.barrier()
        dist.destroy_process_group()


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
    return {"value": round(tokens / dt, 2), "unit": unit_of(args.workload), "cores": oracle.threads(),
            "kind": "oracle",
            "sample": f"{tokens} tokens ({n_tok} sampled rows x {passes} passes) of one "
                      f"{args.workload} batch, all projections, fp64 C loops, OpenMP over rows",
            "seconds": round(dt, 2)}


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
        "config": {"workload": WORKLOAD_DESC[args.workload], "tokens_per_step": n_tok},
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
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args(argv)
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
