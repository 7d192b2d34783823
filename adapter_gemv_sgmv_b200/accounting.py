"""Algorithmic FLOP and byte counts of the multi-LoRA delta.

The per-layer formulas are those of the cost model on "Serving several LoRAs,
ControlNet and IP-Adapter", section "LoRA: merged or alongside": one adapted
linear layer costs 2*N*(d*r + r*d) extra FLOPs unmerged, one adapter weighs
d*r*2 elements, and merging reads and writes the affected weight once.  They
are generalised to d_in != d_out and to per-token adapters:

  F     = 2 * sum_n sum_{(a, s) on n} r_a * (d_in + d_out)
  bytes = 2*N*d_in            (X read once)
        + 4*N*d_out           (Y read and written once; stacked adapters share the pass)
        + sum_{distinct a} 2*r_a*(d_in + d_out)   (each touched adapter read once)
        + metadata (int32 ids / offsets, int64 pool offsets, int32 ranks)

Only tokens that carry at least one adapter count in N.  A round trip of the
rank-r intermediate through global memory between two kernels is not
algorithmic and is not counted.
"""
from __future__ import annotations

import numpy as np

BF16_BYTES = 2


def lora_flops(n_tokens: int, rank: int, d_in: int, d_out: int) -> int:
    """Shrink (2*N*d_in*r) plus expand (2*N*r*d_out)."""
    return 2 * int(n_tokens) * int(rank) * (int(d_in) + int(d_out))


def adapter_elems(rank: int, d_in: int, d_out: int) -> int:
    return int(rank) * (int(d_in) + int(d_out))


def merge_bytes(weight_bytes: int) -> int:
    """Merging or unmerging reads and writes the affected weights once."""
    return 2 * int(weight_bytes)


class Cost:
    __slots__ = ("flops", "bytes", "tokens", "adapter_bytes", "act_bytes")

    def __init__(self, flops=0, nbytes=0, tokens=0, adapter_bytes=0, act_bytes=0):
        self.flops = int(flops)
        self.bytes = int(nbytes)
        self.tokens = int(tokens)
        self.adapter_bytes = int(adapter_bytes)
        self.act_bytes = int(act_bytes)

    def __add__(self, o: "Cost") -> "Cost":
        return Cost(self.flops + o.flops, self.bytes + o.bytes, self.tokens + o.tokens,
                    self.adapter_bytes + o.adapter_bytes, self.act_bytes + o.act_bytes)

    def as_dict(self):
        return {k: getattr(self, k) for k in self.__slots__}


def _finish(n_tok, flops, distinct, ranks, d_in, d_out, meta_bytes):
    ranks = np.asarray(ranks, dtype=np.int64)
    ad_bytes = int(sum(BF16_BYTES * adapter_elems(ranks[a], d_in, d_out) for a in distinct))
    act = BF16_BYTES * n_tok * d_in + 2 * BF16_BYTES * n_tok * d_out
    return Cost(flops, act + ad_bytes + meta_bytes, n_tok, ad_bytes, act)


def bgmv_cost(ids: np.ndarray, ranks: np.ndarray, d_in: int, d_out: int) -> Cost:
    ids = np.asarray(ids)
    ranks = np.asarray(ranks, dtype=np.int64)
    valid = ids[ids >= 0]
    flops = int(sum(lora_flops(1, ranks[a], d_in, d_out) for a in valid))
    distinct = np.unique(valid)
    meta = 4 * ids.shape[0] + (8 + 8 + 4) * len(distinct)
    return _finish(int(valid.shape[0]), flops, distinct, ranks, d_in, d_out, meta)


def sgmv_cost(seg_off: np.ndarray, seg_ad: np.ndarray, ranks: np.ndarray, d_in: int,
              d_out: int) -> Cost:
    seg_off = np.asarray(seg_off, dtype=np.int64)
    seg_ad = np.asarray(seg_ad)
    ranks = np.asarray(ranks, dtype=np.int64)
    lens = np.diff(seg_off)
    n_tok = int(lens.sum())
    flops = int(sum(lora_flops(int(l), ranks[a], d_in, d_out) for a, l in zip(seg_ad, lens)))
    distinct = np.unique(seg_ad[lens > 0])
    meta = 4 * (2 * len(seg_ad) + 1) + (8 + 8 + 4) * len(distinct)
    return _finish(n_tok, flops, distinct, ranks, d_in, d_out, meta)


def multi_cost(req_off: np.ndarray, ad_off: np.ndarray, ad_id: np.ndarray, ranks: np.ndarray,
               d_in: int, d_out: int) -> Cost:
    req_off = np.asarray(req_off, dtype=np.int64)
    ad_off = np.asarray(ad_off, dtype=np.int64)
    ad_id = np.asarray(ad_id)
    ranks = np.asarray(ranks, dtype=np.int64)
    n_tok = 0
    flops = 0
    used = []
    for q in range(len(req_off) - 1):
        L = int(req_off[q + 1] - req_off[q])
        ads = ad_id[ad_off[q]:ad_off[q + 1]]
        if L <= 0 or len(ads) == 0:
            continue
        n_tok += L
        flops += int(sum(lora_flops(L, ranks[a], d_in, d_out) for a in ads))
        used.extend(ads.tolist())
    distinct = np.unique(np.asarray(used, dtype=np.int64))
    meta = 4 * (2 * len(req_off) + len(ad_id)) + 4 * len(ad_id) + (8 + 8 + 4) * len(distinct)
    return _finish(n_tok, flops, distinct, ranks, d_in, d_out, meta)


def linear_cost(seg_off: np.ndarray, seg_ad: np.ndarray, ranks: np.ndarray, d_in: int, d_out: int) -> Cost:
    """The projection with its delta: the rows of every segment take x W^T (2 d_in d_out
    FLOPs each) plus their adapter's delta; bytes: x read once, W read once, y written
    once (not read), each touched adapter once, metadata."""
    seg_off = np.asarray(seg_off, dtype=np.int64)
    seg_ad = np.asarray(seg_ad)
    ranks = np.asarray(ranks, dtype=np.int64)
    lens = np.diff(seg_off)
    n_tok = int(lens.sum())
    flops = 2 * n_tok * int(d_in) * int(d_out)
    flops += int(sum(lora_flops(int(l), ranks[a], d_in, d_out) for a, l in zip(seg_ad, lens) if a >= 0))
    distinct = np.unique(seg_ad[(lens > 0) & (seg_ad >= 0)])
    ad_bytes = int(sum(BF16_BYTES * adapter_elems(ranks[a], d_in, d_out) for a in distinct))
    act = BF16_BYTES * n_tok * (int(d_in) + int(d_out))
    w_bytes = BF16_BYTES * int(d_in) * int(d_out)
    meta = 4 * (2 * len(seg_ad) + 1) + (8 + 8 + 4) * len(distinct)
    return Cost(flops, act + w_bytes + ad_bytes + meta, n_tok, ad_bytes, act)


def call_cost(call) -> Cost:
    """Cost of one workload call (duck-typed on the call's host metadata)."""
    p = call.pool
    if hasattr(call, "W") and hasattr(call, "X"):
        return linear_cost(call.seg_off_h, call.seg_ad_h, p.ranks_h, p.d_in, p.d_out)
    if hasattr(call, "W"):
        return merge_cost(p.d_in, p.d_out, int(p.ranks_h[call.adapter]))
    if hasattr(call, "ids_h"):
        return bgmv_cost(call.ids_h, p.ranks_h, p.d_in, p.d_out)
    if hasattr(call, "seg_off_h"):
        return sgmv_cost(call.seg_off_h, call.seg_ad_h, p.ranks_h, p.d_in, p.d_out)
    return multi_cost(call.req_off_h, call.ad_off_h, call.ad_id_h, p.ranks_h, p.d_in, p.d_out)


def merge_cost(d_in: int, d_out: int, r: int) -> Cost:
    """Merging one adapter into W [d_out, d_in]: W read and written once (bf16), the
    adapter read once; 2 d_out d_in r FLOPs (the rank-r product B A)."""
    return Cost(flops=2 * d_out * d_in * r, nbytes=2 * 2 * d_out * d_in + 2 * r * (d_in + d_out), tokens=d_out,
                adapter_bytes=2 * r * (d_in + d_out), act_bytes=2 * 2 * d_out * d_in)


def workload_cost(wl) -> Cost:
    """Sum of the calls' costs.  Where the path reads an input shared by several
    calls once (projections fused on a shared X), that X counts once."""
    c = Cost()
    seen = set()
    for call in wl.calls:
        cc = call_cost(call)
        X = getattr(call, "X", None)
        if wl.desc.get("x_read_once") and X is not None:
            key = X.data_ptr()
            if key in seen:
                dup = BF16_BYTES * cc.tokens * int(call.pool.d_in)
                cc = Cost(cc.flops, cc.bytes - dup, 0, cc.adapter_bytes, cc.act_bytes - dup)
            seen.add(key)
        c = c + cc
    return c
