"""Seeded synthetic workloads for the unmerged multi-LoRA delta.

Shapes and distributions follow the workloads the source pages discuss:

* "Serving several LoRAs, ControlNet and IP-Adapter" (AI-infra handbook),
  section "LoRA: merged or alongside": A is r x d, B is d x r, r from 8 to 128;
  a batch mixes requests that each carry their own LoRA index; several LoRAs
  may be stacked on one request with a per-LoRA weight.
* "Co-occurrence Patterns of LoRA Adapters in Production Diffusion Model
  Inference Services" (abstract): adapter usage is heavy-tailed and requests
  carry one or a few co-occurring adapters -> Zipf adapter ids, 1..3 adapters
  per image.

Conventions (the readings taken where the pages are silent):

* "N(0, v)" is a variance: A ~ N(0, 1/d_in), B ~ N(0, 1/r_a), x ~ N(0, 1).
* Zipf(s) has finite support: P(k) ~ k^-s for k = 1..M, adapter id = k - 1.
* A pool stores adapter a's A as [r_a, d_in] row-major at element offset
  A_off[a] and its B as [d_out, r_a] row-major at B_off[a]; adapters are
  packed back to back in id order (no padding to the maximum rank).

Metadata comes from numpy's PCG64 seeded with the workload seed; tensors come
from a torch generator on the target device seeded from the same seed.  Only
random draws and layout live here.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional, Sequence

import numpy as np
import torch

BF16 = torch.bfloat16


# ----------------------------------------------------------------------------
# helpers
# ----------------------------------------------------------------------------
def _tgen(seed: int, device) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed) & 0x7FFFFFFFFFFFFFFF)
    return g


def _rng(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(int(seed)))


def bf16_bits(a: np.ndarray) -> np.ndarray:
    """float32 numpy array -> bf16 bit patterns (round to nearest even)."""
    t = torch.from_numpy(np.ascontiguousarray(a, dtype=np.float32)).to(BF16)
    return t.view(torch.int16).numpy().view(np.uint16)


def to_host(t: torch.Tensor) -> np.ndarray:
    """Copy a tensor to host numpy; bf16 comes back as uint16 bit patterns."""
    t = t.detach().contiguous().cpu()
    if t.dtype == BF16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def zipf_ids(rng: np.random.Generator, n_adapters: int, s: float, size: int) -> np.ndarray:
    """Heavy-tailed adapter ids: P(id = k-1) ~ k^-s over k = 1..n_adapters."""
    k = np.arange(1, n_adapters + 1, dtype=np.float64)
    p = k ** (-float(s))
    p /= p.sum()
    return rng.choice(n_adapters, size=size, p=p).astype(np.int32)


def _randn_bf16(n_elem: int, std: float, gen: torch.Generator, device) -> torch.Tensor:
    out = torch.empty(n_elem, dtype=BF16, device=device)
    chunk = 1 << 27
    for s in range(0, n_elem, chunk):
        e = min(n_elem, s + chunk)
        tmp = torch.randn(e - s, generator=gen, device=device, dtype=torch.float32)
        out[s:e] = (tmp * std).to(BF16)
    return out


def _randn_rows_bf16(rows: int, cols: int, std: float, gen, device) -> torch.Tensor:
    return _randn_bf16(rows * cols, std, gen, device).view(rows, cols)


# ----------------------------------------------------------------------------
# adapter pool
# ----------------------------------------------------------------------------
@dataclass
class Pool:
    """One projection's resident adapter pool (all adapters packed, bf16)."""

    A: torch.Tensor          # flat bf16, adapter a = [rank[a], d_in] at A_off[a]
    B: torch.Tensor          # flat bf16, adapter a = [d_out, rank[a]] at B_off[a]
    A_off: torch.Tensor      # int64 [n_adapters], on the pool's device
    B_off: torch.Tensor      # int64 [n_adapters]
    rank: torch.Tensor       # int32 [n_adapters]
    d_in: int
    d_out: int
    ranks_h: np.ndarray      # host copies of the metadata
    A_off_h: np.ndarray
    B_off_h: np.ndarray

    @property
    def n_adapters(self) -> int:
        return int(self.ranks_h.shape[0])

    @property
    def max_rank(self) -> int:
        return int(self.ranks_h.max()) if self.n_adapters else 0

    def adapter_A(self, a: int) -> torch.Tensor:
        r = int(self.ranks_h[a])
        o = int(self.A_off_h[a])
        return self.A[o:o + r * self.d_in].view(r, self.d_in)

    def adapter_B(self, a: int) -> torch.Tensor:
        r = int(self.ranks_h[a])
        o = int(self.B_off_h[a])
        return self.B[o:o + self.d_out * r].view(self.d_out, r)

    def weight_bytes(self, a: int) -> int:
        return 2 * int(self.ranks_h[a]) * (self.d_in + self.d_out)


def make_pool(ranks: Sequence[int], d_in: int, d_out: int, seed: int, device="cpu",
              init: str = "normal") -> Pool:
    """Pack adapters back to back.  init: 'normal' (A~N(0,1/d_in), B~N(0,1/r)) or 'zeros'."""
    ranks_h = np.asarray(ranks, dtype=np.int32).copy()
    n = ranks_h.shape[0]
    a_sz = ranks_h.astype(np.int64) * d_in
    b_sz = ranks_h.astype(np.int64) * d_out
    A_off_h = np.zeros(n, dtype=np.int64)
    B_off_h = np.zeros(n, dtype=np.int64)
    if n:
        A_off_h[1:] = np.cumsum(a_sz)[:-1]
        B_off_h[1:] = np.cumsum(b_sz)[:-1]
    tot_a = int(a_sz.sum())
    tot_b = int(b_sz.sum())
    gen = _tgen(seed * 7919 + 11, device)
    if init == "zeros":
        A = torch.zeros(max(tot_a, 8), dtype=BF16, device=device)
        B = torch.zeros(max(tot_b, 8), dtype=BF16, device=device)
    else:
        A = _randn_bf16(max(tot_a, 8), 1.0 / math.sqrt(d_in), gen, device)
        B = torch.empty(max(tot_b, 8), dtype=BF16, device=device)
        # B ~ N(0, 1/r_a): per-adapter std, generated in chunks of adapters
        stds = torch.tensor(1.0 / np.sqrt(np.maximum(ranks_h, 1)), dtype=torch.float32, device=device)
        counts = torch.tensor(b_sz, dtype=torch.int64, device=device)
        c0 = 0
        while c0 < n:
            c1 = c0
            tot = 0
            while c1 < n and (tot == 0 or tot + b_sz[c1] <= (1 << 27)):
                tot += int(b_sz[c1])
                c1 += 1
            tmp = torch.randn(tot, generator=gen, device=device, dtype=torch.float32)
            std = torch.repeat_interleave(stds[c0:c1], counts[c0:c1])
            s = int(B_off_h[c0])
            B[s:s + tot] = (tmp * std).to(BF16)
            c0 = c1
    dev = torch.device(device)
    return Pool(
        A=A, B=B,
        A_off=torch.tensor(A_off_h, dtype=torch.int64, device=dev),
        B_off=torch.tensor(B_off_h, dtype=torch.int64, device=dev),
        rank=torch.tensor(ranks_h, dtype=torch.int32, device=dev),
        d_in=int(d_in), d_out=int(d_out),
        ranks_h=ranks_h, A_off_h=A_off_h, B_off_h=B_off_h,
    )


# ----------------------------------------------------------------------------
# calls (one op on one projection)
# ----------------------------------------------------------------------------
@dataclass
class BgmvCall:
    """One token per request; ids[n] = adapter of token n (-1: none); unsorted."""

    name: str
    X: torch.Tensor          # bf16 [N, d_in]
    Y: torch.Tensor          # bf16 [N, d_out] (initial y0; the op adds into it)
    pool: Pool
    ids: torch.Tensor        # int32 [N]
    ids_h: np.ndarray
    scale: float

    @property
    def n_tokens(self) -> int:
        return int(self.X.shape[0])


@dataclass
class SgmvCall:
    """Tokens already grouped: rows seg_off[k]..seg_off[k+1] use adapter seg_ad[k]."""

    name: str
    X: torch.Tensor
    Y: torch.Tensor
    pool: Pool
    seg_off: torch.Tensor    # int32 [n_seg + 1]
    seg_ad: torch.Tensor     # int32 [n_seg]
    seg_off_h: np.ndarray
    seg_ad_h: np.ndarray
    scale: float

    @property
    def n_tokens(self) -> int:
        return int(self.X.shape[0])


@dataclass
class MultiCall:
    """Request q = rows req_off[q]..req_off[q+1]; adapters ad_id[ad_off[q]..ad_off[q+1])
    with weights ad_scale[...]; their deltas are summed."""

    name: str
    X: torch.Tensor
    Y: torch.Tensor
    pool: Pool
    req_off: torch.Tensor    # int32 [n_req + 1]
    ad_off: torch.Tensor     # int32 [n_req + 1]
    ad_id: torch.Tensor      # int32 [n_pairs]
    ad_scale: torch.Tensor   # float32 [n_pairs]
    req_off_h: np.ndarray
    ad_off_h: np.ndarray
    ad_id_h: np.ndarray
    ad_scale_h: np.ndarray

    @property
    def n_tokens(self) -> int:
        return int(self.X.shape[0])


@dataclass
class MergeCall:
    """Fold adapter `adapter` of `pool` into the base weight W [d_out, d_in] in place:
    W += scale * B[a] A[a] (unmerge: -scale)."""

    name: str
    W: torch.Tensor          # bf16 [d_out, d_in]
    pool: Pool
    adapter: int
    scale: float

    @property
    def n_tokens(self) -> int:
        # rows of W (the unit the merge streams)
        return int(self.W.shape[0])


@dataclass
class LinearCall:
    """The projection with its LoRA delta: Y = X W^T + scale * (X A^T B^T per segment's
    adapter); Y is the output (overwritten)."""

    name: str
    X: torch.Tensor          # bf16 [N, d_in]
    W: torch.Tensor          # bf16 [d_out, d_in] (the base weight)
    Y: torch.Tensor          # bf16 [N, d_out] (output)
    pool: Pool
    seg_off: torch.Tensor
    seg_ad: torch.Tensor
    seg_off_h: np.ndarray
    seg_ad_h: np.ndarray
    scale: float

    @property
    def n_tokens(self) -> int:
        return int(self.X.shape[0])


@dataclass
class Workload:
    name: str
    calls: list
    desc: dict = field(default_factory=dict)

    @property
    def n_tokens(self) -> int:
        # tokens of one layer pass: calls that share X count once
        return int(self.desc.get("tokens", self.calls[0].n_tokens))


def _x(N: int, d: int, gen, device) -> torch.Tensor:
    return _randn_rows_bf16(N, d, 1.0, gen, device)


def _y0(N: int, d: int, gen, device, y0: str) -> torch.Tensor:
    if y0 == "zeros":
        return torch.zeros(N, d, dtype=BF16, device=device)
    return _randn_rows_bf16(N, d, 1.0, gen, device)


def bgmv_call(name, X, pool, ids_h, scale, device, y0="zeros", seed=0) -> BgmvCall:
    gen = _tgen(seed * 104729 + 3, device)
    N = X.shape[0]
    Y = _y0(N, pool.d_out, gen, device, y0)
    ids_h = np.asarray(ids_h, dtype=np.int32).copy()
    return BgmvCall(name, X, Y, pool, torch.tensor(ids_h, device=device), ids_h, float(scale))


def sgmv_call(name, X, pool, seg_off_h, seg_ad_h, scale, device, y0="zeros", seed=0) -> SgmvCall:
    gen = _tgen(seed * 104729 + 5, device)
    N = X.shape[0]
    Y = _y0(N, pool.d_out, gen, device, y0)
    so = np.asarray(seg_off_h, dtype=np.int32).copy()
    sa = np.asarray(seg_ad_h, dtype=np.int32).copy()
    return SgmvCall(name, X, Y, pool, torch.tensor(so, device=device),
                    torch.tensor(sa, device=device), so, sa, float(scale))


def multi_call(name, X, pool, req_off_h, ad_off_h, ad_id_h, ad_scale_h, device,
               y0="zeros", seed=0) -> MultiCall:
    gen = _tgen(seed * 104729 + 7, device)
    N = X.shape[0]
    Y = _y0(N, pool.d_out, gen, device, y0)
    ro = np.asarray(req_off_h, dtype=np.int32).copy()
    ao = np.asarray(ad_off_h, dtype=np.int32).copy()
    ai = np.asarray(ad_id_h, dtype=np.int32).copy()
    asc = np.asarray(ad_scale_h, dtype=np.float32).copy()
    return MultiCall(name, X, Y, pool, torch.tensor(ro, device=device), torch.tensor(ao, device=device),
                     torch.tensor(ai, device=device), torch.tensor(asc, device=device), ro, ao, ai, asc)


def segments_from_sorted_ids(sorted_ids: np.ndarray, n_adapters: int, keep_empty: bool):
    """Segment offsets of an id array that is already sorted ascending."""
    counts = np.bincount(sorted_ids, minlength=n_adapters)
    ads = np.arange(n_adapters, dtype=np.int32)
    if not keep_empty:
        ads = ads[counts > 0]
        counts = counts[counts > 0]
    seg_off = np.zeros(len(ads) + 1, dtype=np.int32)
    seg_off[1:] = np.cumsum(counts)
    return seg_off, ads.astype(np.int32)


# ----------------------------------------------------------------------------
# the five workloads
# ----------------------------------------------------------------------------
WORKLOAD_NAMES = [
    "tiny_sgmv",          # N=64, 256->256, r8, 4 adapters, 4 contiguous segments
    "decode_bgmv",        # 256 requests x 1 token, 4096->4096, r16, 128 adapters, Zipf(1.1)
    "prefill_sgmv",       # 32 prompts U[128,1024], 4096->14336, r64, 64 adapters, Zipf(1.1)
    "mixed_rank_layer",   # 512 decode tokens, 1000 adapters r in {8..128}, 7 Llama-3-8B projections
    "diffusion_multi",    # 16 images x 4096 tokens, 1280->1280 x QKVO, r32, 200 adapters, 1-3 per image
    "merge_mlp_up",       # fold one rank-64 adapter into W [14336, 4096] (Llama-3-8B MLP up-proj) in place
    "prefill_qkv",        # the prefill segments over Llama-3-8B q/k/v (4096 -> 4096/1024/1024), r64, X shared
    "prefill_linear_up",  # the prefill segments through the MLP up-proj W [14336, 4096] with its LoRA, fused
]

LLAMA3_8B_PROJ = [  # name, d_in, d_out, which input it reads
    ("q", 4096, 4096, "attn"), ("k", 4096, 1024, "attn"), ("v", 4096, 1024, "attn"),
    ("o", 4096, 4096, "o"), ("gate", 4096, 14336, "mlp"), ("up", 4096, 14336, "mlp"),
    ("down", 14336, 4096, "down"),
]


def cooccurrence_requests(seed: int, n_requests: int = 20000, n_adapters: int = 200, n_bundles: int = 64,
                          p_bundle: float = 0.8, zipf_s: float = 1.1):
    """A stream of requests' adapter lists with recurring combinations, standing in
    for the production traces of "Co-occurrence Patterns of LoRA Adapters in
    Production Diffusion Model Inference Services" (not available here).

    Each request carries k in {1, 2, 3} adapters with P = 0.5 / 0.3 / 0.2 (the
    diffusion workload's mix).  A single adapter is Zipf(zipf_s) over the pool.  A
    multi-adapter request, with probability p_bundle, takes the first k adapters of
    one of n_bundles fixed bundles (three distinct adapters each, drawn once; the
    bundle picked Zipf(zipf_s)); otherwise k distinct adapters uniformly.  The first
    adapter of a list is its primary one."""
    rng = _rng(seed)
    bundles = [rng.choice(n_adapters, size=3, replace=False) for _ in range(n_bundles)]
    ks = rng.choice(np.array([1, 2, 3]), size=n_requests, p=[0.5, 0.3, 0.2])
    out = []
    for k in ks:
        if k == 1:
            out.append(zipf_ids(rng, n_adapters, zipf_s, 1).astype(np.int64))
        elif rng.random() < p_bundle:
            b = bundles[int(zipf_ids(rng, n_bundles, zipf_s, 1)[0])]
            out.append(np.asarray(b[:k], np.int64))
        else:
            out.append(rng.choice(n_adapters, size=int(k), replace=False).astype(np.int64))
    return out


def make_workload(which, device="cpu", seed: Optional[int] = None, y0: str = "zeros",
                  **overrides) -> Workload:
    """Build one of the named workloads (index or name).  seed defaults to the index.

    overrides shrink a workload for quick tests (e.g. n_req=4, d_out=512)."""
    idx = which if isinstance(which, int) else WORKLOAD_NAMES.index(which)
    seed = idx if seed is None else int(seed)
    rng = _rng(seed)
    gen = _tgen(seed * 31 + 1, device)
    if idx == 0:
        N = overrides.get("N", 64)
        d = overrides.get("d", 256)
        r = overrides.get("rank", 8)
        n_ad = overrides.get("n_adapters", 4)
        ids = rng.integers(0, n_ad, size=N).astype(np.int32)
        sorted_ids = np.sort(ids, kind="stable")
        seg_off, seg_ad = segments_from_sorted_ids(sorted_ids, n_ad, keep_empty=True)
        pool = make_pool([r] * n_ad, d, d, seed, device)
        X = _x(N, d, gen, device)
        call = sgmv_call("tiny", X, pool, seg_off, seg_ad, 1.0, device, y0, seed)
        return Workload("tiny_sgmv", [call], {"tokens": N, "op": "sgmv"})
    if idx == 1:
        N = overrides.get("N", 256)
        d = overrides.get("d", 4096)
        r = overrides.get("rank", 16)
        n_ad = overrides.get("n_adapters", 128)
        ids = zipf_ids(rng, n_ad, overrides.get("zipf_s", 1.1), N)
        pool = make_pool([r] * n_ad, d, d, seed, device)
        X = _x(N, d, gen, device)
        call = bgmv_call("q", X, pool, ids, overrides.get("scale", 2.0), device, y0, seed)
        return Workload("decode_bgmv", [call], {"tokens": N, "op": "bgmv"})
    if idx == 2:
        n_req = overrides.get("n_req", 32)
        lo, hi = overrides.get("len_range", (128, 1024))
        d_in = overrides.get("d_in", 4096)
        d_out = overrides.get("d_out", 14336)
        r = overrides.get("rank", 64)
        n_ad = overrides.get("n_adapters", 64)
        lens = rng.integers(lo, hi + 1, size=n_req).astype(np.int64)
        req_ids = zipf_ids(rng, n_ad, overrides.get("zipf_s", 1.1), n_req)
        order = np.argsort(req_ids, kind="stable")      # requests laid out by adapter
        tok_ids = np.repeat(req_ids[order], lens[order]).astype(np.int32)
        seg_off, seg_ad = segments_from_sorted_ids(tok_ids, n_ad, keep_empty=False)
        N = int(lens.sum())
        pool = make_pool([r] * n_ad, d_in, d_out, seed, device)
        X = _x(N, d_in, gen, device)
        call = sgmv_call("up", X, pool, seg_off, seg_ad, overrides.get("scale", 1.0), device, y0, seed)
        return Workload("prefill_sgmv", [call], {"tokens": N, "op": "sgmv", "requests": n_req,
                                                 "req_len": lens.tolist()})
    if idx == 3:
        N = overrides.get("N", 512)
        n_ad = overrides.get("n_adapters", 1000)
        rank_set = overrides.get("rank_set", (8, 16, 32, 64, 128))
        ranks = rng.choice(np.asarray(rank_set, dtype=np.int32), size=n_ad).astype(np.int32)
        ids = zipf_ids(rng, n_ad, overrides.get("zipf_s", 1.0), N)
        projs = overrides.get("projections", LLAMA3_8B_PROJ)
        dscale = overrides.get("dim_div", 1)
        xs = {}
        calls = []
        for p_i, (pname, d_in, d_out, xin) in enumerate(projs):
            d_in //= dscale
            d_out //= dscale
            if xin not in xs:
                xs[xin] = _x(N, d_in, gen, device)
            pool = make_pool(ranks, d_in, d_out, seed * 100 + p_i, device)
            calls.append(bgmv_call(pname, xs[xin], pool, ids, overrides.get("scale", 1.0),
                                   device, y0, seed * 100 + p_i))
        return Workload("mixed_rank_layer", calls, {"tokens": N, "op": "bgmv"})
    if idx == 4:
        n_img = overrides.get("n_img", 16)
        tok = overrides.get("tokens_per_img", 4096)
        d = overrides.get("d", 1280)
        r = overrides.get("rank", 32)
        n_ad = overrides.get("n_adapters", 200)
        ks = rng.choice(np.array([1, 2, 3]), size=n_img, p=[0.5, 0.3, 0.2])
        ad_id = []
        ad_scale = []
        for q in range(n_img):
            ad_id.extend(rng.choice(n_ad, size=int(ks[q]), replace=False).tolist())
            ad_scale.extend(rng.uniform(0.5, 1.0, size=int(ks[q])).tolist())
        ad_off = np.zeros(n_img + 1, dtype=np.int32)
        ad_off[1:] = np.cumsum(ks)
        req_off = (np.arange(n_img + 1) * tok).astype(np.int32)
        N = n_img * tok
        calls = []
        for p_i, pname in enumerate(overrides.get("projections", ["q", "k", "v", "o"])):
            pool = make_pool([r] * n_ad, d, d, seed * 100 + p_i, device)
            X = _x(N, d, gen, device)
            calls.append(multi_call(pname, X, pool, req_off, ad_off, np.asarray(ad_id, np.int32),
                                    np.asarray(ad_scale, np.float32), device, y0, seed * 100 + p_i))
        return Workload("diffusion_multi", calls, {"tokens": N, "op": "multi", "images": n_img})
    if idx == 5:
        d_in = overrides.get("d_in", 4096)
        d_out = overrides.get("d_out", 14336)
        r = overrides.get("rank", 64)
        n_ad = overrides.get("n_adapters", 64)
        pool = make_pool([r] * n_ad, d_in, d_out, seed, device)
        # base weight ~ N(0, 1/d_in): the same scale as B A, so the update is not lost in rounding
        W = _randn_rows_bf16(d_out, d_in, 1.0 / math.sqrt(d_in), gen, device)
        a = int(rng.integers(0, n_ad))
        call = MergeCall("up", W, pool, a, overrides.get("scale", 1.0))
        return Workload("merge_mlp_up", [call], {"tokens": d_out, "op": "merge"})
    if idx == 6:
        # the prefill recipe (prompt lengths, Zipf adapters, per-adapter segments) over the
        # three attention projections that read the same input; an adapter fine-tunes all three
        n_req = overrides.get("n_req", 32)
        lo, hi = overrides.get("len_range", (128, 1024))
        d_in = overrides.get("d_in", 4096)
        d_outs = overrides.get("d_outs", (4096, 1024, 1024))
        r = overrides.get("rank", 64)
        n_ad = overrides.get("n_adapters", 64)
        lens = rng.integers(lo, hi + 1, size=n_req).astype(np.int64)
        req_ids = zipf_ids(rng, n_ad, overrides.get("zipf_s", 1.1), n_req)
        order = np.argsort(req_ids, kind="stable")
        tok_ids = np.repeat(req_ids[order], lens[order]).astype(np.int32)
        seg_off, seg_ad = segments_from_sorted_ids(tok_ids, n_ad, keep_empty=False)
        N = int(lens.sum())
        X = _x(N, d_in, gen, device)
        calls = []
        for p_i, (pname, d_out) in enumerate(zip(("q", "k", "v"), d_outs)):
            pool = make_pool([r] * n_ad, d_in, d_out, seed * 100 + p_i, device)
            calls.append(sgmv_call(pname, X, pool, seg_off, seg_ad, overrides.get("scale", 1.0), device, y0,
                                   seed * 100 + p_i))
        return Workload("prefill_qkv", calls, {"tokens": N, "op": "sgmv_proj", "x_read_once": True,
                                               "requests": n_req})
    if idx == 7:
        # the prefill recipe through the whole adapted projection: y = x W^T + s x A^T B^T
        n_req = overrides.get("n_req", 32)
        lo, hi = overrides.get("len_range", (128, 1024))
        d_in = overrides.get("d_in", 4096)
        d_out = overrides.get("d_out", 14336)
        r = overrides.get("rank", 64)
        n_ad = overrides.get("n_adapters", 64)
        lens = rng.integers(lo, hi + 1, size=n_req).astype(np.int64)
        req_ids = zipf_ids(rng, n_ad, overrides.get("zipf_s", 1.1), n_req)
        order = np.argsort(req_ids, kind="stable")
        tok_ids = np.repeat(req_ids[order], lens[order]).astype(np.int32)
        seg_off, seg_ad = segments_from_sorted_ids(tok_ids, n_ad, keep_empty=False)
        N = int(lens.sum())
        pool = make_pool([r] * n_ad, d_in, d_out, seed, device)
        X = _x(N, d_in, gen, device)
        # base weight ~ N(0, 1/d_in), like the adapters' A: x W^T and the delta are both O(1)
        W = _randn_rows_bf16(d_out, d_in, 1.0 / math.sqrt(d_in), gen, device)
        Y = torch.zeros(N, d_out, dtype=BF16, device=device)
        call = LinearCall("up", X, W, Y, pool, torch.tensor(seg_off, device=device),
                          torch.tensor(seg_ad, device=device), seg_off, seg_ad, overrides.get("scale", 1.0))
        return Workload("prefill_linear_up", [call], {"tokens": N, "op": "linear", "requests": n_req})
    raise ValueError(f"unknown workload {which!r}")
