"""Shared test helpers: host copies of workloads, numpy references for the pins,
the parity bound, and compaction of large pools to the adapters a call touches."""
from __future__ import annotations

import numpy as np

from oracle import HostPool
from workloads import bf16_bits, to_host


def widen(bits: np.ndarray) -> np.ndarray:
    """bf16 bits -> float64 through numpy's float32 view (independent of the C oracle)."""
    b = np.asarray(bits, dtype=np.uint16).astype(np.uint32) << np.uint32(16)
    return b.view(np.float32).astype(np.float64)


def host_pool(pool) -> HostPool:
    """workloads.Pool (any device) -> oracle.HostPool."""
    return HostPool(A=to_host(pool.A), B=to_host(pool.B), A_off=pool.A_off_h.copy(),
                    B_off=pool.B_off_h.copy(), rank=pool.ranks_h.copy(), d_in=pool.d_in,
                    d_out=pool.d_out)


def rand_host_pool(rng: np.random.Generator, ranks, d_in: int, d_out: int,
                   zero_B: bool = False) -> HostPool:
    ranks = np.asarray(ranks, dtype=np.int32)
    A_off = np.zeros(len(ranks), np.int64)
    B_off = np.zeros(len(ranks), np.int64)
    A_off[1:] = np.cumsum(ranks.astype(np.int64) * d_in)[:-1]
    B_off[1:] = np.cumsum(ranks.astype(np.int64) * d_out)[:-1]
    na = int(ranks.sum()) * d_in
    nb = int(ranks.sum()) * d_out
    A = bf16_bits(rng.standard_normal(na).astype(np.float32) / np.sqrt(d_in))
    if zero_B:
        B = np.zeros(nb, np.uint16)
    else:
        B = np.concatenate([bf16_bits(rng.standard_normal(d_out * int(r)).astype(np.float32) /
                                      np.sqrt(r)) for r in ranks]) if len(ranks) else np.zeros(0, np.uint16)
    return HostPool(A=A, B=B, A_off=A_off, B_off=B_off, rank=ranks, d_in=d_in, d_out=d_out)


def rand_x(rng: np.random.Generator, N: int, d: int) -> np.ndarray:
    return bf16_bits(rng.standard_normal((N, d)).astype(np.float32))


def A_of(p: HostPool, a: int) -> np.ndarray:
    r = int(p.rank[a])
    return widen(p.A[p.A_off[a]:p.A_off[a] + r * p.d_in]).reshape(r, p.d_in)


def B_of(p: HostPool, a: int) -> np.ndarray:
    r = int(p.rank[a])
    return widen(p.B[p.B_off[a]:p.B_off[a] + p.d_out * r]).reshape(p.d_out, r)


def numpy_delta_rows(X: np.ndarray, p: HostPool, ids: np.ndarray, scale: float) -> np.ndarray:
    """Per-adapter dense numpy products, scattered back to the token rows."""
    Xd = widen(X)
    D = np.zeros((X.shape[0], p.d_out))
    for a in np.unique(ids[ids >= 0]):
        rows = np.nonzero(ids == a)[0]
        D[rows] = scale * ((Xd[rows] @ A_of(p, a).T) @ B_of(p, a).T)
    return D


def bound(y_ref: np.ndarray) -> float:
    """The elementwise parity bound: 1e-2 * rms(y_ref) + 1e-3 over the whole output."""
    y = np.asarray(y_ref, dtype=np.float64)
    rms = float(np.sqrt(np.mean(y * y))) if y.size else 0.0
    return 1e-2 * rms + 1e-3


def compact_pool(hp_full_getter, ranks_h, A_off_h, B_off_h, d_in, d_out, used: np.ndarray):
    """Build a HostPool holding only the adapters in `used` (ascending), fetching each
    adapter's A and B via hp_full_getter(a) -> (A_bits, B_bits).  Returns (pool, remap)
    where remap[a_full] = a_compact (-1 if absent)."""
    used = np.asarray(sorted(set(int(a) for a in used)), dtype=np.int64)
    remap = -np.ones(len(ranks_h), dtype=np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    ranks = ranks_h[used].astype(np.int32)
    As, Bs = [], []
    for a in used:
        Aa, Ba = hp_full_getter(int(a))
        As.append(Aa)
        Bs.append(Ba)
    A_off = np.zeros(len(used), np.int64)
    B_off = np.zeros(len(used), np.int64)
    if len(used):
        A_off[1:] = np.cumsum(ranks.astype(np.int64) * d_in)[:-1]
        B_off[1:] = np.cumsum(ranks.astype(np.int64) * d_out)[:-1]
    A = np.concatenate(As) if As else np.zeros(8, np.uint16)
    B = np.concatenate(Bs) if Bs else np.zeros(8, np.uint16)
    return HostPool(A=A, B=B, A_off=A_off, B_off=B_off, rank=ranks, d_in=d_in, d_out=d_out), remap


def compact_from_device_pool(pool, used):
    """Compact a workloads.Pool (possibly on the GPU, possibly GBs) to the adapters used."""
    def get(a):
        return to_host(pool.adapter_A(a)).reshape(-1), to_host(pool.adapter_B(a)).reshape(-1)
    return compact_pool(get, pool.ranks_h, pool.A_off_h, pool.B_off_h, pool.d_in, pool.d_out, used)
