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


def scatter_pool(hp: HostPool, gap: int = 8) -> HostPool:
    """The same adapters stored in reverse order with `gap` spare elements before
    each one: offsets stay multiples of 8 but are no longer multiples of d_in."""
    n = len(hp.rank)
    A_off = np.zeros(n, np.int64)
    B_off = np.zeros(n, np.int64)
    a_pos = b_pos = 0
    for a in reversed(range(n)):
        r = int(hp.rank[a])
        a_pos += gap
        b_pos += gap
        A_off[a], B_off[a] = a_pos, b_pos
        a_pos += r * hp.d_in
        b_pos += r * hp.d_out
    A = np.full(a_pos + gap, 0x7FC0, np.uint16)       # NaN between adapters: a stray read shows
    B = np.full(b_pos + gap, 0x7FC0, np.uint16)
    for a in range(n):
        r = int(hp.rank[a])
        A[A_off[a]:A_off[a] + r * hp.d_in] = hp.A[hp.A_off[a]:hp.A_off[a] + r * hp.d_in]
        B[B_off[a]:B_off[a] + r * hp.d_out] = hp.B[hp.B_off[a]:hp.B_off[a] + r * hp.d_out]
    return HostPool(A=A, B=B, A_off=A_off, B_off=B_off, rank=hp.rank.copy(), d_in=hp.d_in, d_out=hp.d_out)


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


def compact_from_device_pool(pool, used):
    """Compact a workloads.Pool (possibly on the GPU, possibly GBs) to the adapters used."""
    from oracle import host_pool_subset
    return host_pool_subset(pool, used)


def half_ulp_bf16(y: np.ndarray) -> np.ndarray:
    """Half a bf16 ulp at y's binade: 2**(floor(log2|y|) - 8) (bf16 carries 8
    significant bits), 0 at y = 0.  No bf16 value is closer to y than the nearest
    one, which is at most this far away."""
    a = np.abs(np.asarray(y, np.float64))
    out = np.zeros_like(a)
    nz = a > 0
    out[nz] = np.ldexp(1.0, (np.floor(np.log2(a[nz])) - 8).astype(np.int64))
    return out


def check_parity(y_gpu_f64: np.ndarray, y_exact: np.ndarray, what: str):
    """The parity bar for a bf16 output, elementwise against the oracle's exact value:

        |y_gpu - y_exact| <= 1e-2 * rms(y_exact) + 1e-3 + half_ulp_bf16(y_exact)

    The first two terms are the stated tolerance for the arithmetic (bf16 inputs,
    fp32 accumulation), rms over the whole compared output.  The last term is the
    single rounding of the stored bf16 result: the nearest bf16 value may be up to
    half an ulp of y_exact's binade away, and for |y| >= 4 rms that alone exceeds
    the first two terms.  Returns (max excess ratio err/bound, rms)."""
    y = np.asarray(y_gpu_f64, np.float64)
    ex = np.asarray(y_exact, np.float64)
    rms = float(np.sqrt(np.mean(ex * ex))) if ex.size else 0.0
    b = 1e-2 * rms + 1e-3 + half_ulp_bf16(ex)
    err = np.abs(y - ex)
    ratio = err / b
    m = float(ratio.max()) if ratio.size else 0.0
    if not (m <= 1.0):
        i = np.unravel_index(int(np.argmax(ratio)), ratio.shape)
        raise AssertionError(f"{what}: |err| {err[i]:.4g} > bound {b[i]:.4g} at {i}: gpu {y[i]!r} "
                             f"exact {ex[i]!r} (rms {rms:.4g})")
    return m, rms


def check_rounded(y_gpu_f64: np.ndarray, y_exact: np.ndarray, what: str, min_frac: float = 0.99):
    """With the rank-r intermediate carried to fp32 precision, the stored output is the
    correctly rounded bf16 of the exact value for all but the rare elements whose fp32
    sum lands across a rounding midpoint: at least `min_frac` of them must match."""
    from oracle import round_bf16
    y = np.asarray(y_gpu_f64, np.float64)
    want = round_bf16(np.asarray(y_exact, np.float64))
    frac = float(np.mean(y == want)) if y.size else 1.0
    assert frac >= min_frac, f"{what}: only {frac:.5f} of the outputs are the correctly rounded bf16"
    return frac


def check_close_f32(v_gpu: np.ndarray, v_exact: np.ndarray, what: str):
    """fp32 outputs (the shrink's V): |v - v_exact| <= 1e-2 * rms(v_exact) + 1e-3."""
    b = bound(v_exact)
    err = np.abs(np.asarray(v_gpu, np.float64) - v_exact)
    m = float(err.max()) if err.size else 0.0
    assert m <= b, f"{what}: max |err| {m:.4g} > bound {b:.4g}"
    return m, b


class DevPool:
    """A HostPool copied to a device, shaped like workloads.Pool for the binding."""

    def __init__(self, hp: HostPool, device="cuda", max_rank=None):
        import torch
        def bf(a):
            a = np.ascontiguousarray(a, np.uint16)
            if a.size == 0:
                a = np.zeros(8, np.uint16)
            return torch.from_numpy(a.view(np.int16).copy()).to(device).view(torch.bfloat16)
        self.A = bf(hp.A)
        self.B = bf(hp.B)
        self.A_off = torch.tensor(hp.A_off, dtype=torch.int64, device=device)
        self.B_off = torch.tensor(hp.B_off, dtype=torch.int64, device=device)
        self.rank = torch.tensor(hp.rank, dtype=torch.int32, device=device)
        self.d_in = hp.d_in
        self.d_out = hp.d_out
        self.max_rank = int(max_rank or max(8, int(hp.rank.max()) if hp.rank.size else 8))


def dev_bf16(bits: np.ndarray, device="cuda"):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits, np.uint16).view(np.int16).copy()).to(device).view(torch.bfloat16)
