"""CPU oracle for the unmerged multi-LoRA delta -- TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU-baseline
leg may import this package.  The CUDA library never calls it and it never
calls the CUDA library; the two share no code.

The arithmetic lives in ``lora_oracle.c`` (plain fp64 loops, OpenMP over
rows); this module only builds it with gcc, marshals numpy arrays and
returns float64 results.  Every function follows the definition on
"Serving several LoRAs, ControlNet and IP-Adapter", section "LoRA: merged or
alongside" (W' = W + BA, A is r x d, B is d x r, the unmerged delta
x A^T B^T) and exercise 2's answer on the same page (group by LoRA index,
results back in the original order).  Pins: tests/test_oracle_pins.py.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass
from typing import Optional

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SOURCE = os.path.join(_HERE, "lora_oracle.c")
_LIB = os.path.join(_HERE, "liblora_oracle.so")


class OracleError(RuntimeError):
    pass


def compile_oracle(src: str, out: str) -> str:
    """gcc -O2 -fopenmp a C oracle source into a shared library."""
    tmp = out + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11", "-Wall", "-Wextra",
           "-o", tmp, src]
    subprocess.check_call(cmd)
    os.replace(tmp, out)
    return out


def build(force: bool = False) -> str:
    """Compile lora_oracle.c into liblora_oracle.so when it is missing or stale."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(SOURCE):
        compile_oracle(SOURCE, _LIB)
    return _LIB


def set_threads(n: int) -> None:
    """Number of OpenMP threads the oracle uses (n <= 0: leave the runtime default)."""
    if n > 0:
        os.environ["OMP_NUM_THREADS"] = str(n)
        try:
            ctypes.CDLL("libgomp.so.1").omp_set_num_threads(int(n))
        except OSError:
            pass


def threads() -> int:
    try:
        return int(ctypes.CDLL("libgomp.so.1").omp_get_max_threads())
    except OSError:
        return 1


@dataclass
class HostPool:
    """Adapter pool on the host: A, B as bf16 bit patterns (uint16, flat)."""

    A: np.ndarray
    B: np.ndarray
    A_off: np.ndarray   # int64, element offset of adapter a's A ([rank, d_in] row-major)
    B_off: np.ndarray   # int64, element offset of adapter a's B ([d_out, rank] row-major)
    rank: np.ndarray    # int32
    d_in: int
    d_out: int

    @property
    def n_adapters(self) -> int:
        return int(self.rank.shape[0])


def _p(a: Optional[np.ndarray]):
    return None if a is None else ctypes.c_void_p(a.ctypes.data)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


def _rows(rows, N):
    if rows is None:
        return None, N
    r = _c(rows, np.int32)
    return r, int(r.shape[0])


def _check(rc: int, what: str):
    if rc != 0:
        raise OracleError(f"{what}: oracle rejected the metadata (code {rc})")


class Oracle:
    """The oracle's entry points bound to one compiled library."""

    def __init__(self, path: str):
        lib = ctypes.CDLL(path)
        P = ctypes.c_void_p
        i32, i64, f64 = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
        lib.oracle_bgmv_delta.argtypes = [P, i64, P, P, P, P, P, i32, i32, i32, P, i32, f64, P, i32, P]
        lib.oracle_sgmv_shrink.argtypes = [P, i64, P, P, P, i32, i32, P, P, i32, i32, P, i32, P, i64]
        lib.oracle_sgmv_expand.argtypes = [P, i64, P, P, P, i32, i32, P, P, i32, i32, f64, P, i32, P]
        lib.oracle_sgmv_delta.argtypes = [P, i64, P, P, P, P, P, i32, i32, i32, P, P, i32, i32, f64,
                                          P, i32, P]
        lib.oracle_apply_multi.argtypes = [P, i64, P, P, P, P, P, i32, i32, i32, P, P, P, P, i32, i32,
                                           P, i32, P]
        lib.oracle_route.argtypes = [P, i32, i32, P, P, P, P, P]
        lib.oracle_merge.argtypes = [P, i64, P, P, P, P, P, i32, i32, i32, i32, f64, P, i32, P]
        lib.oracle_linear_sgmv.argtypes = [P, i64, P, i64, P, P, P, P, P, i32, i32, i32, P, P, i32, i32, f64,
                                           P, i32, P]
        for f in (lib.oracle_bgmv_delta, lib.oracle_sgmv_shrink, lib.oracle_sgmv_expand,
                  lib.oracle_sgmv_delta, lib.oracle_apply_multi, lib.oracle_route, lib.oracle_merge,
                  lib.oracle_linear_sgmv):
            f.restype = ctypes.c_int
        self.lib = lib
        self.path = path

    def bgmv_delta(self, X: np.ndarray, pool: HostPool, ids: np.ndarray, scale: float,
                   rows: Optional[np.ndarray] = None) -> np.ndarray:
        """delta[k] = scale * B[a] A[a] x[n] for n = rows[k], a = ids[n] (zero if a == -1)."""
        X = _c(X, np.uint16)
        ids = _c(ids, np.int32)
        N = int(ids.shape[0])
        rows, n_rows = _rows(rows, N)
        D = np.zeros((n_rows, pool.d_out), dtype=np.float64)
        rc = self.lib.oracle_bgmv_delta(_p(X), X.shape[1], _p(pool.A), _p(pool.A_off), _p(pool.B),
                                        _p(pool.B_off), _p(pool.rank), pool.n_adapters, pool.d_in,
                                        pool.d_out, _p(ids), N, float(scale), _p(rows), n_rows, _p(D))
        _check(rc, "bgmv")
        return D

    def sgmv_shrink(self, X: np.ndarray, pool: HostPool, seg_off: np.ndarray, seg_ad: np.ndarray,
                    rows: Optional[np.ndarray] = None, ld: Optional[int] = None,
                    fill: float = np.nan) -> np.ndarray:
        """V[k][j] = sum_i A[a][j][i] x[n][i] (n = rows[k], j < rank[a]); other entries = fill."""
        X = _c(X, np.uint16)
        seg_off = _c(seg_off, np.int32)
        seg_ad = _c(seg_ad, np.int32)
        N = int(X.shape[0])
        rows, n_rows = _rows(rows, N)
        ld = int(ld or max(int(pool.rank.max()), 1))
        V = np.full((n_rows, ld), fill, dtype=np.float64)
        rc = self.lib.oracle_sgmv_shrink(_p(X), X.shape[1], _p(pool.A), _p(pool.A_off), _p(pool.rank),
                                         pool.n_adapters, pool.d_in, _p(seg_off), _p(seg_ad),
                                         int(seg_ad.shape[0]), N, _p(rows), n_rows, _p(V), ld)
        _check(rc, "sgmv_shrink")
        return V

    def sgmv_expand(self, V: np.ndarray, pool: HostPool, seg_off: np.ndarray, seg_ad: np.ndarray,
                    scale: float, rows: Optional[np.ndarray] = None) -> np.ndarray:
        """delta[k][o] = scale * sum_j B[a][o][j] V[n][j]; V is float32, as the GPU receives it."""
        V = _c(V, np.float32)
        seg_off = _c(seg_off, np.int32)
        seg_ad = _c(seg_ad, np.int32)
        N = int(V.shape[0])
        rows, n_rows = _rows(rows, N)
        D = np.zeros((n_rows, pool.d_out), dtype=np.float64)
        rc = self.lib.oracle_sgmv_expand(_p(V), V.shape[1], _p(pool.B), _p(pool.B_off), _p(pool.rank),
                                         pool.n_adapters, pool.d_out, _p(seg_off), _p(seg_ad),
                                         int(seg_ad.shape[0]), N, float(scale), _p(rows), n_rows, _p(D))
        _check(rc, "sgmv_expand")
        return D

    def sgmv_delta(self, X: np.ndarray, pool: HostPool, seg_off: np.ndarray, seg_ad: np.ndarray,
                   scale: float, rows: Optional[np.ndarray] = None) -> np.ndarray:
        """Shrink then expand in double: delta of each row under its segment's adapter."""
        X = _c(X, np.uint16)
        seg_off = _c(seg_off, np.int32)
        seg_ad = _c(seg_ad, np.int32)
        N = int(X.shape[0])
        rows, n_rows = _rows(rows, N)
        D = np.zeros((n_rows, pool.d_out), dtype=np.float64)
        rc = self.lib.oracle_sgmv_delta(_p(X), X.shape[1], _p(pool.A), _p(pool.A_off), _p(pool.B),
                                        _p(pool.B_off), _p(pool.rank), pool.n_adapters, pool.d_in,
                                        pool.d_out, _p(seg_off), _p(seg_ad), int(seg_ad.shape[0]), N,
                                        float(scale), _p(rows), n_rows, _p(D))
        _check(rc, "sgmv")
        return D

    def apply_multi_delta(self, X: np.ndarray, pool: HostPool, req_off: np.ndarray,
                          ad_off: np.ndarray, ad_id: np.ndarray, ad_scale: np.ndarray,
                          rows: Optional[np.ndarray] = None) -> np.ndarray:
        """Sum over a request's adapters of ad_scale * B A x."""
        X = _c(X, np.uint16)
        req_off = _c(req_off, np.int32)
        ad_off = _c(ad_off, np.int32)
        ad_id = _c(ad_id, np.int32)
        ad_scale = _c(ad_scale, np.float32)
        N = int(X.shape[0])
        rows, n_rows = _rows(rows, N)
        D = np.zeros((n_rows, pool.d_out), dtype=np.float64)
        rc = self.lib.oracle_apply_multi(_p(X), X.shape[1], _p(pool.A), _p(pool.A_off), _p(pool.B),
                                         _p(pool.B_off), _p(pool.rank), pool.n_adapters, pool.d_in,
                                         pool.d_out, _p(req_off), _p(ad_off), _p(ad_id), _p(ad_scale),
                                         int(req_off.shape[0]) - 1, N, _p(rows), n_rows, _p(D))
        _check(rc, "apply_multi")
        return D

    def merge(self, W: np.ndarray, pool: HostPool, adapter: int, scale: float,
              rows: Optional[np.ndarray] = None) -> np.ndarray:
        """Wm[k] = W[o] + scale * (B[a] A[a])[o] for o = rows[k] (all rows by default), unrounded."""
        W = _c(W, np.uint16)
        rows, n_rows = _rows(rows, pool.d_out)
        Wm = np.zeros((n_rows, pool.d_in), dtype=np.float64)
        rc = self.lib.oracle_merge(_p(W), W.shape[1], _p(pool.A), _p(pool.A_off), _p(pool.B), _p(pool.B_off),
                                   _p(pool.rank), pool.n_adapters, pool.d_in, pool.d_out, int(adapter),
                                   float(scale), _p(rows), n_rows, _p(Wm))
        _check(rc, "merge")
        return Wm

    def linear_sgmv(self, X: np.ndarray, W: np.ndarray, pool: HostPool, seg_off: np.ndarray,
                    seg_ad: np.ndarray, scale: float, rows: Optional[np.ndarray] = None) -> np.ndarray:
        """Y[k] = W x[n] + scale * B[a] A[a] x[n] (n = rows[k], a = its segment's adapter, -1: none);
        zero rows outside every segment; unrounded."""
        X = _c(X, np.uint16)
        W = _c(W, np.uint16)
        seg_off = _c(seg_off, np.int32)
        seg_ad = _c(seg_ad, np.int32)
        N = int(X.shape[0])
        rows, n_rows = _rows(rows, N)
        Y = np.zeros((n_rows, pool.d_out), dtype=np.float64)
        rc = self.lib.oracle_linear_sgmv(_p(X), X.shape[1], _p(W), W.shape[1], _p(pool.A), _p(pool.A_off),
                                         _p(pool.B), _p(pool.B_off), _p(pool.rank), pool.n_adapters, pool.d_in,
                                         pool.d_out, _p(seg_off), _p(seg_ad), int(seg_ad.shape[0]), N,
                                         float(scale), _p(rows), n_rows, _p(Y))
        _check(rc, "linear_sgmv")
        return Y

    def route(self, ids: np.ndarray, n_adapters: int):
        """Stable counting sort of ids by adapter: (perm, seg_off, seg_ad); id -1 left out."""
        ids = _c(ids, np.int32)
        N = int(ids.shape[0])
        counts = np.zeros(max(n_adapters, 1), dtype=np.int32)
        perm = np.zeros(max(N, 1), dtype=np.int32)
        seg_off = np.zeros(min(N, n_adapters) + 1, dtype=np.int32)
        seg_ad = np.zeros(max(min(N, n_adapters), 1), dtype=np.int32)
        n_seg = np.zeros(1, dtype=np.int32)
        rc = self.lib.oracle_route(_p(ids), N, int(n_adapters), _p(counts), _p(perm), _p(seg_off),
                                   _p(seg_ad), _p(n_seg))
        _check(rc, "route")
        k = int(n_seg[0])
        return perm[: seg_off[k]].copy(), seg_off[: k + 1].copy(), seg_ad[:k].copy()


_default: Optional[Oracle] = None


def default() -> Oracle:
    global _default
    if _default is None:
        _default = Oracle(build())
    return _default


def bgmv_delta(*a, **k):
    return default().bgmv_delta(*a, **k)


def sgmv_shrink(*a, **k):
    return default().sgmv_shrink(*a, **k)


def sgmv_expand(*a, **k):
    return default().sgmv_expand(*a, **k)


def sgmv_delta(*a, **k):
    return default().sgmv_delta(*a, **k)


def apply_multi_delta(*a, **k):
    return default().apply_multi_delta(*a, **k)


def route(*a, **k):
    return default().route(*a, **k)


def merge(*a, **k):
    return default().merge(*a, **k)


def linear_sgmv(*a, **k):
    return default().linear_sgmv(*a, **k)


def widen_bf16(bits: np.ndarray) -> np.ndarray:
    """bf16 bit patterns -> float64, exactly (the same widening the C oracle applies)."""
    return (np.asarray(bits, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def round_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 (ties to even), once, directly from
    float64 (no intermediate float32 rounding); returned as float64.  This models the
    single rounding of the bf16 output y that the library's interface fixes."""
    x = np.asarray(x, dtype=np.float64)
    mag = np.abs(x)
    f = mag.astype(np.float32)                       # near |x|, at most half an fp32 ulp away
    base = (f.view(np.uint32) & np.uint32(0xFFFF0000)).astype(np.int64)
    best = None
    best_err = None
    for step in (-1, 0, 1):
        c_bits = np.clip(base + step * 0x10000, 0, 0x7F7F0000).astype(np.uint32)
        c = c_bits.view(np.float32).astype(np.float64)
        err = np.abs(mag - c)
        if best is None:
            best, best_err, best_bits = c, err, c_bits
            continue
        even = ((c_bits >> np.uint32(16)) & np.uint32(1)) == 0
        take = (err < best_err) | ((err == best_err) & even)
        best = np.where(take, c, best)
        best_err = np.where(take, err, best_err)
        best_bits = np.where(take, c_bits, best_bits)
    return np.copysign(best, x)


def host_pool_subset(pool, used):
    """Copy adapters `used` of a device-resident pool to a HostPool.

    `pool` is any object with A, B (bf16 tensors), A_off_h, B_off_h, ranks_h (numpy),
    d_in, d_out (the seeded workload pools).  Returns (HostPool, remap) with
    remap[a] = index of adapter a in the subset (-1 if absent).  Marshalling only."""
    import torch
    used = np.asarray(sorted(set(int(a) for a in np.asarray(used).ravel())), dtype=np.int64)
    remap = -np.ones(len(pool.ranks_h), dtype=np.int32)
    remap[used] = np.arange(len(used), dtype=np.int32)
    ranks = pool.ranks_h[used].astype(np.int32)
    A_parts, B_parts = [], []
    for a in used:
        r = int(pool.ranks_h[a])
        ao, bo = int(pool.A_off_h[a]), int(pool.B_off_h[a])
        A_parts.append(pool.A[ao:ao + r * pool.d_in].detach().cpu().view(torch.int16).numpy().view(np.uint16))
        B_parts.append(pool.B[bo:bo + r * pool.d_out].detach().cpu().view(torch.int16).numpy().view(np.uint16))
    A_off = np.zeros(len(used), np.int64)
    B_off = np.zeros(len(used), np.int64)
    if len(used):
        A_off[1:] = np.cumsum(ranks.astype(np.int64) * pool.d_in)[:-1]
        B_off[1:] = np.cumsum(ranks.astype(np.int64) * pool.d_out)[:-1]
    A = np.concatenate(A_parts) if A_parts else np.zeros(8, np.uint16)
    B = np.concatenate(B_parts) if B_parts else np.zeros(8, np.uint16)
    return HostPool(A=A, B=B, A_off=A_off, B_off=B_off, rank=ranks, d_in=pool.d_in, d_out=pool.d_out), remap
