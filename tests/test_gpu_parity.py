"""GPU vs oracle parity on the five workloads, through the C ABI.

Every call goes through liblora_sgmv.so via the ctypes binding; the oracle
runs on the host on the same seeded inputs.  The bar (elementwise, against
the oracle's exact fp64 value y_exact):
    |y_gpu - y_exact| <= 1e-2 * rms(y_exact) + 1e-3 + half a bf16 ulp of y_exact
(the stated tolerance plus the one bf16 rounding of the stored output; see
helpers.check_parity).  The shrink's fp32 V is held to 1e-2 * rms + 1e-3
against the oracle's fp64 V.  Every path carries the rank-r intermediate to
fp32 precision, so each must in addition give the correctly rounded bf16 of
y_exact for at least 99% of the outputs.  Full-size workloads are checked on
sampled rows (segment boundaries always included); the small ones on every row.
"""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import (check_close_f32, check_parity, check_rounded, compact_from_device_pool, host_pool,
                     widen)
from workloads import make_workload, to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    torch.cuda.synchronize()
    return widen(to_host(t)) if t.dtype == torch.bfloat16 else to_host(t).astype(np.float64)


def _no_err(ws):
    assert L.lora_get_error(ws) == 0


def _sample_rows(N, bounds, n=160, seed=0):
    rng = np.random.default_rng(seed)
    rows = set(rng.choice(N, size=min(n, N), replace=False).tolist())
    for b in bounds:
        for r in (b - 1, b):
            if 0 <= r < N:
                rows.add(int(r))
    return np.array(sorted(rows), np.int32)


def _sgmv_roundtrip(c, rows=None):
    """GPU shrink then expand; returns (V gpu, Y gpu) on the host as float64."""
    N = c.X.shape[0]
    mr = c.pool.max_rank
    V = torch.full((N, mr), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(c.X, V, c.pool, c.seg_off, c.seg_ad)
    _no_err(ws)
    Y = c.Y.clone()
    ws = L.lora_sgmv_expand(torch.nan_to_num(V), Y, c.pool, c.seg_off, c.seg_ad, c.scale)
    _no_err(ws)
    Vh = to_host(V).astype(np.float64)
    Yh = _f64(Y)
    if rows is not None:
        Vh, Yh = Vh[rows], Yh[rows]
    return Vh, Yh


@pytest.mark.parametrize("y0", ["zeros", "normal"])
def test_tiny_sgmv_every_row(y0):
    wl = make_workload(0, device=DEV, y0=y0)
    c = wl.calls[0]
    hp = host_pool(c.pool)
    X = to_host(c.X)
    Vh, Yh = _sgmv_roundtrip(c)
    Vref = oracle.sgmv_shrink(X, hp, c.seg_off_h, c.seg_ad_h, ld=Vh.shape[1])
    assert np.array_equal(np.isnan(Vh), np.isnan(Vref))
    m = ~np.isnan(Vref)
    check_close_f32(Vh[m], Vref[m], "tiny shrink V")
    y_exact = _f64(c.Y) + oracle.sgmv_delta(X, hp, c.seg_off_h, c.seg_ad_h, c.scale)
    check_parity(Yh, y_exact, f"tiny sgmv y0={y0}")
    check_rounded(Yh, y_exact, f"tiny sgmv y0={y0}")
    # the expand alone, fed the GPU's own fp32 V, against the oracle's expand of that V
    Y2 = c.Y.clone()
    V32 = torch.tensor(np.nan_to_num(Vh).astype(np.float32), device=DEV)
    _no_err(L.lora_sgmv_expand(V32, Y2, c.pool, c.seg_off, c.seg_ad, c.scale))
    check_parity(_f64(Y2), _f64(c.Y) + oracle.sgmv_expand(np.nan_to_num(Vh).astype(np.float32), hp,
                                                            c.seg_off_h, c.seg_ad_h, c.scale),
                 "tiny expand")


@pytest.mark.parametrize("y0", ["zeros", "normal"])
def test_decode_bgmv_full(y0):
    wl = make_workload(1, device=DEV, y0=y0)
    c = wl.calls[0]
    Y = c.Y.clone()
    _no_err(L.lora_bgmv(c.X, Y, c.pool, c.ids, c.scale))
    hp = host_pool(c.pool)
    y_exact = _f64(c.Y) + oracle.bgmv_delta(to_host(c.X), hp, c.ids_h, c.scale)
    got = _f64(Y)
    check_parity(got, y_exact, f"decode bgmv y0={y0}")
    check_rounded(got, y_exact, f"decode bgmv y0={y0}")


def test_prefill_sgmv_full_size_sampled_rows():
    wl = make_workload(2, device=DEV)
    c = wl.calls[0]
    N = c.X.shape[0]
    rows = _sample_rows(N, c.seg_off_h, n=192)
    Vh, Yh = _sgmv_roundtrip(c, rows)
    hp = host_pool(c.pool)
    X = to_host(c.X)
    Vref = oracle.sgmv_shrink(X, hp, c.seg_off_h, c.seg_ad_h, rows=rows, ld=Vh.shape[1])
    check_close_f32(Vh, Vref, "prefill shrink V")
    y_exact = _f64(c.Y)[rows] + oracle.sgmv_delta(X, hp, c.seg_off_h, c.seg_ad_h, c.scale, rows=rows)
    check_parity(Yh, y_exact, "prefill sgmv")
    check_rounded(Yh, y_exact, "prefill sgmv")


def test_mixed_rank_layer_every_row():
    wl = make_workload(3, device=DEV)
    for c in wl.calls:
        Y = c.Y.clone()
        _no_err(L.lora_bgmv(c.X, Y, c.pool, c.ids, c.scale))
        used = np.unique(c.ids_h[c.ids_h >= 0])
        hp, remap = compact_from_device_pool(c.pool, used)
        ids = np.where(c.ids_h >= 0, remap[np.maximum(c.ids_h, 0)], -1).astype(np.int32)
        y_exact = _f64(c.Y) + oracle.bgmv_delta(to_host(c.X), hp, ids, c.scale)
        check_parity(_f64(Y), y_exact, f"mixed-rank layer {c.name}")
        check_rounded(_f64(Y), y_exact, f"mixed-rank layer {c.name}")
        del Y
    del wl
    torch.cuda.empty_cache()


def test_diffusion_multi_sampled_rows():
    wl = make_workload(4, device=DEV)
    for i, c in enumerate(wl.calls):
        Y = c.Y.clone()
        _no_err(L.lora_apply_multi(c.X, Y, c.pool, c.req_off, c.ad_off, c.ad_id, c.ad_scale,
                                   max_ads_per_req=3))
        rows = _sample_rows(c.X.shape[0], c.req_off_h, n=128, seed=i)
        hp = host_pool(c.pool)
        d = oracle.apply_multi_delta(to_host(c.X), hp, c.req_off_h, c.ad_off_h, c.ad_id_h, c.ad_scale_h,
                                     rows=rows)
        check_parity(_f64(Y)[rows], _f64(c.Y)[rows] + d, f"diffusion multi {c.name}")
        check_rounded(_f64(Y)[rows], _f64(c.Y)[rows] + d, f"diffusion multi {c.name}")
