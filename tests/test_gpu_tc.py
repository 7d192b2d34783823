"""The tensor-core (tcgen05) path of the SGMV and multi-adapter ops, through the
C ABI, on shapes chosen to exercise every edge of its tiling: a d_in that is not a
multiple of the 64-column k-block, a d_out that is not a multiple of the 128-output
slice (nor of the 64-column y box), segment tails of 1..255 rows, empty segments,
rows outside every segment, mixed ranks 8..128, stacked adapters (duplicates,
empty lists) and y0 != 0.  Long items on average select this path."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import (DevPool, check_close_f32, check_parity, check_rounded, dev_bf16, rand_host_pool, rand_x,
                     scatter_pool, widen)
from workloads import to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _i32(a):
    return torch.tensor(np.asarray(a, np.int32), device=DEV)


@pytest.mark.parametrize("packed", [True, False])
@pytest.mark.parametrize("d_in,d_out", [(264, 200), (4096, 384), (128, 1000)])
def test_tc_sgmv_ragged(d_in, d_out, packed):
    """packed: adapters back to back (A rows fetched by TMA); else scattered with
    gaps, offsets not multiples of d_in (A rows gathered 16 bytes at a time)."""
    rng = np.random.default_rng(d_in + d_out)
    ranks = [8, 24, 128, 40, 64]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    if not packed:
        hp = scatter_pool(hp)
    lens = [130, 1, 255, 0, 128, 37, 300]
    ads = [2, 0, 4, 1, 3, 2, 1]
    start = 5
    seg_off = np.concatenate([[start], start + np.cumsum(lens)]).astype(np.int32)
    N = int(seg_off[-1]) + 11                     # rows before and after every segment
    assert N >= 64 * len(ads)                     # long segments on average: the tensor-core path
    X = rand_x(rng, N, d_in)
    Y0 = rand_x(rng, N, d_out)
    pool = DevPool(hp)
    V = torch.full((N, 128), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(dev_bf16(X), V, pool, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    Vh = to_host(V).astype(np.float64)
    Vref = oracle.sgmv_shrink(X, hp, seg_off, ads, ld=128)
    assert np.array_equal(np.isnan(Vh), np.isnan(Vref))
    m = ~np.isnan(Vref)
    check_close_f32(Vh[m], Vref[m], "tc shrink")
    Y = dev_bf16(Y0)
    ws = L.lora_sgmv_expand(torch.nan_to_num(V), Y, pool, _i32(seg_off), _i32(ads), 1.25)
    assert L.lora_get_error(ws) == 0
    got = widen(to_host(Y))
    check_parity(got, widen(Y0) + oracle.sgmv_delta(X, hp, seg_off, ads, 1.25), "tc sgmv")
    check_rounded(got, widen(Y0) + oracle.sgmv_delta(X, hp, seg_off, ads, 1.25), "tc sgmv")
    outside = np.r_[0:start, seg_off[-1]:N]
    assert np.array_equal(got[outside], widen(Y0)[outside])


@pytest.mark.parametrize("packed", [True, False])
def test_tc_multi_stacked_adapters(packed):
    rng = np.random.default_rng(7)
    d_in, d_out = 320, 272
    ranks = [8, 16, 32, 24, 32, 8]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    if not packed:
        hp = scatter_pool(hp)
    lens = [300, 0, 129, 64, 200]
    req_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = int(req_off[-1]) + 7                      # a few rows outside every request
    ad_lists = [[0, 5, 5, 2], [1], [], [3, 4, 0], [2, 1]]
    ad_off = np.concatenate([[0], np.cumsum([len(a) for a in ad_lists])]).astype(np.int32)
    ad_id = np.array([a for l in ad_lists for a in l], np.int32)
    ad_sc = rng.uniform(0.5, 1.0, len(ad_id)).astype(np.float32)
    X = rand_x(rng, N, d_in)
    Y0 = rand_x(rng, N, d_out)
    Y = dev_bf16(Y0)
    # max_ads_per_req * max_rank = 4 * 32 = 128: stacked ranks fit one tile
    ws = L.lora_apply_multi(dev_bf16(X), Y, DevPool(hp), _i32(req_off), _i32(ad_off), _i32(ad_id),
                            torch.tensor(ad_sc, device=DEV), max_ads_per_req=4)
    assert L.lora_get_error(ws) == 0
    got = widen(to_host(Y))
    check_parity(got, widen(Y0) + oracle.apply_multi_delta(X, hp, req_off, ad_off, ad_id, ad_sc), "tc multi")
    check_rounded(got, widen(Y0) + oracle.apply_multi_delta(X, hp, req_off, ad_off, ad_id, ad_sc), "tc multi")
    untouched = np.r_[req_off[1]:req_off[2], req_off[-1]:N, req_off[3]:req_off[3]]   # empty list, outside
    assert np.array_equal(got[req_off[2]:req_off[3]], widen(Y0)[req_off[2]:req_off[3]])  # request with no adapters
    assert np.array_equal(got[untouched], widen(Y0)[untouched])


def test_tc_bad_adapter_in_a_segment_is_skipped_and_reported():
    rng = np.random.default_rng(9)
    hp = rand_host_pool(rng, [16, 16], 128, 128)
    seg_off = np.array([0, 200, 400], np.int32)
    ads = np.array([1, 5], np.int32)               # 5 is out of range
    X = rand_x(rng, 400, 128)
    Y0 = rand_x(rng, 400, 128)
    pool = DevPool(hp)
    V = torch.zeros(400, 16, dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(dev_bf16(X), V, pool, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) & 4
    Y = dev_bf16(Y0)
    ws = L.lora_sgmv_expand(V, Y, pool, _i32(seg_off), _i32(ads), 1.0)
    err = L.lora_get_error(ws)
    assert err & 4 or err == 0                     # the shrink reported it; the expand skips it quietly
    got = widen(to_host(Y))
    assert np.array_equal(got[200:], widen(Y0)[200:])
    good = np.array([0, 200, 200], np.int32)
    check_parity(got[:200], widen(Y0)[:200] + oracle.sgmv_delta(X, hp, good, np.array([1, 0], np.int32), 1.0)[:200],
                 "tc sgmv with a bad segment")


@pytest.mark.parametrize("d_in", [192, 328])
def test_tc_more_tiles_than_ctas_every_row(d_in):
    """About 330 tiles of 128 rows, more than the CTAs of either shrink layout (two
    per SM for one pool; one per SM for three projections stacked past 128 ranks):
    every V entry and every output row of one projection against the oracle; the
    output bound holds at |y| up to several rms, where the expand's V precision
    shows (scale 1.5)."""
    rng = np.random.default_rng(d_in)
    ranks = [64, 16, 32, 64, 8, 40]
    hps = [rand_host_pool(rng, ranks, d_in, d) for d in (136, 64, 200)]
    lens = [7001, 5, 6900, 0, 8100, 12000, 7777]
    ads = [2, 0, 4, 1, 3, 5, 2]
    seg_off = np.concatenate([[3], 3 + np.cumsum(lens)]).astype(np.int32)
    N = int(seg_off[-1]) + 9
    X = rand_x(rng, N, d_in)
    Xd = dev_bf16(X)
    pools = [DevPool(hp) for hp in hps]
    # one pool (two CTAs per SM, 296 CTAs)
    V = torch.full((N, 64), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(Xd, V, pools[0], _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    Vref = oracle.sgmv_shrink(X, hps[0], seg_off, ads, ld=64)
    Vh = to_host(V).astype(np.float64)
    assert np.array_equal(np.isnan(Vh), np.isnan(Vref))
    m = ~np.isnan(Vref)
    check_close_f32(Vh[m], Vref[m], "many-tile shrink")
    # three projections, 192 stacked ranks
    W = torch.full((N, 192), float("nan"), dtype=torch.float32, device=DEV)
    ws, cols = L.lora_sgmv_shrink_proj(Xd, W, pools, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    Wh = to_host(W).astype(np.float64)
    for p, c in enumerate(cols):
        Vref = oracle.sgmv_shrink(X, hps[p], seg_off, ads, ld=64)
        got = Wh[:, c:c + 64]
        assert np.array_equal(np.isnan(got), np.isnan(Vref))
        m = ~np.isnan(Vref)
        check_close_f32(got[m], Vref[m], f"many-tile proj shrink p{p}")
    # and the outputs of one projection from the fused V
    Y0 = rand_x(rng, N, hps[2].d_out)
    Y = dev_bf16(Y0)
    ws = L.lora_sgmv_expand(torch.nan_to_num(W)[:, cols[2]:], Y, pools[2], _i32(seg_off), _i32(ads), 1.5)
    assert L.lora_get_error(ws) == 0
    check_parity(widen(to_host(Y)), widen(Y0) + oracle.sgmv_delta(X, hps[2], seg_off, ads, 1.5), "many-tile sgmv")
