"""Projections that share an input (Q, K, V; gate, up): lora_sgmv_shrink_proj
reads X once for all of them, and each projection's expand then reads its own
columns of V.  Compared with the oracle's per-projection shrink and delta, on
pools that differ in d_out, ranks, storage (packed or scattered) and max_rank,
covering the stacked-rank cases: up to 128 (two CTAs per SM), up to 256 (one
wide accumulator), above 256 (split into launches) and short segments (the
CUDA-core shrink, once per projection)."""
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


# per projection: (d_out, ranks of the 5 adapters); the max ranks set the stacking
CASES = {
    "qkv_r64": [(384, [64, 8, 64, 16, 40]), (128, [64, 8, 64, 16, 40]), (128, [32, 8, 64, 16, 40])],
    "qkv_r128": [(264, [128, 8, 24, 64, 128]), (136, [128, 16, 8, 64, 128]), (200, [128, 8, 24, 64, 128])],
    "gate_up_r128": [(1000, [128, 8, 64, 128, 32]), (1000, [128, 8, 64, 128, 32])],
    "four_r16": [(128, [16, 8, 16, 16, 8]), (128, [16, 8, 16, 16, 8]), (128, [8, 8, 16, 16, 8]),
                 (64, [16, 8, 16, 8, 8])],
}


def _segments(long: bool):
    if long:
        lens, ads = [130, 1, 255, 0, 128, 37, 300], [2, 0, 4, 1, 3, 2, 1]
    else:
        lens, ads = [3, 1, 9, 0, 17, 5, 2], [2, 0, 4, 1, 3, 2, 1]
    start = 5
    seg_off = np.concatenate([[start], start + np.cumsum(lens)]).astype(np.int32)
    return seg_off, np.array(ads, np.int32), int(seg_off[-1]) + 11


@pytest.mark.parametrize("packed", [True, False])
@pytest.mark.parametrize("long", [True, False])
@pytest.mark.parametrize("case", sorted(CASES))
def test_shrink_proj_and_expands(case, long, packed):
    rng = np.random.default_rng(len(case) * 7 + long + 2 * packed)
    d_in = 328                                     # not a multiple of the 64-column k-block
    hps = []
    for d_out, ranks in CASES[case]:
        hp = rand_host_pool(rng, ranks, d_in, d_out)
        hps.append(hp if packed else scatter_pool(hp))
    seg_off, ads, N = _segments(long)
    assert (N >= 64 * len(ads)) == long            # long segments select the tensor-core path
    X = rand_x(rng, N, d_in)
    pools = [DevPool(hp) for hp in hps]
    width = sum(p.max_rank for p in pools)
    V = torch.full((N, width + 8), float("nan"), dtype=torch.float32, device=DEV)
    ws, cols = L.lora_sgmv_shrink_proj(dev_bf16(X), V, pools, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    assert cols == list(np.cumsum([0] + [p.max_rank for p in pools])[:-1])
    Vh = to_host(V).astype(np.float64)
    assert np.isnan(Vh[:, width:]).all()           # nothing written past the last projection
    for p, (hp, c) in enumerate(zip(hps, cols)):
        mr = pools[p].max_rank
        Vref = oracle.sgmv_shrink(X, hp, seg_off, ads, ld=mr)
        got = Vh[:, c:c + mr]
        assert np.array_equal(np.isnan(got), np.isnan(Vref)), f"projection {p}: written entries"
        m = ~np.isnan(Vref)
        check_close_f32(got[m], Vref[m], f"proj shrink {case} p{p}")
    # each projection's expand from its own columns of V
    Vz = torch.nan_to_num(V)
    for p, (hp, c) in enumerate(zip(hps, cols)):
        Y0 = rand_x(rng, N, hp.d_out)
        Y = dev_bf16(Y0)
        ws = L.lora_sgmv_expand(Vz[:, c:], Y, pools[p], _i32(seg_off), _i32(ads), 0.75)
        assert L.lora_get_error(ws) == 0
        check_parity(widen(to_host(Y)), widen(Y0) + oracle.sgmv_delta(X, hp, seg_off, ads, 0.75),
                     f"proj {case} p{p}")


def test_shrink_proj_bad_adapter_is_skipped_and_reported():
    rng = np.random.default_rng(11)
    d_in = 256
    hps = [rand_host_pool(rng, [64, 32, 64, 64, 8], d_in, 128) for _ in range(3)]
    seg_off, ads, N = _segments(True)
    ads = ads.copy()
    ads[2] = 9                                      # out of range in every pool
    X = rand_x(rng, N, d_in)
    pools = [DevPool(hp) for hp in hps]
    V = torch.full((N, 192), float("nan"), dtype=torch.float32, device=DEV)
    ws, cols = L.lora_sgmv_shrink_proj(dev_bf16(X), V, pools, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 4                # LORA_ERR_BAD_ADAPTER
    Vh = to_host(V).astype(np.float64)
    good = np.ones(len(ads), bool)
    good[2] = False
    for p, (hp, c) in enumerate(zip(hps, cols)):
        Vref = oracle.sgmv_shrink(X, hp, seg_off, np.where(good, ads, 0), ld=64)
        for k in range(len(ads)):
            rows = slice(seg_off[k], seg_off[k + 1])
            if good[k]:
                m = ~np.isnan(Vref[rows])
                check_close_f32(Vh[rows, c:c + 64][m], Vref[rows][m], f"proj p{p} segment {k}")
            else:
                assert np.isnan(Vh[rows, c:c + 64]).all()


def test_shrink_proj_equals_separate_shrinks_at_full_size():
    """Prefill shape (4096 -> Q 4096, K 1024, V 1024 at rank 64, 8 segments): the fused
    shrink and three separate shrinks take the same products in the same k-block
    order, so their V's agree to a few fp32 roundings."""
    rng = np.random.default_rng(5)
    d_in, n_ad = 4096, 8
    hps = [rand_host_pool(rng, [64] * n_ad, d_in, d) for d in (4096, 1024, 1024)]
    lens = rng.integers(256, 2048, n_ad)
    seg_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    N = int(seg_off[-1])
    ads = rng.permutation(n_ad).astype(np.int32)
    X = dev_bf16(rand_x(rng, N, d_in))
    pools = [DevPool(hp) for hp in hps]
    V = torch.zeros((N, 192), dtype=torch.float32, device=DEV)
    ws, cols = L.lora_sgmv_shrink_proj(X, V, pools, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    for p, c in enumerate(cols):
        Vs = torch.zeros((N, 64), dtype=torch.float32, device=DEV)
        ws = L.lora_sgmv_shrink(X, Vs, pools[p], _i32(seg_off), _i32(ads))
        assert L.lora_get_error(ws) == 0
        diff = float((V[:, c:c + 64] - Vs).abs().max())
        assert diff <= 1e-5 * float(Vs.abs().max()), f"projection {p}: {diff}"
    # and sampled rows against the oracle
    rows = np.sort(rng.choice(N, 64, replace=False)).astype(np.int32)
    Xh = to_host(X)
    for p, c in enumerate(cols):
        Vref = oracle.sgmv_shrink(Xh, hps[p], seg_off, ads, rows=rows, ld=64)
        check_close_f32(to_host(V[:, c:c + 64]).astype(np.float64)[rows], Vref, f"sampled p{p}")


def test_prefill_qkv_full_size_sampled_rows():
    """The bench's prefill_qkv step (the same closure bench.py times) at full size:
    sampled rows of every projection's output against the oracle."""
    import bench
    from helpers import host_pool
    from workloads import make_workload
    wl = make_workload("prefill_qkv", device=DEV)
    Y0 = [to_host(c.Y) for c in wl.calls]
    ws_map = {id(c): bench.workspace_for(c) for c in wl.calls}
    stream = torch.cuda.current_stream()
    bench.make_step(wl, ws_map, stream)()
    for ws in ws_map.values():
        assert L.lora_get_error(ws) == 0
    c0 = wl.calls[0]
    N = c0.X.shape[0]
    rng = np.random.default_rng(1)
    rows = np.sort(rng.choice(N, 160, replace=False)).astype(np.int32)
    X = to_host(c0.X)
    for c, y0 in zip(wl.calls, Y0):
        hp = host_pool(c.pool)
        y_exact = widen(y0)[rows] + oracle.sgmv_delta(X, hp, c.seg_off_h, c.seg_ad_h, c.scale, rows=rows)
        check_parity(widen(to_host(c.Y))[rows], y_exact, f"prefill_qkv {c.name}")
        check_rounded(widen(to_host(c.Y))[rows], y_exact, f"prefill_qkv {c.name}")


def test_shrink_proj_only_empty_segments_writes_nothing():
    rng = np.random.default_rng(12)
    hps = [rand_host_pool(rng, [64, 64], 128, d) for d in (128, 64, 64)]
    N = 300
    X = rand_x(rng, N, 128)
    V = torch.full((N, 192), float("nan"), dtype=torch.float32, device=DEV)
    ws, _ = L.lora_sgmv_shrink_proj(dev_bf16(X), V, [DevPool(hp) for hp in hps], _i32([0, 0, 0]), _i32([0, 1]))
    assert L.lora_get_error(ws) == 0
    assert torch.isnan(V).all()


@pytest.mark.parametrize("long", [True, False])
@pytest.mark.parametrize("case", ["qkv_r64", "qkv_r128", "four_r16"])
def test_apply_proj_every_output(case, long):
    """One call for the whole delta of projections sharing X: each projection's y against
    the oracle's delta, with its own scale; rows outside every segment untouched."""
    rng = np.random.default_rng(len(case) * 11 + long)
    d_in = 328
    hps = [rand_host_pool(rng, ranks, d_in, d_out) for d_out, ranks in CASES[case]]
    seg_off, ads, N = _segments(long)
    X = rand_x(rng, N, d_in)
    Y0 = [rand_x(rng, N, hp.d_out) for hp in hps]
    Ys = [dev_bf16(y) for y in Y0]
    scales = [0.5 + 0.25 * p for p in range(len(hps))]
    ws = L.lora_sgmv_apply_proj(dev_bf16(X), Ys, [DevPool(hp) for hp in hps], _i32(seg_off), _i32(ads), scales)
    assert L.lora_get_error(ws) == 0
    outside = np.r_[0:seg_off[0], seg_off[-1]:N]
    for p, (hp, y0, Y) in enumerate(zip(hps, Y0, Ys)):
        got = widen(to_host(Y))
        want = widen(y0) + oracle.sgmv_delta(X, hp, seg_off, ads, scales[p])
        check_parity(got, want, f"apply {case} p{p}")
        check_rounded(got, want, f"apply {case} p{p}")
        assert np.array_equal(got[outside], widen(y0)[outside])
