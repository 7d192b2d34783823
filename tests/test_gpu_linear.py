"""The projection with its LoRA delta in one tensor-core pass (lora_linear_sgmv),
through the C ABI, against the oracle's unmerged projection: ragged shapes (d_in
not a multiple of the 64-column k-block, d_out not a multiple of the 256-output
slice), segment tails of 1..255 rows, empty segments, segments without an adapter
(-1), rows outside every segment (left untouched), every rank the fused path takes
(16, 32, 64, 128, mixed in one pool), a rank it does not take (reported, base
product only), and the full prefill shape on sampled rows."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import DevPool, check_parity, check_rounded, dev_bf16, rand_host_pool, rand_x, widen
from workloads import bf16_bits, to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _i32(a):
    return torch.tensor(np.asarray(a, np.int32), device=DEV)


def _rand_w(rng, d_out, d_in):
    """A base weight ~ N(0, 1/d_in) as bf16 bits: x W^T is O(1), like the delta."""
    return bf16_bits(rng.standard_normal((d_out, d_in)).astype(np.float32) / np.sqrt(d_in))


@pytest.mark.parametrize("d_in,d_out", [(328, 200), (256, 520), (4096, 264)])
def test_linear_ragged(d_in, d_out):
    rng = np.random.default_rng(d_in * 7 + d_out)
    ranks = [16, 32, 128, 64, 16]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    lens = [130, 1, 255, 0, 128, 37, 300, 64]
    ads = [2, 0, 4, 1, 3, -1, 1, 2]
    start = 5
    seg_off = np.concatenate([[start], start + np.cumsum(lens)]).astype(np.int32)
    N = int(seg_off[-1]) + 11
    X = rand_x(rng, N, d_in)
    W = _rand_w(rng, d_out, d_in)
    sentinel = np.full((N, d_out), 0x3F80, np.uint16)          # 1.0 everywhere
    Y = dev_bf16(sentinel)
    ws = L.lora_linear_sgmv(dev_bf16(X), dev_bf16(W), Y, DevPool(hp), _i32(seg_off), _i32(ads), 0.75)
    assert L.lora_get_error(ws) == 0
    got = widen(to_host(Y))
    inside = np.r_[seg_off[0]:seg_off[-1]]
    want = oracle.linear_sgmv(X, W, hp, seg_off, np.array(ads, np.int32), 0.75)
    check_parity(got[inside], want[inside], f"linear {d_in}x{d_out}")
    check_rounded(got[inside], want[inside], f"linear {d_in}x{d_out}")
    outside = np.r_[0:start, seg_off[-1]:N]
    assert np.all(got[outside] == 1.0)


@pytest.mark.parametrize("scatter", [False, True])
def test_linear_any_rank_multiple_of_8(scatter):
    """Ranks 8, 24, 40, 96 and 120 (no pool view: B gathered row by row) next to
    16/64/128 (views), mixed in one call -- and, on a scattered pool (offsets no
    longer multiples of the rank), every adapter through the gather -- against the
    oracle's x (W + s B_a A_a)^T."""
    from helpers import scatter_pool
    rng = np.random.default_rng(3 + scatter)
    d_in, d_out = 192, 264
    ranks = [8, 24, 40, 16, 96, 64, 120, 128]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    if scatter:
        hp = scatter_pool(hp)
    lens = [130, 200, 64, 150, 129, 90, 200, 140]
    seg_off = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    ads = np.arange(len(ranks), dtype=np.int32)
    N = int(seg_off[-1])
    X = rand_x(rng, N, d_in)
    W = _rand_w(rng, d_out, d_in)
    Y = torch.zeros((N, d_out), dtype=torch.bfloat16, device=DEV)
    ws = L.lora_linear_sgmv(dev_bf16(X), dev_bf16(W), Y, DevPool(hp), _i32(seg_off), _i32(ads), 1.5)
    assert L.lora_get_error(ws) == 0
    want = oracle.linear_sgmv(X, W, hp, seg_off, ads, 1.5)
    got = widen(to_host(Y))
    check_parity(got, want, f"linear, ranks {ranks} scatter={scatter}")
    check_rounded(got, want, f"linear, ranks {ranks} scatter={scatter}")


def test_linear_scale_zero_and_no_adapter_are_the_base_product():
    rng = np.random.default_rng(4)
    d_in, d_out = 128, 256
    hp = rand_host_pool(rng, [64, 16], d_in, d_out)
    seg_off = np.array([0, 300, 640], np.int32)
    X = rand_x(rng, 640, d_in)
    W = _rand_w(rng, d_out, d_in)
    base = oracle.linear_sgmv(X, W, hp, seg_off, np.array([-1, -1], np.int32), 0.0)
    for ads, s in (([0, 1], 0.0), ([-1, -1], 2.0)):
        Y = torch.zeros((640, d_out), dtype=torch.bfloat16, device=DEV)
        ws = L.lora_linear_sgmv(dev_bf16(X), dev_bf16(W), Y, DevPool(hp), _i32(seg_off), _i32(ads), s)
        assert L.lora_get_error(ws) == 0
        check_parity(widen(to_host(Y)), base, f"base product {ads} s={s}")


def test_prefill_linear_full_size_sampled_rows():
    """The bench's prefill_linear_up step (the same closure bench.py times): sampled
    rows of y = x W^T + s x A^T B^T against the oracle."""
    import bench
    from helpers import host_pool
    from workloads import make_workload
    wl = make_workload("prefill_linear_up", device=DEV)
    c = wl.calls[0]
    ws_map = {id(c): bench.workspace_for(c)}
    bench.make_step(wl, ws_map, torch.cuda.current_stream())()
    assert L.lora_get_error(ws_map[id(c)]) == 0
    N = c.X.shape[0]
    rng = np.random.default_rng(2)
    rows = np.sort(rng.choice(N, 96, replace=False)).astype(np.int32)
    want = oracle.linear_sgmv(to_host(c.X), to_host(c.W), host_pool(c.pool), c.seg_off_h, c.seg_ad_h, c.scale,
                              rows=rows)
    check_parity(widen(to_host(c.Y))[rows], want, "prefill_linear_up")
    check_rounded(widen(to_host(c.Y))[rows], want, "prefill_linear_up")


def test_linear_degenerate_segments():
    """Only empty segments: nothing is written and nothing is reported.  One row in one
    segment (a tile of one row, boxes reading past the end of x): that row is exact."""
    rng = np.random.default_rng(6)
    d_in, d_out = 64, 256
    hp = rand_host_pool(rng, [16, 32], d_in, d_out)
    W = _rand_w(rng, d_out, d_in)
    X = rand_x(rng, 100, d_in)
    sentinel = np.full((100, d_out), 0x4000, np.uint16)          # 2.0
    Y = dev_bf16(sentinel)
    ws = L.lora_linear_sgmv(dev_bf16(X), dev_bf16(W), Y, DevPool(hp), _i32([0, 0, 0]), _i32([0, 1]), 1.0)
    assert L.lora_get_error(ws) == 0
    assert np.all(widen(to_host(Y)) == 2.0)
    X1 = rand_x(rng, 1, d_in)
    Y1 = torch.zeros((1, d_out), dtype=torch.bfloat16, device=DEV)
    ws = L.lora_linear_sgmv(dev_bf16(X1), dev_bf16(W), Y1, DevPool(hp), _i32([0, 1]), _i32([1]), 0.5)
    assert L.lora_get_error(ws) == 0
    want = oracle.linear_sgmv(X1, W, hp, np.array([0, 1], np.int32), np.array([1], np.int32), 0.5)
    check_parity(widen(to_host(Y1)), want, "linear, one row")
