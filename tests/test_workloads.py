"""The seeded generators: deterministic, the stated shapes, and metadata that
satisfies each op's contract (sorted segments, CSR bounds, Zipf skew)."""
import numpy as np
import torch

from workloads import make_workload, zipf_ids, make_pool


def test_deterministic_and_shapes():
    a = make_workload(0)
    b = make_workload(0)
    ca, cb = a.calls[0], b.calls[0]
    assert torch.equal(ca.X, cb.X) and torch.equal(ca.pool.A, cb.pool.A)
    assert ca.X.shape == (64, 256) and ca.pool.ranks_h.tolist() == [8] * 4
    so = ca.seg_off_h
    assert so[0] == 0 and so[-1] == 64 and np.all(np.diff(so) >= 0) and len(ca.seg_ad_h) == 4


def test_zipf_is_heavy_tailed():
    rng = np.random.Generator(np.random.PCG64(0))
    ids = zipf_ids(rng, 128, 1.1, 200000)
    cnt = np.bincount(ids, minlength=128)
    p = np.arange(1, 129) ** -1.1
    p /= p.sum()
    assert abs(cnt[0] / 200000 - p[0]) < 0.01
    assert cnt[0] > cnt[1] > cnt[10] > cnt[100]


def test_small_variants_of_each_workload():
    wl = make_workload(1, N=32, d=64, n_adapters=8)
    c = wl.calls[0]
    assert c.X.shape == (32, 64) and c.ids_h.min() >= 0 and c.ids_h.max() < 8
    wl = make_workload(2, n_req=4, len_range=(3, 9), d_in=32, d_out=48, rank=16, n_adapters=5)
    c = wl.calls[0]
    assert c.seg_off_h[-1] == c.X.shape[0] and np.all(np.diff(c.seg_ad_h) > 0)
    wl = make_workload(3, N=16, n_adapters=20, dim_div=64)
    assert len(wl.calls) == 7 and all(cc.pool.ranks_h.tolist() == wl.calls[0].pool.ranks_h.tolist()
                                       for cc in wl.calls)
    assert wl.calls[0].X.data_ptr() == wl.calls[1].X.data_ptr()  # q, k share their input
    wl = make_workload(4, n_img=5, tokens_per_img=8, d=32, n_adapters=10)
    c = wl.calls[0]
    k = np.diff(c.ad_off_h)
    assert np.all((k >= 1) & (k <= 3)) and np.all((c.ad_scale_h >= 0.5) & (c.ad_scale_h <= 1.0))
    for q in range(5):
        ids = c.ad_id_h[c.ad_off_h[q]:c.ad_off_h[q + 1]]
        assert len(set(ids.tolist())) == len(ids)


def test_pool_layout_packed_without_padding():
    p = make_pool([8, 128, 16], 32, 24, seed=3)
    assert p.A_off_h.tolist() == [0, 8 * 32, (8 + 128) * 32]
    assert p.B_off_h.tolist() == [0, 8 * 24, (8 + 128) * 24]
    assert p.A.numel() == (8 + 128 + 16) * 32
    B1 = p.adapter_B(1).float()
    assert abs(B1.std().item() - 128 ** -0.5) < 0.02


def test_merge_workload_shapes():
    wl = make_workload("merge_mlp_up", d_in=64, d_out=32, rank=16, n_adapters=4)
    c = wl.calls[0]
    assert tuple(c.W.shape) == (32, 64) and c.W.dtype == torch.bfloat16
    assert 0 <= c.adapter < 4 and wl.n_tokens == 32
    from adapter_gemv_sgmv_b200 import accounting
    cost = accounting.workload_cost(wl)
    assert cost.bytes == 2 * 2 * 32 * 64 + 2 * 16 * (64 + 32) and cost.flops == 2 * 32 * 64 * 16



def test_qkv_workload_shares_x_and_counts_it_once():
    wl = make_workload("prefill_qkv", n_req=3, len_range=(4, 9), d_in=64, d_outs=(64, 16, 16), rank=8,
                       n_adapters=5)
    q, k, v = wl.calls
    assert q.X.data_ptr() == k.X.data_ptr() == v.X.data_ptr()
    assert [c.pool.d_out for c in wl.calls] == [64, 16, 16]
    assert np.array_equal(q.seg_off_h, v.seg_off_h) and np.array_equal(q.seg_ad_h, k.seg_ad_h)
    assert q.seg_off_h[-1] == wl.n_tokens == q.X.shape[0]
    from adapter_gemv_sgmv_b200 import accounting
    N = wl.n_tokens
    separate = sum(accounting.call_cost(c).bytes for c in wl.calls)
    assert accounting.workload_cost(wl).bytes == separate - 2 * 2 * N * 64
    assert accounting.workload_cost(wl).tokens == N


def test_bench_counts_the_fused_calls():
    """Launch counts the bench claims for the shared-input and fused-projection steps
    follow the library's own rule (one tensor-core shrink per run of projections whose
    max ranks sum to at most 256)."""
    import bench
    assert bench.shrink_proj_passes([64, 64, 64]) == 1
    assert bench.shrink_proj_passes([128, 128, 128]) == 2
    assert bench.shrink_proj_passes([128, 8, 128]) == 2
    assert bench.shrink_proj_passes([16, 16, 16, 16]) == 1
    wl = make_workload("prefill_qkv", n_req=3, len_range=(200, 300), d_in=64, d_outs=(64, 16, 16), rank=8,
                       n_adapters=5)
    assert bench.launches_per_step(wl) == 1 + 1 + 1              # one plan, one shrink, one expand launch
    wl = make_workload("prefill_linear_up", n_req=3, len_range=(4, 9), d_in=64, d_out=48, rank=16,
                       n_adapters=5)
    assert bench._is_linear(wl.calls[0]) and bench.launches_per_step(wl) == 3
    merge = make_workload("merge_mlp_up", d_in=64, d_out=32, rank=16, n_adapters=4).calls[0]
    assert not bench._is_linear(merge)
