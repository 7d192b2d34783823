"""lora_merge on the GPU against the oracle: W <- bf16(W + s B_a A_a) in place.

Shapes exercise both expand paths (d_out >= 128: tcgen05 tiles with A^T by TMA
for ranks 16/32/64/128 and by cp.async otherwise; d_out < 128: CUDA cores),
ragged d_in / d_out, packed and scattered pools, a large scale (the update then
dominates W, so errors of the product itself show), merge then unmerge, an
invalid adapter, and the full-size up-projection weight on sampled rows."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import DevPool, dev_bf16, half_ulp_bf16, rand_host_pool, rand_x, scatter_pool, widen
from workloads import make_workload, to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _check_merge(got, exact, what):
    """One bf16 rounding of the exact result: within half an ulp plus fp32 accumulation
    slack everywhere, and the correctly rounded value for >= 99 % of the elements."""
    got = np.asarray(got, np.float64)
    exact = np.asarray(exact, np.float64)
    rnd = oracle.round_bf16(exact)
    bound = half_ulp_bf16(exact) + 1e-4 * (np.sqrt(np.mean(exact ** 2)) + 1e-30)
    bad = np.abs(got - exact) > bound
    assert not bad.any(), f"{what}: {int(bad.sum())} elements off, worst {np.max(np.abs(got - exact)):.3e}"
    frac = float(np.mean(got == rnd))
    assert frac >= 0.99, f"{what}: only {frac:.4f} correctly rounded"


@pytest.mark.parametrize("packed", [True, False])
@pytest.mark.parametrize("d_in,d_out", [(264, 200), (4096, 384), (128, 64)])
def test_merge_matches_oracle(d_in, d_out, packed):
    rng = np.random.default_rng(d_in * 7 + d_out)
    ranks = [8, 24, 64, 128, 16, 32]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    if not packed:
        hp = scatter_pool(hp)
    pool = DevPool(hp)
    W0 = (rand_x(rng, d_out, d_in))
    for a, s in enumerate([1.0, -0.75, 2.5, 0.5, -1.25, 1.5]):
        W = dev_bf16(W0)
        ws = L.lora_merge(W, pool, a, s)
        assert L.lora_get_error(ws) == 0
        _check_merge(widen(to_host(W)), oracle.merge(W0, hp, a, s), f"merge a={a} r={ranks[a]}")


def test_merge_large_scale_shows_the_product():
    """With s = 64 the update dwarfs W: the merged weight is checked against the exact
    product to the same bf16-rounding bar, so an error in B A itself would show."""
    rng = np.random.default_rng(11)
    hp = rand_host_pool(rng, [64, 16], 512, 256)
    pool = DevPool(hp)
    W0 = rand_x(rng, 256, 512)
    for a in (0, 1):
        W = dev_bf16(W0)
        L.lora_merge(W, pool, a, 64.0)
        _check_merge(widen(to_host(W)), oracle.merge(W0, hp, a, 64.0), "large scale")


def test_merge_then_unmerge_restores_within_rounding():
    rng = np.random.default_rng(12)
    hp = rand_host_pool(rng, [32], 384, 256)
    pool = DevPool(hp)
    W0 = rand_x(rng, 256, 384)
    W = dev_bf16(W0)
    L.lora_merge(W, pool, 0, 0.9)
    L.lora_merge(W, pool, 0, -0.9)
    got = widen(to_host(W))
    w0 = widen(W0)
    # two roundings of a value near W: within one bf16 ulp of W each way
    assert np.all(np.abs(got - w0) <= 2.0 ** -7 * np.abs(w0) + 2.0 ** -7 * np.sqrt(np.mean(w0 ** 2)))


def test_merge_invalid_adapter_leaves_w_and_reports():
    rng = np.random.default_rng(13)
    hp = rand_host_pool(rng, [16, 16], 256, 256)
    hp.rank[1] = 12                                   # not a multiple of 8: rejected on the device
    pool = DevPool(hp, max_rank=16)
    W0 = rand_x(rng, 256, 256)
    W = dev_bf16(W0)
    ws = L.lora_merge(W, pool, 1, 1.0)
    assert L.lora_get_error(ws) & 4
    assert np.array_equal(to_host(W), W0)
    L.lora_workspace_init(ws)


def test_merge_full_size_sampled_rows():
    """The up-projection weight [14336, 4096] with a rank-64 adapter; 24 sampled rows."""
    wl = make_workload("merge_mlp_up", device=DEV)
    c = wl.calls[0]
    rows = np.sort(np.random.default_rng(0).choice(c.pool.d_out, 24, replace=False)).astype(np.int32)
    W0_rows = to_host(c.W[torch.from_numpy(rows).long().to(DEV)])
    hp, remap = oracle.host_pool_subset(c.pool, [c.adapter])
    W0 = np.zeros((c.pool.d_out, c.pool.d_in), np.uint16)
    W0[rows] = W0_rows
    ws = L.lora_merge(c.W, c.pool, c.adapter, c.scale)
    assert L.lora_get_error(ws) == 0
    got = widen(to_host(c.W[torch.from_numpy(rows).long().to(DEV)]))
    _check_merge(got, oracle.merge(W0, hp, int(remap[c.adapter]), c.scale, rows=rows), "full-size merge")
