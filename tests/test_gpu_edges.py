"""GPU edge cases, routing and device-side error reporting, through the C ABI.

Routing is checked bit-exact twice: lora_route's permutation and segment
tables against the oracle's stable counting sort, and integer-coded adapters
whose every output spells the id of the adapter the kernel actually applied.
"""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import (DevPool, check_parity, dev_bf16, rand_host_pool, rand_x, widen)
from oracle_pins import integer_coded_expect, integer_coded_pool, integer_coded_x
from workloads import to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(t):
    torch.cuda.synchronize()
    return widen(to_host(t))


def _i32(a):
    return torch.tensor(np.asarray(a, np.int32), device=DEV)


@pytest.mark.parametrize("N,n_ad", [(1, 1), (31, 7), (256, 128), (512, 1000), (5000, 30000), (0, 5)])
def test_route_bit_exact(N, n_ad):
    rng = np.random.default_rng(N + n_ad)
    ids = rng.integers(-1, n_ad, N).astype(np.int32)
    cap = min(N, n_ad)
    perm = torch.full((max(N, 1),), -7, dtype=torch.int32, device=DEV)
    seg_off = torch.full((cap + 1,), -7, dtype=torch.int32, device=DEV)
    seg_ad = torch.full((max(cap, 1),), -7, dtype=torch.int32, device=DEV)
    n_seg = torch.zeros(1, dtype=torch.int32, device=DEV)
    ws = L.lora_route(_i32(ids) if N else torch.zeros(1, dtype=torch.int32, device=DEV)[:0], n_ad,
                      perm, seg_off, seg_ad, n_seg)
    assert L.lora_get_error(ws) == 0
    p_ref, so_ref, sa_ref = oracle.route(ids, n_ad)
    k = int(n_seg.item())
    assert k == len(sa_ref)
    assert np.array_equal(to_host(seg_ad)[:k], sa_ref)
    assert np.array_equal(to_host(seg_off)[:k + 1], so_ref)
    assert np.array_equal(to_host(perm)[:len(p_ref)], p_ref)


@pytest.mark.parametrize("n_ad,N,scale", [(300, 64, 2.0), (1000, 512, 1.0), (4, 1, 0.5)])
def test_integer_coded_bgmv_exact(n_ad, N, scale):
    rng = np.random.default_rng(n_ad)
    n_bits = int(np.ceil(np.log2(n_ad + 1)))
    ranks = rng.choice([8, 16, 32, 128], n_ad)
    hp = integer_coded_pool(n_ad, ranks, 64, 48, n_bits)
    pool = DevPool(hp)
    ids = rng.integers(-1, n_ad, N).astype(np.int32)
    X = dev_bf16(integer_coded_x(N, 64))
    Y = torch.zeros(N, 48, dtype=torch.bfloat16, device=DEV)
    ws = L.lora_bgmv(X, Y, pool, _i32(ids), scale)
    assert L.lora_get_error(ws) == 0
    assert np.array_equal(_f64(Y), integer_coded_expect(ids, 48, n_bits, scale))


def test_integer_coded_multi_exact():
    n_ad, n_bits = 40, 6
    hp = integer_coded_pool(n_ad, [8] * 20 + [16] * 20, 32, 24, n_bits)
    pool = DevPool(hp)
    N = 20
    X = dev_bf16(integer_coded_x(N, 32))
    req_off = np.array([0, 3, 3, 11, 20], np.int32)
    ad_off = np.array([0, 2, 3, 3, 6], np.int32)
    ad_id = np.array([5, 39, 7, 12, 12, 0], np.int32)
    ad_sc = np.array([1.0, 2.0, 0.5, 1.0, 0.25, 4.0], np.float32)
    Y = torch.zeros(N, 24, dtype=torch.bfloat16, device=DEV)
    ws = L.lora_apply_multi(X, Y, pool, _i32(req_off), _i32(ad_off), _i32(ad_id),
                            torch.tensor(ad_sc, device=DEV), max_ads_per_req=3)
    assert L.lora_get_error(ws) == 0
    want = np.zeros((N, 24))
    for q in range(4):
        for p in range(ad_off[q], ad_off[q + 1]):
            ids = np.full(N, -1, np.int32)
            ids[req_off[q]:req_off[q + 1]] = ad_id[p]
            want += integer_coded_expect(ids, 24, n_bits, float(ad_sc[p]))
    assert np.array_equal(_f64(Y), want)


def _ragged_case(seed=0, N=37, d_in=264, d_out=136, ranks=(8, 24, 128, 40, 16)):
    rng = np.random.default_rng(seed)
    hp = rand_host_pool(rng, list(ranks), d_in, d_out)
    X = rand_x(rng, N, d_in)
    Y0 = rand_x(rng, N, d_out)
    return rng, hp, X, Y0


def test_ragged_bgmv_with_no_adapter_rows():
    rng, hp, X, Y0 = _ragged_case()
    ids = rng.integers(-1, 5, 37).astype(np.int32)
    ids[:4] = [-1, 2, 2, -1]
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, DevPool(hp), _i32(ids), 1.5)
    assert L.lora_get_error(ws) == 0
    got = _f64(Y)
    check_parity(got, widen(Y0) + oracle.bgmv_delta(X, hp, ids, 1.5), "ragged bgmv")
    assert np.array_equal(got[ids == -1], widen(Y0)[ids == -1])


@pytest.mark.parametrize("d_out", [136, 4096])
def test_bgmv_every_rank(d_out):
    """Every rank the pool allows (8 .. 128 in steps of 8: one to four 32-rank blocks,
    the k16 path at ranks <= 16), with adapters used by 1 to 40 tokens (several
    16-token items per adapter), on the staged path (small d_out) and the unstaged one
    (d_out = 4096: the B chunk per CTA exceeds the shared-memory stage)."""
    rng = np.random.default_rng(7 + d_out)
    ranks = list(range(8, 129, 8))
    hp = rand_host_pool(rng, ranks, 520, d_out)
    n_ad = len(ranks)
    counts = np.concatenate([[40, 17, 16], rng.integers(1, 6, n_ad - 3)])
    ids = np.concatenate([np.full(c, a, np.int32) for a, c in enumerate(counts)] + [np.full(5, -1, np.int32)])
    ids = ids[rng.permutation(ids.size)]
    N = ids.size
    X = rand_x(rng, N, 520)
    Y0 = rand_x(rng, N, d_out)
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, DevPool(hp), _i32(ids), 0.75)
    assert L.lora_get_error(ws) == 0
    check_parity(_f64(Y), widen(Y0) + oracle.bgmv_delta(X, hp, ids, 0.75), f"bgmv every rank, d_out {d_out}")


def test_ragged_sgmv_empty_segments_and_uncovered_rows():
    rng, hp, X, Y0 = _ragged_case(1)
    seg_off = np.array([3, 3, 10, 11, 30, 30], np.int32)   # rows 0-2 and 30-36 outside
    seg_ad = np.array([4, 2, 0, 2, 1], np.int32)
    V = torch.full((37, 128), float("nan"), dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(dev_bf16(X), V, DevPool(hp), _i32(seg_off), _i32(seg_ad))
    assert L.lora_get_error(ws) == 0
    Vh = to_host(V).astype(np.float64)
    Vref = oracle.sgmv_shrink(X, hp, seg_off, seg_ad, ld=128)
    assert np.array_equal(np.isnan(Vh), np.isnan(Vref))
    Y = dev_bf16(Y0)
    ws = L.lora_sgmv_expand(torch.nan_to_num(V), Y, DevPool(hp), _i32(seg_off), _i32(seg_ad), -0.75)
    assert L.lora_get_error(ws) == 0
    got = _f64(Y)
    check_parity(got, widen(Y0) + oracle.sgmv_delta(X, hp, seg_off, seg_ad, -0.75), "ragged sgmv")
    assert np.array_equal(got[:3], widen(Y0)[:3]) and np.array_equal(got[30:], widen(Y0)[30:])


def test_ragged_multi_duplicates_and_empty_lists():
    rng, hp, X, Y0 = _ragged_case(2)
    req_off = np.array([0, 5, 5, 20, 33], np.int32)     # rows 33-36 outside
    ad_off = np.array([0, 3, 4, 4, 8], np.int32)        # request 2 has no adapter
    ad_id = np.array([1, 1, 4, 0, 2, 3, 0, 4], np.int32)
    ad_sc = rng.uniform(0.5, 1.0, 8).astype(np.float32)
    Y = dev_bf16(Y0)
    ws = L.lora_apply_multi(dev_bf16(X), Y, DevPool(hp), _i32(req_off), _i32(ad_off), _i32(ad_id),
                            torch.tensor(ad_sc, device=DEV), max_ads_per_req=4)
    assert L.lora_get_error(ws) == 0
    got = _f64(Y)
    check_parity(got, widen(Y0) + oracle.apply_multi_delta(X, hp, req_off, ad_off, ad_id, ad_sc), "ragged multi")
    assert np.array_equal(got[5:20], widen(Y0)[5:20]) and np.array_equal(got[33:], widen(Y0)[33:])


def test_strided_x_and_y():
    rng, hp, X, Y0 = _ragged_case(3, N=9)
    Xw = torch.zeros(9, 264 + 40, dtype=torch.bfloat16, device=DEV)
    Xw[:, :264] = dev_bf16(X)
    Yw = torch.zeros(9, 136 + 24, dtype=torch.bfloat16, device=DEV)
    Yw[:, :136] = dev_bf16(Y0)
    ids = np.array([0, 4, -1, 3, 3, 2, 1, 0, 4], np.int32)
    ws = L.lora_bgmv(Xw[:, :264], Yw[:, :136], DevPool(hp), _i32(ids), 2.0)
    assert L.lora_get_error(ws) == 0
    check_parity(_f64(Yw[:, :136].contiguous()), widen(Y0) + oracle.bgmv_delta(X, hp, ids, 2.0), "strided")
    assert torch.count_nonzero(Yw[:, 136:]).item() == 0


def test_deterministic():
    rng, hp, X, Y0 = _ragged_case(4, N=300)
    ids = rng.integers(0, 5, 300).astype(np.int32)
    outs = []
    for _ in range(2):
        Y = dev_bf16(Y0)
        L.lora_bgmv(dev_bf16(X), Y, DevPool(hp), _i32(ids), 1.0)
        outs.append(to_host(Y))
    assert np.array_equal(outs[0], outs[1])


def test_bad_adapter_id_sets_error_and_skips_only_that_row():
    rng, hp, X, Y0 = _ragged_case(5, N=12)
    ids = np.array([0, 1, 7, 2, -1, 3, 4, 0, -5, 1, 2, 3], np.int32)   # 7 and -5 are invalid
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, DevPool(hp), _i32(ids), 1.0)
    assert L.lora_get_error(ws) & 4
    assert L.lora_get_error(ws) == 0          # the read cleared it
    ok = (ids >= 0) & (ids < 5)
    got = _f64(Y)
    clean = np.where(ok, ids, -1).astype(np.int32)
    check_parity(got, widen(Y0) + oracle.bgmv_delta(X, hp, clean, 1.0), "bad id rows")
    assert np.array_equal(got[~ok], widen(Y0)[~ok])


def test_bad_rank_in_pool_sets_error():
    rng, hp, X, Y0 = _ragged_case(6, N=6)
    hp.rank = hp.rank.copy()
    hp.rank[1] = 12                           # not a multiple of 8
    ids = np.array([0, 1, 1, 2, 3, 4], np.int32)
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, DevPool(hp, max_rank=128), _i32(ids), 1.0)
    assert L.lora_get_error(ws) & 4
    got = _f64(Y)
    assert np.array_equal(got[1:3], widen(Y0)[1:3])


def test_bad_segments_set_error_and_change_nothing():
    rng, hp, X, Y0 = _ragged_case(7, N=10)
    Y = dev_bf16(Y0)
    ws = L.lora_sgmv_expand(torch.zeros(10, 128, device=DEV), Y, DevPool(hp), _i32([0, 6, 4]),
                            _i32([0, 1]), 1.0)
    assert L.lora_get_error(ws) & 8
    assert np.array_equal(_f64(Y), widen(Y0))
    ws = L.lora_apply_multi(dev_bf16(X), Y, DevPool(hp), _i32([0, 10]), _i32([0, 5]), _i32([0] * 5),
                            torch.ones(5, device=DEV), max_ads_per_req=3)   # 5 adapters > 3
    assert L.lora_get_error(ws) & 8
    assert np.array_equal(_f64(Y), widen(Y0))


@pytest.mark.parametrize("N,n_ad", [(9000, 40), (6000, 9000)])
def test_bgmv_three_kernel_path_beyond_fused_limits(N, n_ad):
    """Batches beyond the single-launch kernel's shared-memory limits take the
    plan/shrink/expand path; both must agree with the oracle."""
    assert L.lora_kernel_launches(L.OP_BGMV, N, n_ad, 64) == 3
    assert L.lora_kernel_launches(L.OP_BGMV, 256, 128, 4096) == 1
    rng = np.random.default_rng(N)
    ranks = rng.choice([8, 16, 32], n_ad)
    hp = rand_host_pool(rng, ranks, 64, 48)
    X = rand_x(rng, N, 64)
    Y0 = rand_x(rng, N, 48)
    ids = rng.integers(-1, n_ad, N).astype(np.int32)
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, DevPool(hp), _i32(ids), 0.5)
    assert L.lora_get_error(ws) == 0
    check_parity(_f64(Y), widen(Y0) + oracle.bgmv_delta(X, hp, ids, 0.5), f"3-kernel bgmv N={N}")


def test_output_ties_round_to_even():
    """Outputs that land exactly halfway between two bf16 values come back rounded to
    the even one (round to nearest even), through the decode path and the tensor-core
    SGMV path.  A[a] row 0 holds (256, v1) so v_0 = 256 + v1 exactly; B[a][o][0] = 1;
    scale 2^-8: y = y0 + (256 + v1) / 256, with v1 = 1 giving 1 + 2^-8 (a tie, even
    neighbour 1.0) and v1 = 3 giving 1 + 3 * 2^-8 (a tie, even neighbour 1 + 2^-6)."""
    from workloads import bf16_bits
    d_in, d_out, r = 64, 48, 8
    ranks = np.array([r, r], np.int32)
    A = np.zeros((2, r, d_in), np.float32)
    A[0, 0, 0], A[0, 0, 1] = 256.0, 1.0
    A[1, 0, 0], A[1, 0, 1] = 256.0, 3.0
    B = np.zeros((2, d_out, r), np.float32)
    B[:, :, 0] = 1.0
    hp = oracle.HostPool(A=bf16_bits(A.reshape(-1)), B=bf16_bits(B.reshape(-1)),
                         A_off=np.array([0, r * d_in], np.int64), B_off=np.array([0, r * d_out], np.int64),
                         rank=ranks, d_in=d_in, d_out=d_out)
    N = 300
    X = np.zeros((N, d_in), np.float32)
    X[:, 0] = X[:, 1] = 1.0
    Xb = bf16_bits(X)
    ids = (np.arange(N) % 2).astype(np.int32)
    want = np.where(ids[:, None] == 0, 1.0, 1.0 + 2.0 ** -6) * np.ones((1, d_out))
    # y0 = 0: the delta itself is the tie
    Y = torch.zeros(N, d_out, dtype=torch.bfloat16, device=DEV)
    ws = L.lora_bgmv(dev_bf16(Xb), Y, DevPool(hp), _i32(ids), 2.0 ** -8)
    assert L.lora_get_error(ws) == 0
    assert np.array_equal(_f64(Y), want)
    # the same through the SGMV tensor-core path (segments of 150 rows)
    order = np.argsort(ids, kind="stable")
    seg_off = np.array([0, 150, 300], np.int32)
    Xs = Xb[order]
    V = torch.zeros(N, r, dtype=torch.float32, device=DEV)
    ws = L.lora_sgmv_shrink(dev_bf16(Xs), V, DevPool(hp), _i32(seg_off), _i32([0, 1]))
    assert L.lora_get_error(ws) == 0
    Y = torch.zeros(N, d_out, dtype=torch.bfloat16, device=DEV)
    ws = L.lora_sgmv_expand(V, Y, DevPool(hp), _i32(seg_off), _i32([0, 1]), 2.0 ** -8)
    assert L.lora_get_error(ws) == 0
    assert np.array_equal(_f64(Y), want[order])
    # a nonzero y0 in the same pass: y = -2 - (256 + v1) / 256, rounded once
    Y0 = np.full((N, d_out), bf16_bits(np.float32(-2.0)), np.uint16)
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(Xb), Y, DevPool(hp), _i32(ids), -2.0 ** -8)
    assert L.lora_get_error(ws) == 0
    exact = -2.0 - np.where(ids[:, None] == 0, 257.0, 259.0) / 256.0 * np.ones((1, d_out))
    assert np.array_equal(_f64(Y), oracle.round_bf16(exact))
