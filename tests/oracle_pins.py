"""The oracle's pins: facts fixed by the pages and by mathematics, checked
against something other than the oracle itself.

Each pin takes an ``oracle.Oracle`` and raises AssertionError when it fails,
so the same battery runs against the real oracle (test_oracle_pins.py) and
against deliberately broken builds of it (test_oracle_mutants.py).

Sources of the facts (all on "Serving several LoRAs, ControlNet and
IP-Adapter", section "LoRA: merged or alongside", unless stated):
* W' = W + BA with A r x d, B d x r; unmerged each layer adds x A^T B^T
  to x W^T  -> dense special case, merged-weight identity, zero B.
* the LoRA weight is a runtime scalar swapped per step -> linearity in s.
* exercise 2's answer (tokens sorted stably by adapter, one kernel over all
  runs, results returned in token order; tokens sharing an adapter share a
  run) -> permutation invariance, segment-split independence, SGMV == BGMV,
  the stable grouping (route) and integer-coded routing.
* table row "Stacking several LoRAs": a few more alongside computations
  -> additivity and rank stacking.
* merging folds s B A into W (and switching unmerges it) -> the merge pins.
"""
from __future__ import annotations

import numpy as np

from oracle import HostPool, OracleError
from helpers import (A_of, B_of, numpy_delta_rows, rand_host_pool, rand_x, widen)

TIGHT = 1e-12


def _close(got, want, rel=TIGHT):
    got = np.asarray(got, np.float64)
    want = np.asarray(want, np.float64)
    assert got.shape == want.shape, (got.shape, want.shape)
    scale = max(float(np.max(np.abs(want))) if want.size else 0.0, 1e-300)
    err = float(np.max(np.abs(got - want))) if want.size else 0.0
    assert err <= rel * scale, f"max err {err:.3e} > {rel:.0e} * {scale:.3e}"


def pin_dense_single_adapter(orc):
    """One adapter over the whole batch is one dense product s * X A^T B^T
    (numpy float64 matmul), for BGMV, SGMV and multi alike.  d_in != d_out
    and a rank distinct from both, so a transposed operand cannot pass."""
    rng = np.random.default_rng(1)
    N, d_in, d_out, r, s = 13, 40, 24, 16, 0.75
    p = rand_host_pool(rng, [r], d_in, d_out)
    X = rand_x(rng, N, d_in)
    want = s * (widen(X) @ A_of(p, 0).T) @ B_of(p, 0).T
    _close(orc.bgmv_delta(X, p, np.zeros(N, np.int32), s), want)
    _close(orc.sgmv_delta(X, p, np.array([0, N], np.int32), np.array([0], np.int32), s), want)
    _close(orc.apply_multi_delta(X, p, np.array([0, N], np.int32), np.array([0, 1], np.int32),
                                 np.array([0], np.int32), np.array([s], np.float32)), want)


def pin_merged_weight_identity(orc):
    """x (W + s B_a A_a)^T - x W^T equals the unmerged delta, per token."""
    rng = np.random.default_rng(2)
    N, d_in, d_out = 11, 32, 48
    ranks = [8, 24, 16]
    s = 1.5
    p = rand_host_pool(rng, ranks, d_in, d_out)
    X = rand_x(rng, N, d_in)
    ids = rng.integers(0, len(ranks), N).astype(np.int32)
    W = rng.standard_normal((d_out, d_in))
    D = orc.bgmv_delta(X, p, ids, s)
    Xd = widen(X)
    for n in range(N):
        a = ids[n]
        Wm = W + s * (B_of(p, a) @ A_of(p, a))
        want = Xd[n] @ Wm.T - Xd[n] @ W.T
        assert np.max(np.abs(D[n] - want)) <= 1e-10 * max(1.0, np.max(np.abs(want)))


def pin_mixed_ranks_per_token(orc):
    """Mixed ranks, ids in any order, id -1 = no adapter: each row equals the
    numpy product with that row's own adapter."""
    rng = np.random.default_rng(3)
    N, d_in, d_out = 29, 24, 40
    ranks = [8, 24, 128, 16, 40]
    p = rand_host_pool(rng, ranks, d_in, d_out)
    X = rand_x(rng, N, d_in)
    ids = rng.integers(-1, len(ranks), N).astype(np.int32)
    ids[:3] = [-1, 2, 4]
    s = 2.0
    _close(orc.bgmv_delta(X, p, ids, s), numpy_delta_rows(X, p, ids, s))
    assert np.all(orc.bgmv_delta(X, p, ids, s)[ids == -1] == 0.0)


def pin_merge_is_the_dense_rank_r_update(orc):
    """Merging adapter a into W is W + s B_a A_a (numpy float64 matmul), on every row
    or on a subset of rows; d_in != d_out != rank so a transposed operand fails."""
    rng = np.random.default_rng(21)
    d_in, d_out = 40, 24
    p = rand_host_pool(rng, [8, 16, 24], d_in, d_out)
    W = rand_x(rng, d_out, d_in)
    for a, s in ((1, 0.75), (2, -1.25)):
        want = widen(W) + s * (B_of(p, a) @ A_of(p, a))
        _close(orc.merge(W, p, a, s), want)
        rows = np.array([5, 0, 23], np.int32)
        _close(orc.merge(W, p, a, s, rows=rows), want[rows])


def pin_merge_agrees_with_the_unmerged_delta(orc):
    """The merged-weight identity through the oracle's two paths: x Wm^T - x W^T
    (merge) equals the unmerged delta s B_a A_a x (bgmv) for every token."""
    rng = np.random.default_rng(22)
    N, d_in, d_out = 9, 32, 48
    p = rand_host_pool(rng, [16, 8], d_in, d_out)
    W = rand_x(rng, d_out, d_in)
    X = rand_x(rng, N, d_in)
    for a, s in ((0, 1.5), (1, 0.5)):
        Wm = orc.merge(W, p, a, s)
        via_merge = widen(X) @ Wm.T - widen(X) @ widen(W).T
        delta = orc.bgmv_delta(X, p, np.full(N, a, np.int32), s)
        _close(via_merge, delta, rel=1e-10)


def pin_merge_zero_B_and_unmerge(orc):
    """B = 0 leaves W exactly as it was; merging with s and with -s averages to W."""
    rng = np.random.default_rng(23)
    p0 = rand_host_pool(rng, [8], 16, 24, zero_B=True)
    W = rand_x(rng, 24, 16)
    assert np.array_equal(orc.merge(W, p0, 0, 2.0), widen(W))
    p = rand_host_pool(rng, [8], 16, 24)
    _close(0.5 * (orc.merge(W, p, 0, 0.7) + orc.merge(W, p, 0, -0.7)), widen(W))


def pin_zero_B(orc):
    """B = 0 gives a delta of exactly zero."""
    rng = np.random.default_rng(4)
    p = rand_host_pool(rng, [8, 16], 16, 24, zero_B=True)
    X = rand_x(rng, 7, 16)
    ids = np.array([0, 1, 1, 0, -1, 1, 0], np.int32)
    assert np.all(orc.bgmv_delta(X, p, ids, 3.0) == 0.0)
    assert np.all(orc.apply_multi_delta(X, p, np.array([0, 7], np.int32), np.array([0, 2], np.int32),
                                        np.array([0, 1], np.int32), np.array([1.0, 2.0], np.float32)) == 0.0)


def pin_scale_linearity(orc):
    """The weight is a plain multiplier: s = 2 doubles and s = -0.5 negates and
    halves the delta bit for bit (powers of two are exact)."""
    rng = np.random.default_rng(5)
    p = rand_host_pool(rng, [16, 8], 32, 16)
    X = rand_x(rng, 9, 32)
    ids = rng.integers(0, 2, 9).astype(np.int32)
    d1 = orc.bgmv_delta(X, p, ids, 1.0)
    assert np.array_equal(orc.bgmv_delta(X, p, ids, 2.0), 2.0 * d1)
    assert np.array_equal(orc.bgmv_delta(X, p, ids, -0.5), -0.5 * d1)
    assert np.max(np.abs(d1)) > 0


def pin_permutation_invariance(orc):
    """Results go back in the original order: permuting tokens (with their ids)
    permutes the output rows exactly."""
    rng = np.random.default_rng(6)
    p = rand_host_pool(rng, [8, 16, 8, 32], 24, 40)
    N = 31
    X = rand_x(rng, N, 24)
    ids = rng.integers(-1, 4, N).astype(np.int32)
    D = orc.bgmv_delta(X, p, ids, 1.25)
    perm = rng.permutation(N)
    Dp = orc.bgmv_delta(X[perm], p, ids[perm], 1.25)
    assert np.array_equal(Dp, D[perm])


def integer_coded_pool(n_adapters: int, ranks, d_in: int, d_out: int, n_bits: int) -> HostPool:
    """Adapters whose output spells their id: x = e_0 + e_1 gives v_0 = v_1 = 1,
    and B[a][o] = (1 + bit_{o mod n_bits}(a), 1) so delta[o] = s*(2 + bit).
    Every value is a small integer, exact in bf16, fp32 and fp64."""
    ranks = np.asarray(ranks, np.int32)
    A_off = np.zeros(n_adapters, np.int64)
    B_off = np.zeros(n_adapters, np.int64)
    A_off[1:] = np.cumsum(ranks.astype(np.int64) * d_in)[:-1]
    B_off[1:] = np.cumsum(ranks.astype(np.int64) * d_out)[:-1]
    A = np.zeros(int(ranks.sum()) * d_in, np.float32)
    B = np.zeros(int(ranks.sum()) * d_out, np.float32)
    for a in range(n_adapters):
        r = int(ranks[a])
        Aa = A[A_off[a]:A_off[a] + r * d_in].reshape(r, d_in)
        Aa[0, 0] = 1.0
        Aa[1, 1] = 1.0
        Ba = B[B_off[a]:B_off[a] + d_out * r].reshape(d_out, r)
        for o in range(d_out):
            Ba[o, 0] = 1.0 + ((a >> (o % n_bits)) & 1)
            Ba[o, 1] = 1.0
    from workloads import bf16_bits
    return HostPool(A=bf16_bits(A), B=bf16_bits(B), A_off=A_off, B_off=B_off, rank=ranks,
                    d_in=d_in, d_out=d_out)


def integer_coded_x(N: int, d_in: int):
    from workloads import bf16_bits
    X = np.zeros((N, d_in), np.float32)
    X[:, 0] = 1.0
    X[:, 1] = 1.0
    return bf16_bits(X)


def integer_coded_expect(ids: np.ndarray, d_out: int, n_bits: int, scale: float) -> np.ndarray:
    """Closed form of the integer-coded delta: s * (2 + bit_{o mod n_bits}(id)), 0 for id -1."""
    o = np.arange(d_out)
    out = np.zeros((len(ids), d_out))
    for n, a in enumerate(ids):
        if a >= 0:
            out[n] = scale * (2.0 + ((int(a) >> (o % n_bits)) & 1))
    return out


def pin_integer_coded_routing(orc):
    """Routing is exact: every token's output spells its own adapter id."""
    rng = np.random.default_rng(7)
    n_ad, d_in, d_out, n_bits = 300, 16, 24, 9
    ranks = rng.choice([8, 16, 32], n_ad)
    p = integer_coded_pool(n_ad, ranks, d_in, d_out, n_bits)
    N = 64
    ids = rng.integers(-1, n_ad, N).astype(np.int32)
    X = integer_coded_x(N, d_in)
    assert np.array_equal(orc.bgmv_delta(X, p, ids, 2.0), integer_coded_expect(ids, d_out, n_bits, 2.0))


def pin_multi_additivity(orc):
    """Stacked LoRAs add: multi(a1 s1, a2 s2) = s1 single(a1) + s2 single(a2);
    a repeated adapter counts twice."""
    rng = np.random.default_rng(8)
    p = rand_host_pool(rng, [8, 16, 24], 32, 20)
    N = 10
    X = rand_x(rng, N, 32)
    req_off = np.array([0, 4, 4, 10], np.int32)   # a zero-length request in the middle
    ad_off = np.array([0, 2, 3, 6], np.int32)
    ad_id = np.array([0, 2, 1, 1, 2, 1], np.int32)
    ad_sc = np.array([0.5, 1.5, 3.0, 0.75, -1.0, 0.25], np.float32)
    got = orc.apply_multi_delta(X, p, req_off, ad_off, ad_id, ad_sc)
    want = np.zeros_like(got)
    for q in range(3):
        rows = np.arange(req_off[q], req_off[q + 1])
        for k in range(ad_off[q], ad_off[q + 1]):
            ids = np.full(N, -1, np.int32)
            ids[rows] = ad_id[k]
            want += orc.bgmv_delta(X, p, ids, float(ad_sc[k]))
    _close(got, want)


def pin_rank_stacking(orc):
    """Two adapters on one request equal one adapter of rank r1 + r2 with
    A = [A1; A2] and B = [s1 B1 | s2 B2] (s1, s2 powers of two, so exact)."""
    rng = np.random.default_rng(9)
    d_in, d_out = 24, 16
    p = rand_host_pool(rng, [8, 16], d_in, d_out)
    s1, s2 = 0.5, 2.0
    A = np.concatenate([p.A[p.A_off[0]:p.A_off[0] + 8 * d_in], p.A[p.A_off[1]:p.A_off[1] + 16 * d_in]])
    from workloads import bf16_bits
    Bst = np.concatenate([s1 * B_of(p, 0), s2 * B_of(p, 1)], axis=1).astype(np.float32)
    stacked = HostPool(A=A, B=bf16_bits(Bst.reshape(-1)), A_off=np.array([0], np.int64),
                       B_off=np.array([0], np.int64), rank=np.array([24], np.int32),
                       d_in=d_in, d_out=d_out)
    X = rand_x(rng, 6, d_in)
    got = orc.apply_multi_delta(X, p, np.array([0, 6], np.int32), np.array([0, 2], np.int32),
                                np.array([0, 1], np.int32), np.array([s1, s2], np.float32))
    _close(got, orc.bgmv_delta(X, stacked, np.zeros(6, np.int32), 1.0))


def pin_segment_split(orc):
    """Two requests on the same LoRA fall in one group: splitting a segment in
    two changes nothing, bit for bit."""
    rng = np.random.default_rng(10)
    p = rand_host_pool(rng, [8, 32], 16, 24)
    X = rand_x(rng, 20, 16)
    a = orc.sgmv_delta(X, p, np.array([0, 5, 20], np.int32), np.array([1, 0], np.int32), 1.0)
    b = orc.sgmv_delta(X, p, np.array([0, 5, 12, 20], np.int32), np.array([1, 0, 0], np.int32), 1.0)
    assert np.array_equal(a, b)


def pin_sgmv_equals_bgmv(orc):
    """SGMV over sorted segments equals BGMV with each token's segment id, and
    rows outside every segment get nothing; shrink then expand through an fp32
    intermediate agrees with the all-fp64 path to fp32 rounding."""
    rng = np.random.default_rng(11)
    p = rand_host_pool(rng, [16, 8, 24], 40, 32)
    N = 27
    X = rand_x(rng, N, 40)
    seg_off = np.array([2, 9, 9, 20, 25], np.int32)    # rows 0-1 and 25-26 outside; an empty segment
    seg_ad = np.array([2, 0, 1, 2], np.int32)
    ids = np.full(N, -1, np.int32)
    for k in range(4):
        ids[seg_off[k]:seg_off[k + 1]] = seg_ad[k]
    full = orc.sgmv_delta(X, p, seg_off, seg_ad, 1.5)
    assert np.array_equal(full, orc.bgmv_delta(X, p, ids, 1.5))
    V = orc.sgmv_shrink(X, p, seg_off, seg_ad, fill=np.nan)
    Xd = widen(X)
    for k in range(4):
        a = seg_ad[k]
        r = int(p.rank[a])
        rows = slice(seg_off[k], seg_off[k + 1])
        _close(V[rows, :r], Xd[rows] @ A_of(p, a).T)
        assert np.all(np.isnan(V[rows, r:]))
    assert np.all(np.isnan(V[:2])) and np.all(np.isnan(V[25:]))
    V32 = np.nan_to_num(V, nan=0.0).astype(np.float32)
    ex = orc.sgmv_expand(V32, p, seg_off, seg_ad, 1.5)
    for k in range(4):
        a = seg_ad[k]
        r = int(p.rank[a])
        rows = slice(seg_off[k], seg_off[k + 1])
        _close(ex[rows], 1.5 * (V32[rows, :r].astype(np.float64) @ B_of(p, a).T))
    assert np.max(np.abs(ex - full)) <= 1e-5 * np.max(np.abs(full))


def pin_route(orc):
    """The grouping is a stable counting sort: numpy's stable argsort and
    bincount give the same permutation, bounds and adapters; id -1 is left out."""
    rng = np.random.default_rng(12)
    for n_ad, N in [(1000, 512), (4, 64), (7, 1), (5, 0)]:
        ids = rng.integers(-1, n_ad, N).astype(np.int32)
        perm, seg_off, seg_ad = orc.route(ids, n_ad)
        valid = np.nonzero(ids >= 0)[0]
        order = valid[np.argsort(ids[valid], kind="stable")]
        assert np.array_equal(perm, order)
        cnt = np.bincount(ids[valid], minlength=n_ad)
        assert np.array_equal(seg_ad, np.nonzero(cnt)[0])
        assert np.array_equal(np.diff(seg_off), cnt[cnt > 0])
        assert seg_off[0] == 0


def pin_rows_subset(orc):
    """A subset of rows equals the same rows of the full result, exactly."""
    rng = np.random.default_rng(13)
    p = rand_host_pool(rng, [8, 16], 16, 24)
    X = rand_x(rng, 15, 16)
    ids = rng.integers(-1, 2, 15).astype(np.int32)
    rows = np.array([14, 0, 7, 7, 3], np.int32)
    assert np.array_equal(orc.bgmv_delta(X, p, ids, 1.0, rows=rows), orc.bgmv_delta(X, p, ids, 1.0)[rows])
    so, sa = np.array([0, 6, 15], np.int32), np.array([1, 0], np.int32)
    assert np.array_equal(orc.sgmv_delta(X, p, so, sa, 1.0, rows=rows), orc.sgmv_delta(X, p, so, sa, 1.0)[rows])


def pin_bad_metadata(orc):
    """Out-of-range ids and non-monotone segments are rejected, not computed."""
    rng = np.random.default_rng(14)
    p = rand_host_pool(rng, [8], 16, 16)
    X = rand_x(rng, 4, 16)
    for bad in ([0, 1, 0, 0], [0, -2, 0, 0]):
        try:
            orc.bgmv_delta(X, p, np.array(bad, np.int32), 1.0)
        except OracleError:
            pass
        else:
            raise AssertionError(f"ids {bad} accepted")
    try:
        orc.sgmv_delta(X, p, np.array([0, 3, 2], np.int32), np.array([0, 0], np.int32), 1.0)
    except OracleError:
        pass
    else:
        raise AssertionError("non-monotone segments accepted")
    # the projection: an adapter id past the pool (not -1) and non-monotone segments
    W = rand_x(rng, 16, 16)
    for seg_off, seg_ad in (([0, 4], [1]), ([0, 3, 2], [0, 0])):
        try:
            orc.linear_sgmv(X, W, p, np.array(seg_off, np.int32), np.array(seg_ad, np.int32), 1.0)
        except OracleError:
            pass
        else:
            raise AssertionError(f"linear segments {seg_off} / adapters {seg_ad} accepted")


def pin_linear_is_the_merged_weight_product(orc):
    """The projection with its LoRA delta equals x (W + s B_a A_a)^T (numpy float64), row
    by row, for each segment's adapter -- the merged-weight identity of the handbook page
    -- and the base product x W^T alone for a segment with adapter -1; rows outside every
    segment are zero.  d_in != d_out != rank, so a transposed W or B fails."""
    rng = np.random.default_rng(31)
    d_in, d_out = 40, 24
    p = rand_host_pool(rng, [16, 8, 24], d_in, d_out)
    W = rand_x(rng, d_out, d_in)
    seg_off = np.array([2, 7, 7, 12, 17], np.int32)
    seg_ad = np.array([2, 0, -1, 1], np.int32)
    N = 19
    X = rand_x(rng, N, d_in)
    s = 0.625
    Y = orc.linear_sgmv(X, W, p, seg_off, seg_ad, s)
    Xd, Wd = widen(X), widen(W)
    want = np.zeros((N, d_out))
    for k, a in enumerate(seg_ad):
        Wm = Wd if a == -1 else Wd + s * (B_of(p, a) @ A_of(p, a))
        for n in range(seg_off[k], seg_off[k + 1]):
            want[n] = Xd[n] @ Wm.T
    _close(Y, want)
    rows = np.array([12, 0, 3, 18], np.int32)
    _close(orc.linear_sgmv(X, W, p, seg_off, seg_ad, s, rows=rows), want[rows])


def pin_linear_zero_B_is_the_base_product(orc):
    """With every B zero the LoRA part vanishes: y = x W^T exactly as numpy computes it."""
    rng = np.random.default_rng(32)
    d_in, d_out = 24, 56
    p = rand_host_pool(rng, [8, 16], d_in, d_out, zero_B=True)
    W = rand_x(rng, d_out, d_in)
    X = rand_x(rng, 10, d_in)
    seg_off = np.array([0, 4, 10], np.int32)
    Y = orc.linear_sgmv(X, W, p, seg_off, np.array([1, 0], np.int32), 3.0)
    _close(Y, widen(X) @ widen(W).T)


ALL_PINS = [v for k, v in sorted(globals().items()) if k.startswith("pin_")]
