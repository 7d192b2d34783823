"""The resident pool manager on the GPU: batches of decode tokens over a registry of
more adapters than slots, each batch made resident by acquire() and run through
lora_bgmv on the managed pool, against the oracle on the registry itself; eviction,
reloading and re-registration; and the host -> device load throughput."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import check_parity, dev_bf16, rand_host_pool, rand_x, widen
from workloads import to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _host_ab(hp, a):
    r = int(hp.rank[a])
    A = hp.A[hp.A_off[a]:hp.A_off[a] + r * hp.d_in].reshape(r, hp.d_in)
    B = hp.B[hp.B_off[a]:hp.B_off[a] + hp.d_out * r].reshape(hp.d_out, r)
    to_t = lambda m: torch.from_numpy(np.ascontiguousarray(m).view(np.int16)).view(torch.bfloat16).pin_memory()
    return to_t(A), to_t(B)


def test_pool_manager_batches_match_the_oracle():
    rng = np.random.default_rng(31)
    d_in, d_out = 512, 384
    ranks = [16, 32, 8, 64, 16, 24, 48, 16, 32, 8, 64, 40]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    pm = L.PoolManager(5, d_in, d_out, 64)
    for a in range(len(ranks)):
        pm.register(a, *_host_ab(hp, a))
    resident = {}
    for step in range(10):
        keys = rng.choice(len(ranks), size=int(rng.integers(1, 6)), replace=False)
        tok_keys = rng.choice(keys, size=48).astype(np.int64)
        before = set(resident.values())
        slots, n_loaded = pm.acquire(tok_keys)
        assert n_loaded == len(set(int(k) for k in keys) - before)
        for sl, k in zip(slots, tok_keys):
            resident[int(sl)] = int(k)                  # a reassigned slot no longer holds its old key
        X = rand_x(rng, 48, d_in)
        Y0 = rand_x(rng, 48, d_out)
        Y = dev_bf16(Y0)
        ws = L.lora_bgmv(dev_bf16(X), Y, pm, torch.tensor(slots, dtype=torch.int32, device=DEV), 1.25)
        assert L.lora_get_error(ws) == 0
        want = widen(Y0) + oracle.bgmv_delta(X, hp, tok_keys.astype(np.int32), 1.25)
        check_parity(widen(to_host(Y)), want, f"managed pool step {step}")


def test_reregistering_replaces_the_adapter():
    rng = np.random.default_rng(32)
    hp = rand_host_pool(rng, [16, 16], 256, 256)
    pm = L.PoolManager(2, 256, 256, 16)
    pm.register(7, *_host_ab(hp, 0))
    slots, n = pm.acquire([7, 7])
    assert n == 1
    slots, n = pm.acquire([7])
    assert n == 0                                       # resident: nothing loads
    pm.register(7, *_host_ab(hp, 1))                    # new host copy: reloaded next time
    slots, n = pm.acquire([7])
    assert n == 1
    X = rand_x(rng, 4, 256)
    Y = dev_bf16(np.zeros((4, 256), np.uint16))
    L.lora_bgmv(dev_bf16(X), Y, pm, torch.tensor(np.repeat(slots, 4), dtype=torch.int32, device=DEV), 1.0)
    want = oracle.bgmv_delta(X, hp, np.ones(4, np.int32), 1.0)
    check_parity(widen(to_host(Y)), want, "re-registered adapter")


def test_preloaded_partners_give_oracle_exact_batches():
    """Co-occurrence preloading on the GPU: after requests that pair adapter 0 with 3 and
    1 with 4, acquiring {0, 1} also brings 3 and 4 in (on the same stream); a batch over
    3 and 4 then loads nothing, and its decode through the managed pool matches the oracle."""
    rng = np.random.default_rng(35)
    d_in, d_out = 384, 256
    ranks = [16, 32, 8, 64, 24, 16]
    hp = rand_host_pool(rng, ranks, d_in, d_out)
    pm = L.PoolManager(4, d_in, d_out, 64)
    for a in range(len(ranks)):
        pm.register(a, *_host_ab(hp, a))
    for req in ([0, 3], [0, 3], [1, 4], [0, 5], [1, 4, 2]):
        pm.observe(req)
    pm.set_preload(1)
    slots01, n = pm.acquire([0, 1, 0])
    assert n == 2 and pm.preloaded() == 2              # partners 3 (of 0) and 4 (of 1)
    slots34, n = pm.acquire([3, 4, 4, 3])
    assert n == 0 and pm.preloaded() == 0              # already resident; their partners 0 and 1 too
    tok = np.array([3, 4, 4, 3, 3, 4, 3, 3], np.int64)
    slot_of = {3: int(slots34[0]), 4: int(slots34[1])}
    ids = np.array([slot_of[int(k)] for k in tok], np.int32)
    X = rand_x(rng, len(tok), d_in)
    Y0 = rand_x(rng, len(tok), d_out)
    Y = dev_bf16(Y0)
    ws = L.lora_bgmv(dev_bf16(X), Y, pm, torch.tensor(ids, device=DEV), 0.75)
    assert L.lora_get_error(ws) == 0
    want = widen(Y0) + oracle.bgmv_delta(X, hp, tok.astype(np.int32), 0.75)
    check_parity(widen(to_host(Y)), want, "preloaded adapters")
    pm.set_preload(0)
    pm.acquire([5])
    assert pm.preloaded() == 0


def test_oversize_batch_and_unknown_key_change_nothing():
    rng = np.random.default_rng(33)
    hp = rand_host_pool(rng, [8, 8, 8], 64, 64)
    pm = L.PoolManager(2, 64, 64, 8)
    for a in range(3):
        pm.register(a, *_host_ab(hp, a))
    with pytest.raises(L.LoraError):
        pm.acquire([0, 1, 2])                           # three distinct keys, two slots
    with pytest.raises(L.LoraError):
        pm.acquire([0, 99])
    slots, n = pm.acquire([0, 1])
    assert n == 2 and sorted(slots.tolist()) == [0, 1]


def test_load_throughput():
    """16 cold rank-64 adapters of a 4096 x 4096 projection (1 MB each) from pinned memory."""
    rng = np.random.default_rng(34)
    d, r, n = 4096, 64, 16
    pm = L.PoolManager(n, d, d, r)
    for k in range(n):
        A = torch.from_numpy(rng.standard_normal((r, d)).astype(np.float32)).to(torch.bfloat16).pin_memory()
        B = torch.from_numpy(rng.standard_normal((d, r)).astype(np.float32)).to(torch.bfloat16).pin_memory()
        pm.register(k, A, B)
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    torch.cuda.synchronize()
    e0.record(s)
    _, loaded = pm.acquire(list(range(n)), stream=s)
    e1.record(s)
    torch.cuda.synchronize()
    ms = e0.elapsed_time(e1)
    gbs = n * 2 * r * d * 2 / (ms * 1e-3) / 1e9
    print(f"adapter loads: {loaded} x {2 * r * d * 2 / 1e6:.2f} MB in {ms:.3f} ms = {gbs:.1f} GB/s")
    assert loaded == n and gbs > 1.0
