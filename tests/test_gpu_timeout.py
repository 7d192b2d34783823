"""The timeout path of the pipelined (tensor-core) kernels, made to run on purpose without a
broken kernel: with the testing hook lora_test_stall set, each kernel's producer
issues no loads, so its consumers' first wait runs out after a few microseconds.
The call must then report LORA_ERR_TIMEOUT, leave its outputs untouched, and free
everything it held (shared memory fills, TMEM): the same call right after, with
the hook off, must succeed and match the oracle."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import DevPool, check_parity, dev_bf16, rand_host_pool, rand_x, widen
from workloads import to_host

pytestmark = pytest.mark.gpu
DEV = "cuda"
TIMEOUT = 64


def _i32(a):
    return torch.tensor(np.asarray(a, np.int32), device=DEV)


def _stalled(fn):
    """Run fn() with the hook on (20 us waits); return the workspace's error word."""
    L.lora_test_stall(True, 20e-6)
    try:
        ws = fn()
        torch.cuda.synchronize()
    finally:
        L.lora_test_stall(False)
    return L.lora_get_error(ws)


def _segments():
    seg_off = np.array([0, 300, 700], np.int32)
    return seg_off, np.array([1, 0], np.int32), 700


def test_tensor_core_shrink_and_expand_time_out_and_recover():
    rng = np.random.default_rng(42)
    hp = rand_host_pool(rng, [64, 32], 256, 320)
    seg_off, ads, N = _segments()
    X = rand_x(rng, N, 256)
    pool = DevPool(hp)
    V = torch.full((N, 64), float("nan"), dtype=torch.float32, device=DEV)
    err = _stalled(lambda: L.lora_sgmv_shrink(dev_bf16(X), V, pool, _i32(seg_off), _i32(ads)))
    assert err & TIMEOUT
    assert torch.isnan(V).all()                               # nothing written
    ws = L.lora_sgmv_shrink(dev_bf16(X), V, pool, _i32(seg_off), _i32(ads))
    assert L.lora_get_error(ws) == 0
    Vh = to_host(V).astype(np.float32)
    Y0 = rand_x(rng, N, 320)
    Y = dev_bf16(Y0)
    err = _stalled(lambda: L.lora_sgmv_expand(V, Y, pool, _i32(seg_off), _i32(ads), 0.5))
    assert err & TIMEOUT
    assert np.array_equal(to_host(Y), Y0)
    ws = L.lora_sgmv_expand(V, Y, pool, _i32(seg_off), _i32(ads), 0.5)
    assert L.lora_get_error(ws) == 0
    check_parity(widen(to_host(Y)), widen(Y0) + oracle.sgmv_expand(np.nan_to_num(Vh), hp, seg_off, ads, 0.5),
                 "expand after a timeout")


def test_fused_projection_times_out_and_recovers():
    rng = np.random.default_rng(43)
    d_in, d_out = 256, 264
    hp = rand_host_pool(rng, [32, 64], d_in, d_out)
    seg_off, ads, N = _segments()
    X = rand_x(rng, N, d_in)
    W = (rng.standard_normal((d_out, d_in)) / np.sqrt(d_in)).astype(np.float32)
    from workloads import bf16_bits
    Wb = bf16_bits(W)
    sentinel = np.full((N, d_out), 0x3F80, np.uint16)
    Y = dev_bf16(sentinel)
    pool = DevPool(hp)
    err = _stalled(lambda: L.lora_linear_sgmv(dev_bf16(X), dev_bf16(Wb), Y, pool, _i32(seg_off), _i32(ads), 0.75))
    assert err & TIMEOUT
    assert np.array_equal(to_host(Y), sentinel)
    ws = L.lora_linear_sgmv(dev_bf16(X), dev_bf16(Wb), Y, pool, _i32(seg_off), _i32(ads), 0.75)
    assert L.lora_get_error(ws) == 0
    check_parity(widen(to_host(Y)), oracle.linear_sgmv(X, Wb, hp, seg_off, ads, 0.75), "projection after a timeout")
