"""lora_apply_multi_static: the entry point for callers that cannot allocate
device memory (graph-capture regions without allocation, processes whose device
memory belongs to another allocator, plugins handed only their inputs and
outputs).  It must give what lora_apply_multi gives with a caller workspace,
call after call, while its scratch lives in a fixed array inside the library.

This file is collected last on purpose, and also passes on its own in a fresh
process (the library's scratch set-up happens on the first call on a device)."""
import numpy as np
import pytest
import torch

import adapter_gemv_sgmv_b200 as L
import oracle
from helpers import check_parity, check_rounded, host_pool, widen
from workloads import make_pool, make_workload, to_host

pytestmark = pytest.mark.gpu


def _case(seed):
    return make_workload(4, device="cuda", seed=seed, n_img=6, tokens_per_img=200, d=256, n_adapters=20,
                         projections=["q"], y0="normal").calls[0]


def test_static_scratch_matches_the_oracle_on_two_calls():
    """Two calls in a row on the one fixed scratch, each against the oracle's exact
    multi-adapter delta (the bar every parity test uses), and against what
    lora_apply_multi gives with a caller workspace on the same inputs."""
    for seed in (11, 12):
        c = _case(seed)
        y = c.Y.clone()
        err = torch.full((1,), -1, dtype=torch.int32, device="cuda")
        L.lora_apply_multi_static(c.X, y, c.pool, c.req_off, c.ad_off, c.ad_id, c.ad_scale, max_ads_per_req=3,
                                  err_out=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        y_exact = widen(to_host(c.Y)) + oracle.apply_multi_delta(to_host(c.X), host_pool(c.pool), c.req_off_h,
                                                                 c.ad_off_h, c.ad_id_h, c.ad_scale_h)
        got = widen(to_host(y))
        check_parity(got, y_exact, f"static scratch, call seed {seed}")
        check_rounded(got, y_exact, f"static scratch, call seed {seed}")
        assert np.max(np.abs(got - widen(to_host(c.Y)))) > 0   # the call did change y
        y_ws = c.Y.clone()
        ws = L.lora_apply_multi(c.X, y_ws, c.pool, c.req_off, c.ad_off, c.ad_id, c.ad_scale, max_ads_per_req=3)
        assert L.lora_get_error(ws) == 0
        check_parity(widen(to_host(y_ws)), y_exact, f"workspace entry point, call seed {seed}")


def test_static_scratch_rejects_calls_that_do_not_fit():
    pool = make_pool([128] * 4, 8, 8, seed=0, device="cuda")
    N = 1 << 16                 # 65536 tokens x 8 adapters x rank 128 x 4 B = 256 MiB of scratch
    X = torch.zeros(N, 8, dtype=torch.bfloat16, device="cuda")
    Y = torch.zeros(N, 8, dtype=torch.bfloat16, device="cuda")
    req_off = torch.tensor([0, N], dtype=torch.int32, device="cuda")
    ad_off = torch.tensor([0, 1], dtype=torch.int32, device="cuda")
    ad_id = torch.zeros(1, dtype=torch.int32, device="cuda")
    ad_scale = torch.ones(1, dtype=torch.float32, device="cuda")
    with pytest.raises(L.LoraError) as ei:
        L.lora_apply_multi_static(X, Y, pool, req_off, ad_off, ad_id, ad_scale, max_ads_per_req=8)
    assert ei.value.code == 32
    torch.cuda.synchronize()
    assert torch.count_nonzero(Y).item() == 0
