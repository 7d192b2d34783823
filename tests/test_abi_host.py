"""The C ABI without a GPU: the library loads, exports every entry point the
header declares, sizes workspaces, and rejects bad arguments on the host.

Every rejected call below carries at least one defect the host checks catch
before the first CUDA call, and each case also passes a null workspace, so no
case can reach a kernel launch even if the check under test were missing
(the call would then fail on the workspace check instead, and the test would
report the wrong status code).
"""
import ctypes
import os
import re

import pytest

import adapter_gemv_sgmv_b200 as L
from adapter_gemv_sgmv_b200 import build as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lora_sgmv.h")

OK, INVALID, UNSUPPORTED, WORKSPACE = 0, 1, 2, 32


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load()


def declared():
    src = open(HEADER).read()
    return re.findall(r"LORA_API\s+[\w\s\*]+?\b(lora_\w+)\s*\(", src)


def test_header_declares_the_entry_points():
    names = set(declared())
    assert {"lora_bgmv", "lora_sgmv_shrink", "lora_sgmv_expand", "lora_apply_multi", "lora_route",
            "lora_workspace_size", "lora_workspace_init", "lora_get_error", "lora_version",
            "lora_merge", "lora_sgmv_shrink_proj", "lora_linear_sgmv", "lora_sgmv_apply_proj"} <= names


def test_every_declared_symbol_is_exported(lib):
    raw = ctypes.CDLL(L.library_path())
    for name in declared():
        assert hasattr(raw, name), name
    assert "sm_100a" in L.lora_version()


def test_workspace_size(lib):
    s1 = L.lora_workspace_size(L.OP_BGMV, 256, 128, 4096, 4096, 16)
    s2 = L.lora_workspace_size(L.OP_BGMV, 512, 128, 4096, 4096, 16)
    assert 0 < s1 < s2 and s1 % 256 == 0
    assert L.lora_workspace_size(L.OP_SGMV_SHRINK, 1000, 64, 4096, 14336, 64, n_items=16) > 0
    assert L.lora_workspace_size(L.OP_APPLY_MULTI, 100, 8, 64, 64, 32, 4, 3) >= 100 * 3 * 32 * 4
    # rejected shapes size to 0
    assert L.lora_workspace_size(L.OP_BGMV, -1, 128, 4096, 4096, 16) == 0
    assert L.lora_workspace_size(L.OP_BGMV, 4, 128, 4096, 4096, 256) == 0
    assert L.lora_workspace_size(L.OP_APPLY_MULTI, 4, 8, 64, 64, 16, 1, 9) == 0
    assert L.lora_workspace_size(99, 4, 8, 64, 64, 16) == 0
    # merge: N is d_out; the workspace holds A^T (bf16) and B (fp32) of one adapter
    m = L.lora_workspace_size(L.OP_MERGE, 14336, 64, 4096, 14336, 64)
    assert m >= 4096 * 64 * 2 + 14336 * 64 * 4 and m % 256 == 0
    assert L.lora_workspace_size(L.OP_MERGE, 100, 64, 4096, 14336, 64) == 0
    assert L.lora_kernel_launches(L.OP_MERGE, 14336, 64, 4096) == 2
    assert L.lora_kernel_launches(L.OP_MERGE, 64, 64, 4096) == 3


FAKE = 0x10000          # a 256-byte-aligned address that is never dereferenced


def _pool(**kw):
    d = dict(A=FAKE, B=FAKE, A_off=FAKE, B_off=FAKE, rank=FAKE, A_elems=1 << 20, B_elems=1 << 20,
             n_adapters=4, d_in=64, d_out=32, max_rank=16)
    d.update(kw)
    return L.LoraPoolStruct(**d)


def _bgmv(lib, pool, X=FAKE, ldx=64, Y=FAKE, ldy=32, ids=FAKE, N=4, ws=None, ws_bytes=0):
    return lib.lora_bgmv(X, ldx, Y, ldy, ctypes.byref(pool) if pool is not None else None, ids, N, 1.0,
                         ws, ws_bytes, None)


@pytest.mark.parametrize("case,want", [
    (dict(pool=None), INVALID),
    (dict(pool=_pool(A=0)), INVALID),
    (dict(pool=_pool(rank=0)), INVALID),
    (dict(pool=_pool(A_elems=-1)), INVALID),
    (dict(pool=_pool(n_adapters=0)), UNSUPPORTED),
    (dict(pool=_pool(n_adapters=40000)), UNSUPPORTED),
    (dict(pool=_pool(d_in=60)), UNSUPPORTED),
    (dict(pool=_pool(d_out=0)), UNSUPPORTED),
    (dict(pool=_pool(max_rank=4)), UNSUPPORTED),
    (dict(pool=_pool(max_rank=136)), UNSUPPORTED),
    (dict(pool=_pool(max_rank=20)), UNSUPPORTED),
    (dict(pool=_pool(A=FAKE + 8)), UNSUPPORTED),
    (dict(ids=0), INVALID),
    (dict(N=-1), INVALID),
    (dict(X=0), INVALID),
    (dict(ldx=32), INVALID),
    (dict(ldx=68), UNSUPPORTED),
    (dict(X=FAKE + 2), UNSUPPORTED),
    (dict(Y=FAKE + 4), UNSUPPORTED),
    (dict(ldy=16), INVALID),
    (dict(ws=None), WORKSPACE),
    (dict(ws=FAKE + 16, ws_bytes=1 << 30), WORKSPACE),
    (dict(ws=FAKE, ws_bytes=256), WORKSPACE),
])
def test_bgmv_host_validation(lib, case, want):
    kw = dict(pool=_pool())
    kw.update(case)
    assert _bgmv(lib, **kw) == want


def test_other_entry_points_validate(lib):
    p = ctypes.byref(_pool())
    # sgmv shrink: ldv below max_rank / null segments / negative n_seg
    assert lib.lora_sgmv_shrink(FAKE, 64, FAKE, 8, p, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert lib.lora_sgmv_shrink(FAKE, 64, FAKE, 16, p, None, FAKE, 2, 4, None, 0, None) == INVALID
    assert lib.lora_sgmv_shrink(FAKE, 64, FAKE, 16, p, FAKE, FAKE, -1, 4, None, 0, None) == INVALID
    assert lib.lora_sgmv_shrink(FAKE, 64, FAKE, 16, p, FAKE, FAKE, 2, 4, None, 0, None) == WORKSPACE
    # sgmv expand
    assert lib.lora_sgmv_expand(FAKE, 8, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert lib.lora_sgmv_expand(FAKE, 16, FAKE + 2, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == UNSUPPORTED
    assert lib.lora_sgmv_expand(FAKE, 16, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == WORKSPACE
    # multi: max_ads_per_req out of range, null adapter list
    assert lib.lora_apply_multi(FAKE, 64, FAKE, 32, p, FAKE, FAKE, FAKE, FAKE, 2, 4, 9, None, 0, None) == UNSUPPORTED
    assert lib.lora_apply_multi(FAKE, 64, FAKE, 32, p, FAKE, FAKE, None, FAKE, 2, 4, 3, None, 0, None) == INVALID
    assert lib.lora_apply_multi(FAKE, 64, FAKE, 32, p, FAKE, FAKE, FAKE, FAKE, 2, 4, 3, None, 0, None) == WORKSPACE
    # route
    assert lib.lora_route(FAKE, 4, 0, FAKE, FAKE, FAKE, FAKE, None, 0, None) == UNSUPPORTED
    assert lib.lora_route(None, 4, 8, FAKE, FAKE, FAKE, FAKE, None, 0, None) == INVALID
    assert lib.lora_route(FAKE, 4, 8, FAKE, FAKE, FAKE, FAKE, None, 0, None) == WORKSPACE
    # merge: adapter out of range, W below one row / misaligned, no workspace
    assert lib.lora_merge(FAKE, 64, p, 4, 1.0, None, 0, None) == INVALID
    assert lib.lora_merge(FAKE, 64, p, -1, 1.0, None, 0, None) == INVALID
    assert lib.lora_merge(FAKE, 32, p, 1, 1.0, None, 0, None) == INVALID
    assert lib.lora_merge(FAKE + 2, 64, p, 1, 1.0, None, 0, None) == UNSUPPORTED
    assert lib.lora_merge(FAKE, 64, p, 1, 1.0, None, 0, None) == WORKSPACE
    assert lib.lora_merge(FAKE, 64, None, 1, 1.0, None, 0, None) == INVALID
    # workspace helpers reject a null / misaligned workspace before touching CUDA
    assert lib.lora_workspace_init(None, None) == WORKSPACE
    assert lib.lora_get_error(FAKE + 8, None) == WORKSPACE


def _pools(*ps):
    return (L.LoraPoolStruct * len(ps))(*ps)


def test_shrink_proj_validates(lib):
    q, k, v = _pool(), _pool(d_out=16, max_rank=8), _pool(max_rank=32)
    three = _pools(q, k, v)
    sh = lib.lora_sgmv_shrink_proj
    # no pools / too many projections
    assert sh(FAKE, 64, FAKE, 56, None, 3, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 64, FAKE, 56, three, 0, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    five = _pools(q, q, q, q, q)
    assert sh(FAKE, 64, FAKE, 80, five, 5, FAKE, FAKE, 2, 4, None, 0, None) == UNSUPPORTED
    # a bad pool anywhere in the list
    assert sh(FAKE, 64, FAKE, 56, _pools(q, _pool(A=0), v), 3, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 64, FAKE, 56, _pools(q, k, _pool(max_rank=12)), 3, FAKE, FAKE, 2, 4, None, 0,
              None) == UNSUPPORTED
    # the pools must share d_in and n_adapters
    assert sh(FAKE, 64, FAKE, 56, _pools(q, _pool(d_in=128), v), 3, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 64, FAKE, 56, _pools(q, _pool(n_adapters=5), v), 3, FAKE, FAKE, 2, 4, None, 0,
              None) == INVALID
    # V holds the ranks side by side: ldv >= 16 + 8 + 32
    assert sh(FAKE, 64, FAKE, 48, three, 3, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 64, FAKE, 56, three, 3, None, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 32, FAKE, 56, three, 3, FAKE, FAKE, 2, 4, None, 0, None) == INVALID
    assert sh(FAKE, 64, FAKE, 56, three, 3, FAKE, FAKE, 2, 4, None, 0, None) == WORKSPACE
    # two projections only: ldv 24 is enough
    assert sh(FAKE, 64, FAKE, 24, three, 2, FAKE, FAKE, 2, 4, None, 0, None) == WORKSPACE


def test_linear_validates(lib):
    p = ctypes.byref(_pool())          # d_in 64, d_out 32, max_rank 16
    ln = lib.lora_linear_sgmv
    # W missing / W leading dimension below d_in / misaligned W
    assert ln(FAKE, 64, None, 64, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert ln(FAKE, 64, FAKE, 32, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert ln(FAKE, 64, FAKE + 2, 64, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == UNSUPPORTED
    # Y and X as elsewhere; segments; workspace
    assert ln(FAKE, 64, FAKE, 64, FAKE, 16, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert ln(FAKE, 64, FAKE, 64, FAKE, 32, p, None, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert ln(FAKE, 64, FAKE, 64, FAKE, 32, None, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == INVALID
    assert ln(FAKE, 64, FAKE, 64, FAKE, 32, p, FAKE, FAKE, 2, 4, 1.0, None, 0, None) == WORKSPACE


def test_linear_workspace_and_launches(lib):
    # header + tiles + s V as bf16 high and low parts, max_rank rounded up to 64 per part
    n = L.lora_workspace_size(L.OP_LINEAR, 1000, 64, 4096, 14336, 64, 8)
    assert n >= 1000 * 2 * 64 * 2
    assert L.lora_workspace_size(L.OP_LINEAR, 1000, 64, 4096, 14336, 128, 8) - n >= 1000 * 2 * 64 * 2
    assert L.lora_kernel_launches(L.OP_LINEAR, 1000, 64, 4096, 8) == 3
    assert L.lora_kernel_launches(L.OP_LINEAR, 1000, 64, 4096, 0) == 0


def test_empty_calls_return_before_any_launch(lib):
    """N = 0 or no segments: the new entry points validate, then return LORA_OK without
    touching the device (a fake but large, aligned workspace is never dereferenced)."""
    p = ctypes.byref(_pool())
    ws, nb = FAKE, 1 << 20
    assert lib.lora_linear_sgmv(FAKE, 64, FAKE, 64, FAKE, 32, p, FAKE, FAKE, 2, 0, 1.0, ws, nb, None) == OK
    assert lib.lora_linear_sgmv(FAKE, 64, FAKE, 64, FAKE, 32, p, FAKE, FAKE, 0, 4, 1.0, ws, nb, None) == OK
    pools = _pools(_pool(), _pool(max_rank=32))
    assert lib.lora_sgmv_shrink_proj(FAKE, 64, FAKE, 48, pools, 2, FAKE, FAKE, 2, 0, ws, nb, None) == OK
    assert lib.lora_sgmv_shrink_proj(FAKE, 64, FAKE, 48, pools, 2, FAKE, FAKE, 0, 4, ws, nb, None) == OK


def test_apply_proj_validates(lib):
    q, k = _pool(), _pool(d_out=16, max_rank=8)
    two = _pools(q, k)
    ap = lib.lora_sgmv_apply_proj
    ys = (ctypes.c_void_p * 2)(FAKE, FAKE)
    lds = (ctypes.c_int64 * 2)(32, 16)
    sc = (ctypes.c_float * 2)(1.0, 0.5)
    # host arrays missing
    assert ap(FAKE, 64, None, lds, two, 2, FAKE, FAKE, 2, 4, sc, None, 0, None) == INVALID
    assert ap(FAKE, 64, ys, None, two, 2, FAKE, FAKE, 2, 4, sc, None, 0, None) == INVALID
    assert ap(FAKE, 64, ys, lds, two, 2, FAKE, FAKE, 2, 4, None, None, 0, None) == INVALID
    # a projection's leading dimension below its d_out; a misaligned output
    bad_ld = (ctypes.c_int64 * 2)(32, 8)
    assert ap(FAKE, 64, ys, bad_ld, two, 2, FAKE, FAKE, 2, 4, sc, None, 0, None) == INVALID
    bad_y = (ctypes.c_void_p * 2)(FAKE, FAKE + 2)
    assert ap(FAKE, 64, bad_y, lds, two, 2, FAKE, FAKE, 2, 4, sc, None, 0, None) == UNSUPPORTED
    # pools that do not share d_in
    assert ap(FAKE, 64, ys, lds, _pools(q, _pool(d_in=128, d_out=16)), 2, FAKE, FAKE, 2, 4, sc, None, 0,
              None) == INVALID
    assert ap(FAKE, 64, ys, lds, two, 2, FAKE, FAKE, 2, 4, sc, None, 0, None) == WORKSPACE
    # empty: validated, then nothing launched
    assert ap(FAKE, 64, ys, lds, two, 2, FAKE, FAKE, 2, 0, sc, FAKE, 1 << 20, None) == OK
    # the workspace holds V for all projections side by side (16 + 8 columns)
    assert L.lora_workspace_size(L.OP_APPLY_PROJ, 1000, 4, 64, 0, 24, 2) >= 1000 * 24 * 4
    assert L.lora_workspace_size(L.OP_APPLY_PROJ, 1000, 4, 64, 0, 4 * 128 + 8, 2) == 0
