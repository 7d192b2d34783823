"""Multi-LoRA delta (SGMV / BGMV) for B200 -- Python binding of liblora_sgmv.so.

The binding only marshals arguments (tensor pointers, sizes, the current CUDA
stream) into the C ABI declared in include/lora_sgmv.h; every step of the
computation runs in the library's kernels.  There is no fallback: if the
shared library is missing or cannot be loaded, every call raises LoraError.

Tensors: bf16 activations and pools on one CUDA device, int32 metadata, int64
pool offsets, fp32 intermediate and per-adapter weights.  The workspace is a
uint8 CUDA tensor; if none is given, one is taken from a per-device cache.
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = [
    "LoraError", "load", "library_path", "lora_version", "lora_workspace_size", "lora_workspace_init",
    "lora_kernel_launches",
    "lora_get_error", "lora_route", "lora_bgmv", "lora_sgmv_shrink", "lora_sgmv_shrink_proj", "lora_sgmv_apply_proj",
    "lora_sgmv_expand",
    "lora_apply_multi", "lora_apply_multi_static", "make_pool_struct", "Workspace", "OP_BGMV", "OP_SGMV_SHRINK", "OP_SGMV_EXPAND",
    "OP_APPLY_MULTI", "OP_ROUTE", "OP_MERGE", "OP_LINEAR", "OP_APPLY_PROJ", "STATUS", "lora_merge", "lora_linear_sgmv",
    "PoolManager", "lora_test_stall",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_LIBNAME = "liblora_sgmv.so"

OP_BGMV, OP_SGMV_SHRINK, OP_SGMV_EXPAND, OP_APPLY_MULTI, OP_ROUTE, OP_MERGE, OP_LINEAR, OP_APPLY_PROJ = range(8)
STATUS = {0: "LORA_OK", 1: "LORA_ERR_INVALID_ARG", 2: "LORA_ERR_UNSUPPORTED", 4: "LORA_ERR_BAD_ADAPTER",
          8: "LORA_ERR_BAD_SEGMENT", 16: "LORA_ERR_CUDA", 32: "LORA_ERR_WORKSPACE", 64: "LORA_ERR_TIMEOUT"}
MAX_ADS_PER_REQ = 8


class LoraError(RuntimeError):
    def __init__(self, what: str, code: int = -1):
        self.code = code
        names = [v for k, v in STATUS.items() if k and (code > 0 and code & k)]
        super().__init__(f"{what}: {'|'.join(names) or code}")


class LoraPoolStruct(ctypes.Structure):
    _fields_ = [("A", ctypes.c_void_p), ("B", ctypes.c_void_p), ("A_off", ctypes.c_void_p),
                ("B_off", ctypes.c_void_p), ("rank", ctypes.c_void_p), ("A_elems", ctypes.c_int64),
                ("B_elems", ctypes.c_int64), ("n_adapters", ctypes.c_int32), ("d_in", ctypes.c_int32),
                ("d_out", ctypes.c_int32), ("max_rank", ctypes.c_int32)]


_lib = None
_lock = threading.Lock()


def library_path() -> str:
    return os.environ.get("LORA_SGMV_LIB", os.path.join(_PKG, _LIBNAME))


def load():
    """Load liblora_sgmv.so (built in-tree by adapter_gemv_sgmv_b200.build)."""
    global _lib
    if _lib is not None:
        return _lib
    with _lock:
        if _lib is not None:
            return _lib
        path = library_path()
        if not os.path.exists(path):
            raise LoraError(f"{path} not found; build it with `python -m adapter_gemv_sgmv_b200.build`")
        lib = ctypes.CDLL(path)
        P, i32, i64, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float, ctypes.c_size_t
        PP = ctypes.POINTER(LoraPoolStruct)
        lib.lora_version.restype = ctypes.c_char_p
        lib.lora_version.argtypes = []
        lib.lora_test_stall.restype = None
        lib.lora_test_stall.argtypes = [ctypes.c_int, ctypes.c_double]
        lib.lora_workspace_size.restype = sz
        lib.lora_workspace_size.argtypes = [ctypes.c_int, i32, i32, i32, i32, i32, i32, i32]
        lib.lora_kernel_launches.restype = ctypes.c_int
        lib.lora_kernel_launches.argtypes = [ctypes.c_int, i32, i32, i32, i32]
        lib.lora_workspace_init.restype = ctypes.c_int
        lib.lora_workspace_init.argtypes = [P, P]
        lib.lora_get_error.restype = ctypes.c_int
        lib.lora_get_error.argtypes = [P, P]
        lib.lora_route.restype = ctypes.c_int
        lib.lora_route.argtypes = [P, i32, i32, P, P, P, P, P, sz, P]
        lib.lora_bgmv.restype = ctypes.c_int
        lib.lora_bgmv.argtypes = [P, i64, P, i64, PP, P, i32, f32, P, sz, P]
        lib.lora_sgmv_shrink.restype = ctypes.c_int
        lib.lora_sgmv_shrink.argtypes = [P, i64, P, i64, PP, P, P, i32, i32, P, sz, P]
        lib.lora_sgmv_shrink_proj.restype = ctypes.c_int
        lib.lora_linear_sgmv.restype = ctypes.c_int
        lib.lora_sgmv_apply_proj.restype = ctypes.c_int
        lib.lora_sgmv_apply_proj.argtypes = [P, i64, P, P, PP, i32, P, P, i32, i32, P, P, sz, P]
        lib.lora_linear_sgmv.argtypes = [P, i64, P, i64, P, i64, PP, P, P, i32, i32, f32, P, sz, P]
        lib.lora_sgmv_shrink_proj.argtypes = [P, i64, P, i64, PP, i32, P, P, i32, i32, P, sz, P]
        lib.lora_sgmv_expand.restype = ctypes.c_int
        lib.lora_sgmv_expand.argtypes = [P, i64, P, i64, PP, P, P, i32, i32, f32, P, sz, P]
        lib.lora_apply_multi.restype = ctypes.c_int
        lib.lora_apply_multi.argtypes = [P, i64, P, i64, PP, P, P, P, P, i32, i32, i32, P, sz, P]
        lib.lora_apply_multi_static.restype = ctypes.c_int
        lib.lora_apply_multi_static.argtypes = [P, i64, P, i64, PP, P, P, P, P, i32, i32, i32, P, P]
        lib.lora_merge.restype = ctypes.c_int
        lib.lora_merge.argtypes = [P, i64, PP, i32, f32, P, sz, P]
        lib.lora_pm_create.restype = ctypes.c_int
        lib.lora_pm_create.argtypes = [PP, P, ctypes.POINTER(ctypes.c_void_p)]
        lib.lora_pm_destroy.restype = None
        lib.lora_pm_destroy.argtypes = [P]
        lib.lora_pm_register.restype = ctypes.c_int
        lib.lora_pm_register.argtypes = [P, i64, P, P, i32]
        lib.lora_pm_acquire.restype = ctypes.c_int
        lib.lora_pm_acquire.argtypes = [P, P, i32, P, P, P]
        lib.lora_pm_observe.restype = ctypes.c_int
        lib.lora_pm_observe.argtypes = [P, P, i32]
        lib.lora_pm_set_preload.restype = ctypes.c_int
        lib.lora_pm_set_preload.argtypes = [P, i32]
        lib.lora_pm_preloaded.restype = ctypes.c_int32
        lib.lora_pm_preloaded.argtypes = [P]
        _lib = lib
    return _lib


def lora_test_stall(stall: bool, wait_seconds: float = 0.0) -> None:
    """Testing hook: while set, the pipelined kernels issue no loads and every wait
    inside a kernel gives up after wait_seconds (the call reports LORA_ERR_TIMEOUT)."""
    load().lora_test_stall(1 if stall else 0, float(wait_seconds))


def lora_version() -> str:
    return load().lora_version().decode()


def lora_workspace_size(op: int, N: int, n_adapters: int, d_in: int, d_out: int, max_rank: int,
                        n_items: int = 0, max_ads_per_req: int = 1) -> int:
    return int(load().lora_workspace_size(op, N, n_adapters, d_in, d_out, max_rank, n_items,
                                          max_ads_per_req))


def lora_kernel_launches(op: int, N: int, n_adapters: int, d_in: int, n_items: int = 0) -> int:
    return int(load().lora_kernel_launches(op, N, n_adapters, d_in, n_items))


# ----------------------------------------------------------------------------
# marshalling helpers
# ----------------------------------------------------------------------------
def _torch():
    import torch
    return torch


def _stream_ptr(stream=None) -> int:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return int(stream.cuda_stream)


def _ptr(t) -> int:
    return 0 if t is None else int(t.data_ptr())


def _check_dev(*ts):
    for t in ts:
        if t is not None and not t.is_cuda:
            raise LoraError("tensors must live on a CUDA device", 1)


def make_pool_struct(pool, max_rank: int | None = None) -> LoraPoolStruct:
    """lora_pool from an object with A, B (bf16), A_off, B_off (int64), rank (int32), d_in, d_out."""
    torch = _torch()
    for name, dt in (("A", torch.bfloat16), ("B", torch.bfloat16), ("A_off", torch.int64),
                     ("B_off", torch.int64), ("rank", torch.int32)):
        t = getattr(pool, name)
        if t.dtype != dt or not t.is_contiguous():
            raise LoraError(f"pool.{name} must be a contiguous {dt} tensor", 1)
    _check_dev(pool.A, pool.B, pool.A_off, pool.B_off, pool.rank)
    if max_rank is None:
        max_rank = int(getattr(pool, "max_rank"))
    return LoraPoolStruct(_ptr(pool.A), _ptr(pool.B), _ptr(pool.A_off), _ptr(pool.B_off), _ptr(pool.rank),
                          int(pool.A.numel()), int(pool.B.numel()), int(pool.rank.numel()),
                          int(pool.d_in), int(pool.d_out), int(max_rank))


class Workspace:
    """A caller-owned workspace tensor, zeroed once (its error word starts clear)."""

    def __init__(self, nbytes: int, device=None):
        torch = _torch()
        self.tensor = torch.zeros(max(int(nbytes), 256), dtype=torch.uint8, device=device or "cuda")

    @property
    def nbytes(self) -> int:
        return int(self.tensor.numel())

    def ptr(self) -> int:
        return int(self.tensor.data_ptr())


_ws_cache: dict = {}


def _workspace(nbytes: int, device) -> Workspace:
    torch = _torch()
    dev = torch.device(device)
    key = (dev.type, dev.index if dev.index is not None else torch.cuda.current_device())
    ws = _ws_cache.get(key)
    if ws is None or ws.nbytes < nbytes:
        ws = Workspace(max(nbytes, 2 * (ws.nbytes if ws else 0)), device=dev)
        _ws_cache[key] = ws
    return ws


def _rc(rc: int, what: str):
    if rc != 0:
        raise LoraError(what, rc)


def _mat(t, d: int, name: str):
    torch = _torch()
    if t.dtype != torch.bfloat16 or t.dim() != 2 or t.stride(1) != 1 or t.shape[1] != d:
        raise LoraError(f"{name} must be a 2-D bf16 tensor with {d} unit-stride columns", 1)
    return t.stride(0)


def lora_workspace_init(ws: Workspace, stream=None):
    _rc(load().lora_workspace_init(ws.ptr(), _stream_ptr(stream)), "lora_workspace_init")


def lora_get_error(ws: Workspace, stream=None) -> int:
    """Device error bits of the workspace (cleared by the read); 0 if none."""
    return int(load().lora_get_error(ws.ptr(), _stream_ptr(stream)))


# ----------------------------------------------------------------------------
# the entry points
# ----------------------------------------------------------------------------
def lora_route(ids, n_adapters: int, perm, seg_off, seg_ad, n_seg, ws: Workspace | None = None,
               stream=None):
    """Stable grouping of ids by adapter into caller tensors (see lora_route in the header)."""
    lib = load()
    _check_dev(ids, perm, seg_off, seg_ad, n_seg)
    N = int(ids.numel())
    need = lora_workspace_size(OP_ROUTE, N, n_adapters, 8, 8, 8)
    ws = ws or _workspace(need, ids.device)
    _rc(lib.lora_route(_ptr(ids), N, int(n_adapters), _ptr(perm), _ptr(seg_off), _ptr(seg_ad), _ptr(n_seg),
                       ws.ptr(), ws.nbytes, _stream_ptr(stream)), "lora_route")
    return ws


def lora_bgmv(X, Y, pool, ids, scale: float, ws: Workspace | None = None, stream=None,
              max_rank: int | None = None):
    """Y[n] += scale * B[ids[n]] A[ids[n]] X[n] in place (ids[n] == -1: untouched)."""
    lib = load()
    _check_dev(X, Y, ids)
    ps = make_pool_struct(pool, max_rank)
    ldx = _mat(X, ps.d_in, "X")
    ldy = _mat(Y, ps.d_out, "Y")
    N = int(ids.numel())
    need = lora_workspace_size(OP_BGMV, N, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank)
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_bgmv(_ptr(X), ldx, _ptr(Y), ldy, ctypes.byref(ps), _ptr(ids), N, float(scale),
                      ws.ptr(), ws.nbytes, _stream_ptr(stream)), "lora_bgmv")
    return ws


def lora_sgmv_shrink(X, V, pool, seg_off, seg_ad, ws: Workspace | None = None, stream=None,
                     max_rank: int | None = None):
    """V[n, :rank[a]] = A[a] X[n] for rows of segment k (a = seg_ad[k]); V is fp32 [N, >= max_rank]."""
    lib = load()
    torch = _torch()
    _check_dev(X, V, seg_off, seg_ad)
    ps = make_pool_struct(pool, max_rank)
    ldx = _mat(X, ps.d_in, "X")
    if V.dtype != torch.float32 or V.dim() != 2 or V.stride(1) != 1:
        raise LoraError("V must be a 2-D fp32 tensor with unit-stride columns", 1)
    N = int(X.shape[0])
    n_seg = int(seg_ad.numel())
    need = lora_workspace_size(OP_SGMV_SHRINK, N, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank, n_seg)
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_sgmv_shrink(_ptr(X), ldx, _ptr(V), V.stride(0), ctypes.byref(ps), _ptr(seg_off),
                             _ptr(seg_ad), n_seg, N, ws.ptr(), ws.nbytes, _stream_ptr(stream)),
        "lora_sgmv_shrink")
    return ws


def lora_sgmv_shrink_proj(X, V, pools, seg_off, seg_ad, ws: Workspace | None = None, stream=None,
                          max_ranks=None):
    """Shrinks of projections sharing the input X (Q, K, V; gate, up) in one pass over X.

    Projection p's rank vector lands in V columns [c_p, c_p + rank_p[a]), where
    c_p is the sum of the earlier pools' max_rank; returns (ws, [c_p]).  Every
    pool has the same d_in and n_adapters; V is fp32 [N, >= sum of max_rank]."""
    lib = load()
    torch = _torch()
    pools = list(pools)
    _check_dev(X, V, seg_off, seg_ad)
    if max_ranks is None:
        max_ranks = [None] * len(pools)
    structs = [make_pool_struct(p, m) for p, m in zip(pools, max_ranks)]
    arr = (LoraPoolStruct * max(len(structs), 1))(*structs)
    ldx = _mat(X, structs[0].d_in if structs else X.shape[1], "X")
    if V.dtype != torch.float32 or V.dim() != 2 or V.stride(1) != 1:
        raise LoraError("V must be a 2-D fp32 tensor with unit-stride columns", 1)
    N = int(X.shape[0])
    n_seg = int(seg_ad.numel())
    cols, c = [], 0
    for ps in structs:
        cols.append(c)
        c += ps.max_rank
    ps0 = structs[0] if structs else None
    need = lora_workspace_size(OP_SGMV_SHRINK, N, ps0.n_adapters, ps0.d_in, ps0.d_out, ps0.max_rank,
                               n_seg) if ps0 else 256
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_sgmv_shrink_proj(_ptr(X), ldx, _ptr(V), V.stride(0), arr, len(structs), _ptr(seg_off),
                                  _ptr(seg_ad), n_seg, N, ws.ptr(), ws.nbytes, _stream_ptr(stream)),
        "lora_sgmv_shrink_proj")
    return ws, cols


def lora_sgmv_apply_proj(X, Ys, pools, seg_off, seg_ad, scales, ws: Workspace | None = None, stream=None,
                         max_ranks=None):
    """Ys[p][n] += scales[p] * B_p[a] A_p[a] X[n] for projections sharing X (q/k/v; gate/up):
    one plan, one stacked shrink, one expand per projection; V stays in the workspace."""
    lib = load()
    pools = list(pools)
    Ys = list(Ys)
    _check_dev(X, seg_off, seg_ad, *Ys)
    if max_ranks is None:
        max_ranks = [None] * len(pools)
    structs = [make_pool_struct(p, m) for p, m in zip(pools, max_ranks)]
    n = len(structs)
    if n < 1 or len(Ys) != n or len(scales) != n:
        raise LoraError("one output and one scale per pool", 1)
    arr = (LoraPoolStruct * n)(*structs)
    ldx = _mat(X, structs[0].d_in, "X")
    ys = (ctypes.c_void_p * n)(*[_ptr(Y) for Y in Ys])
    lds = (ctypes.c_int64 * n)(*[_mat(Y, ps.d_out, "Y") for Y, ps in zip(Ys, structs)])
    sc = (ctypes.c_float * n)(*[float(s) for s in scales])
    N = int(X.shape[0])
    n_seg = int(seg_ad.numel())
    vcols = sum(ps.max_rank for ps in structs)
    need = lora_workspace_size(OP_APPLY_PROJ, N, structs[0].n_adapters, structs[0].d_in, 0, vcols, n_seg)
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_sgmv_apply_proj(_ptr(X), ldx, ys, lds, arr, n, _ptr(seg_off), _ptr(seg_ad), n_seg, N, sc,
                                 ws.ptr(), ws.nbytes, _stream_ptr(stream)), "lora_sgmv_apply_proj")
    return ws


def lora_linear_sgmv(X, W, Y, pool, seg_off, seg_ad, scale: float, ws: Workspace | None = None, stream=None,
                     max_rank: int | None = None):
    """Y[n] = W X[n] + scale * B[a] A[a] X[n] for rows of segment k (a = seg_ad[k]; -1: W X[n] only).

    W is the projection's bf16 weight [d_out, d_in]; Y is overwritten (rows outside every
    segment are left as they are)."""
    lib = load()
    _check_dev(X, W, Y, seg_off, seg_ad)
    ps = make_pool_struct(pool, max_rank)
    ldx = _mat(X, ps.d_in, "X")
    ldw = _mat(W, ps.d_in, "W")
    ldy = _mat(Y, ps.d_out, "Y")
    if W.shape[0] != ps.d_out:
        raise LoraError(f"W must have d_out = {ps.d_out} rows", 1)
    N = int(X.shape[0])
    n_seg = int(seg_ad.numel())
    need = lora_workspace_size(OP_LINEAR, N, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank, n_seg)
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_linear_sgmv(_ptr(X), ldx, _ptr(W), ldw, _ptr(Y), ldy, ctypes.byref(ps), _ptr(seg_off),
                             _ptr(seg_ad), n_seg, N, float(scale), ws.ptr(), ws.nbytes, _stream_ptr(stream)),
        "lora_linear_sgmv")
    return ws


def lora_sgmv_expand(V, Y, pool, seg_off, seg_ad, scale: float, ws: Workspace | None = None,
                     stream=None, max_rank: int | None = None):
    """Y[n] += scale * B[a] V[n, :rank[a]] for rows of segment k (a = seg_ad[k])."""
    lib = load()
    torch = _torch()
    _check_dev(V, Y, seg_off, seg_ad)
    ps = make_pool_struct(pool, max_rank)
    ldy = _mat(Y, ps.d_out, "Y")
    if V.dtype != torch.float32 or V.dim() != 2 or V.stride(1) != 1:
        raise LoraError("V must be a 2-D fp32 tensor with unit-stride columns", 1)
    N = int(Y.shape[0])
    n_seg = int(seg_ad.numel())
    need = lora_workspace_size(OP_SGMV_EXPAND, N, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank, n_seg)
    ws = ws or _workspace(need, Y.device)
    _rc(lib.lora_sgmv_expand(_ptr(V), V.stride(0), _ptr(Y), ldy, ctypes.byref(ps), _ptr(seg_off),
                             _ptr(seg_ad), n_seg, N, float(scale), ws.ptr(), ws.nbytes, _stream_ptr(stream)),
        "lora_sgmv_expand")
    return ws


def lora_apply_multi(X, Y, pool, req_off, ad_off, ad_id, ad_scale, max_ads_per_req: int = 3,
                     ws: Workspace | None = None, stream=None, max_rank: int | None = None):
    """Y[n] += sum_p ad_scale[p] B[ad_id[p]] A[ad_id[p]] X[n] over request q's adapters."""
    lib = load()
    _check_dev(X, Y, req_off, ad_off, ad_id, ad_scale)
    ps = make_pool_struct(pool, max_rank)
    ldx = _mat(X, ps.d_in, "X")
    ldy = _mat(Y, ps.d_out, "Y")
    N = int(X.shape[0])
    n_req = int(req_off.numel()) - 1
    need = lora_workspace_size(OP_APPLY_MULTI, N, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank, n_req,
                               max_ads_per_req)
    ws = ws or _workspace(need, X.device)
    _rc(lib.lora_apply_multi(_ptr(X), ldx, _ptr(Y), ldy, ctypes.byref(ps), _ptr(req_off), _ptr(ad_off),
                             _ptr(ad_id), _ptr(ad_scale), n_req, N, int(max_ads_per_req), ws.ptr(),
                             ws.nbytes, _stream_ptr(stream)), "lora_apply_multi")
    return ws


def lora_apply_multi_static(X, Y, pool, req_off, ad_off, ad_id, ad_scale, max_ads_per_req: int = 3,
                            err_out=None, stream=None, max_rank: int | None = None):
    """lora_apply_multi without a workspace, for callers that cannot allocate device memory.

    The scratch is a fixed array inside the library (see lora_apply_multi_static in the
    header): calls must not overlap on the GPU, the first call on a device should come
    before any stream capture, and too-large calls raise LoraError (LORA_ERR_WORKSPACE).
    err_out: optional 1-element int32/uint32 CUDA tensor that receives the device status bits."""
    lib = load()
    _check_dev(X, Y, req_off, ad_off, ad_id, ad_scale, err_out)
    ps = make_pool_struct(pool, max_rank)
    ldx = _mat(X, ps.d_in, "X")
    ldy = _mat(Y, ps.d_out, "Y")
    N = int(X.shape[0])
    n_req = int(req_off.numel()) - 1
    _rc(lib.lora_apply_multi_static(_ptr(X), ldx, _ptr(Y), ldy, ctypes.byref(ps), _ptr(req_off), _ptr(ad_off),
                                    _ptr(ad_id), _ptr(ad_scale), n_req, N, int(max_ads_per_req), _ptr(err_out),
                                    _stream_ptr(stream)), "lora_apply_multi_static")


def lora_merge(W, pool, adapter: int, scale: float, ws: Workspace | None = None, stream=None,
               max_rank: int | None = None):
    """W[o] += scale * (B[a] A[a])[o] in place for the base weight W [d_out, d_in] (bf16);
    unmerge with -scale.  Returns the workspace (its error word: lora_get_error)."""
    lib = load()
    _check_dev(W)
    ps = make_pool_struct(pool, max_rank)
    ldw = _mat(W, ps.d_in, "W")
    if int(W.shape[0]) != ps.d_out:
        raise LoraError("W must have pool.d_out rows", 1)
    need = lora_workspace_size(OP_MERGE, ps.d_out, ps.n_adapters, ps.d_in, ps.d_out, ps.max_rank)
    ws = ws or _workspace(need, W.device)
    _rc(lib.lora_merge(_ptr(W), ldw, ctypes.byref(ps), int(adapter), float(scale), ws.ptr(), ws.nbytes,
                       _stream_ptr(stream)), "lora_merge")
    return ws


class PoolManager:
    """A resident pool of n_slots adapter slots with on-demand loads (lora_pm_*).

    Owns the pool's device tensors (A, B, A_off, B_off, rank) and is itself the pool
    the ops take (slot indices are the adapter ids).  register() records an adapter's
    host copy (CPU bf16 tensors A [r, d_in], B [d_out, r]; pinned memory makes the
    loads asynchronous); acquire(keys) makes a batch's adapters resident and returns
    their slots, loading missing ones on `stream` over least recently used slots."""

    def __init__(self, n_slots: int, d_in: int, d_out: int, max_rank: int, device="cuda", stream=None):
        torch = _torch()
        self.d_in, self.d_out, self.max_rank = int(d_in), int(d_out), int(max_rank)
        self.A = torch.zeros(n_slots * max_rank * d_in, dtype=torch.bfloat16, device=device)
        self.B = torch.zeros(n_slots * d_out * max_rank, dtype=torch.bfloat16, device=device)
        self.A_off = torch.zeros(n_slots, dtype=torch.int64, device=device)
        self.B_off = torch.zeros(n_slots, dtype=torch.int64, device=device)
        self.rank = torch.zeros(n_slots, dtype=torch.int32, device=device)
        self._host = {}
        self._h = ctypes.c_void_p()
        ps = make_pool_struct(self)
        _rc(load().lora_pm_create(ctypes.byref(ps), _stream_ptr(stream), ctypes.byref(self._h)), "lora_pm_create")

    @property
    def n_adapters(self) -> int:
        return int(self.rank.numel())

    def register(self, key: int, A_host, B_host):
        torch = _torch()
        r = int(A_host.shape[0])
        if (A_host.dtype != torch.bfloat16 or B_host.dtype != torch.bfloat16 or A_host.device.type != "cpu" or
                B_host.device.type != "cpu" or tuple(A_host.shape) != (r, self.d_in) or
                tuple(B_host.shape) != (self.d_out, r) or not A_host.is_contiguous() or not B_host.is_contiguous()):
            raise LoraError("register: A [r, d_in] and B [d_out, r] contiguous bf16 CPU tensors", 1)
        self._host[int(key)] = (A_host, B_host)        # kept alive while a copy may be in flight
        _rc(load().lora_pm_register(self._h, int(key), A_host.data_ptr(), B_host.data_ptr(), r), "lora_pm_register")

    def acquire(self, keys, stream=None):
        """slots (int32 numpy array, one per key) and the number of adapters loaded."""
        import numpy as np
        keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
        slots = np.zeros(max(len(keys), 1), dtype=np.int32)
        n_loaded = ctypes.c_int32(0)
        _rc(load().lora_pm_acquire(self._h, keys.ctypes.data, len(keys), slots.ctypes.data,
                                   ctypes.byref(n_loaded), _stream_ptr(stream)), "lora_pm_acquire")
        return slots[:len(keys)], int(n_loaded.value)

    def observe(self, keys):
        """Record one request's adapter keys for co-occurrence preloading."""
        import numpy as np
        keys = np.ascontiguousarray(np.asarray(keys, dtype=np.int64))
        _rc(load().lora_pm_observe(self._h, keys.ctypes.data, len(keys)), "lora_pm_observe")

    def set_preload(self, top_k: int):
        """Preload the top_k co-occurring partners of every acquired key (0: off)."""
        _rc(load().lora_pm_set_preload(self._h, int(top_k)), "lora_pm_set_preload")

    def preloaded(self) -> int:
        """Adapters the last acquire preloaded."""
        return int(load().lora_pm_preloaded(self._h))

    def close(self):
        if self._h:
            load().lora_pm_destroy(self._h)
            self._h = ctypes.c_void_p()

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass

