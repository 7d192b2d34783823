// The C ABI (include/lora_sgmv.h): host-side validation, workspace layout and
// kernel launches.  No entry point allocates memory; every validation below
// runs before the first CUDA call, so a rejected call touches no device.

#include <stdlib.h>
#include <string.h>

#include <atomic>

#include "lora_internal.cuh"

using namespace lora;

namespace lora {

// Programmatic dependent launch for the single-launch decode kernel: on
// unless LORA_SGMV_NO_PDL is set in the environment (read once).
bool pdl_enabled()
{
    static const bool on = [] {
        const char *v = getenv("LORA_SGMV_NO_PDL");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

// Tensor-core (tcgen05) path for long segments / requests: on unless
// LORA_SGMV_NO_TC is set in the environment (read once).
bool tc_enabled()
{
    static const bool on = [] {
        const char *v = getenv("LORA_SGMV_NO_TC");
        return !(v && v[0] && v[0] != '0');
    }();
    return on;
}

namespace {
std::atomic<int> g_test_stall{0};
std::atomic<unsigned long long> g_wait_ns{kWaitBoundNs};
}  // namespace

int test_stall_mode() { return g_test_stall.load(std::memory_order_relaxed); }
unsigned long long wait_bound_ns() { return g_wait_ns.load(std::memory_order_relaxed); }

}  // namespace lora

extern "C" LORA_API void lora_test_stall(int stall, double wait_seconds)
{
    using namespace lora;
    if (stall) {
        const double ns = wait_seconds > 0 ? wait_seconds * 1e9 : 0.0;
        g_wait_ns.store(ns < 1e3 ? 1000ull : (ns > 2e9 ? kWaitBoundNs : (unsigned long long)ns));
        g_test_stall.store(1);
    } else {
        g_test_stall.store(0);
        g_wait_ns.store(kWaitBoundNs);
    }
}

namespace {

constexpr size_t kAlign = 256;

// Items long enough on average for 128-row tensor-core tiles to pay off.
bool long_items(int32_t N, int32_t n_items)
{
    return tc_enabled() && N >= kTcGroup && (int64_t)N >= 64LL * (n_items > 0 ? n_items : 1);
}

bool aligned_v(const void *V, int64_t ldv) { return ((uintptr_t)V & 15) == 0 && (ldv & 3) == 0; }

size_t align_up(size_t x) { return (x + kAlign - 1) & ~(kAlign - 1); }

bool misaligned(const void *p, size_t a) { return ((uintptr_t)p) & (a - 1); }

int32_t n_chunks_for(int op, int32_t d_in)
{
    return op == LORA_OP_BGMV ? (d_in + kBgmvChunk - 1) / kBgmvChunk : 1;
}

struct Layout {
    size_t hdr, perm, seg_off, seg_ad, groups, V, total;
    int32_t max_groups, n_chunks;
    int32_t kv;      // LORA_OP_LINEAR: column of the low parts of s V (max_rank rounded up to 64)
};

bool layout(int op, int32_t N, int32_t n_adapters, int32_t d_in, int32_t max_rank, int32_t n_items,
            int32_t max_ads, Layout *L)
{
    // LORA_OP_APPLY_PROJ: max_rank is the V width, the projections' max ranks summed
    const int32_t rank_cap = op == LORA_OP_APPLY_PROJ ? LORA_MAX_PROJ * LORA_MAX_RANK : LORA_MAX_RANK;
    if (N < 0 || n_adapters < 1 || n_adapters > LORA_MAX_ADAPTERS || d_in <= 0 || max_rank < 8 ||
        max_rank > rank_cap)
        return false;
    const bool routed = op == LORA_OP_BGMV || op == LORA_OP_ROUTE;
    if (!routed && n_items < 0)
        return false;
    if (op == LORA_OP_APPLY_MULTI && (max_ads < 1 || max_ads > LORA_MAX_ADS_PER_REQ))
        return false;
    const int64_t items = routed ? (int64_t)(N < n_adapters ? N : n_adapters) : n_items;
    memset(L, 0, sizeof *L);
    L->max_groups = (int32_t)((int64_t)N / kGroup + items + 1);
    L->n_chunks = n_chunks_for(op, d_in);
    size_t off = 0;
    L->hdr = off;
    off = align_up(off + sizeof(WsHeader));
    L->perm = off;
    off = align_up(off + (routed ? (size_t)N * 4 : 0));
    L->seg_off = off;
    off = align_up(off + (op == LORA_OP_BGMV ? (size_t)(items + 1) * 4 : 0));
    L->seg_ad = off;
    off = align_up(off + (op == LORA_OP_BGMV ? (size_t)items * 4 : 0));
    L->groups = off;
    off = align_up(off + (size_t)L->max_groups * sizeof(Group));
    L->V = off;
    size_t v = 0;
    if (op == LORA_OP_BGMV)
        v = (size_t)L->n_chunks * N * max_rank * 4;
    else if (op == LORA_OP_APPLY_MULTI)
        v = (size_t)N * max_ads * max_rank * 4;
    else if (op == LORA_OP_APPLY_PROJ)
        v = (size_t)N * max_rank * 4;       // V of all the projections side by side
    else if (op == LORA_OP_LINEAR) {
        L->kv = (max_rank + 63) & ~63;
        v = (size_t)N * 2 * L->kv * 2;      // s V, bf16 high and low parts
    }
    off = align_up(off + v);
    L->total = off;
    return true;
}

lora_status check_pool(const lora_pool *p)
{
    if (!p || !p->A || !p->B || !p->A_off || !p->B_off || !p->rank)
        return LORA_ERR_INVALID_ARG;
    if (p->A_elems < 0 || p->B_elems < 0)
        return LORA_ERR_INVALID_ARG;
    if (p->n_adapters < 1 || p->n_adapters > LORA_MAX_ADAPTERS)
        return LORA_ERR_UNSUPPORTED;
    if (p->d_in <= 0 || p->d_out <= 0 || (p->d_in & 7) || (p->d_out & 7))
        return LORA_ERR_UNSUPPORTED;
    if (p->max_rank < 8 || p->max_rank > LORA_MAX_RANK || (p->max_rank & 7))
        return LORA_ERR_UNSUPPORTED;
    if (misaligned(p->A, 16) || misaligned(p->B, 16))
        return LORA_ERR_UNSUPPORTED;
    return LORA_OK;
}

lora_status check_mat(const void *M, int64_t ld, int32_t d, int32_t N)
{
    if (N > 0 && !M)
        return LORA_ERR_INVALID_ARG;
    if (ld < d)
        return LORA_ERR_INVALID_ARG;
    if ((ld & 7) || misaligned(M, 16))
        return LORA_ERR_UNSUPPORTED;
    return LORA_OK;
}

lora_status check_ws(void *ws, size_t ws_bytes, const Layout &L)
{
    if (!ws || misaligned(ws, kAlign) || ws_bytes < L.total)
        return LORA_ERR_WORKSPACE;
    return LORA_OK;
}

PoolDev pool_dev(const lora_pool *p)
{
    PoolDev d;
    d.A = static_cast<const __nv_bfloat16 *>(p->A);
    d.B = static_cast<const __nv_bfloat16 *>(p->B);
    d.A_off = p->A_off;
    d.B_off = p->B_off;
    d.rank = p->rank;
    d.A_elems = p->A_elems;
    d.B_elems = p->B_elems;
    d.n_adapters = p->n_adapters;
    d.max_rank = p->max_rank;
    d.d_in = p->d_in;
    d.d_out = p->d_out;
    return d;
}

template <class T>
T *at(void *ws, size_t off) { return reinterpret_cast<T *>(static_cast<char *>(ws) + off); }

#define LORA_TRY(x)                         \
    do {                                    \
        lora_status _s = (x);               \
        if (_s != LORA_OK)                  \
            return _s;                      \
    } while (0)

#define LORA_CUDA(x)                        \
    do {                                    \
        if ((x) != cudaSuccess)             \
            return LORA_ERR_CUDA;           \
    } while (0)

// Projections sharing one input: the pools must share d_in and n_adapters; vcol[p]
// is projection p's first column in V (the earlier pools' max_rank summed).
lora_status check_proj_pools(const lora_pool *pools, int32_t n_proj, int32_t *vcol, int64_t *vcols)
{
    if (!pools || n_proj < 1)
        return LORA_ERR_INVALID_ARG;
    if (n_proj > LORA_MAX_PROJ)
        return LORA_ERR_UNSUPPORTED;
    *vcols = 0;
    for (int p = 0; p < n_proj; ++p) {
        LORA_TRY(check_pool(&pools[p]));
        if (pools[p].d_in != pools[0].d_in || pools[p].n_adapters != pools[0].n_adapters)
            return LORA_ERR_INVALID_ARG;
        vcol[p] = (int32_t)*vcols;
        *vcols += pools[p].max_rank;
    }
    return LORA_OK;
}

// The plan and the shrinks of projections sharing X into V.  tc (with ta's x map
// encoded): tiles of 128 rows and one tensor-core launch per run of consecutive
// projections whose max ranks fit one stacked accumulator (each launch reads X once);
// else 8-row groups and the CUDA-core shrink once per projection.
cudaError_t run_proj_shrinks(bool tc, const TcArgs &ta0, const void *X, int64_t ldx, float *V, int64_t ldv,
                             const lora_pool *pools, int32_t n_proj, const int32_t *vcol, const int32_t *seg_off,
                             const int32_t *seg_ad, int32_t n_seg, int32_t N, const Layout &L, void *ws,
                             cudaStream_t s)
{
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);
    const int32_t d_in = pools[0].d_in;
    cudaError_t e;
    PlanArgs pa = {};
    pa.mode = kModeSgmv;
    pa.N = N;
    pa.item_off = seg_off;
    pa.n_items = n_seg;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = tc ? kTcGroup : kGroup;
    pa.hdr = hdr;
    if ((e = launch_plan(pa, s)) != cudaSuccess)
        return e;
    if (tc) {
        TcArgs ta = ta0;
        ta.mode = kModeProj;
        ta.groups = groups;
        ta.hdr = hdr;
        ta.seg_ad = seg_ad;
        ta.max_ads = 1;
        ta.scale = 1.0f;
        ta.V = V;
        ta.ldv = ldv;
        ta.slot_stride = 0;
        ta.err = &hdr->err;
        for (int p0 = 0; p0 < n_proj;) {
            int p1 = p0, kk = 0;
            while (p1 < n_proj && kk + pools[p1].max_rank <= kKMaxShrink)
                kk += pools[p1++].max_rank;
            TcArgs tp = ta;
            tp.a_tma = 0;
            tp.n_proj = p1 - p0;
            for (int q = p0; q < p1; ++q) {
                tp.proj[q - p0] = pool_dev(&pools[q]);
                tp.proj_vcol[q - p0] = vcol[q];
                tc_encode_a(tp, pools[q].A, pools[q].A_elems, d_in, q - p0);
            }
            tp.pool = tp.proj[0];
            if ((e = launch_tc_shrink(tp, N / kTcGroup + n_seg + 1, kk, s)) != cudaSuccess)
                return e;
            p0 = p1;
        }
        return cudaSuccess;
    }
    for (int p = 0; p < n_proj; ++p) {
        ShrinkArgs sa = {};
        sa.X = static_cast<const __nv_bfloat16 *>(X);
        sa.ldx = ldx;
        sa.perm = nullptr;
        sa.groups = groups;
        sa.hdr = hdr;
        sa.mode = kModeSgmv;
        sa.seg_ad = seg_ad;
        sa.pool = pool_dev(&pools[p]);
        sa.kc = d_in;
        sa.V = V + vcol[p];
        sa.ldv = ldv;
        sa.chunk_stride = 0;
        sa.slot_stride = 0;
        sa.err = &hdr->err;
        if ((e = launch_shrink(sa, L.max_groups, 1, 1, s)) != cudaSuccess)
            return e;
    }
    return cudaSuccess;
}

}  // namespace

extern "C" {

const char *lora_version(void) { return "lora_sgmv_b200 0.1 (sm_100a)"; }

size_t lora_workspace_size(int op, int32_t N, int32_t n_adapters, int32_t d_in, int32_t d_out,
                           int32_t max_rank, int32_t n_items, int32_t max_ads_per_req)
{
    if (op == LORA_OP_MERGE)
        return n_adapters >= 1 && n_adapters <= LORA_MAX_ADAPTERS && N == d_out
                   ? merge_workspace_size(d_in, d_out, max_rank) : 0;
    if (op < LORA_OP_BGMV || op > LORA_OP_APPLY_PROJ || op == LORA_OP_MERGE)
        return 0;
    Layout L;
    if (!layout(op, N, n_adapters, d_in, max_rank, n_items, max_ads_per_req, &L))
        return 0;
    return L.total;
}

int lora_kernel_launches(int op, int32_t N, int32_t n_adapters, int32_t d_in, int32_t n_items)
{
    if (N <= 0 || n_adapters < 1 || n_adapters > LORA_MAX_ADAPTERS || d_in <= 0)
        return 0;
    switch (op) {
    case LORA_OP_BGMV:
        return fused_bgmv_supported(N, n_adapters, d_in) ? 1 : 3;
    case LORA_OP_SGMV_SHRINK:
    case LORA_OP_SGMV_EXPAND:
        return n_items > 0 ? 2 : 0;
    case LORA_OP_APPLY_MULTI:
        return n_items > 0 ? 3 : 0;
    case LORA_OP_ROUTE:
        return 1;
    case LORA_OP_MERGE:   // preparation + expand (tensor cores), or + plan + expand
        return tc_enabled() && N >= kTcGroup ? 2 : 3;
    case LORA_OP_LINEAR:  // plan + shrink + projection
        return n_items > 0 ? 3 : 0;
    default:
        return 0;
    }
}

lora_status lora_workspace_init(void *ws, void *stream)
{
    if (!ws || misaligned(ws, kAlign))
        return LORA_ERR_WORKSPACE;
    LORA_CUDA(cudaMemsetAsync(ws, 0, sizeof(WsHeader), (cudaStream_t)stream));
    return LORA_OK;
}

int lora_get_error(void *ws, void *stream)
{
    if (!ws || misaligned(ws, kAlign))
        return LORA_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    uint32_t err = 0;
    if (cudaMemcpyAsync(&err, ws, sizeof err, cudaMemcpyDeviceToHost, s) != cudaSuccess)
        return LORA_ERR_CUDA;
    if (cudaStreamSynchronize(s) != cudaSuccess)
        return LORA_ERR_CUDA;
    if (err) {
        if (cudaMemsetAsync(ws, 0, sizeof err, s) != cudaSuccess || cudaStreamSynchronize(s) != cudaSuccess)
            return LORA_ERR_CUDA;
    }
    return (int)err;
}

lora_status lora_route(const int32_t *ids, int32_t N, int32_t n_adapters, int32_t *perm,
                       int32_t *seg_off, int32_t *seg_ad, int32_t *n_seg_out,
                       void *ws, size_t ws_bytes, void *stream)
{
    if (N < 0 || (N > 0 && (!ids || !perm || !seg_ad)) || !seg_off || !n_seg_out)
        return LORA_ERR_INVALID_ARG;
    if (n_adapters < 1 || n_adapters > LORA_MAX_ADAPTERS)
        return LORA_ERR_UNSUPPORTED;
    Layout L;
    if (!layout(LORA_OP_ROUTE, N, n_adapters, 8, 8, 0, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    PlanArgs pa = {};
    pa.mode = kModeRoute;
    pa.N = N;
    pa.ids = ids;
    pa.n_adapters = n_adapters;
    pa.perm = perm;
    pa.seg_off = seg_off;
    pa.seg_ad = seg_ad;
    pa.n_seg_out = n_seg_out;
    pa.groups = at<Group>(ws, L.groups);
    pa.max_groups = L.max_groups;
    pa.group = kGroup;
    pa.hdr = at<WsHeader>(ws, L.hdr);
    LORA_CUDA(launch_plan(pa, (cudaStream_t)stream));
    return LORA_OK;
}

lora_status lora_bgmv(const void *X, int64_t ldx, void *Y, int64_t ldy, const lora_pool *pool,
                      const int32_t *ids, int32_t N, float scale,
                      void *ws, size_t ws_bytes, void *stream)
{
    LORA_TRY(check_pool(pool));
    if (N < 0 || (N > 0 && !ids))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(X, ldx, pool->d_in, N));
    LORA_TRY(check_mat(Y, ldy, pool->d_out, N));
    Layout L;
    if (!layout(LORA_OP_BGMV, N, pool->n_adapters, pool->d_in, pool->max_rank, 0, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0)
        return LORA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    if (fused_bgmv_supported(N, pool->n_adapters, pool->d_in)) {
        FusedBgmvArgs fa = {};
        fa.X = static_cast<const __nv_bfloat16 *>(X);
        fa.ldx = ldx;
        fa.Y = static_cast<__nv_bfloat16 *>(Y);
        fa.ldy = ldy;
        fa.ids = ids;
        fa.N = N;
        fa.pool = pool_dev(pool);
        fa.scale = scale;
        fa.Wk = fused_chunk(pool->d_in);
        fa.Wo = fused_chunk(pool->d_out);
        fa.err = &hdr->err;
        fa.sched = hdr->sched;
        LORA_CUDA(launch_bgmv_fused(fa, s, pdl_enabled()));
        return LORA_OK;
    }
    int32_t *perm = at<int32_t>(ws, L.perm);
    int32_t *seg_off = at<int32_t>(ws, L.seg_off);
    int32_t *seg_ad = at<int32_t>(ws, L.seg_ad);
    Group *groups = at<Group>(ws, L.groups);
    float *V = at<float>(ws, L.V);

    PlanArgs pa = {};
    pa.mode = kModeRoute;
    pa.N = N;
    pa.ids = ids;
    pa.n_adapters = pool->n_adapters;
    pa.perm = perm;
    pa.seg_off = seg_off;
    pa.seg_ad = seg_ad;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = kGroup;
    pa.hdr = hdr;
    LORA_CUDA(launch_plan(pa, s));

    ShrinkArgs sa = {};
    sa.X = static_cast<const __nv_bfloat16 *>(X);
    sa.ldx = ldx;
    sa.perm = perm;
    sa.groups = groups;
    sa.hdr = hdr;
    sa.mode = kModeRoute;
    sa.seg_ad = seg_ad;
    sa.pool = pool_dev(pool);
    sa.kc = kBgmvChunk;
    sa.V = V;
    sa.ldv = pool->max_rank;
    sa.chunk_stride = (int64_t)N * pool->max_rank;
    sa.slot_stride = 0;
    sa.err = &hdr->err;
    LORA_CUDA(launch_shrink(sa, L.max_groups, L.n_chunks, 1, s));

    ExpandArgs ea = {};
    ea.Y = static_cast<__nv_bfloat16 *>(Y);
    ea.ldy = ldy;
    ea.perm = perm;
    ea.groups = groups;
    ea.hdr = hdr;
    ea.mode = kModeRoute;
    ea.seg_ad = seg_ad;
    ea.scale = scale;
    ea.pool = pool_dev(pool);
    ea.V = V;
    ea.ldv = pool->max_rank;
    ea.chunk_stride = (int64_t)N * pool->max_rank;
    ea.n_chunks = L.n_chunks;
    ea.slot_stride = 0;
    ea.max_ads = 1;
    ea.err = &hdr->err;
    LORA_CUDA(launch_expand(ea, L.max_groups, s));
    return LORA_OK;
}

lora_status lora_sgmv_shrink(const void *X, int64_t ldx, float *V, int64_t ldv,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, void *ws, size_t ws_bytes, void *stream)
{
    LORA_TRY(check_pool(pool));
    if (N < 0 || n_seg < 0 || !seg_off || (n_seg > 0 && !seg_ad))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(X, ldx, pool->d_in, N));
    if ((N > 0 && !V) || ldv < pool->max_rank)
        return LORA_ERR_INVALID_ARG;
    Layout L;
    if (!layout(LORA_OP_SGMV_SHRINK, N, pool->n_adapters, pool->d_in, pool->max_rank, n_seg, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_seg == 0)
        return LORA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);

    if (long_items(N, n_seg) && aligned_v(V, ldv)) {
        TcArgs ta = {};
        tc_encode_a(ta, pool->A, pool->A_elems, pool->d_in);
        if (tc_encode_x(ta, X, N, pool->d_in, ldx)) {
            PlanArgs pa = {};
            pa.mode = kModeSgmv;
            pa.N = N;
            pa.item_off = seg_off;
            pa.n_items = n_seg;
            pa.groups = groups;
            pa.max_groups = L.max_groups;
            pa.group = kTcGroup;
            pa.hdr = hdr;
            LORA_CUDA(launch_plan(pa, s));
            ta.mode = kModeSgmv;
            ta.groups = groups;
            ta.hdr = hdr;
            ta.seg_ad = seg_ad;
            ta.max_ads = 1;
            ta.scale = 1.0f;
            ta.pool = pool_dev(pool);
            ta.V = V;
            ta.ldv = ldv;
            ta.slot_stride = 0;
            ta.err = &hdr->err;
            LORA_CUDA(launch_tc_shrink(ta, N / kTcGroup + n_seg + 1, pool->max_rank, s));
            return LORA_OK;
        }
    }

    PlanArgs pa = {};
    pa.mode = kModeSgmv;
    pa.N = N;
    pa.item_off = seg_off;
    pa.n_items = n_seg;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = kGroup;
    pa.hdr = hdr;
    LORA_CUDA(launch_plan(pa, s));

    ShrinkArgs sa = {};
    sa.X = static_cast<const __nv_bfloat16 *>(X);
    sa.ldx = ldx;
    sa.perm = nullptr;
    sa.groups = groups;
    sa.hdr = hdr;
    sa.mode = kModeSgmv;
    sa.seg_ad = seg_ad;
    sa.pool = pool_dev(pool);
    sa.kc = pool->d_in;
    sa.V = V;
    sa.ldv = ldv;
    sa.chunk_stride = 0;
    sa.slot_stride = 0;
    sa.err = &hdr->err;
    LORA_CUDA(launch_shrink(sa, L.max_groups, 1, 1, s));
    return LORA_OK;
}

lora_status lora_sgmv_shrink_proj(const void *X, int64_t ldx, float *V, int64_t ldv,
                                  const lora_pool *pools, int32_t n_proj, const int32_t *seg_off,
                                  const int32_t *seg_ad, int32_t n_seg, int32_t N,
                                  void *ws, size_t ws_bytes, void *stream)
{
    int32_t vcol[LORA_MAX_PROJ];
    int64_t vcols = 0;
    LORA_TRY(check_proj_pools(pools, n_proj, vcol, &vcols));
    const int32_t d_in = pools[0].d_in;
    if (N < 0 || n_seg < 0 || !seg_off || (n_seg > 0 && !seg_ad))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(X, ldx, d_in, N));
    if ((N > 0 && !V) || ldv < vcols)
        return LORA_ERR_INVALID_ARG;
    Layout L;
    if (!layout(LORA_OP_SGMV_SHRINK, N, pools[0].n_adapters, d_in, pools[0].max_rank, n_seg, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_seg == 0)
        return LORA_OK;
    TcArgs ta = {};
    const bool tc = long_items(N, n_seg) && aligned_v(V, ldv) && tc_encode_x(ta, X, N, d_in, ldx);
    LORA_CUDA(run_proj_shrinks(tc, ta, X, ldx, V, ldv, pools, n_proj, vcol, seg_off, seg_ad, n_seg, N, L, ws,
                               (cudaStream_t)stream));
    return LORA_OK;
}

lora_status lora_sgmv_apply_proj(const void *X, int64_t ldx, void *const *Y, const int64_t *ldy,
                                 const lora_pool *pools, int32_t n_proj, const int32_t *seg_off,
                                 const int32_t *seg_ad, int32_t n_seg, int32_t N, const float *scale,
                                 void *ws, size_t ws_bytes, void *stream)
{
    int32_t vcol[LORA_MAX_PROJ];
    int64_t vcols = 0;
    LORA_TRY(check_proj_pools(pools, n_proj, vcol, &vcols));
    if (!Y || !ldy || !scale)
        return LORA_ERR_INVALID_ARG;
    const int32_t d_in = pools[0].d_in;
    if (N < 0 || n_seg < 0 || !seg_off || (n_seg > 0 && !seg_ad))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(X, ldx, d_in, N));
    for (int p = 0; p < n_proj; ++p)
        LORA_TRY(check_mat(Y[p], ldy[p], pools[p].d_out, N));
    Layout L;
    if (!layout(LORA_OP_APPLY_PROJ, N, pools[0].n_adapters, d_in, (int32_t)vcols, n_seg, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_seg == 0)
        return LORA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);
    float *V = at<float>(ws, L.V);
    const int64_t ldv = vcols;

    // every tensor map is built before the first launch: the path is chosen once
    TcArgs ta = {};
    TcArgs te[LORA_MAX_PROJ];
    bool tc = long_items(N, n_seg) && tc_encode_x(ta, X, N, d_in, ldx);
    for (int p = 0; p < n_proj && tc; ++p) {
        te[p] = TcArgs{};
        tc_encode_b(te[p], pools[p].B, pools[p].B_elems);
        tc = tc_encode_y(te[p], Y[p], N, pools[p].d_out, ldy[p]);
    }
    LORA_CUDA(run_proj_shrinks(tc, ta, X, ldx, V, ldv, pools, n_proj, vcol, seg_off, seg_ad, n_seg, N, L, ws, s));
    if (tc) {
        // every projection's expand in one launch, the GPU's CTAs split among them
        int kk = 0;
        for (int p = 0; p < n_proj; ++p) {
            TcArgs &e = te[p];
            e.mode = kModeSgmv;
            e.groups = groups;
            e.hdr = hdr;
            e.seg_ad = seg_ad;
            e.max_ads = 1;
            e.scale = scale[p];
            e.pool = pool_dev(&pools[p]);
            e.V = V + vcol[p];
            e.ldv = ldv;
            e.slot_stride = 0;
            e.Y = static_cast<__nv_bfloat16 *>(Y[p]);
            e.ldy = ldy[p];
            e.err = &hdr->err;
            kk = pools[p].max_rank > kk ? pools[p].max_rank : kk;
        }
        LORA_CUDA(launch_tc_expand_multi(te, n_proj, kk, s));
        return LORA_OK;
    }
    for (int p = 0; p < n_proj; ++p) {
        {
            ExpandArgs ea = {};
            ea.Y = static_cast<__nv_bfloat16 *>(Y[p]);
            ea.ldy = ldy[p];
            ea.perm = nullptr;
            ea.groups = groups;
            ea.hdr = hdr;
            ea.mode = kModeSgmv;
            ea.seg_ad = seg_ad;
            ea.scale = scale[p];
            ea.pool = pool_dev(&pools[p]);
            ea.V = V + vcol[p];
            ea.ldv = ldv;
            ea.chunk_stride = 0;
            ea.n_chunks = 1;
            ea.slot_stride = 0;
            ea.max_ads = 1;
            ea.err = &hdr->err;
            LORA_CUDA(launch_expand(ea, L.max_groups, s));
        }
    }
    return LORA_OK;
}

lora_status lora_linear_sgmv(const void *X, int64_t ldx, const void *W, int64_t ldw, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, float scale, void *ws, size_t ws_bytes, void *stream)
{
    LORA_TRY(check_pool(pool));
    if (N < 0 || n_seg < 0 || !seg_off || (n_seg > 0 && !seg_ad))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(X, ldx, pool->d_in, N));
    LORA_TRY(check_mat(Y, ldy, pool->d_out, N));
    if (!W)
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(W, ldw, pool->d_in, pool->d_out));
    Layout L;
    if (!layout(LORA_OP_LINEAR, N, pool->n_adapters, pool->d_in, pool->max_rank, n_seg, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_seg == 0)
        return LORA_OK;
    if (!tc_enabled())
        return LORA_ERR_UNSUPPORTED;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);
    __nv_bfloat16 *Vb = at<__nv_bfloat16>(ws, L.V);
    const int64_t ldvb = 2 * (int64_t)L.kv;

    TcArgs ta = {};
    tc_encode_a(ta, pool->A, pool->A_elems, pool->d_in);
    LinArgs la = {};
    la.kv = L.kv;
    if (!tc_encode_x(ta, X, N, pool->d_in, ldx) ||
        !lin_encode(la, X, ldx, N, W, ldw, Vb, ldvb, pool->B, pool->B_elems, pool->d_in, pool->d_out))
        return LORA_ERR_UNSUPPORTED;

    PlanArgs pa = {};
    pa.mode = kModeSgmv;
    pa.N = N;
    pa.item_off = seg_off;
    pa.n_items = n_seg;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = kTcGroup;
    pa.hdr = hdr;
    LORA_CUDA(launch_plan(pa, s));

    // s V for every tile, as bf16 high and low parts
    ta.mode = kModeSgmv;
    ta.groups = groups;
    ta.hdr = hdr;
    ta.seg_ad = seg_ad;
    ta.max_ads = 1;
    ta.scale = scale;
    ta.pool = pool_dev(pool);
    ta.V = nullptr;
    ta.ldv = 0;
    ta.slot_stride = 0;
    ta.Vb = Vb;
    ta.ldvb = ldvb;
    ta.vb_lo = L.kv;
    ta.allow_none = 1;
    ta.err = &hdr->err;
    const int max_tiles = N / kTcGroup + n_seg + 1;
    LORA_CUDA(launch_tc_shrink(ta, max_tiles, pool->max_rank, s));

    la.groups = groups;
    la.hdr = hdr;
    la.seg_ad = seg_ad;
    la.pool = pool_dev(pool);
    la.Y = static_cast<__nv_bfloat16 *>(Y);
    la.ldy = ldy;
    la.err = &hdr->err;
    const int64_t n_ns = (pool->d_out + 255) / 256;
    const int64_t max_units = (int64_t)max_tiles * n_ns;
    LORA_CUDA(launch_tc_linear(la, (int)(max_units < (1 << 30) ? max_units : (1 << 30)), s));
    return LORA_OK;
}

lora_status lora_sgmv_expand(const float *V, int64_t ldv, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *seg_off, const int32_t *seg_ad,
                             int32_t n_seg, int32_t N, float scale,
                             void *ws, size_t ws_bytes, void *stream)
{
    LORA_TRY(check_pool(pool));
    if (N < 0 || n_seg < 0 || !seg_off || (n_seg > 0 && !seg_ad))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_mat(Y, ldy, pool->d_out, N));
    if ((N > 0 && !V) || ldv < pool->max_rank)
        return LORA_ERR_INVALID_ARG;
    Layout L;
    if (!layout(LORA_OP_SGMV_EXPAND, N, pool->n_adapters, pool->d_in, pool->max_rank, n_seg, 1, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_seg == 0)
        return LORA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);

    if (long_items(N, n_seg) && aligned_v(V, ldv)) {
        TcArgs ta = {};
        tc_encode_b(ta, pool->B, pool->B_elems);
        if (tc_encode_y(ta, Y, N, pool->d_out, ldy)) {
            PlanArgs pa = {};
            pa.mode = kModeSgmv;
            pa.N = N;
            pa.item_off = seg_off;
            pa.n_items = n_seg;
            pa.groups = groups;
            pa.max_groups = L.max_groups;
            pa.group = kTcGroup;
            pa.hdr = hdr;
            LORA_CUDA(launch_plan(pa, s));
            ta.mode = kModeSgmv;
            ta.groups = groups;
            ta.hdr = hdr;
            ta.seg_ad = seg_ad;
            ta.max_ads = 1;
            ta.scale = scale;
            ta.pool = pool_dev(pool);
            ta.V = const_cast<float *>(V);
            ta.ldv = ldv;
            ta.slot_stride = 0;
            ta.Y = static_cast<__nv_bfloat16 *>(Y);
            ta.ldy = ldy;
            ta.err = &hdr->err;
            LORA_CUDA(launch_tc_expand(ta, pool->max_rank, s));
            return LORA_OK;
        }
    }

    PlanArgs pa = {};
    pa.mode = kModeSgmv;
    pa.N = N;
    pa.item_off = seg_off;
    pa.n_items = n_seg;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = kGroup;
    pa.hdr = hdr;
    LORA_CUDA(launch_plan(pa, s));

    ExpandArgs ea = {};
    ea.Y = static_cast<__nv_bfloat16 *>(Y);
    ea.ldy = ldy;
    ea.perm = nullptr;
    ea.groups = groups;
    ea.hdr = hdr;
    ea.mode = kModeSgmv;
    ea.seg_ad = seg_ad;
    ea.scale = scale;
    ea.pool = pool_dev(pool);
    ea.V = V;
    ea.ldv = ldv;
    ea.chunk_stride = 0;
    ea.n_chunks = 1;
    ea.slot_stride = 0;
    ea.max_ads = 1;
    ea.err = &hdr->err;
    LORA_CUDA(launch_expand(ea, L.max_groups, s));
    return LORA_OK;
}

lora_status lora_apply_multi(const void *X, int64_t ldx, void *Y, int64_t ldy,
                             const lora_pool *pool, const int32_t *req_off, const int32_t *ad_off,
                             const int32_t *ad_id, const float *ad_scale, int32_t n_req, int32_t N,
                             int32_t max_ads_per_req, void *ws, size_t ws_bytes, void *stream)
{
    LORA_TRY(check_pool(pool));
    if (N < 0 || n_req < 0 || !req_off || !ad_off || (n_req > 0 && (!ad_id || !ad_scale)))
        return LORA_ERR_INVALID_ARG;
    if (max_ads_per_req < 1 || max_ads_per_req > LORA_MAX_ADS_PER_REQ)
        return LORA_ERR_UNSUPPORTED;
    LORA_TRY(check_mat(X, ldx, pool->d_in, N));
    LORA_TRY(check_mat(Y, ldy, pool->d_out, N));
    Layout L;
    if (!layout(LORA_OP_APPLY_MULTI, N, pool->n_adapters, pool->d_in, pool->max_rank, n_req,
                max_ads_per_req, &L))
        return LORA_ERR_INVALID_ARG;
    LORA_TRY(check_ws(ws, ws_bytes, L));
    if (N == 0 || n_req == 0)
        return LORA_OK;
    cudaStream_t s = (cudaStream_t)stream;
    WsHeader *hdr = at<WsHeader>(ws, L.hdr);
    Group *groups = at<Group>(ws, L.groups);
    float *V = at<float>(ws, L.V);
    const int32_t ldv = max_ads_per_req * pool->max_rank;

    if (long_items(N, n_req) && max_ads_per_req * pool->max_rank <= kKMax) {
        TcArgs ta = {};
        tc_encode_a(ta, pool->A, pool->A_elems, pool->d_in);
        tc_encode_b(ta, pool->B, pool->B_elems);
        if (tc_encode_x(ta, X, N, pool->d_in, ldx) && tc_encode_y(ta, Y, N, pool->d_out, ldy)) {
            PlanArgs pa = {};
            pa.mode = kModeMulti;
            pa.N = N;
            pa.item_off = req_off;
            pa.n_items = n_req;
            pa.ad_off = ad_off;
            pa.max_ads = max_ads_per_req;
            pa.groups = groups;
            pa.max_groups = L.max_groups;
            pa.group = kTcGroup;
            pa.hdr = hdr;
            LORA_CUDA(launch_plan(pa, s));
            ta.mode = kModeMulti;
            ta.groups = groups;
            ta.hdr = hdr;
            ta.ad_off = ad_off;
            ta.ad_id = ad_id;
            ta.ad_scale = ad_scale;
            ta.max_ads = max_ads_per_req;
            ta.scale = 1.0f;
            ta.pool = pool_dev(pool);
            ta.V = V;
            ta.ldv = ldv;
            ta.slot_stride = pool->max_rank;
            ta.Y = static_cast<__nv_bfloat16 *>(Y);
            ta.ldy = ldy;
            ta.err = &hdr->err;
            LORA_CUDA(launch_tc_shrink(ta, N / kTcGroup + n_req + 1, max_ads_per_req * pool->max_rank, s));
            LORA_CUDA(launch_tc_expand(ta, max_ads_per_req * pool->max_rank, s));
            return LORA_OK;
        }
    }

    PlanArgs pa = {};
    pa.mode = kModeMulti;
    pa.N = N;
    pa.item_off = req_off;
    pa.n_items = n_req;
    pa.ad_off = ad_off;
    pa.max_ads = max_ads_per_req;
    pa.groups = groups;
    pa.max_groups = L.max_groups;
    pa.group = kGroup;
    pa.hdr = hdr;
    LORA_CUDA(launch_plan(pa, s));

    ShrinkArgs sa = {};
    sa.X = static_cast<const __nv_bfloat16 *>(X);
    sa.ldx = ldx;
    sa.perm = nullptr;
    sa.groups = groups;
    sa.hdr = hdr;
    sa.mode = kModeMulti;
    sa.ad_off = ad_off;
    sa.ad_id = ad_id;
    sa.pool = pool_dev(pool);
    sa.kc = pool->d_in;
    sa.V = V;
    sa.ldv = ldv;
    sa.chunk_stride = 0;
    sa.slot_stride = pool->max_rank;
    sa.err = &hdr->err;
    LORA_CUDA(launch_shrink(sa, L.max_groups, 1, max_ads_per_req, s));

    ExpandArgs ea = {};
    ea.Y = static_cast<__nv_bfloat16 *>(Y);
    ea.ldy = ldy;
    ea.perm = nullptr;
    ea.groups = groups;
    ea.hdr = hdr;
    ea.mode = kModeMulti;
    ea.ad_off = ad_off;
    ea.ad_id = ad_id;
    ea.ad_scale = ad_scale;
    ea.scale = 1.0f;
    ea.pool = pool_dev(pool);
    ea.V = V;
    ea.ldv = ldv;
    ea.chunk_stride = 0;
    ea.n_chunks = 1;
    ea.slot_stride = pool->max_rank;
    ea.max_ads = max_ads_per_req;
    ea.err = &hdr->err;
    LORA_CUDA(launch_expand(ea, L.max_groups, s));
    return LORA_OK;
}

}  // extern "C"
