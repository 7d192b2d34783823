// lora_merge: W <- W + s B_a A_a in place ("Serving several LoRAs, ControlNet
// and IP-Adapter", section "LoRA: merged or alongside": merging folds B A into
// the weight; switching adapters unmerges one and merges another).
//
// The update is the expand of the unmerged path with the roles renamed: the
// rows of W are the "tokens" (one segment of d_out rows), B_a [d_out, r] is
// their rank-r "intermediate", and A_a^T [d_in, r] is the "B" of a one-adapter
// pool whose outputs are W's columns.  A small kernel writes A_a^T (bf16,
// row stride r) and B_a widened to fp32 into the workspace, with the metadata
// of that one-adapter pool; lora_sgmv_expand then does the streaming update
// (tcgen05 tiles for d_out >= 128, CUDA cores below).

#include <cstring>

#include "lora_internal.cuh"

using namespace lora;

namespace {

constexpr int kPrepThreads = 256;
constexpr int kPrepCols = 64;     // A columns (or B rows) per block

struct MergeMeta {                // the one-adapter pool and its single segment
    int32_t seg_off[2];
    int32_t seg_ad[1];
    int32_t rank[1];
    int64_t A_off[1];
    int64_t B_off[1];
};

struct PrepArgs {
    PoolDev pool;
    int32_t a;
    int32_t ld;                   // row stride of the fp32 copy of B_a (= max_rank)
    int32_t nbA;                  // blocks transposing A_a; the rest widen B_a
    MergeMeta *meta;
    uint32_t *err;                // the workspace's error word
    WsHeader *hdr;                // direct tensor-core path: the tiles of W's rows (else nullptr)
    Group *groups;
    int32_t n_tiles;
    __nv_bfloat16 *At;            // [d_in][r]
    float *Bf;                    // [d_out][ld]
};

__device__ bool merge_adapter_ok(const PoolDev &P, int32_t a, int32_t *r_out, int64_t *ao, int64_t *bo)
{
    if (a < 0 || a >= P.n_adapters)
        return false;
    const int32_t r = P.rank[a];
    const int64_t A0 = P.A_off[a], B0 = P.B_off[a];
    if (r < 8 || r > P.max_rank || (r & 7))
        return false;
    if (A0 < 0 || (A0 & 7) || A0 + (int64_t)r * P.d_in > P.A_elems)
        return false;
    if (B0 < 0 || (B0 & 7) || B0 + (int64_t)r * P.d_out > P.B_elems)
        return false;
    *r_out = r;
    *ao = A0;
    *bo = B0;
    return true;
}

__global__ void __launch_bounds__(kPrepThreads) k_merge_prep(PrepArgs p)
{
    __shared__ __nv_bfloat16 tile[kMaxRank][kPrepCols + 2];
    __shared__ int32_t s_r;
    __shared__ int64_t s_ao, s_bo;
    const int tid = threadIdx.x;
    // programmatic dependent launch: the previous kernel (which may still use W or the
    // workspace) completes first; the next one may start its prologue
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    if (blockIdx.x == 0 && p.hdr) {
        // W's rows as one segment, cut into tiles of kTcGroup rows
        for (int t = tid; t < p.n_tiles; t += kPrepThreads) {
            Group g;
            g.p0 = t * kTcGroup;
            g.cnt = min(kTcGroup, p.pool.d_out - t * kTcGroup);
            g.item = 0;
            g.pad = 0;
            p.groups[t] = g;
        }
        if (tid == 0)
            p.hdr->n_groups = p.n_tiles;
    }
    if (tid == 0) {
        int32_t r = 0;
        int64_t ao = 0, bo = 0;
        if (!merge_adapter_ok(p.pool, p.a, &r, &ao, &bo)) {
            r = 0;                // the expand then finds no valid adapter: W stays as it is
            if (blockIdx.x == 0)
                atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        }
        s_r = r;
        s_ao = ao;
        s_bo = bo;
        if (blockIdx.x == 0) {
            p.meta->seg_off[0] = 0;
            p.meta->seg_off[1] = p.pool.d_out;
            p.meta->seg_ad[0] = 0;
            p.meta->rank[0] = r;
            p.meta->A_off[0] = 0;
            p.meta->B_off[0] = 0;
        }
    }
    __syncthreads();
    const int r = s_r;
    if (r == 0)
        return;
    const int d_in = p.pool.d_in, d_out = p.pool.d_out;
    if ((int)blockIdx.x < p.nbA) {
        // A_a^T: columns i0 .. i0 + 63 of A_a's r rows, through shared memory
        const int i0 = blockIdx.x * kPrepCols;
        const __nv_bfloat16 *Aa = p.pool.A + s_ao;
        for (int e = tid; e < r * kPrepCols; e += kPrepThreads) {
            const int j = e / kPrepCols, ii = e - j * kPrepCols;
            tile[j][ii] = i0 + ii < d_in ? Aa[(int64_t)j * d_in + i0 + ii] : __float2bfloat16(0.f);
        }
        __syncthreads();
        for (int e = tid; e < r * kPrepCols; e += kPrepThreads) {
            const int ii = e / r, j = e - ii * r;
            if (i0 + ii < d_in)
                p.At[(int64_t)(i0 + ii) * r + j] = tile[j][ii];
        }
    } else {
        // B_a rows o0 .. o0 + 63 widened to fp32, 8 elements (16 bytes in, 32 out) at a time
        const int o0 = (blockIdx.x - p.nbA) * kPrepCols;
        const __nv_bfloat16 *Ba = p.pool.B + s_bo;
        const int cpr = r / 8;
        for (int e = tid; e < cpr * kPrepCols; e += kPrepThreads) {
            const int oo = e / cpr, j = (e - oo * cpr) * 8;
            if (o0 + oo < d_out) {
                const uint4 v = *reinterpret_cast<const uint4 *>(Ba + (int64_t)(o0 + oo) * r + j);
                const __nv_bfloat162 *h = reinterpret_cast<const __nv_bfloat162 *>(&v);
                const float2 f0 = __bfloat1622float2(h[0]), f1 = __bfloat1622float2(h[1]);
                const float2 f2 = __bfloat1622float2(h[2]), f3 = __bfloat1622float2(h[3]);
                float4 *dst = reinterpret_cast<float4 *>(p.Bf + (int64_t)(o0 + oo) * p.ld + j);
                dst[0] = make_float4(f0.x, f0.y, f1.x, f1.y);
                dst[1] = make_float4(f2.x, f2.y, f3.x, f3.y);
            }
        }
    }
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

struct MergeLayout {
    size_t expand_ws, meta, At, Bf, total;
};

bool merge_layout(int32_t d_in, int32_t d_out, int32_t max_rank, MergeLayout *L)
{
    if (d_in <= 0 || d_out <= 0 || max_rank < 8 || max_rank > LORA_MAX_RANK)
        return false;
    // the expand runs over a one-adapter pool: 8 "input" columns, d_in outputs
    const size_t e = lora_workspace_size(LORA_OP_SGMV_EXPAND, d_out, 1, 8, d_in, max_rank, 1, 1);
    if (e == 0)
        return false;
    L->expand_ws = 0;
    size_t off = align256(e);
    L->meta = off;
    off = align256(off + sizeof(MergeMeta));
    L->At = off;
    off = align256(off + (size_t)d_in * max_rank * 2);
    L->Bf = off;
    off = align256(off + (size_t)d_out * max_rank * 4);
    L->total = off;
    return true;
}

}  // namespace

namespace lora {
size_t merge_workspace_size(int32_t d_in, int32_t d_out, int32_t max_rank)
{
    MergeLayout L;
    return merge_layout(d_in, d_out, max_rank, &L) ? L.total : 0;
}
}  // namespace lora

extern "C" lora_status lora_merge(void *W, int64_t ldw, const lora_pool *pool, int32_t adapter, float scale,
                                  void *ws, size_t ws_bytes, void *stream)
{
    if (!pool || !pool->A || !pool->B || !pool->A_off || !pool->B_off || !pool->rank || pool->A_elems < 0 ||
        pool->B_elems < 0)
        return LORA_ERR_INVALID_ARG;
    if (pool->n_adapters < 1 || pool->n_adapters > LORA_MAX_ADAPTERS || pool->d_in <= 0 || pool->d_out <= 0 ||
        (pool->d_in & 7) || (pool->d_out & 7) || pool->max_rank < 8 || pool->max_rank > LORA_MAX_RANK ||
        (pool->max_rank & 7) || ((uintptr_t)pool->A & 15) || ((uintptr_t)pool->B & 15))
        return LORA_ERR_UNSUPPORTED;
    if (adapter < 0 || adapter >= pool->n_adapters || !W || ldw < pool->d_in)
        return LORA_ERR_INVALID_ARG;
    if ((ldw & 7) || ((uintptr_t)W & 15))
        return LORA_ERR_UNSUPPORTED;
    MergeLayout L;
    if (!merge_layout(pool->d_in, pool->d_out, pool->max_rank, &L))
        return LORA_ERR_INVALID_ARG;
    if (!ws || ((uintptr_t)ws & 255) || ws_bytes < L.total)
        return LORA_ERR_WORKSPACE;
    cudaStream_t s = (cudaStream_t)stream;
    char *w = static_cast<char *>(ws);
    MergeMeta *meta = reinterpret_cast<MergeMeta *>(w + L.meta);
    __nv_bfloat16 *At = reinterpret_cast<__nv_bfloat16 *>(w + L.At);
    float *Bf = reinterpret_cast<float *>(w + L.Bf);

    PrepArgs pa = {};
    pa.pool.A = static_cast<const __nv_bfloat16 *>(pool->A);
    pa.pool.B = static_cast<const __nv_bfloat16 *>(pool->B);
    pa.pool.A_off = pool->A_off;
    pa.pool.B_off = pool->B_off;
    pa.pool.rank = pool->rank;
    pa.pool.A_elems = pool->A_elems;
    pa.pool.B_elems = pool->B_elems;
    pa.pool.n_adapters = pool->n_adapters;
    pa.pool.max_rank = pool->max_rank;
    pa.pool.d_in = pool->d_in;
    pa.pool.d_out = pool->d_out;
    pa.a = adapter;
    pa.ld = pool->max_rank;
    pa.nbA = (pool->d_in + kPrepCols - 1) / kPrepCols;
    pa.meta = meta;
    WsHeader *hdr = reinterpret_cast<WsHeader *>(w + L.expand_ws);
    pa.err = &hdr->err;
    // the tensor-core expand is launched directly on W's tiles (written by the
    // preparation kernel where lora_sgmv_expand's plan kernel would put them)
    const bool direct = tc_enabled() && pool->d_out >= kTcGroup;
    Group *groups = reinterpret_cast<Group *>(w + L.expand_ws + sizeof(WsHeader));
    pa.n_tiles = (pool->d_out + kTcGroup - 1) / kTcGroup;
    pa.hdr = direct ? hdr : nullptr;
    pa.groups = groups;
    pa.At = At;
    pa.Bf = Bf;
    const int nbB = (pool->d_out + kPrepCols - 1) / kPrepCols;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(pa.nbA + nbB);
    cfg.blockDim = dim3(kPrepThreads);
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    if (cudaLaunchKernelEx(&cfg, k_merge_prep, pa) != cudaSuccess)
        return LORA_ERR_CUDA;

    // the one-adapter pool: its "B" is A_a^T ([d_in, r], offset 0), 8 dummy inputs
    lora_pool tmp;
    std::memset(&tmp, 0, sizeof tmp);
    tmp.A = At;
    tmp.B = At;
    tmp.A_off = meta->A_off;
    tmp.B_off = meta->B_off;
    tmp.rank = meta->rank;
    tmp.A_elems = (int64_t)pool->d_in * pool->max_rank;
    tmp.B_elems = (int64_t)pool->d_in * pool->max_rank;
    tmp.n_adapters = 1;
    tmp.d_in = 8;
    tmp.d_out = pool->d_in;
    tmp.max_rank = pool->max_rank;
    if (direct) {
        TcArgs ta = {};
        tc_encode_b(ta, At, tmp.B_elems);
        if (tc_encode_y(ta, W, pool->d_out, pool->d_in, ldw)) {
            ta.mode = kModeSgmv;
            ta.groups = groups;
            ta.hdr = hdr;
            ta.seg_ad = meta->seg_ad;
            ta.max_ads = 1;
            ta.scale = scale;
            ta.pool.A = At;
            ta.pool.B = At;
            ta.pool.A_off = meta->A_off;
            ta.pool.B_off = meta->B_off;
            ta.pool.rank = meta->rank;
            ta.pool.A_elems = tmp.A_elems;
            ta.pool.B_elems = tmp.B_elems;
            ta.pool.n_adapters = 1;
            ta.pool.max_rank = tmp.max_rank;
            ta.pool.d_in = tmp.d_in;
            ta.pool.d_out = tmp.d_out;
            ta.V = Bf;
            ta.ldv = pool->max_rank;
            ta.slot_stride = 0;
            ta.Y = static_cast<__nv_bfloat16 *>(W);
            ta.ldy = ldw;
            ta.err = &hdr->err;
            return launch_tc_expand(ta, pool->max_rank, s) == cudaSuccess ? LORA_OK : LORA_ERR_CUDA;
        }
        // no tensor map: the tiles are written, but the general path re-plans them
    }
    return lora_sgmv_expand(Bf, pool->max_rank, W, ldw, &tmp, meta->seg_off, meta->seg_ad, 1, pool->d_out, scale,
                            w + L.expand_ws, L.meta, stream);
}
