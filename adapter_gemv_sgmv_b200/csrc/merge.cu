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
        // B_a rows o0 .. o0 + 63 widened to fp32
        const int o0 = (blockIdx.x - p.nbA) * kPrepCols;
        const __nv_bfloat16 *Ba = p.pool.B + s_bo;
        for (int e = tid; e < r * kPrepCols; e += kPrepThreads) {
            const int oo = e / r, j = e - oo * r;
            if (o0 + oo < d_out)
                p.Bf[(int64_t)(o0 + oo) * p.ld + j] = __bfloat162float(Ba[(int64_t)(o0 + oo) * r + j]);
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
    pa.err = &reinterpret_cast<WsHeader *>(w + L.expand_ws)->err;
    pa.At = At;
    pa.Bf = Bf;
    const int nbB = (pool->d_out + kPrepCols - 1) / kPrepCols;
    k_merge_prep<<<pa.nbA + nbB, kPrepThreads, 0, s>>>(pa);
    if (cudaGetLastError() != cudaSuccess)
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
    return lora_sgmv_expand(Bf, pool->max_rank, W, ldw, &tmp, meta->seg_off, meta->seg_ad, 1, pool->d_out, scale,
                            w + L.expand_ws, L.meta, stream);
}
