// CUDA-core shrink and expand over work groups of at most kGroup tokens that
// share one item (a decode adapter group, a prefill segment or a request).
//
// The operation ("Serving several LoRAs, ControlNet and IP-Adapter", section
// "LoRA: merged or alongside"): the unmerged LoRA adds x A^T B^T, i.e. per
// token v = A x (shrink, d_in -> r) and y += s B v (expand, r -> d_out).  For
// decode this is a gather matrix-vector product ("Punica: multi-tenant LoRA
// serving", contribution 1: segmented gather matrix-vector kernels) and is
// bound by streaming each distinct adapter's A and B rows from HBM:
//
// * shrink: CTA (group, d_in chunk, stacked adapter).  The group's X rows for
//   the chunk are staged in shared memory as fp32; each warp owns rank rows
//   of A, streams them with 16-byte non-allocating loads, and reduces each
//   token's dot product with warp shuffles.  The rank-r partial stays in
//   shared memory until it is written once per (token, rank row).
// * expand: CTA (group, 1024 outputs).  The rank-r vectors of the group's
//   tokens (summed over the shrink's d_in chunks) sit in shared memory; each
//   thread owns 8 consecutive outputs, streams their B rows with 16-byte
//   loads, and updates y with one 16-byte read and one 16-byte write per
//   token, adding every stacked adapter's contribution before the single
//   bf16 rounding.

#include "lora_internal.cuh"

namespace lora {
namespace {

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    // weights are read once per CTA: keep them out of L1
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

__device__ __forceinline__ void unpack8(uint4 u, float *f)
{
    f[0] = __uint_as_float(u.x << 16);
    f[1] = __uint_as_float(u.x & 0xffff0000u);
    f[2] = __uint_as_float(u.y << 16);
    f[3] = __uint_as_float(u.y & 0xffff0000u);
    f[4] = __uint_as_float(u.z << 16);
    f[5] = __uint_as_float(u.z & 0xffff0000u);
    f[6] = __uint_as_float(u.w << 16);
    f[7] = __uint_as_float(u.w & 0xffff0000u);
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi)
{
    const uint32_t l = __bfloat16_as_ushort(__float2bfloat16_rn(lo));
    const uint32_t h = __bfloat16_as_ushort(__float2bfloat16_rn(hi));
    return l | (h << 16);
}

__device__ __forceinline__ float warp_sum(float v)
{
#pragma unroll
    for (int off = 16; off > 0; off >>= 1)
        v += __shfl_xor_sync(0xffffffffu, v, off);
    return v;
}

// Adapter a is usable: id in range, rank a multiple of 8 in [8, max_rank],
// both matrix offsets non-negative multiples of 8 with the matrices inside
// the pool.  Shrink and expand apply the same test, so an adapter is either
// computed by both or skipped by both.
__device__ __forceinline__ bool adapter_ok(const PoolDev &P, int32_t a, int32_t *r_out,
                                           int64_t *aoff_out, int64_t *boff_out)
{
    if (a < 0 || a >= P.n_adapters)
        return false;
    const int32_t r = P.rank[a];
    if (r < 8 || r > P.max_rank || (r & 7))
        return false;
    const int64_t ao = P.A_off[a], bo = P.B_off[a];
    if (ao < 0 || (ao & 7) || ao + (int64_t)r * P.d_in > P.A_elems)
        return false;
    if (bo < 0 || (bo & 7) || bo + (int64_t)r * P.d_out > P.B_elems)
        return false;
    *r_out = r;
    *aoff_out = ao;
    *boff_out = bo;
    return true;
}

__global__ void __launch_bounds__(kThreads) k_shrink(ShrinkArgs p)
{
    __shared__ __align__(16) float xs[kGroup][kStageK];
    __shared__ float vacc[kGroup][kMaxRank];
    __shared__ int32_t tok[kGroup];

    const int g = blockIdx.x;
    if (g >= p.hdr->n_groups)
        return;
    const Group grp = p.groups[g];
    const int c = blockIdx.y;
    const int k = blockIdx.z;
    int32_t a;
    if (p.mode == kModeMulti) {
        const int32_t lo = p.ad_off[grp.item];
        if (k >= p.ad_off[grp.item + 1] - lo)
            return;
        a = p.ad_id[lo + k];
    } else {
        if (k > 0)
            return;
        a = p.seg_ad[grp.item];
    }
    int32_t r;
    int64_t aoff, boff;
    if (!adapter_ok(p.pool, a, &r, &aoff, &boff)) {
        if (threadIdx.x == 0)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        return;
    }
    const int i0 = c * p.kc;
    const int i1 = min(p.pool.d_in, i0 + p.kc);
    const int cnt = grp.cnt;
    if (threadIdx.x < cnt)
        tok[threadIdx.x] = p.perm ? p.perm[grp.p0 + threadIdx.x] : grp.p0 + threadIdx.x;
    for (int e = threadIdx.x; e < kGroup * kMaxRank; e += kThreads)
        (&vacc[0][0])[e] = 0.f;
    __syncthreads();

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const __nv_bfloat16 *Aa = p.pool.A + aoff;
    for (int s0 = i0; s0 < i1; s0 += kStageK) {
        const int nv = min(kStageK, i1 - s0) >> 3;   // 8-element vectors in this stage
        for (int idx = threadIdx.x; idx < cnt * nv; idx += kThreads) {
            const int t = idx / nv, v = idx - t * nv;
            const uint4 u = __ldg(reinterpret_cast<const uint4 *>(p.X + (int64_t)tok[t] * p.ldx + s0 + v * 8));
            float f[8];
            unpack8(u, f);
            *reinterpret_cast<float4 *>(&xs[t][v * 8]) = make_float4(f[0], f[1], f[2], f[3]);
            *reinterpret_cast<float4 *>(&xs[t][v * 8 + 4]) = make_float4(f[4], f[5], f[6], f[7]);
        }
        __syncthreads();
        for (int j = warp; j < r; j += kThreads / 32) {
            float acc[kGroup];
#pragma unroll
            for (int t = 0; t < kGroup; ++t)
                acc[t] = 0.f;
            const __nv_bfloat16 *Arow = Aa + (int64_t)j * p.pool.d_in + s0;
            for (int v = lane; v < nv; v += 32) {
                float af[8];
                unpack8(ld_stream(Arow + v * 8), af);
#pragma unroll
                for (int t = 0; t < kGroup; ++t) {
                    if (t < cnt) {
                        const float4 x0 = *reinterpret_cast<const float4 *>(&xs[t][v * 8]);
                        const float4 x1 = *reinterpret_cast<const float4 *>(&xs[t][v * 8 + 4]);
                        float s = acc[t];
                        s = fmaf(af[0], x0.x, s);
                        s = fmaf(af[1], x0.y, s);
                        s = fmaf(af[2], x0.z, s);
                        s = fmaf(af[3], x0.w, s);
                        s = fmaf(af[4], x1.x, s);
                        s = fmaf(af[5], x1.y, s);
                        s = fmaf(af[6], x1.z, s);
                        s = fmaf(af[7], x1.w, s);
                        acc[t] = s;
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kGroup; ++t)
                if (t < cnt)
                    acc[t] = warp_sum(acc[t]);
            if (lane == 0) {
#pragma unroll
                for (int t = 0; t < kGroup; ++t)
                    if (t < cnt)
                        vacc[t][j] += acc[t];
            }
        }
        __syncthreads();
    }
    float *V = p.V + (int64_t)c * p.chunk_stride + (int64_t)k * p.slot_stride;
    for (int idx = threadIdx.x; idx < cnt * r; idx += kThreads) {
        const int t = idx / r, j = idx - t * r;
        V[(int64_t)(grp.p0 + t) * p.ldv + j] = vacc[t][j];
    }
}

__global__ void __launch_bounds__(kThreads) k_expand(ExpandArgs p)
{
    __shared__ float vs[LORA_MAX_ADS_PER_REQ][kGroup][kMaxRank];
    __shared__ int32_t tok[kGroup];
    __shared__ int32_t s_r[LORA_MAX_ADS_PER_REQ];
    __shared__ int64_t s_off[LORA_MAX_ADS_PER_REQ];
    __shared__ float s_scale[LORA_MAX_ADS_PER_REQ];
    __shared__ int32_t s_np;

    const int g = blockIdx.x;
    if (g >= p.hdr->n_groups)
        return;
    const Group grp = p.groups[g];
    const int cnt = grp.cnt;
    if (threadIdx.x == 0) {
        int32_t np, lo = 0;
        if (p.mode == kModeMulti) {
            lo = p.ad_off[grp.item];
            np = min(p.ad_off[grp.item + 1] - lo, p.max_ads);
        } else {
            np = 1;
        }
        bool bad = false;
        for (int k = 0; k < np; ++k) {
            const int32_t a = p.mode == kModeMulti ? p.ad_id[lo + k] : p.seg_ad[grp.item];
            int32_t r = 0;
            int64_t aoff = 0, off = 0;
            if (!adapter_ok(p.pool, a, &r, &aoff, &off)) {
                r = 0;
                bad = true;
            }
            s_r[k] = r;
            s_off[k] = off;
            s_scale[k] = p.mode == kModeMulti ? p.ad_scale[lo + k] : p.scale;
        }
        s_np = np;
        if (bad && blockIdx.y == 0)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
    }
    if (threadIdx.x < cnt)
        tok[threadIdx.x] = p.perm ? p.perm[grp.p0 + threadIdx.x] : grp.p0 + threadIdx.x;
    __syncthreads();
    const int np = s_np;
    for (int k = 0; k < np; ++k) {
        const int r = s_r[k];
        for (int idx = threadIdx.x; idx < cnt * r; idx += kThreads) {
            const int t = idx / r, j = idx - t * r;
            const float *src = p.V + (int64_t)(grp.p0 + t) * p.ldv + (int64_t)k * p.slot_stride + j;
            float s = 0.f;
            for (int c = 0; c < p.n_chunks; ++c)
                s += src[(int64_t)c * p.chunk_stride];
            vs[k][t][j] = s;
        }
    }
    __syncthreads();

    const int o0 = blockIdx.y * kExpandTile + threadIdx.x * kExpandPerThread;
    if (o0 >= p.pool.d_out)
        return;
    float acc[kExpandPerThread][kGroup];
#pragma unroll
    for (int e = 0; e < kExpandPerThread; ++e)
#pragma unroll
        for (int t = 0; t < kGroup; ++t)
            acc[e][t] = 0.f;
    for (int k = 0; k < np; ++k) {
        const int r = s_r[k];
        if (r == 0)
            continue;
        const float sc = s_scale[k];
        const __nv_bfloat16 *Bk = p.pool.B + s_off[k];
#pragma unroll
        for (int e = 0; e < kExpandPerThread; ++e) {
            const __nv_bfloat16 *row = Bk + (int64_t)(o0 + e) * r;
            float part[kGroup];
#pragma unroll
            for (int t = 0; t < kGroup; ++t)
                part[t] = 0.f;
            for (int jv = 0; jv < r; jv += 8) {
                float bf[8];
                unpack8(ld_stream(row + jv), bf);
#pragma unroll
                for (int t = 0; t < kGroup; ++t) {
                    if (t < cnt) {
                        float s = part[t];
#pragma unroll
                        for (int q = 0; q < 8; ++q)
                            s = fmaf(bf[q], vs[k][t][jv + q], s);
                        part[t] = s;
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kGroup; ++t)
                acc[e][t] = fmaf(sc, part[t], acc[e][t]);
        }
    }
#pragma unroll
    for (int t = 0; t < kGroup; ++t) {
        if (t < cnt) {
            __nv_bfloat16 *yp = p.Y + (int64_t)tok[t] * p.ldy + o0;
            const uint4 u = *reinterpret_cast<const uint4 *>(yp);
            float y[8];
            unpack8(u, y);
            uint4 w;
            w.x = pack2(y[0] + acc[0][t], y[1] + acc[1][t]);
            w.y = pack2(y[2] + acc[2][t], y[3] + acc[3][t]);
            w.z = pack2(y[4] + acc[4][t], y[5] + acc[5][t]);
            w.w = pack2(y[6] + acc[6][t], y[7] + acc[7][t]);
            *reinterpret_cast<uint4 *>(yp) = w;
        }
    }
}

}  // namespace

cudaError_t launch_shrink(const ShrinkArgs &a, int grid_groups, int n_chunks, int max_ads, cudaStream_t s)
{
    if (grid_groups <= 0)
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_groups, n_chunks, max_ads);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, k_shrink, a);
}

cudaError_t launch_expand(const ExpandArgs &a, int grid_groups, cudaStream_t s)
{
    if (grid_groups <= 0)
        return cudaSuccess;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid_groups, (a.pool.d_out + kExpandTile - 1) / kExpandTile, 1);
    cfg.blockDim = dim3(kThreads);
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, k_expand, a);
}

}  // namespace lora
