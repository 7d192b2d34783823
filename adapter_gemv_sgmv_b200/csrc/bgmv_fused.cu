// Decode BGMV in one launch: grouping, shrink and expand fused; one
// thread-block cluster per (adapter, group of <= kFT tokens) item.
//
// The operation ("Serving several LoRAs, ControlNet and IP-Adapter", section
// "LoRA: merged or alongside" and exercise 2's answer): y[n] += s B[a] A[a] x[n]
// for a batch whose tokens carry their own adapter ids, grouped by adapter so
// that each distinct adapter's A and B are streamed from HBM once (the
// segmented gather matrix-vector product of "Punica: multi-tenant LoRA
// serving", contribution 1).
//
// Work layout on B200:
// * every CTA rebuilds the grouping in shared memory (ids -> per-adapter
//   counts -> exclusive scan of groups per adapter); item k is the k-th
//   (adapter, group) pair in adapter order.  Clusters are persistent: the
//   grid holds as many clusters as fit on the GPU at once, and cluster c
//   takes items c, c + n_clusters, ...;
// * the kFC CTAs of a cluster split d_in for the shrink: CTA c reduces its
//   d_in chunk for all tokens of the item with 16-byte streaming loads of A,
//   packed fp32x2 FMAs over token pairs and a warp reduce-scatter, leaving a
//   partial rank-r vector per token in its shared memory;
// * after a cluster barrier every CTA sums the kFC partials through
//   distributed shared memory (fixed order, so the result is deterministic)
//   and expands its own d_out chunk: B rows streamed with 16-byte loads, y
//   read and written once, two outputs per thread per step;
// * the item's B chunk and y rows are bulk-prefetched into L2 before the
//   shrink, so their HBM latency hides behind the shrink and the exchange;
// * programmatic dependent launch: the grouping and the L2 prefetch of the
//   first item's adapter weights (immutable inputs) run before
//   griddepcontrol.wait, i.e. while the previous kernel on the stream is
//   still finishing; x, y and the workspace are touched only after it.

#include <cooperative_groups.h>

#include <mutex>

#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kXPad = 68;   // floats per 8-column vector of staged x (64 + 4: no bank conflicts)

__device__ __forceinline__ uint4 ld_stream(const void *p)
{
    uint4 r;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
                 : "l"(p));
    return r;
}

// element e (0..7) of 8 packed bf16 values, widened exactly to fp32
__device__ __forceinline__ float bf_at(const uint4 &u, int e)
{
    const uint32_t w = e < 2 ? u.x : e < 4 ? u.y : e < 6 ? u.z : u.w;
    return (e & 1) ? __uint_as_float(w & 0xffff0000u) : __uint_as_float(w << 16);
}

// (d0, d1) += (a0, a1) * (b0, b1), one rounding per lane (Blackwell packed FMA)
__device__ __forceinline__ void ffma2(float &d0, float &d1, float a0, float a1, float b0, float b1)
{
    asm("{\n\t.reg .b64 ra, rb, rc;\n\tmov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "mov.b64 rc, {%0, %1};\n\tfma.rn.f32x2 rc, ra, rb, rc;\n\tmov.b64 {%0, %1}, rc;\n\t}"
        : "+f"(d0), "+f"(d1)
        : "f"(a0), "f"(a1), "f"(b0), "f"(b1));
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    // p 16-byte aligned, bytes a non-zero multiple of 16
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint32_t cluster_ctarank()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t cluster_id_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ uint32_t n_clusters_x()
{
    uint32_t r;
    asm volatile("mov.u32 %0, %%nclusterid.x;" : "=r"(r));
    return r;
}

__device__ __forceinline__ void cluster_arrive() { asm volatile("barrier.cluster.arrive.release.aligned;" ::: "memory"); }
__device__ __forceinline__ void cluster_wait() { asm volatile("barrier.cluster.wait.acquire.aligned;" ::: "memory"); }
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

#ifdef LORA_PHASE_TIMING
// Development aid: per-CTA %globaltimer stamps at phase boundaries of the first item.
__device__ unsigned long long g_phase[65536 * 12];
#define PHASE(i)                                                                     \
    do {                                                                             \
        if (threadIdx.x == 0 && first && blockIdx.x < 65536) {                       \
            unsigned long long t_;                                                   \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                   \
            g_phase[blockIdx.x * 12 + (i)] = t_;                                     \
        }                                                                            \
    } while (0)
#else
#define PHASE(i) \
    do {         \
    } while (0)
#endif

// Sum 32 per-lane values v[0..31] over the 32 lanes of a warp so that lane l
// ends with the total of value l (31 shuffles instead of 32 x 5).
__device__ __forceinline__ float reduce_scatter32(float (&v)[32], int lane)
{
#pragma unroll
    for (int s = 16; s >= 1; s >>= 1) {
        const bool upper = (lane & s) != 0;
#pragma unroll
        for (int i = 0; i < s; ++i) {
            const float send = upper ? v[i] : v[i + s];
            const float keep = upper ? v[i + s] : v[i];
            v[i] = keep + __shfl_xor_sync(0xffffffffu, send, s);
        }
    }
    return v[0];
}

__device__ __forceinline__ bool adapter_ok(const PoolDev &P, int32_t a, int32_t *r_out, int64_t *aoff,
                                           int64_t *boff)
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
    *aoff = ao;
    *boff = bo;
    return true;
}

__global__ void __launch_bounds__(kFThreads, 6) k_bgmv_fused(FusedBgmvArgs p)
{
    extern __shared__ __align__(16) unsigned char sm_raw[];
    const FusedSmem L = fused_smem_layout(p.N, p.pool.n_adapters, p.Wk);
    int32_t *ids_s = reinterpret_cast<int32_t *>(sm_raw + L.ids);
    int32_t *ipre = reinterpret_cast<int32_t *>(sm_raw + L.cnt);    // [n_ad + 1]
    float *xs = reinterpret_cast<float *>(sm_raw + L.xs);           // [Wk/8][kXPad]
    float *vpart = reinterpret_cast<float *>(sm_raw + L.vpart);     // [kMaxRank][kFT], read by the cluster
    float *vsum = reinterpret_cast<float *>(sm_raw + L.vsum);       // [kMaxRank][kFT]
    __shared__ int32_t tok[kFT];
    __shared__ int32_t s_ad, s_g, s_cnt, s_bad;
    __shared__ int32_t sm_scan[kFWarps + 1];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const uint32_t crank = cluster_ctarank();
    const int N = p.N, n_ad = p.pool.n_adapters;
    const int d_in = p.pool.d_in, d_out = p.pool.d_out;
    [[maybe_unused]] bool first = true;
    PHASE(0);

    // ---- grouping, rebuilt by every CTA in shared memory (immutable inputs only)
    for (int a = tid; a < n_ad; a += kFThreads)
        ipre[a] = 0;
    if (tid == 0)
        s_bad = 0;
    __syncthreads();
    for (int n = tid; n < N; n += kFThreads) {
        const int32_t a = p.ids[n];
        ids_s[n] = a;
        if (a >= 0 && a < n_ad)
            atomicAdd(&ipre[a], 1);
        else if (a != -1)
            s_bad = 1;
    }
    __syncthreads();
    PHASE(1);
    {
        // counts -> exclusive prefix of groups per adapter, ipre[n_ad] = total
        const int per = (n_ad + kFThreads - 1) / kFThreads;
        const int b = tid * per, e = min(n_ad, b + per);
        int local = 0;
        for (int a = b; a < e; ++a)
            local += (ipre[a] + kFT - 1) / kFT;
        int incl = local;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            if (lane >= off)
                incl += v;
        }
        if (lane == 31)
            sm_scan[warp] = incl;
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            for (int w = 0; w < kFWarps; ++w) {
                const int t = sm_scan[w];
                sm_scan[w] = run;
                run += t;
            }
            sm_scan[kFWarps] = run;
        }
        __syncthreads();
        int run = sm_scan[warp] + incl - local;
        for (int a = b; a < e; ++a) {
            const int g = (ipre[a] + kFT - 1) / kFT;
            ipre[a] = run;
            run += g;
        }
        if (tid == 0)
            ipre[n_ad] = sm_scan[kFWarps];
        __syncthreads();
    }
    PHASE(2);
    const int n_items = ipre[n_ad];
    const int n_cl = (int)n_clusters_x();
    int item = (int)cluster_id_x();

    // prefetch the first item's adapter weights into L2 before waiting on the
    // previous kernel: they are immutable inputs
    const int k0 = min(d_in, (int)crank * p.Wk), k1 = min(d_in, k0 + p.Wk);
    const int o0 = min(d_out, (int)crank * p.Wo), o1 = min(d_out, o0 + p.Wo);
    if (item < n_items && warp == 1) {
        int lo = 0, hi = n_ad;   // last adapter with ipre[a] <= item
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (ipre[mid] <= item)
                lo = mid;
            else
                hi = mid;
        }
        int32_t r;
        int64_t aoff, boff;
        if (adapter_ok(p.pool, lo, &r, &aoff, &boff)) {
            if (k1 > k0)
                for (int j = lane; j < r; j += 32)
                    prefetch_l2(p.pool.A + aoff + (int64_t)j * d_in + k0, (uint32_t)((k1 - k0) * 2));
            if (lane == 0 && o1 > o0)
                prefetch_l2(p.pool.B + boff + (int64_t)o0 * r, (uint32_t)((o1 - o0) * r * 2));
        }
    }
    pdl_trigger();
    pdl_wait();   // from here on x, y and the workspace may be touched
    PHASE(3);
    if (s_bad && blockIdx.x == 0 && tid == 0)
        atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);

    for (; item < n_items; item += n_cl) {
        // ---- the item's adapter and tokens
        if (tid == 0) {
            int lo = 0, hi = n_ad;
            while (hi - lo > 1) {
                const int mid = (lo + hi) >> 1;
                if (ipre[mid] <= item)
                    lo = mid;
                else
                    hi = mid;
            }
            s_ad = lo;
            s_g = item - ipre[lo];
        }
        __syncthreads();
        const int a = s_ad;
        int32_t r;
        int64_t aoff, boff;
        if (!adapter_ok(p.pool, a, &r, &aoff, &boff)) {
            if (crank == 0 && tid == 0)
                atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
            __syncthreads();
            continue;   // the same decision in every CTA of the cluster
        }
        if (warp == 0) {
            const int lo = s_g * kFT;
            int seen = 0;
            for (int base = 0; base < N && seen < lo + kFT; base += 32) {
                const int n = base + lane;
                const bool m = n < N && ids_s[n] == a;
                const unsigned bal = __ballot_sync(0xffffffffu, m);
                if (m) {
                    const int rk = seen + __popc(bal & ((1u << lane) - 1u));
                    if (rk >= lo && rk < lo + kFT)
                        tok[rk - lo] = n;
                }
                seen += __popc(bal);
            }
            if (lane == 0)
                s_cnt = min(kFT, seen - lo);
        }
        for (int e = tid; e < kFT * kMaxRank; e += kFThreads)
            vpart[e] = 0.f;
        __syncthreads();
        PHASE(4);
        const int cnt = s_cnt;
        const int npair = (cnt + 1) >> 1;
        const __nv_bfloat16 *Bc = p.pool.B + boff + (int64_t)o0 * r;

        // ---- expand operands towards L2: B chunk and the tokens' y rows
        if (o1 > o0) {
            if (tid == 0)
                prefetch_l2(Bc, (uint32_t)((o1 - o0) * r * 2));
            if (tid >= 32 && tid < 32 + cnt)
                prefetch_l2(p.Y + (int64_t)tok[tid - 32] * p.ldy + o0, (uint32_t)((o1 - o0) * 2));
        }

        // ---- stage x for this CTA's d_in chunk, token-contiguous, zero-padded to kFT tokens
        const int nv = (k1 - k0) >> 3;
        for (int idx = tid; idx < kFT * nv; idx += kFThreads) {
            const int t = idx & (kFT - 1), v = idx >> 3;
            uint4 u = make_uint4(0, 0, 0, 0);
            if (t < cnt)
                u = __ldg(reinterpret_cast<const uint4 *>(p.X + (int64_t)tok[t] * p.ldx + k0 + v * 8));
            float *dst = xs + v * kXPad + t;
#pragma unroll
            for (int e = 0; e < 8; ++e)
                dst[e * kFT] = bf_at(u, e);
        }
        __syncthreads();
        PHASE(5);

        // ---- shrink: a warp owns 4 rank rows and a share of the chunk's vectors
        {
            const int n_rb = r >> 2;
            const int kparts = max(1, kFWarps / n_rb);
            const int units = n_rb * kparts;
            const __nv_bfloat16 *Aa = p.pool.A + aoff + k0;
            for (int u = warp; u < units; u += kFWarps) {
                const int rb = u / kparts, kp = u - rb * kparts;
                const int v0 = kp * nv / kparts, v1 = (kp + 1) * nv / kparts;
                float acc[32];
#pragma unroll
                for (int q = 0; q < 32; ++q)
                    acc[q] = 0.f;
                const __nv_bfloat16 *A0 = Aa + (int64_t)(rb * 4) * d_in;
#pragma unroll 2
                for (int v = v0 + lane; v < v1; v += 32) {
                    uint4 ar[4];
#pragma unroll
                    for (int i = 0; i < 4; ++i)
                        ar[i] = ld_stream(A0 + (int64_t)i * d_in + v * 8);
                    const float4 *x4 = reinterpret_cast<const float4 *>(xs + v * kXPad);
#pragma unroll
                    for (int e = 0; e < 8; ++e) {
                        const float4 xa = x4[e * 2], xb = x4[e * 2 + 1];
#pragma unroll
                        for (int i = 0; i < 4; ++i) {
                            const float av = bf_at(ar[i], e);
                            ffma2(acc[i * 8 + 0], acc[i * 8 + 1], av, av, xa.x, xa.y);
                            if (npair > 1)
                                ffma2(acc[i * 8 + 2], acc[i * 8 + 3], av, av, xa.z, xa.w);
                            if (npair > 2) {
                                ffma2(acc[i * 8 + 4], acc[i * 8 + 5], av, av, xb.x, xb.y);
                                ffma2(acc[i * 8 + 6], acc[i * 8 + 7], av, av, xb.z, xb.w);
                            }
                        }
                    }
                }
                const float val = reduce_scatter32(acc, lane);
                const int i = lane >> 3, t = lane & 7;
                if (t < cnt)
                    atomicAdd(&vpart[(rb * 4 + i) * kFT + t], val);
            }
        }
        __syncthreads();
        PHASE(6);

        // ---- exchange partials across the cluster (fixed summation order)
        cluster_arrive();
        cluster_wait();
        {
            namespace cg = cooperative_groups;
            cg::cluster_group cl = cg::this_cluster();
            for (int idx = tid; idx < kFT * r; idx += kFThreads) {
                const int t = idx & (kFT - 1), j = idx >> 3;
                float s = 0.f;
                if (t < cnt) {
#pragma unroll
                    for (int c = 0; c < kFC; ++c)
                        s += cl.map_shared_rank(vpart, c)[j * kFT + t];
                }
                vsum[j * kFT + t] = s;
            }
        }
        cluster_arrive();   // our reads of the other CTAs' partials are done
        __syncthreads();
        PHASE(7);

        // ---- expand this CTA's d_out chunk, two outputs per thread per step
        const float sc = p.scale;
        for (int o = o0 + 2 * tid; o < o1; o += 2 * kFThreads) {
            float c0[kFT], c1[kFT];
#pragma unroll
            for (int t = 0; t < kFT; ++t) {
                c0[t] = 0.f;
                c1[t] = 0.f;
            }
            const __nv_bfloat16 *b0 = Bc + (int64_t)(o - o0) * r;
#pragma unroll 2
            for (int jc = 0; jc < r; jc += 8) {
                const uint4 u0 = ld_stream(b0 + jc), u1 = ld_stream(b0 + r + jc);
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    const float f0 = bf_at(u0, e), f1 = bf_at(u1, e);
                    const float4 *v4 = reinterpret_cast<const float4 *>(vsum + (jc + e) * kFT);
                    const float4 va = v4[0], vb = v4[1];
                    ffma2(c0[0], c0[1], f0, f0, va.x, va.y);
                    ffma2(c1[0], c1[1], f1, f1, va.x, va.y);
                    if (npair > 1) {
                        ffma2(c0[2], c0[3], f0, f0, va.z, va.w);
                        ffma2(c1[2], c1[3], f1, f1, va.z, va.w);
                    }
                    if (npair > 2) {
                        ffma2(c0[4], c0[5], f0, f0, vb.x, vb.y);
                        ffma2(c1[4], c1[5], f1, f1, vb.x, vb.y);
                        ffma2(c0[6], c0[7], f0, f0, vb.z, vb.w);
                        ffma2(c1[6], c1[7], f1, f1, vb.z, vb.w);
                    }
                }
            }
#pragma unroll
            for (int t = 0; t < kFT; ++t) {
                if (t < cnt) {
                    __nv_bfloat162 *yp = reinterpret_cast<__nv_bfloat162 *>(p.Y + (int64_t)tok[t] * p.ldy + o);
                    const float2 y = __bfloat1622float2(*yp);
                    *yp = __floats2bfloat162_rn(y.x + sc * c0[t], y.y + sc * c1[t]);
                }
            }
        }
        __syncthreads();
        PHASE(8);
        cluster_wait();     // no CTA reuses its partials while another may still read them
        PHASE(9);
        first = false;
    }
}

}  // namespace

size_t fused_smem_bytes(int32_t N, int32_t n_adapters, int32_t Wk)
{
    return fused_smem_layout(N, n_adapters, Wk).total;
}

bool fused_bgmv_supported(int32_t N, int32_t n_adapters, int32_t d_in)
{
    const int32_t Wk = fused_chunk(d_in);
    return N <= kFMaxTokens && n_adapters <= kFMaxAdapters && Wk <= kFMaxChunk &&
           fused_smem_bytes(N, n_adapters, Wk) <= kFMaxSmem;
}

namespace {

struct OccCache {
    int dev = -1;
    size_t smem = 0;
    int clusters = 0;
};

// Clusters of this kernel that fit on the device at once for a given
// dynamic shared-memory size (a handful of sizes occur per process).
int max_active_clusters(int dev, size_t smem, cudaStream_t s)
{
    static OccCache cache[16];
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &c : cache)
        if (c.dev == dev && c.smem == smem)
            return c.clusters;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kFC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(kFC * 1024);
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    int n = 0;
    if (cudaOccupancyMaxActiveClusters(&n, k_bgmv_fused, &cfg) != cudaSuccess || n <= 0)
        n = 0;
    for (auto &c : cache)
        if (c.dev < 0) {
            c.dev = dev;
            c.smem = smem;
            c.clusters = n;
            break;
        }
    return n;
}

}  // namespace

cudaError_t launch_bgmv_fused(const FusedBgmvArgs &a, cudaStream_t s, bool pdl)
{
    const size_t smem = fused_smem_bytes(a.N, a.pool.n_adapters, a.Wk);
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_bgmv_fused, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kFMaxSmem);
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    // at most min(N, n_adapters) adapters plus one extra group per kFT further tokens
    const int64_t items = (int64_t)(a.N < a.pool.n_adapters ? a.N : a.pool.n_adapters) + a.N / kFT;
    if (items <= 0)
        return cudaSuccess;
    int64_t clusters = items;
    const int cap = max_active_clusters(dev, smem, s);
    if (cap > 0 && clusters > cap)
        clusters = cap;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = kFC;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)(clusters * kFC));
    cfg.blockDim = dim3(kFThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 2 : 1;
    return cudaLaunchKernelEx(&cfg, k_bgmv_fused, a);
}

}  // namespace lora

#ifdef LORA_PHASE_TIMING
extern "C" LORA_API int lora_debug_phases(unsigned long long *host, int n)
{
    return (int)cudaMemcpyFromSymbol(host, lora::g_phase, sizeof(unsigned long long) * (size_t)n);
}
#endif
