// Decode BGMV in one launch: grouping, shrink and expand fused; one
// thread-block cluster per (adapter, group of <= kFT tokens) item.
//
// The operation ("Serving several LoRAs, ControlNet and IP-Adapter", section
// "LoRA: merged or alongside" and exercise 2's answer): y[n] += s B[a] A[a] x[n]
// for a batch whose tokens carry their own adapter ids, grouped by adapter so
// that each distinct adapter's A and B are streamed from HBM once per group
// (the segmented gather matrix-vector product of "Punica: multi-tenant LoRA
// serving", contribution 1).
//
// Work layout on B200:
// * every CTA rebuilds the grouping in shared memory (ids -> per-adapter
//   counts -> exclusive scan of groups per adapter); item k is the k-th
//   (adapter, group of up to 16 tokens) pair in adapter order.  Clusters are
//   persistent: the grid holds as many clusters as fit on the GPU at once.  The
//   items are dealt out heaviest first: ordered by rank class (ranks 65-128,
//   33-64, 17-32, 8-16; adapter order inside a class), cluster c starts with
//   position c and then takes the next free position from a counter in the
//   workspace header (rank 0 of the cluster draws it during the item and writes
//   it into every CTA of the cluster before the cluster barrier that ends the
//   item).  With cluster c taking items c, c + n_clusters, ... instead, the
//   mixed-rank gate projection (about 230 items on 86 clusters) ran 1.6x longer
//   than its average cluster load.  The last cluster to finish puts the counter
//   back to zero; a launch draws from it only after griddepcontrol.wait, i.e.
//   after the previous launch on the stream has finished.
// * an item is a 16-row tile of tokens, so both halves are tiny dense
//   contractions done with warp-level tensor-core MMAs (m16n8k16, bf16 in,
//   fp32 accumulate): with CUDA-core FMAs the instruction issue, not HBM,
//   bounds decode.  Inside each 32-wide block of the reduction dimension the
//   k order is permuted identically for both operands, so every thread's
//   operand fragments are plain 16-byte global loads (no shared-memory
//   staging, no bf16 unpacking): quad position q owns columns 8q..8q+7.
// * shrink: the kFC CTAs of a cluster split d_in; CTA c computes its partial
//   V_c = X_tile A[:, chunk]^T (16 tokens x r), its warps splitting the rank
//   tiles and/or the chunk, reduced into shared memory;
// * the cluster sums the kFC partials through distributed shared memory
//   (fixed order: deterministic) and splits V into bf16 hi + lo parts, so the
//   expand MMAs see V to ~16 significant bits instead of bf16's 8; V is kept
//   in MMA fragment order, so a lane's 16-byte read is one A operand as the
//   MMA takes it;
// * expand: CTA c owns a d_out chunk; its warps walk 8-output tiles,
//   Y_tile += s * (V_hi + V_lo) B[tile]^T, and update y in place;
// * when a CTA's B chunk and the item's y rows fit 16 KB each (decode shapes)
//   both are copied to shared memory as soon as the item is known; otherwise
//   the CTA's A rows are requested into L2 line by line before the shrink; the
//   grouping, the item metadata and those requests come before
//   griddepcontrol.wait (programmatic dependent launch), i.e. while the
//   previous kernel on the stream is still finishing -- they only read
//   immutable inputs.

#include <cooperative_groups.h>

#include <mutex>

#include "lora_internal.cuh"

namespace lora {
namespace {

// Read-only 16-byte load that does not allocate in L1 (weights are used once
// per CTA), or zeros when ok is false.  The predicate is inside the asm so that
// the compiler needs no branch around it.  Not volatile: the compiler may batch
// independent loads.
__device__ __forceinline__ uint4 ld_stream(const void *p, bool ok)
{
    uint4 r = make_uint4(0, 0, 0, 0);
    asm("{\n\t.reg .pred q;\n\tsetp.ne.b32 q, %5, 0;\n\t"
        "@q ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n\t}"
        : "+r"(r.x), "+r"(r.y), "+r"(r.z), "+r"(r.w)
        : "l"(p), "r"((int)ok));
    return r;
}

// D += A * B for one m16n8k16 tile, bf16 inputs, fp32 accumulators.
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
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

// 16-byte asynchronous copy global -> shared (both 16-byte aligned), and the wait for all of them
__device__ __forceinline__ void cp_async16(void *dst, const void *src)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"((uint32_t)__cvta_generic_to_shared(dst)), "l"(src)
                 : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
__device__ __forceinline__ void cp_async_wait_all() { asm volatile("cp.async.wait_group 0;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

#ifdef LORA_PHASE_TIMING
// Development aid: per-CTA %globaltimer stamps at phase boundaries of the first item.
__device__ unsigned long long g_phase[65536 * 16];
#define PHASE(i)                                                                     \
    do {                                                                             \
        if (threadIdx.x == 0 && first && blockIdx.x < 65536) {                       \
            unsigned long long t_;                                                   \
            asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t_));                   \
            g_phase[blockIdx.x * 16 + (i)] = t_;                                     \
        }                                                                            \
    } while (0)
#else
#define PHASE(i) \
    do {         \
    } while (0)
#endif

__device__ __forceinline__ bool adapter_ok(const PoolDev &P, int32_t a, int32_t *r_out, int64_t *aoff,
                                           int64_t *boff)
{
    if (a < 0 || a >= P.n_adapters)
        return false;
    const int32_t r = P.rank[a];
    const int64_t ao = P.A_off[a], bo = P.B_off[a];
    if (r < 8 || r > P.max_rank || (r & 7))
        return false;
    if (ao < 0 || (ao & 7) || ao + (int64_t)r * P.d_in > P.A_elems)
        return false;
    if (bo < 0 || (bo & 7) || bo + (int64_t)r * P.d_out > P.B_elems)
        return false;
    *r_out = r;
    *aoff = ao;
    *boff = bo;
    return true;
}

// Scheduling class of a rank: 3 for ranks 65-128 .. 0 for 8-16 and for a rank that
// fails the checks.
__device__ __forceinline__ int rank_class(const PoolDev &P, int r)
{
    if (r < 8 || r > P.max_rank || (r & 7))
        return 0;
    return r <= 16 ? 0 : r <= 32 ? 1 : r <= 64 ? 2 : 3;
}

// The ranks of adapters a0 .. a0 + 7 (below e), eight loads in flight together.
__device__ __forceinline__ void load_ranks8(const PoolDev &P, int a0, int e, int (&rk)[8])
{
#pragma unroll
    for (int u = 0; u < 8; ++u)
        rk[u] = a0 + u < e ? __ldg(P.rank + a0 + u) : 0;
}

// Shrink of one warp: NT rank tiles (8 ranks each, from rank tile nt0) over
// the 32-column blocks [b0, b1) starting at column kb0; all A and x
// fragments of a batch of BPB blocks are requested before any MMA runs.
template <int NT>
__device__ __forceinline__ void shrink_tiles(const __nv_bfloat16 *Aa, int d_in, int nt0, int kb0, int k1,
                                             int b0, int b1, const __nv_bfloat16 *x0, const __nv_bfloat16 *x1,
                                             bool row0, bool row1, int g, int qd, float (&acc)[4][4])
{
    constexpr int BPB = NT == 1 ? 4 : 2;   // blocks per batch (register budget)
    for (int bb = b0; bb < b1; bb += BPB) {
        uint4 aw[BPB][NT], xa[BPB], xb[BPB];
#pragma unroll
        for (int k = 0; k < BPB; ++k) {
            const int col = kb0 + (bb + k) * 32 + qd * 8;
            const bool ok = bb + k < b1 && col < k1;
#pragma unroll
            for (int i = 0; i < NT; ++i)
                aw[k][i] = ld_stream(Aa + (int64_t)((nt0 + i) * 8 + g) * d_in + col, ok);
            xa[k] = (ok && row0) ? __ldg(reinterpret_cast<const uint4 *>(x0 + col)) : make_uint4(0, 0, 0, 0);
            xb[k] = (ok && row1) ? __ldg(reinterpret_cast<const uint4 *>(x1 + col)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int k = 0; k < BPB; ++k) {
#pragma unroll
            for (int i = 0; i < NT; ++i) {
                // two k16 steps: low and high 8 bytes of each 16-byte fragment
                mma16816(acc[i], xa[k].x, xb[k].x, xa[k].y, xb[k].y, aw[k][i].x, aw[k][i].y);
                mma16816(acc[i], xa[k].z, xb[k].z, xa[k].w, xb[k].w, aw[k][i].z, aw[k][i].w);
            }
        }
    }
}

// Position (in bf16 elements) of V[t][j] (token t < 16, rank j) in the fragment-
// ordered V buffer, hi part (the lo part follows: +512 per 32-rank block, +256 for
// ranks <= 16).  For an m16n8k16 A operand, lane (g, qd) holds rows g and g + 8 at
// k-slot pairs {2qd, 2qd+1} and {2qd+8, 2qd+9}; inside a 32-rank block quad qd
// owns ranks 8qd .. 8qd+7 (pairs 0, 1 for MMA 0 and pairs 2, 3 for MMA 1), and for
// ranks <= 16 ranks 4qd .. 4qd+3 (pairs 0, 1 of the single MMA).  Each quad is
// stored as the four registers the MMA takes: (row g, pair p), (row g+8, pair p),
// (row g, pair p+1), (row g+8, pair p+1), so one 16-byte load yields an operand.
__device__ __forceinline__ int vfrag_index(int t, int j, bool r16)
{
    const int g = t & 7, hi8 = t >> 3;
    if (r16) {
        const int qd = j >> 2, w = j & 3;
        return (g * 4 + qd) * 8 + (((w >> 1) << 1) | hi8) * 2 + (w & 1);
    }
    const int kb = j >> 5, jj = j & 31, qd = jj >> 3, w = jj & 7, pair = w >> 1;
    const int m = pair >> 1;
    return ((kb * 4 + m) * 32 + g * 4 + qd) * 8 + (((pair & 1) << 1) | hi8) * 2 + (w & 1);
}

// Expand of one warp over its output tiles ot = warp, warp + nw, ... < n_ot
// (8 outputs each, from output o0): Y += s (V_hi + V_lo) B^T with NKB
// 32-rank blocks; a batch's B fragments and y values are all requested
// before its MMAs, and the V fragments are read from shared memory once.
// vq: V_hi and V_lo in fragment order (vfrag_index): quad vq[((kb * 2 + hl) * 2
// + m) * 32 + lane] is the A operand of MMA m of block kb as it stands.
// ST: B and y come from the staged copies in shared memory (bst: [Wo][r] from
// output o0; yst: [kFT][Wo]), else from global memory.
template <int NKB, bool ST>
__device__ __forceinline__ void expand_tiles(const __nv_bfloat16 *Ba, int r, int o0, int n_ot, int warp, int nw,
                                             const uint4 *vq, int lane, int g, int qd, __nv_bfloat16 *y0row,
                                             __nv_bfloat16 *y1row, bool row0, bool row1, float sc,
                                             const __nv_bfloat16 *bst, const __nv_bfloat16 *yst, int Wo)
{
    constexpr int TPB = ST ? 16 : (NKB == 1 ? 8 : NKB == 2 ? 4 : 2);   // tiles per batch
    constexpr bool HOIST = NKB <= 2;                                  // keep V fragments in registers
    uint4 qv[HOIST ? NKB : 1][2][2];     // [kb][hi, lo][MMA]
    if (HOIST) {
#pragma unroll
        for (int kb = 0; kb < (HOIST ? NKB : 1); ++kb)
#pragma unroll
            for (int hl = 0; hl < 2; ++hl)
#pragma unroll
                for (int m = 0; m < 2; ++m)
                    qv[kb][hl][m] = vq[((kb * 2 + hl) * 2 + m) * 32 + lane];
    }
    for (int ot0 = warp; ot0 < n_ot; ot0 += TPB * nw) {
        uint4 bw[ST ? 1 : TPB][NKB];
        __nv_bfloat162 ya[ST ? 1 : TPB], yb[ST ? 1 : TPB];
        if (!ST) {
#pragma unroll
            for (int t = 0; t < TPB; ++t) {
                const int ot = ot0 + t * nw;
                const bool ok = ot < n_ot;
                const int ob = o0 + ot * 8;
                const __nv_bfloat16 *brow = Ba + (int64_t)(ob + g) * r;
#pragma unroll
                for (int kb = 0; kb < NKB; ++kb) {
                    const int kc = kb * 32 + qd * 8;   // r and kc are multiples of 8
                    bw[ST ? 0 : t][kb] = ld_stream(brow + kc, ok && kc < r);
                }
                const __nv_bfloat162 z = __floats2bfloat162_rn(0.f, 0.f);
                ya[ST ? 0 : t] = (ok && row0) ? *reinterpret_cast<const __nv_bfloat162 *>(y0row + ob + 2 * qd) : z;
                yb[ST ? 0 : t] = (ok && row1) ? *reinterpret_cast<const __nv_bfloat162 *>(y1row + ob + 2 * qd) : z;
            }
        }
#pragma unroll
        for (int t = 0; t < TPB; ++t) {
            const int ot = ot0 + t * nw;
            if (ot < n_ot) {
                const int ol = ot * 8;          // output offset within this CTA's chunk
                uint4 bfr[NKB];
                __nv_bfloat162 yva, yvb;
                if (ST) {
#pragma unroll
                    for (int kb = 0; kb < NKB; ++kb) {
                        const int kc = kb * 32 + qd * 8;
                        bfr[kb] = kc < r ? *reinterpret_cast<const uint4 *>(bst + (ol + g) * r + kc)
                                         : make_uint4(0, 0, 0, 0);
                    }
                    yva = *reinterpret_cast<const __nv_bfloat162 *>(yst + g * Wo + ol + 2 * qd);
                    yvb = *reinterpret_cast<const __nv_bfloat162 *>(yst + (g + 8) * Wo + ol + 2 * qd);
                } else {
#pragma unroll
                    for (int kb = 0; kb < NKB; ++kb)
                        bfr[kb] = bw[ST ? 0 : t][kb];
                    yva = ya[ST ? 0 : t];
                    yvb = yb[ST ? 0 : t];
                }
                float d[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int kb = 0; kb < NKB; ++kb) {
                    uint4 h0, h1, l0, l1;     // hi / lo quads of the two MMAs
                    if (HOIST) {
                        h0 = qv[HOIST ? kb : 0][0][0];
                        h1 = qv[HOIST ? kb : 0][0][1];
                        l0 = qv[HOIST ? kb : 0][1][0];
                        l1 = qv[HOIST ? kb : 0][1][1];
                    } else {
                        h0 = vq[(kb * 4 + 0) * 32 + lane];
                        h1 = vq[(kb * 4 + 1) * 32 + lane];
                        l0 = vq[(kb * 4 + 2) * 32 + lane];
                        l1 = vq[(kb * 4 + 3) * 32 + lane];
                    }
                    mma16816(d, h0.x, h0.y, h0.z, h0.w, bfr[kb].x, bfr[kb].y);
                    mma16816(d, l0.x, l0.y, l0.z, l0.w, bfr[kb].x, bfr[kb].y);
                    mma16816(d, h1.x, h1.y, h1.z, h1.w, bfr[kb].z, bfr[kb].w);
                    mma16816(d, l1.x, l1.y, l1.z, l1.w, bfr[kb].z, bfr[kb].w);
                }
                // D fragment: tokens g, g+8; outputs ob + 2qd, ob + 2qd + 1
                const int o = o0 + ol + 2 * qd;
                __nv_bfloat16 *d0 = y0row + o;
                __nv_bfloat16 *d1 = y1row + o;
                if (row0) {
                    const float2 y = __bfloat1622float2(yva);
                    *reinterpret_cast<__nv_bfloat162 *>(d0) =
                        __floats2bfloat162_rn(fmaf(sc, d[0], y.x), fmaf(sc, d[1], y.y));
                }
                if (row1) {
                    const float2 y = __bfloat1622float2(yvb);
                    *reinterpret_cast<__nv_bfloat162 *>(d1) =
                        __floats2bfloat162_rn(fmaf(sc, d[2], y.x), fmaf(sc, d[3], y.y));
                }
            }
        }
    }
}

// Expand for ranks <= 16: one k16 step per tile.  Inside the 16 ranks the k order
// is permuted identically for both operands so that thread quad qd holds ranks
// 4qd .. 4qd+3 (8-byte fragments of V and B), and the two MMAs per tile are the
// V_hi and V_lo halves.
template <bool ST>
__device__ __forceinline__ void expand_tiles16(const __nv_bfloat16 *Ba, int r, int o0, int n_ot, int warp, int nw,
                                               const uint4 *vq, int lane, int g, int qd, __nv_bfloat16 *y0row,
                                               __nv_bfloat16 *y1row, bool row0, bool row1, float sc,
                                               const __nv_bfloat16 *bst, const __nv_bfloat16 *yst, int Wo)
{
    // global operands: a batch's B fragments and y values are requested before its MMAs;
    // staged operands (shared memory) are read tile by tile
    constexpr int TPB = ST ? 1 : 8;
    const int kc = qd * 4;
    const bool kin = kc < r;
    const uint4 qh = vq[lane], ql = vq[32 + lane];     // hi / lo quads (ranks <= 16 order)
    const __nv_bfloat162 z = __floats2bfloat162_rn(0.f, 0.f);
    for (int ot0 = warp; ot0 < n_ot; ot0 += TPB * nw) {
        uint2 bw[TPB];
        __nv_bfloat162 ya[TPB], yb[TPB];
#pragma unroll
        for (int t = 0; t < TPB; ++t) {
            const int ot = ot0 + t * nw;
            const bool ok = ot < n_ot;
            const int ol = ot * 8;
            if (ST) {
                bw[t] = (ok && kin) ? *reinterpret_cast<const uint2 *>(bst + (ol + g) * r + kc) : make_uint2(0, 0);
                ya[t] = ok ? *reinterpret_cast<const __nv_bfloat162 *>(yst + g * Wo + ol + 2 * qd) : z;
                yb[t] = ok ? *reinterpret_cast<const __nv_bfloat162 *>(yst + (g + 8) * Wo + ol + 2 * qd) : z;
            } else {
                bw[t] = (ok && kin) ? *reinterpret_cast<const uint2 *>(Ba + (int64_t)(o0 + ol + g) * r + kc)
                                    : make_uint2(0, 0);
                ya[t] = (ok && row0) ? *reinterpret_cast<const __nv_bfloat162 *>(y0row + o0 + ol + 2 * qd) : z;
                yb[t] = (ok && row1) ? *reinterpret_cast<const __nv_bfloat162 *>(y1row + o0 + ol + 2 * qd) : z;
            }
        }
#pragma unroll
        for (int t = 0; t < TPB; ++t) {
            const int ot = ot0 + t * nw;
            if (ot < n_ot) {
                float d[4] = {0.f, 0.f, 0.f, 0.f};
                mma16816(d, qh.x, qh.y, qh.z, qh.w, bw[t].x, bw[t].y);
                mma16816(d, ql.x, ql.y, ql.z, ql.w, bw[t].x, bw[t].y);
                const int o = o0 + ot * 8 + 2 * qd;
                if (row0) {
                    const float2 y = __bfloat1622float2(ya[t]);
                    *reinterpret_cast<__nv_bfloat162 *>(y0row + o) =
                        __floats2bfloat162_rn(fmaf(sc, d[0], y.x), fmaf(sc, d[1], y.y));
                }
                if (row1) {
                    const float2 y = __bfloat1622float2(yb[t]);
                    *reinterpret_cast<__nv_bfloat162 *>(y1row + o) =
                        __floats2bfloat162_rn(fmaf(sc, d[2], y.x), fmaf(sc, d[3], y.y));
                }
            }
        }
    }
}

__global__ void __launch_bounds__(kFThreads, 5) k_bgmv_fused(FusedBgmvArgs p)
{
    extern __shared__ __align__(16) unsigned char sm_raw[];
    const FusedSmem L = fused_smem_layout(p.N, p.pool.n_adapters, p.pool.max_rank, p.Wo);
    int16_t *item_ad = reinterpret_cast<int16_t *>(sm_raw + L.items);   // adapter of items < L.n_tab
    int16_t *order = reinterpret_cast<int16_t *>(sm_raw + L.order);    // item at each schedule position
    const int mr = p.pool.max_rank < kMaxRank ? p.pool.max_rank : kMaxRank;
    int32_t *ids_s = reinterpret_cast<int32_t *>(sm_raw + L.ids);
    int32_t *ipre = reinterpret_cast<int32_t *>(sm_raw + L.cnt);    // [n_ad + 1]
    float *vpart = reinterpret_cast<float *>(sm_raw + L.vpart);     // [max_rank][kFT], read by the cluster
    // V split into bf16 hi and lo parts, in MMA fragment order (vfrag_index)
    __nv_bfloat16 *vfr = reinterpret_cast<__nv_bfloat16 *>(sm_raw + L.vsum);
    const uint4 *vq = reinterpret_cast<const uint4 *>(sm_raw + L.vsum);
    // staged (when L.staged): this CTA's B chunk [Wo][r] and the item's y rows [kFT][Wo]
    __nv_bfloat16 *bst = reinterpret_cast<__nv_bfloat16 *>(sm_raw + L.bst);
    __nv_bfloat16 *yst = reinterpret_cast<__nv_bfloat16 *>(sm_raw + L.yst);
    __shared__ int32_t tok[kFT];
    __shared__ int32_t s_ad, s_g, s_cnt, s_bad, s_r;
    __shared__ int64_t s_aoff, s_boff;
    __shared__ int32_t sm_scan[kFWarps + 1];
    __shared__ unsigned long long sm_cls[kFWarps + 1];
    __shared__ int s_next;          // the cluster's next schedule position (written by cluster rank 0)

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int g = lane >> 2, qd = lane & 3;    // MMA fragment row group and quad position
    const uint32_t crank = cluster_ctarank();
    const int N = p.N, n_ad = p.pool.n_adapters;
    const int d_in = p.pool.d_in, d_out = p.pool.d_out;
    [[maybe_unused]] bool first = true;
    PHASE(0);

    // pool metadata towards L2 while the ids arrive (whole 16-byte lines only)
    if (tid == 0) {
        const uint32_t rb = (uint32_t)(n_ad * 4) & ~15u, ob = (uint32_t)(n_ad * 8) & ~15u;
        if (rb)
            prefetch_l2(p.pool.rank, rb);
        if (ob) {
            prefetch_l2(p.pool.A_off, ob);
            prefetch_l2(p.pool.B_off, ob);
        }
    }

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
        // counts -> exclusive prefix of groups per adapter, ipre[n_ad] = total; and the
        // same prefix per rank class (four 16-bit fields of one 64-bit scan: class 3 =
        // ranks 65-128 .. class 0 = ranks 8-16, or an adapter that fails its checks)
        const int per = (n_ad + kFThreads - 1) / kFThreads;
        const int b = tid * per, e = min(n_ad, b + per);
        int local = 0;
        unsigned long long lcls = 0;
        for (int a0 = b; a0 < e; a0 += 8) {
            int rk[8];
            load_ranks8(p.pool, a0, e, rk);
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int a = a0 + u;
                if (a < e) {
                    const int gr = (ipre[a] + kFT - 1) / kFT;
                    local += gr;
                    if (gr)
                        lcls += (unsigned long long)gr << (16 * rank_class(p.pool, rk[u]));
                }
            }
        }
        int incl = local;
        unsigned long long icls = lcls;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            const int v = __shfl_up_sync(0xffffffffu, incl, off);
            const unsigned long long w = __shfl_up_sync(0xffffffffu, icls, off);
            if (lane >= off) {
                incl += v;
                icls += w;
            }
        }
        if (lane == 31) {
            sm_scan[warp] = incl;
            sm_cls[warp] = icls;
        }
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            unsigned long long runc = 0;
            for (int w = 0; w < kFWarps; ++w) {
                const int t = sm_scan[w];
                const unsigned long long tc = sm_cls[w];
                sm_scan[w] = run;
                sm_cls[w] = runc;
                run += t;
                runc += tc;
            }
            sm_scan[kFWarps] = run;
            sm_cls[kFWarps] = runc;
        }
        __syncthreads();
        int run = sm_scan[warp] + incl - local;
        unsigned long long runc = sm_cls[warp] + icls - lcls;
        // schedule position of the first item of each class: heaviest class first
        const unsigned long long tot = sm_cls[kFWarps];
        int cbase[4];
        cbase[3] = 0;
        cbase[2] = (int)(tot >> 48);
        cbase[1] = cbase[2] + (int)((tot >> 32) & 0xFFFF);
        cbase[0] = cbase[1] + (int)((tot >> 16) & 0xFFFF);
        for (int a0 = b; a0 < e; a0 += 8) {
            int rk[8];
            load_ranks8(p.pool, a0, e, rk);       // L1 hits now
#pragma unroll
            for (int u = 0; u < 8; ++u) {
                const int a = a0 + u;
                if (a < e) {
                    const int gr = (ipre[a] + kFT - 1) / kFT;
                    ipre[a] = run;
                    if (gr) {
                        const int c = rank_class(p.pool, rk[u]);
                        const int pos = cbase[c] + (int)((runc >> (16 * c)) & 0xFFFF);
                        for (int j = 0; j < gr && run + j < L.n_tab; ++j) {
                            item_ad[run + j] = (int16_t)a;
                            if (pos + j < L.n_tab)
                                order[pos + j] = (int16_t)(run + j);
                        }
                        runc += (unsigned long long)gr << (16 * c);
                    }
                    run += gr;
                }
            }
        }
        if (tid == 0)
            ipre[n_ad] = sm_scan[kFWarps];
        __syncthreads();
    }
    PHASE(2);
    const int n_items = ipre[n_ad];
    const int n_cl = (int)n_clusters_x();
    const int k0 = min(d_in, (int)crank * p.Wk), k1 = min(d_in, k0 + p.Wk);
    const int o0 = min(d_out, (int)crank * p.Wo), o1 = min(d_out, o0 + p.Wo);
    bool waited = false;

    // the schedule (above) needs every item in the tables; else items in index order
    const bool sched = n_items <= L.n_tab;
    const int cid = (int)cluster_id_x();
    // rank 0 of the cluster draws the next position (early, so that the atomic's round
    // trip overlaps the shrink) and later hands it to every CTA of the cluster, which
    // read it after the next cluster barrier
    int drawn = -1;
    auto draw = [&]() {
        if (crank == 0 && tid == 0 && drawn < 0)
            drawn = (int)atomicAdd(p.sched, 1u) + n_cl;
    };
    auto publish = [&]() {
        if (crank == 0 && tid == 0) {
            namespace cg = cooperative_groups;
            cg::cluster_group cl = cg::this_cluster();
#pragma unroll
            for (int c = 0; c < kFC; ++c)
                *cl.map_shared_rank(&s_next, c) = drawn;
            drawn = -1;
        }
    };
    int pos = cid;                  // the first round: the heaviest items, one per cluster
    for (bool first_item = true; pos < n_items; first_item = false) {
        const int item = sched ? order[pos] : pos;
        // ---- the item's adapter, metadata and tokens (immutable inputs only)
        if (tid == 0) {
            int lo = 0;
            if (item < L.n_tab) {
                lo = item_ad[item];      // written by the grouping
            } else {
                int hi = n_ad;           // last adapter with ipre[a] <= item
                while (hi - lo > 1) {
                    const int mid = (lo + hi) >> 1;
                    if (ipre[mid] <= item)
                        lo = mid;
                    else
                        hi = mid;
                }
            }
            s_ad = lo;
            s_g = item - ipre[lo];
        }
        __syncthreads();
        PHASE(9);
        const int a = s_ad;
        // warp 1 fetches the adapter's metadata while warp 0 finds the item's tokens
        if (tid == 32) {
            int32_t r = 0;
            int64_t ao = 0, bo = 0;
            const bool ok = adapter_ok(p.pool, a, &r, &ao, &bo);
            s_r = ok ? r : 0;
            s_aoff = ao;
            s_boff = bo;
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
        for (int e = tid; e < mr * kFT; e += kFThreads)
            vpart[e] = 0.f;
        __syncthreads();
        PHASE(10);
        const int r = s_r;
        const int cnt = s_cnt;
        if (r == 0) {
            // the same decision in every CTA of the cluster
            if (!waited) {
                pdl_trigger();
                pdl_wait();
                waited = true;
            }
            if (crank == 0 && tid == 0)
                atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
            draw();
            publish();
            cluster_arrive();
            cluster_wait();
            pos = s_next;
            __syncthreads();
            continue;
        }
        const __nv_bfloat16 *Aa = p.pool.A + s_aoff;
        const __nv_bfloat16 *Ba = p.pool.B + s_boff;
        if (L.staged) {
            // this CTA's B chunk into shared memory (immutable input): lands during the shrink
            const int nch = (o1 - o0) * r / 8;
            const __nv_bfloat16 *src = Ba + (int64_t)o0 * r;
            for (int c = tid; c < nch; c += kFThreads)
                cp_async16(bst + c * 8, src + c * 8);
        }
        // (a chunk too large to stage is not prefetched: its expand streams at the
        // HBM rate anyway, and one bulk prefetch of a few hundred KB holds the SM's copy
        // engine for microseconds, blocking every copy and prefetch issued after it)
        PHASE(3);

        // ---- shrink work split: rank tiles of 8 in groups of up to 4 per warp;
        // warps left over split this CTA's d_in chunk (32-column blocks)
        const int n_nt = r >> 3;                        // rank tiles
        const int ngrp = (n_nt + 3) >> 2;               // warp groups of <= 4 rank tiles
        const int kparts = max(1, kFWarps / ngrp);
        const int nblk = (k1 - k0 + 31) >> 5;           // 32-column blocks of the chunk
        const int my_grp = warp / kparts, my_kp = warp - (warp / kparts) * kparts;
        const int b0 = my_kp * nblk / kparts, b1 = (my_kp + 1) * nblk / kparts;

        // ---- shrink: V_c[16 x r] = X_tile[16 x chunk] A[:, chunk]^T; this
        // CTA's A rows are requested into L2 first (immutable input), one 128-byte
        // line per prefetch instruction (these do not queue behind bulk copies)
        if (k1 > k0) {
            const uint32_t lpr = (uint32_t)((k1 - k0) * 2 + 127) >> 7;    // lines per row
            for (uint32_t e = (uint32_t)tid; e < (uint32_t)r * lpr; e += kFThreads) {
                const uint32_t j = e / lpr, l = e - j * lpr;
                asm volatile("prefetch.global.L2 [%0];" ::"l"(reinterpret_cast<const char *>(
                                                            Aa + (int64_t)j * d_in + k0) + ((size_t)l << 7))
                             : "memory");
            }
        }
        if (!waited) {
            pdl_trigger();
            pdl_wait();   // from here on x, y and the workspace may be touched
            waited = true;
        }
        draw();
        PHASE(11);
        if (L.staged) {
            // the item's y rows into shared memory: land during the shrink and the exchange
            const int cpr = (o1 - o0) / 8;
            for (int c = tid; c < cnt * cpr; c += kFThreads) {
                const int t = c / cpr, j = c - t * cpr;
                cp_async16(yst + t * p.Wo + j * 8, p.Y + (int64_t)tok[t] * p.ldy + o0 + j * 8);
            }
        }
        cp_async_commit();
        {
            const bool row0 = g < cnt, row1 = g + 8 < cnt;
            const __nv_bfloat16 *x0 = p.X + (int64_t)(row0 ? tok[g] : 0) * p.ldx;
            const __nv_bfloat16 *x1 = p.X + (int64_t)(row1 ? tok[g + 8] : 0) * p.ldx;
            for (int grp = my_grp; grp < ngrp; grp += kFWarps / kparts) {
                const int gt0 = grp * 4, nt = min(n_nt, gt0 + 4) - gt0;
                float acc[4][4];
#pragma unroll
                for (int i = 0; i < 4; ++i)
#pragma unroll
                    for (int j = 0; j < 4; ++j)
                        acc[i][j] = 0.f;
                switch (nt) {
                case 1: shrink_tiles<1>(Aa, d_in, gt0, k0, k1, b0, b1, x0, x1, row0, row1, g, qd, acc); break;
                case 2: shrink_tiles<2>(Aa, d_in, gt0, k0, k1, b0, b1, x0, x1, row0, row1, g, qd, acc); break;
                case 3: shrink_tiles<3>(Aa, d_in, gt0, k0, k1, b0, b1, x0, x1, row0, row1, g, qd, acc); break;
                default: shrink_tiles<4>(Aa, d_in, gt0, k0, k1, b0, b1, x0, x1, row0, row1, g, qd, acc); break;
                }
                // D fragment: rows (tokens) g, g+8; cols (ranks) 2qd, 2qd+1 of each rank tile
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    if (i < nt) {
                        const int j = (gt0 + i) * 8 + 2 * qd;
                        if (row0) {
                            atomicAdd(&vpart[j * kFT + g], acc[i][0]);
                            atomicAdd(&vpart[(j + 1) * kFT + g], acc[i][1]);
                        }
                        if (row1) {
                            atomicAdd(&vpart[j * kFT + g + 8], acc[i][2]);
                            atomicAdd(&vpart[(j + 1) * kFT + g + 8], acc[i][3]);
                        }
                    }
                }
            }
        }
        if (!waited) {
            pdl_trigger();
            pdl_wait();
            waited = true;
        }
        if (s_bad && blockIdx.x == 0 && tid == 0 && first_item)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        PHASE(4);
        __syncthreads();
        PHASE(5);

        // ---- exchange partials across the cluster (fixed summation order),
        // then split V into bf16 hi + lo, token-major, zero beyond cnt and r
        cluster_arrive();
        cluster_wait();
        PHASE(13);
        {
            namespace cg = cooperative_groups;
            cg::cluster_group cl = cg::this_cluster();
            const int rp = (r + 31) & ~31;
            // kFT * rp <= 16 * 128 elements: at most 16 per thread, 4 at a time
            for (int base = 0; base < kFT * rp; base += 4 * kFThreads) {
                float s[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
                for (int c = 0; c < kFC; ++c) {
                    const float *rv = cl.map_shared_rank(vpart, c);
#pragma unroll
                    for (int u = 0; u < 4; ++u) {
                        const int idx = base + u * kFThreads + tid;
                        const int t = idx & (kFT - 1), j = idx >> 4;
                        if (idx < kFT * rp && t < cnt && j < r)
                            s[u] += rv[j * kFT + t];
                    }
                }
#pragma unroll
                for (int u = 0; u < 4; ++u) {
                    const int idx = base + u * kFThreads + tid;
                    if (idx < kFT * rp) {
                        const int t = idx & (kFT - 1), j = idx >> 4;
                        const __nv_bfloat16 h = __float2bfloat16_rn(s[u]);
                        if (r > 16 || j < 16) {
                            const int e = vfrag_index(t, j, r <= 16);
                            vfr[e] = h;
                            vfr[e + (r <= 16 ? 256 : 512)] = __float2bfloat16_rn(s[u] - __bfloat162float(h));
                        }
                    }
                }
            }
        }
        publish();          // lands before the barrier that ends this item
        cluster_arrive();   // our reads of the other CTAs' partials are done
        cp_async_wait_all();
        __syncthreads();
        PHASE(6);

        // ---- expand: Y[16 x o-tile] += s (V_hi + V_lo) B[o-tile]^T, 8 outputs per tile
        {
            const int n_ot = (o1 - o0) >> 3;
            const bool row0 = g < cnt, row1 = g + 8 < cnt;
            __nv_bfloat16 *y0row = p.Y + (int64_t)(row0 ? tok[g] : 0) * p.ldy;
            __nv_bfloat16 *y1row = p.Y + (int64_t)(row1 ? tok[g + 8] : 0) * p.ldy;
#define LORA_EXPAND(NKB, ST)                                                                             \
    expand_tiles<NKB, ST>(Ba, r, o0, n_ot, warp, kFWarps, vq, lane, g, qd, y0row, y1row, row0, row1, p.scale, \
                          bst, yst, p.Wo)
            if (r <= 16) {
                if (L.staged)
                    expand_tiles16<true>(Ba, r, o0, n_ot, warp, kFWarps, vq, lane, g, qd, y0row, y1row, row0,
                                         row1, p.scale, bst, yst, p.Wo);
                else
                    expand_tiles16<false>(Ba, r, o0, n_ot, warp, kFWarps, vq, lane, g, qd, y0row, y1row, row0,
                                          row1, p.scale, bst, yst, p.Wo);
            } else if (L.staged) {
                switch ((r + 31) >> 5) {
                case 1: LORA_EXPAND(1, true); break;
                case 2: LORA_EXPAND(2, true); break;
                case 3: LORA_EXPAND(3, true); break;
                default: LORA_EXPAND(4, true); break;
                }
            } else {
                switch ((r + 31) >> 5) {
                case 1: LORA_EXPAND(1, false); break;
                case 2: LORA_EXPAND(2, false); break;
                case 3: LORA_EXPAND(3, false); break;
                default: LORA_EXPAND(4, false); break;
                }
            }
#undef LORA_EXPAND
        }
        PHASE(12);
        __syncthreads();
        PHASE(7);
        cluster_wait();     // no CTA reuses its partials while another may still read them
        PHASE(8);
        first = false;
        pos = s_next;
    }
    if (!waited) {
        pdl_trigger();
        pdl_wait();
        if (s_bad && blockIdx.x == 0 && tid == 0)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
    }
    // the last cluster out puts the item counter back to zero for the next launch
    if (crank == 0 && tid == 0) {
        __threadfence();
        if (atomicAdd(p.sched + 1, 1u) == (unsigned)n_cl - 1u) {
            atomicExch(p.sched, 0u);
            atomicExch(p.sched + 1, 0u);
        }
    }
}

}  // namespace

size_t fused_smem_bytes(int32_t N, int32_t n_adapters, int32_t max_rank, int32_t Wo)
{
    return fused_smem_layout(N, n_adapters, max_rank, Wo).total;
}

bool fused_bgmv_supported(int32_t N, int32_t n_adapters, int32_t d_in)
{
    // the layout at the largest rank, without staging (staging is dropped when it does not fit)
    const int32_t Wk = fused_chunk(d_in);
    return N <= kFMaxTokens && n_adapters <= kFMaxAdapters && Wk <= kFMaxChunk &&
           fused_smem_bytes(N, n_adapters, kMaxRank, 0) <= kFMaxSmem;
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
    const size_t smem = fused_smem_bytes(a.N, a.pool.n_adapters, a.pool.max_rank, a.Wo);
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
