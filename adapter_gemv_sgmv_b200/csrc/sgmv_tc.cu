// Tensor-core (tcgen05) shrink and expand for long segments and multi-adapter
// requests: the prefill SGMV and the diffusion multi-adapter workloads.
//
// The operation ("Serving several LoRAs, ControlNet and IP-Adapter", section
// "LoRA: merged or alongside"; exercise 2's answer; table row "Stacking
// several LoRAs"): V = X A^T (shrink, d_in -> r) then Y += s V B^T (expand,
// r -> d_out) for the rows of each segment (one adapter) or request (several
// adapters, their deltas summed).  Segments of a prefill batch and images of
// a diffusion batch hold hundreds to thousands of rows, so both halves are
// dense contractions with M = 128 rows per tile.
//
// Tiles never straddle an item: the plan kernel cuts every segment/request
// into tiles of at most 128 rows, so the rows of a tile share one adapter
// list.  A request's adapters are stacked along the rank axis (at most kKMax
// ranks in total): the shrink produces all of them in one accumulator
// (N = stacked rank), and the expand contracts over all of them at once
// (K = stacked rank, each adapter's scale folded into its V columns), so y is
// read, updated and rounded to bf16 once.  The shrink also stacks the A rows of
// projections that share x (up to 256 ranks), and can write s V as bf16 high
// and low parts for the fused projection kernel.
//
// Both kernels are persistent and warp specialised:
//   warp 0     producer: TMA for every operand -- x tiles (shrink) and y tiles
//              (expand) with 128-byte swizzle, A rows through the A pool seen
//              as [A_elems / d_in, d_in] and B slices through the B pool seen as
//              [B_elems / r, r] per rank r (an adapter whose offset does not fit
//              those views is gathered with cp.async into the same layout);
//   warp 1     one thread issues tcgen05.mma (bf16 x bf16 -> fp32 in TMEM,
//              M = 128) and tracks completion with tcgen05.commit;
//   others     epilogue: tcgen05.ld of the accumulator (a warp reads the TMEM
//              lane quarter of its warp index mod 4) -- four warps writing V
//              rows in the shrink (192 threads, two CTAs per SM), sixteen
//              adding D into y in the expand (576 threads, one CTA per SM).
// Stages hand over through mbarriers; every wait is bounded in time and, if it
// expires, records LORA_ERR_TIMEOUT and winds the CTA down (TMEM is freed).

#include <cuda.h>

#include "lora_internal.cuh"
#include "tc_ptx.cuh"

namespace lora {
namespace {

constexpr int kTcThreads = 192;       // shrink: producer, MMA, 4 epilogue warps
constexpr int kExpandThreads = 576;   // expand: producer, MMA, 16 epilogue warps
constexpr int kEpiWarps = 16;
// heights of the A-pool TMA boxes (map_a[m])
__host__ __device__ constexpr int abox_rows(int m) { return m == 0 ? 64 : (m == 1 ? 32 : 8); }
constexpr int kBN = 128;            // expand: outputs per unit
constexpr int kZeroCol = 1 << 30;          // shrink epilogue: a V column written as zeros
constexpr int kMaxShrinkStages = 6;
constexpr int kExpandBStages = 2;

// The adapter stack of one tile: entry i covers ranks [kb[i], kb[i] + r[i]) of
// the stacked axis, maps to V columns vc0[i] + j, is scaled by s[i] and reads
// its A rows from pool pool[i] (0 except for projections sharing an input).
// The roles work on different tiles at any moment, so every warp keeps its own
// copy in shared memory.
struct StackSm {
    int n;                                  // entries
    int ktot;                               // stacked rank
    int kpad;                               // stacked rank rounded up to 16 (MMA N or K)
    int a_tma;                              // every entry's A offset is a multiple of d_in
    int b_tma;                              // every entry's B slice can come by TMA (see b_map)
    int r[LORA_MAX_ADS_PER_REQ];
    int kb[LORA_MAX_ADS_PER_REQ];
    int vc0[LORA_MAX_ADS_PER_REQ];
    signed char pool[LORA_MAX_ADS_PER_REQ];
    float s[LORA_MAX_ADS_PER_REQ];
    long long aoff[LORA_MAX_ADS_PER_REQ];
    long long boff[LORA_MAX_ADS_PER_REQ];
};

// the entry holding stacked rank k (k < ktot)
__device__ __forceinline__ int stack_entry(const StackSm &st, int k)
{
    int e = 0;
    for (int i = 1; i < st.n; ++i)
        if (k >= st.kb[i])
            e = i;
    return e;
}

// One warp builds the stack of item `item`; lane e looks at the item's adapter
// e (for projections sharing an input: the segment's adapter in pool e).
// Adapters failing validation are left out (and reported when `report`); the
// shrink and the expand leave out the same ones.  The host sends only calls
// whose stacks fit in kmax ranks; an entry that would not fit is left out and
// reported as a bad segment.
__device__ void warp_build_stack(const TcArgs &p, int item, StackSm &st, bool report, int kmax = kKMax)
{
    const int lane = threadIdx.x & 31;
    __syncwarp();                           // this warp's readers of the previous stack are done
    int lo = 0, n = 1;
    if (p.mode == kModeMulti) {
        lo = p.ad_off[item];
        n = min(p.ad_off[item + 1] - lo, p.max_ads);
    } else if (p.mode == kModeProj) {
        n = p.n_proj;
    }
    const int pl = p.mode == kModeProj && lane < n ? lane : 0;   // this lane's pool
    int32_t r = 0;
    int64_t ao = 0, bo = 0;
    float sc = 0.f;
    bool ok = false;
    if (lane < n) {
        const int32_t a = p.mode == kModeMulti ? p.ad_id[lo + lane] : p.seg_ad[item];
        ok = pool_adapter_ok(p.mode == kModeProj ? p.proj[pl] : p.pool, a, &r, &ao, &bo);
        if (!ok && report && !(p.allow_none && a == -1))
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        sc = p.mode == kModeMulti ? p.ad_scale[lo + lane] : p.scale;
    }
    if (!ok)
        r = 0;
    int incl = r;                           // inclusive prefix of the ranks over the item's adapters
#pragma unroll
    for (int d = 1; d < LORA_MAX_ADS_PER_REQ; d <<= 1) {
        const int t = __shfl_up_sync(0xffffffffu, incl, d);
        if (lane >= d)
            incl += t;
    }
    const bool fits = ok && incl <= kmax;
    if (ok && !fits && report)
        atomicOr(p.err, (uint32_t)LORA_ERR_BAD_SEGMENT);
    const unsigned m = __ballot_sync(0xffffffffu, fits);
    const int ktot = (int)__reduce_max_sync(0xffffffffu, fits ? (unsigned)incl : 0u);
    const bool a_tma = __all_sync(0xffffffffu, !fits || ((ao % p.pool.d_in) == 0 && ((p.a_tma >> pl) & 1)));
    const int bm = b_map(r);
    const bool b_tma = __all_sync(0xffffffffu, !fits || (bm >= 0 && ((p.b_tma >> bm) & 1) && (bo % r) == 0));
    if (fits) {
        const int i = __popc(m & ((1u << lane) - 1u));
        st.r[i] = r;
        st.kb[i] = incl - r;
        st.vc0[i] = p.mode == kModeProj ? p.proj_vcol[pl] : lane * p.slot_stride;
        st.pool[i] = (signed char)pl;
        st.s[i] = sc;
        st.aoff[i] = ao;
        st.boff[i] = bo;
    }
    if (lane == 0) {
        st.n = __popc(m);
        st.ktot = ktot;
        st.kpad = (ktot + 15) & ~15;
        st.a_tma = a_tma ? 1 : 0;
        st.b_tma = b_tma ? 1 : 0;
    }
    __syncwarp();
}

#ifdef LORA_TC_TRACE
// Development aid: %globaltimer stamps of the last CTA, [role][unit][point].
__device__ unsigned long long g_tc_trace[3 * 1024 * 8];
#define TC_STAMP(role, iter, point)                                                          \
    do {                                                                                     \
        if (blockIdx.x == gridDim.x - 1 && (threadIdx.x & 31) == 0 && (iter) < 1024)         \
            g_tc_trace[((role) * 1024 + (iter)) * 8 + (point)] = now_ns();                   \
    } while (0)
#else
#define TC_STAMP(role, iter, point) \
    do {                            \
    } while (0)
#endif

// ============================================================ shrink kernel
//
// Unit = one tile of <= 128 rows of one item.  D[128 x kpad] = X_tile A_stack^T
// over d_in in 64-column k-blocks; the epilogue writes V rows (fp32).  The A
// rows of a k-block come by TMA in 64-, 32- and 8-row boxes over the A pool
// seen as a [A_elems / d_in, d_in] matrix (every adapter packed at a multiple
// of d_in), else by cp.async, 16 bytes at a time.  A stage holds the x atom and
// as many A rows as the call's largest stacked rank (rounded to 16): at rank
// 64, 24 KB, and four stages fit twice per SM, so two tiles can stream through
// one SM at once.  Projections that share X stack their A rows (from their own
// pools) up to 256 ranks: then one CTA per SM, as many 40-48 KB stages as fit,
// and MMA N up to 256.

__global__ void __launch_bounds__(kTcThreads, 2) k_tc_shrink(const __grid_constant__ TcArgs p)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    // 1024-byte alignment for the swizzle atoms
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[kMaxShrinkStages], empty_bar[kMaxShrinkStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2], mma_drain;
    __shared__ __align__(8) StackSm stk[kTcThreads / 32];
    __shared__ const __nv_bfloat16 *arow[kKMaxShrink];   // producer, cp.async path: stacked row j's A row
    __shared__ int4 abox[kKMaxShrink / 8];   // producer, TMA path: (stacked row, pool row, map) of each A box
    __shared__ int vcol[4][kKMaxShrink / 4]; // epilogue warp q: V column of stacked columns 4g..4g+3 (-1: none)
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int d_in = p.pool.d_in;
    const int n_kb = (d_in + kBK - 1) / kBK;
    const int n_st = p.s_stages;
    const int acc = p.s_acc;                     // TMEM columns per accumulator (two of them)

    if (tid == 0) {
        for (int s = 0; s < kMaxShrinkStages; ++s) {
            mbar_init(&full_bar[s], 33);     // producer lane 0's expect_tx + 32 cp.async arrivals
            mbar_init(&empty_bar[s], 1);     // MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);      // MMA commit
            mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
        }
        mbar_init(&mma_drain, 1);            // the MMA issuer's last commit before TMEM is freed
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1)
        tmem_alloc(&tmem_base, 2 * acc);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    pdl_wait();                                  // the plan kernel's tiles are complete
    pdl_trigger();
    const int n_units = p.hdr->n_groups;
    const int u0 = (int)((int64_t)blockIdx.x * n_units / G), u1 = (int)((int64_t)(blockIdx.x + 1) * n_units / G);
    int issued = 0;                              // producer: stage fills issued

    if (warp == 0) {
        // ------------------------------------------------ producer
        StackSm &st = stk[0];
        int it = 0;
        if (p.test_stall)
            goto done;
        for (int u = u0; u < u1; ++u) {
            const Group gr = p.groups[u];
            warp_build_stack(p, gr.item, st, false, kKMaxShrink);
            const bool use_tma = st.a_tma;
            // A boxes: each entry's rows cut into 64-, 32- and 8-row boxes (at most 32 boxes)
            int nbox = 0;
            int box_j = 0, box_row = 0, box_m = 0;   // this lane's box: stacked row, pool row, map
            if (use_tma) {
                if (lane == 0) {
                    for (int e = 0; e < st.n; ++e) {
                        const int row0 = (int)(st.aoff[e] / d_in);
                        for (int j = 0; j < st.r[e];) {
                            const int m = st.r[e] - j >= 64 ? 0 : (st.r[e] - j >= 32 ? 1 : 2);
                            abox[nbox] = make_int4(st.kb[e] + j, row0 + j, 3 * st.pool[e] + m, 0);
                            ++nbox;
                            j += abox_rows(m);
                        }
                    }
                }
                nbox = __shfl_sync(0xffffffffu, nbox, 0);
                __syncwarp();
                if (lane < nbox) {
                    const int4 bx = abox[lane];
                    box_j = bx.x;
                    box_row = bx.y;
                    box_m = bx.z;
                }
            } else {
                for (int j = lane; j < kKMaxShrink; j += 32) {
                    const __nv_bfloat16 *o = p.pool.A;
                    if (j < st.ktot) {
                        const int e = stack_entry(st, j);
                        const __nv_bfloat16 *A = p.mode == kModeProj ? p.proj[st.pool[e]].A : p.pool.A;
                        o = A + st.aoff[e] + (long long)(j - st.kb[e]) * d_in;
                    }
                    arow[j] = o;
                }
                __syncwarp();
            }
            const uint32_t tx = (uint32_t)kAtom + (use_tma ? (uint32_t)st.ktot * 128u : 0u);
            const uint64_t pol_x = policy_evict_first(), pol_a = policy_evict_last();
            for (int kb = 0; kb < n_kb; ++kb, ++it) {
                const int s = it % n_st;
                const uint32_t ph = (it / n_st) & 1;
                TC_STAMP(0, it, 0);
                if (!warp_wait(&empty_bar[s], ph ^ 1, &abort_flag, p.err, p.wait_ns))
                    goto done;
                TC_STAMP(0, it, 1);
                unsigned char *xs = sm + s * p.s_stage;
                unsigned char *as = xs + kAtom;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_bar[s], tx);
                    tma_load_2d_hint(xs, &p.map_x, &full_bar[s], kb * kBK, gr.p0, pol_x);
                }
                __syncwarp();
                if (use_tma) {
                    if (lane < nbox)
                        tma_load_2d_hint(as + box_j * 128, &p.map_a[box_m], &full_bar[s], kb * kBK, box_row, pol_a);
                } else {
                    // stacked row j, 16-byte chunk c; rows past the stack feed only
                    // accumulator columns that are never stored
                    const int c = lane & 7, col = kb * kBK + c * 8;
                    const bool in = col < d_in;
                    const uint32_t abase = smem_u32(as);
                    for (int j = lane >> 3; j < st.ktot; j += 4)
                        cp_async16(abase + sw128_off(j, c), in ? arow[j] + col : p.pool.A, in);
                }
                cp_async_arrive(&full_bar[s]);
                issued = it + 1;
                TC_STAMP(0, it, 2);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        StackSm &st = stk[1];
        int it = 0, t = 0;
        for (int u = u0; u < u1; ++u, ++t) {
            const Group gr = p.groups[u];
            warp_build_stack(p, gr.item, st, false, kKMaxShrink);
            const int kpad = st.kpad;
            const bool a_tma = st.a_tma;
            const int b = t & 1;
            if (!warp_wait(&acc_empty[b], ((t >> 1) & 1) ^ 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(kBM, kpad > 0 ? kpad : 16);
            for (int kb = 0; kb < n_kb; ++kb, ++it) {
                const int s = it % n_st;
                const uint32_t ph = (it / n_st) & 1;
                TC_STAMP(1, it, 0);
                if (!warp_wait(&full_bar[s], ph, &abort_flag, p.err, p.wait_ns))
                    goto done;
                TC_STAMP(1, it, 1);
                if (!a_tma)
                    fence_async_smem();         // A written by cp.async (generic proxy)
                tc_fence_after();
                if (lane == 0 && kpad > 0) {
                    const uint32_t xa = smem_u32(sm + s * p.s_stage);
                    const uint32_t aa = xa + kAtom;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        tc_mma(tmem + b * acc, sw128_desc(xa + k * 32), sw128_desc(aa + k * 32), idesc,
                               (kb > 0 || k > 0) ? 1u : 0u);
                    TC_STAMP(1, it, 2);
                }
                __syncwarp();
                if (lane == 0)
                    tc_commit(&empty_bar[s]);
                TC_STAMP(1, it, 3);
                __syncwarp();
            }
            if (lane == 0)
                tc_commit(&acc_full[b]);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue: D -> V rows
        const int q = warp & 3;                 // TMEM lane quarter owned by this warp
        const int row = q * 32 + lane;
        StackSm &st = stk[warp];
        int *vc = vcol[q];
        int t = 0;
        for (int u = u0; u < u1; ++u, ++t) {
            const Group gr = p.groups[u];
            warp_build_stack(p, gr.item, st, warp == 2, kKMaxShrink);
            for (int g = lane; g < kKMaxShrink / 4; g += 32) {
                const int k = g * 4;
                int c = -1;
                if (k < st.ktot) {
                    const int e = stack_entry(st, k);
                    c = st.vc0[e] + (k - st.kb[e]);
                } else if (p.Vb && st.n == 1 && k < ((st.ktot + 15) & ~15)) {
                    // bf16-pair output: the columns up to the next 16 are written as zeros,
                    // since the projection's MMAs read V in steps of 16 ranks
                    c = (st.vc0[0] + k) | kZeroCol;
                }
                vc[g] = c;
            }
            __syncwarp();
            const int b = t & 1;
            if (!warp_wait(&acc_full[b], (t >> 1) & 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            tc_fence_after();
            const bool valid = row < gr.cnt;
            const int64_t vr = gr.p0 + (valid ? row : 0);
            float *vrow = p.Vb ? nullptr : p.V + vr * p.ldv;
            __nv_bfloat16 *brow = p.Vb ? p.Vb + vr * p.ldvb : nullptr;
            for (int c0 = 0; c0 < st.kpad; c0 += 32) {
                float v[32];
                tmem_ld32(tmem + b * acc + ((uint32_t)(q * 32) << 16) + c0, v);
                if (valid) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        int col = vc[(c0 >> 2) + g];
                        if (col < 0)
                            continue;
                        if (col & kZeroCol) {
                            col &= ~kZeroCol;
                            *reinterpret_cast<uint2 *>(brow + col) = make_uint2(0u, 0u);
                            *reinterpret_cast<uint2 *>(brow + p.vb_lo + col) = make_uint2(0u, 0u);
                            continue;
                        }
                        if (brow) {
                            // s v as a high and a low bf16 part (the fused projection's LoRA operand)
                            uint32_t hi[2], lo[2];
#pragma unroll
                            for (int j = 0; j < 2; ++j) {
                                const float x0 = p.scale * v[4 * g + 2 * j], x1 = p.scale * v[4 * g + 2 * j + 1];
                                const __nv_bfloat162 h = __floats2bfloat162_rn(x0, x1);
                                const float2 hf = __bfloat1622float2(h);
                                const __nv_bfloat162 l = __floats2bfloat162_rn(x0 - hf.x, x1 - hf.y);
                                hi[j] = *reinterpret_cast<const uint32_t *>(&h);
                                lo[j] = *reinterpret_cast<const uint32_t *>(&l);
                            }
                            *reinterpret_cast<uint2 *>(brow + col) = make_uint2(hi[0], hi[1]);
                            *reinterpret_cast<uint2 *>(brow + p.vb_lo + col) = make_uint2(lo[0], lo[1]);
                        } else {
                            *reinterpret_cast<float4 *>(vrow + col) =
                                make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[b]);
        }
    }
done:
    // nothing may land in shared memory or TMEM after this CTA lets go of them:
    // the producer waits for its fills, the MMA issuer for its last MMAs
    if (warp == 0)
        drain_fills(full_bar, n_st, issued, p.err, p.wait_ns);
    if (warp == 1 && lane == 0)
        drain_mma(&mma_drain, 0, p.err, p.wait_ns);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * acc);
    }
}


// ============================================================ expand kernel
//
// Unit = (tile, 128-output slice).  D[128 x 128] = V_tile B_stack[slice]^T over
// the stacked rank (V staged once per tile as a pair of bf16 matrices, high and
// low parts, so the product sees V to about 2^-17 relative for one extra MMA per
// 16 ranks; each adapter's scale folded in when a request stacks several, a
// single adapter's scale multiplying the fp32 accumulator instead);
// the epilogue adds D to the y tile (TMA-loaded; threads only read it, so a
// stage goes back to the producer as soon as it is read) and each epilogue
// warp stores its rows through a small staging area with coalesced 16-byte
// stores.
//
// Shared memory is laid out at run time: each half of V and every B stage take
// one 16 KB atom per 64 stacked ranks the call can carry (1 or 2), and the y
// stages fill the rest (up to kMaxYStages): four 32 KB y tiles in flight at rank
// 64, two at 128.
constexpr int kY = kBM * kBN * 2;                  // y: 128 rows x 128 outputs (two 64-column atoms)
constexpr int kMaxYStages = 6;
constexpr int kStaging = kEpiWarps * 1024;         // per epilogue warp: 32 rows x 16 outputs of bf16

// The expand of one CTA: block bid of G working on p's units.  p must refer to
// kernel-parameter memory (its tensor maps are read by the copy engine).
__device__ __forceinline__ void tc_expand_cta(const TcArgs &p, int bid, int G)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t b_full[kExpandBStages], b_empty[kExpandBStages];
    __shared__ __align__(8) uint64_t y_full[kMaxYStages], y_empty[kMaxYStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ __align__(8) uint64_t v_full, v_empty;
    __shared__ __align__(8) StackSm stk[kExpandThreads / 32];
    __shared__ long long cb_off[kKMax / 8];  // producer: B element offset of stacked 8-rank chunk c in output row 0
    __shared__ int cb_r[kKMax / 8];          // its row stride (the adapter's rank); 0 = padding chunk
    __shared__ int vsrc[kEpiWarps][kKMax / 8];   // epilogue warp e: V column of stacked chunk c (-1: zero)
    __shared__ float vsc[kEpiWarps][kKMax / 8];  // and its adapter's scale
    __shared__ uint32_t tmem_base;
    __shared__ __align__(8) uint64_t mma_drain;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d_out = p.pool.d_out;
    const int n_ns = (d_out + kBN - 1) / kBN;           // output slices
    const int n_ys = p.e_ystages;
    const int szB = p.e_natoms * kAtom;                 // one B stage (and each half of V)
    unsigned char *const smV = sm;                      // V high parts, then V low parts
    unsigned char *const smB = sm + 2 * szB;
    unsigned char *const smS = smB + kExpandBStages * szB;   // epilogue warps' output staging
    unsigned char *const smY = smS + kStaging;

    if (tid == 0) {
        for (int s = 0; s < kExpandBStages; ++s) {
            mbar_init(&b_full[s], 33);       // lane 0 (expect_tx or plain) + 32 cp.async arrivals
            mbar_init(&b_empty[s], 1);       // MMA commit
        }
        for (int s = 0; s < kMaxYStages; ++s) {
            mbar_init(&y_full[s], 1);        // expect_tx
            mbar_init(&y_empty[s], kEpiWarps);   // epilogue warps: the tile is read
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], kEpiWarps); // epilogue warps
        }
        mbar_init(&v_full, kEpiWarps);       // epilogue warps, after staging V
        mbar_init(&v_empty, 1);              // MMA commit after a tile's last unit
        mbar_init(&mma_drain, 1);            // the MMA issuer's last commit before TMEM is freed
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1)
        tmem_alloc(&tmem_base, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    pdl_wait();                                  // tiles and V of the previous kernels are complete
    pdl_trigger();
    const int64_t n_units = (int64_t)p.hdr->n_groups * n_ns;
    const int64_t u0 = (int64_t)bid * n_units / G, u1 = (int64_t)(bid + 1) * n_units / G;
    int y_issued = 0, b_issued = 0;              // producer: y and B stage fills issued

    if (warp == 0) {
        // ------------------------------------------------ producer: y tiles and B slices
        StackSm &st = stk[0];
        int it = 0;
        if (p.test_stall)
            goto done;
        int64_t prev_tile = -1;
        int nch = 0, o_l = 0, c_l = 0, dq = 0, dr = 0;
        int p0 = 0;
        int bx_m = 0, bx_y = 0, bx_dst = 0, bx_two = 0;   // this lane's B box (TMA path, lane < n)
        const uint64_t pol_y = policy_evict_first(), pol_b = policy_evict_last();
        for (int64_t u = u0; u < u1; ++u, ++it) {
            const int tile = (int)(u / n_ns), ns = (int)(u - (int64_t)tile * n_ns);
            if (tile != prev_tile) {
                const Group gr = p.groups[tile];
                p0 = gr.p0;
                warp_build_stack(p, gr.item, st, false);
                prev_tile = tile;
                if (st.b_tma) {
                    if (lane < st.n) {
                        const int r = st.r[lane];
                        bx_m = b_map(r);
                        bx_y = (int)(st.boff[lane] / r);
                        bx_dst = st.kb[lane] * 256;
                        bx_two = r == 128;
                    }
                } else {
                    if (lane < kKMax / 8) {
                        const int k = lane * 8;
                        long long o = 0;
                        int rr = 0;
                        if (k < st.ktot) {
                            const int e = stack_entry(st, k);
                            o = st.boff[e] + (k - st.kb[e]);
                            rr = st.r[e];
                        }
                        cb_off[lane] = o;
                        cb_r[lane] = rr;
                    }
                    __syncwarp();
                    // this lane walks chunk indices lane, lane + 32, ... of the (output, chunk) grid
                    nch = st.kpad >> 3;
                    if (nch > 0) {
                        o_l = lane / nch;
                        c_l = lane - o_l * nch;
                        dq = 32 / nch;
                        dr = 32 - dq * nch;
                    }
                }
            }
            const int o0 = ns * kBN;
            const int sy = it % n_ys;
            TC_STAMP(0, it, 0);
            if (!warp_wait(&y_empty[sy], ((it / n_ys) & 1) ^ 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            TC_STAMP(0, it, 1);
            unsigned char *ys = smY + sy * kY;
            if (lane == 0) {
                mbar_arrive_expect_tx(&y_full[sy], kY);
                tma_load_2d_hint(ys, &p.map_y, &y_full[sy], o0, p0, pol_y);
                tma_load_2d_hint(ys + kAtom, &p.map_y, &y_full[sy], o0 + 64, p0, pol_y);
            }
            y_issued = it + 1;
            const int sb = it % kExpandBStages;
            if (!warp_wait(&b_empty[sb], ((it / kExpandBStages) & 1) ^ 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            TC_STAMP(0, it, 2);
            unsigned char *bs = smB + sb * szB;
            if (st.b_tma) {
                // one box per entry (two for rank 128): outputs o0 .. o0 + 127 of its B, in the
                // entry's own region (kb * 256 bytes in), swizzled to its row width; rows past
                // d_out feed only accumulator columns that are never stored
                if (lane == 0)
                    mbar_arrive_expect_tx(&b_full[sb], (uint32_t)st.ktot * 256u);
                __syncwarp();
                if (lane < st.n) {
                    tma_load_2d_hint(bs + bx_dst, &p.map_b[bx_m], &b_full[sb], 0, bx_y + o0, pol_b);
                    if (bx_two)
                        tma_load_2d_hint(bs + bx_dst + kAtom, &p.map_b[bx_m], &b_full[sb], 64, bx_y + o0, pol_b);
                }
            } else {
                if (lane == 0)
                    mbar_arrive(&b_full[sb]);
                // cp.async: output o of the slice, 16-byte chunk c of the stacked rank axis
                // (atom c / 8); padding chunks and outputs past d_out are zero-filled
                const uint32_t bbase = smem_u32(bs);
                int o = o_l, c = c_l;
                for (int idx = lane; idx < kBN * nch; idx += 32) {
                    const int rr = cb_r[c];
                    const bool ok = rr > 0 && o0 + o < d_out;
                    const __nv_bfloat16 *src = ok ? p.pool.B + cb_off[c] + (long long)(o0 + o) * rr : p.pool.B;
                    cp_async16(bbase + (c >> 3) * kAtom + sw128_off(o, c & 7), src, ok);
                    c += dr;
                    o += dq;
                    if (c >= nch) {
                        c -= nch;
                        ++o;
                    }
                }
            }
            cp_async_arrive(&b_full[sb]);
            b_issued = it + 1;
            TC_STAMP(0, it, 3);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        // Per tile, the operand descriptors of every 16-rank step (at most 8) are worked
        // out once: V's are absolute, B's relative to the stage (the stage base, >> 4, is
        // added to the start-address field per unit).
        StackSm &st = stk[1];
        int it = 0, vt = 0;
        int64_t prev_tile = -1;
        int nsteps = 0;
        bool b_tma = false;
        uint64_t ad[kKMax / 16], bd[kKMax / 16];
        const uint32_t va = smem_u32(smV);
        const uint64_t lo_step = (uint64_t)((szB >> 4) & 0x3FFF);   // descriptor start field: V high -> V low
        for (int64_t u = u0; u < u1; ++u, ++it) {
            const int tile = (int)(u / n_ns);
            if (tile != prev_tile) {
                warp_build_stack(p, p.groups[tile].item, st, false);
                prev_tile = tile;
                b_tma = st.b_tma;
                nsteps = st.kpad / 16;
                int e = 0;
#pragma unroll
                for (int k16 = 0; k16 < kKMax / 16; ++k16) {
                    const int k = k16 * 16;
                    ad[k16] = sw128_desc(va + (k >> 6) * kAtom + ((k & 63) >> 4) * 32);
                    if (b_tma) {
                        // B: entry e's region at kb_e * 256 bytes, swizzled to its rank
                        while (e + 1 < st.n && k >= st.kb[e + 1])
                            ++e;
                        const int kl = k - st.kb[e];
                        const int re = st.r[e];
                        const uint32_t reg = st.kb[e] * 256;
                        bd[k16] = re >= 64 ? sw128_desc(reg + (kl >> 6) * kAtom + ((kl & 63) >> 4) * 32)
                                           : (re == 32 ? sw64_desc(reg + (kl >> 4) * 32) : sw32_desc(reg));
                    } else {
                        bd[k16] = sw128_desc((k >> 6) * kAtom + ((k & 63) >> 4) * 32);
                    }
                }
                if (!warp_wait(&v_full, vt & 1, &abort_flag, p.err, p.wait_ns))
                    goto done;
                ++vt;
            }
            const int b = it & 1;
            TC_STAMP(1, it, 0);
            if (!warp_wait(&acc_empty[b], ((it >> 1) & 1) ^ 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            TC_STAMP(1, it, 1);
            const int sb = it % kExpandBStages;
            if (!warp_wait(&b_full[sb], (it / kExpandBStages) & 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            TC_STAMP(1, it, 2);
            if (!b_tma)
                fence_async_smem();             // B written by cp.async (generic proxy)
            tc_fence_after();
            if (lane == 0) {
                const uint64_t bbase = (smem_u32(smB + sb * szB) >> 4) & 0x3FFFu;
                const uint32_t idesc = idesc_bf16(kBM, kBN);
#pragma unroll
                for (int k16 = 0; k16 < kKMax / 16; ++k16)
                    if (k16 < nsteps) {
                        tc_mma(tmem + b * 128, ad[k16], bd[k16] + bbase, idesc, k16 > 0 ? 1u : 0u);
                        tc_mma(tmem + b * 128, ad[k16] + lo_step, bd[k16] + bbase, idesc, 1u);
                    }
                TC_STAMP(1, it, 3);
                tc_commit(&b_empty[sb]);
                tc_commit(&acc_full[b]);
                const bool last_of_tile = u + 1 >= u1 || (int)((u + 1) / n_ns) != tile;
                if (last_of_tile)
                    tc_commit(&v_empty);
                TC_STAMP(1, it, 4);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue: V staging, y += D, store
        // Sixteen warps: warp w reads TMEM lane quarter w % 4 (rows 32 (w % 4) ..) and
        // owns output quarter cq (32 columns: half cq / 2 of a 64-column y atom) of every
        // unit -- 64 values per thread, so the sixteen warps keep twice as many
        // independent update chains in flight as eight warps of 64 columns could.
        const int e8 = warp - 2;                // 0..15
        const int q = warp & 3;
        const int cq = e8 >> 2;
        const int h = cq >> 1;
        const int row = q * 32 + lane;
        const int et = tid - 64;                // 0..511 over the epilogue warps
        StackSm &st = stk[warp];
        int it = 0, vt = 0;
        int64_t prev_tile = -1;
        Group gr = {0, 0, 0, 0};
        const uint64_t pol_st = policy_evict_first();
        for (int64_t u = u0; u < u1; ++u, ++it) {
            const int tile = (int)(u / n_ns), ns = (int)(u - (int64_t)tile * n_ns);
            if (tile != prev_tile) {
                gr = p.groups[tile];
                warp_build_stack(p, gr.item, st, false);   // the shrink kernel reports bad adapters
                prev_tile = tile;
                if (lane < kKMax / 8) {
                    const int k = lane * 8;
                    int c = -1;
                    float sc = 0.f;
                    if (k < st.ktot) {
                        const int e = stack_entry(st, k);
                        c = st.vc0[e] + (k - st.kb[e]);
                        // several adapters: each one's scale goes into its V columns; one
                        // adapter: V is staged as it is and D is scaled in fp32 (for the merge,
                        // whose V is exactly bf16 -- low part zero -- this keeps a single
                        // rounding of W)
                        sc = p.mode == kModeMulti ? st.s[e] : 1.f;
                    }
                    vsrc[e8][lane] = c;
                    vsc[e8][lane] = sc;
                }
                __syncwarp();
                // wait until the MMAs of the previous tile stopped reading V
                if (vt > 0 && !warp_wait(&v_empty, (vt - 1) & 1, &abort_flag, p.err, p.wait_ns))
                    goto done;
                // V[vr][stacked k] = s_e * V_e[vr][k - kb_e] (s_e = 1 for one adapter), zero outside the
                // tile's rows and the stack, as two bf16 parts: hi = bf16(v) and lo = bf16(v - hi), so
                // hi + lo carries v to about 2^-17 and the MMA sums both; thread et stages row
                // et % 128, stacked ranks 32 (et / 128) .. + 31
                const int vr = et & 127, vq = et >> 7;
                const bool valid = vr < gr.cnt;
                const float *vrow = p.V + (int64_t)(gr.p0 + (valid ? vr : 0)) * p.ldv;
                const uint32_t vbase = smem_u32(smV);
                const int c_end = min(st.kpad / 8, vq * 4 + 4);
                for (int c = vq * 4; c < c_end; ++c) {
                    const int col = vsrc[e8][c];
                    uint32_t w[4] = {0u, 0u, 0u, 0u}, wl[4] = {0u, 0u, 0u, 0u};
                    if (valid && col >= 0) {
                        const float sc = vsc[e8][c];
                        const float4 a = *reinterpret_cast<const float4 *>(vrow + col);
                        const float4 bq = *reinterpret_cast<const float4 *>(vrow + col + 4);
                        const float v[8] = {sc * a.x, sc * a.y, sc * a.z, sc * a.w,
                                            sc * bq.x, sc * bq.y, sc * bq.z, sc * bq.w};
#pragma unroll
                        for (int j = 0; j < 4; ++j) {
                            const __nv_bfloat162 hi = __floats2bfloat162_rn(v[2 * j], v[2 * j + 1]);
                            const float2 hf = __bfloat1622float2(hi);
                            const __nv_bfloat162 lo = __floats2bfloat162_rn(v[2 * j] - hf.x, v[2 * j + 1] - hf.y);
                            w[j] = *reinterpret_cast<const uint32_t *>(&hi);
                            wl[j] = *reinterpret_cast<const uint32_t *>(&lo);
                        }
                    }
                    const uint32_t dst = vbase + (c >> 3) * kAtom + sw128_off(vr, c & 7);
                    st_shared_v4(dst, w[0], w[1], w[2], w[3]);
                    st_shared_v4(dst + szB, wl[0], wl[1], wl[2], wl[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&v_full);
                ++vt;
            }
            const int b = it & 1;
            const int sy = it % n_ys;
            if (warp == 2)
                TC_STAMP(2, it, 0);
            if (!warp_wait(&acc_full[b], (it >> 1) & 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            if (warp == 2)
                TC_STAMP(2, it, 1);
            if (!warp_wait(&y_full[sy], (it / n_ys) & 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            if (warp == 2)
                TC_STAMP(2, it, 2);
            tc_fence_after();
            const int o0 = ns * kBN;
            const uint32_t atom = smem_u32(smY + sy * kY) + h * kAtom;
            const int c0 = (cq & 1) * 4;            // this quarter's first 16-byte chunk in the atom
            // this row's 32 y values (four 16-byte chunks); the stage is then free again:
            // threads only read the TMA-loaded tiles, never write them
            uint32_t yw[4][4];
#pragma unroll
            for (int c = 0; c < 4; ++c)
                ld_shared_v4(atom + sw128_off(row, c0 + c), yw[c]);
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&y_empty[sy]);
            if (warp == 2)
                TC_STAMP(2, it, 3);
            float d[32];
            tmem_ld32(tmem + b * 128 + ((uint32_t)(q * 32) << 16) + cq * 32, d);
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty[b]);
            if (warp == 2)
                TC_STAMP(2, it, 4);
            const bool none = st.kpad == 0;     // no valid adapter: no MMA ran, y is stored unchanged
            const float dsc = p.mode == kModeMulti ? 1.f : p.scale;
            uint32_t ow[4][4];
#pragma unroll
            for (int c = 0; c < 4; ++c) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&yw[c][e]));
                    const float d0 = none ? 0.f : dsc * d[c * 8 + 2 * e];
                    const float d1 = none ? 0.f : dsc * d[c * 8 + 2 * e + 1];
                    const __nv_bfloat162 r2 = __floats2bfloat162_rn(yf.x + d0, yf.y + d1);
                    ow[c][e] = *reinterpret_cast<const uint32_t *>(&r2);
                }
            }
            if (warp == 2)
                TC_STAMP(2, it, 5);
            // store through this warp's 1 KB staging area, 16 columns at a time: rows of 32
            // bytes (2 chunks, XOR-swizzled by row / 4), read back 2 lanes per row so every
            // store instruction writes 16 rows x 32 contiguous bytes (whole sectors)
            const uint32_t stg = smem_u32(smS) + e8 * 1024;
            const int n_rows = min(gr.cnt - q * 32, 32);
#pragma unroll
            for (int pass = 0; pass < 2; ++pass) {
#pragma unroll
                for (int c = 0; c < 2; ++c)
                    st_shared_v4(stg + lane * 32 + ((c ^ ((lane >> 2) & 1)) << 4), ow[2 * pass + c][0],
                                 ow[2 * pass + c][1], ow[2 * pass + c][2], ow[2 * pass + c][3]);
                __syncwarp();
                const int cc = lane & 1;
                const int o = o0 + cq * 32 + pass * 16 + cc * 8;
                if (o < d_out) {
#pragma unroll
                    for (int j = 0; j < 2; ++j) {
                        const int rl = 16 * j + (lane >> 1);
                        if (rl < n_rows) {
                            uint32_t w[4];
                            ld_shared_v4(stg + rl * 32 + ((cc ^ ((rl >> 2) & 1)) << 4), w);
                            st_global_v4_hint(p.Y + (int64_t)(gr.p0 + q * 32 + rl) * p.ldy + o, w[0], w[1], w[2],
                                              w[3], pol_st);
                        }
                    }
                }
                __syncwarp();
            }
            if (warp == 2)
                TC_STAMP(2, it, 6);
        }
    }
done:
    // nothing may land in shared memory or TMEM after this CTA lets go of them
    if (warp == 0) {
        drain_fills(y_full, n_ys, y_issued, p.err, p.wait_ns);
        drain_fills(b_full, kExpandBStages, b_issued, p.err, p.wait_ns);
    }
    if (warp == 1 && lane == 0)
        drain_mma(&mma_drain, 0, p.err, p.wait_ns);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

__global__ void __launch_bounds__(kExpandThreads, 1) k_tc_expand(const __grid_constant__ TcArgs p)
{
    tc_expand_cta(p, blockIdx.x, gridDim.x);
}

// The expands of projections that share V's tiles (q, k, v of one x) in one launch:
// CTAs [cta0[i], cta0[i + 1]) take projection i's units, the split proportional to
// each projection's output slices, so that the small projections no longer run
// alone on the whole GPU with a few units per CTA.
struct TcExpandMulti {
    TcArgs a[kMaxProj];
    int32_t n;
    int32_t cta0[kMaxProj + 1];
};

__global__ void __launch_bounds__(kExpandThreads, 1) k_tc_expand_multi(const __grid_constant__ TcExpandMulti m)
{
    int i = 0;
    while (i + 1 < m.n && (int)blockIdx.x >= m.cta0[i + 1])
        ++i;
    tc_expand_cta(m.a[i], (int)blockIdx.x - m.cta0[i], m.cta0[i + 1] - m.cta0[i]);
}

// attr_set: this kernel's per-device "shared-memory opt-in done" flags (one
// array per kernel: the kernels share a type, so they cannot share the flags)
cudaError_t launch_tc(void (*kernel)(TcArgs), bool *attr_set, const TcArgs &a, int threads, int smem, int grid,
                      cudaStream_t s)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace

bool tc_encode_a(TcArgs &a, const void *A, int64_t A_elems, int32_t d_in, int pool_index)
{
    // the A pool as a [A_elems / d_in, d_in] matrix, boxes of 64 columns x 64, 32 and 8 rows
    if (pool_index < 0 || pool_index >= kMaxProj)
        return false;
    a.a_tma &= ~(1 << pool_index);
    const int64_t rows = A_elems / d_in;
    if (rows < 1 || rows > 0x7fffffffLL)
        return false;
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
    const cuuint32_t estr[2] = {1, 1};
    for (int i = 0; i < 3; ++i) {
        const cuuint32_t box[2] = {64, (cuuint32_t)abox_rows(i)};
        if (fn(&a.map_a[3 * pool_index + i], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(A), dims,
               strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
               CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return false;
    }
    a.a_tma |= 1 << pool_index;
    return true;
}

bool tc_encode_b(TcArgs &a, const void *B, int64_t B_elems)
{
    a.b_tma = encode_b_views(a.map_b, B, B_elems);
    return a.b_tma != 0;
}

bool tc_encode_x(TcArgs &a, const void *X, int32_t N, int32_t d_in, int64_t ldx)
{
    return encode_rows(&a.map_x, X, N, d_in, ldx);
}

bool tc_encode_y(TcArgs &a, const void *Y, int32_t N, int32_t d_out, int64_t ldy)
{
    return encode_rows(&a.map_y, Y, N, d_out, ldy);
}

cudaError_t launch_tc_shrink(const TcArgs &args, int max_tiles, int kk, cudaStream_t s)
{
    // a stage: the x atom and round16(kk) A rows of 128 bytes.  Up to 128
    // stacked ranks: two CTAs per SM, each with two 128-column accumulators;
    // above (projections sharing X): one CTA per SM (its four stages take
    // more than half the SM's shared memory) with two 256-column accumulators
    static bool attr_set[64] = {};
    if (kk < 1 || kk > kKMaxShrink)
        return cudaErrorInvalidValue;
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, k_tc_shrink)) != cudaSuccess)
        return e;
    const int room = optin - (int)fa.sharedSizeBytes - 1024;
    TcArgs a = args;
    a.wait_ns = wait_bound_ns();
    a.test_stall = test_stall_mode();
    const int a_rows = (kk + 15) & ~15;
    const bool wide = kk > kKMax;
    a.s_stage = kAtom + a_rows * 128;
    // wide: as many stages as one CTA's shared memory holds (5 at 192 ranks, 4 at 256)
    a.s_stages = wide ? (room / a.s_stage < kMaxShrinkStages ? room / a.s_stage : kMaxShrinkStages)
                      : (kk > 64 ? 3 : 4);
    if (a.s_stages < 2)
        return cudaErrorInvalidConfiguration;
    a.s_acc = wide ? 256 : 128;
    const int smem = a.s_stages * a.s_stage + 1024;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(k_tc_shrink, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      optin - (int)fa.sharedSizeBytes)) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    int grid = (wide ? 1 : 2) * sm_count();
    if (max_tiles > 0 && max_tiles < grid)
        grid = max_tiles;
    bool done = true;
    return launch_tc(k_tc_shrink, &done, a, kTcThreads, smem, grid, s);
}

cudaError_t launch_tc_expand(const TcArgs &args, int kk, cudaStream_t s)
{
    // shared memory: V (high and low parts) and two B stages of one atom per 64
    // stacked ranks, then as many 32 KB y stages as fit (at least two)
    static bool attr_set[64] = {};
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, k_tc_expand)) != cudaSuccess)
        return e;
    TcArgs a = args;
    a.wait_ns = wait_bound_ns();
    a.test_stall = test_stall_mode();
    a.e_natoms = kk > 64 ? 2 : 1;
    const int fixed = (2 + kExpandBStages) * a.e_natoms * kAtom + kStaging + 1024;
    const int room = optin - (int)fa.sharedSizeBytes - fixed;
    a.e_ystages = room / kY < kMaxYStages ? room / kY : kMaxYStages;
    if (a.e_ystages < 2)
        return cudaErrorInvalidConfiguration;
    const int smem = fixed + a.e_ystages * kY;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(k_tc_expand, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      optin - (int)fa.sharedSizeBytes)) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    bool done = true;
    return launch_tc(k_tc_expand, &done, a, kExpandThreads, smem, sm_count(), s);
}

cudaError_t launch_tc_expand_multi(const TcArgs *args, int n, int kk, cudaStream_t s)
{
    constexpr int kTileCost = 4;     // per-tile overhead of a CTA, in output slices (measured: 0 and 8 slower)
    if (n < 1 || n > kMaxProj)
        return cudaErrorInvalidValue;
    static bool attr_set[64] = {};
    int dev = 0, optin = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if ((e = cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
        return e;
    cudaFuncAttributes fa;
    if ((e = cudaFuncGetAttributes(&fa, k_tc_expand_multi)) != cudaSuccess)
        return e;
    TcExpandMulti m = {};
    m.n = n;
    // one shared-memory layout for all: the largest stacked rank of any projection
    const int natoms = kk > 64 ? 2 : 1;
    const int fixed = (2 + kExpandBStages) * natoms * kAtom + kStaging + 1024;
    const int room = optin - (int)fa.sharedSizeBytes - fixed;
    const int ys = room / kY < kMaxYStages ? room / kY : kMaxYStages;
    if (ys < 2)
        return cudaErrorInvalidConfiguration;
    const int smem = fixed + ys * kY;
    const int G = sm_count();
    int64_t slices = 0;
    for (int i = 0; i < n; ++i) {
        m.a[i] = args[i];
        m.a[i].wait_ns = wait_bound_ns();
        m.a[i].test_stall = test_stall_mode();
        m.a[i].e_natoms = natoms;
        m.a[i].e_ystages = ys;
        slices += (m.a[i].pool.d_out + kBN - 1) / kBN + kTileCost;
    }
    if (G < n)
        return cudaErrorInvalidConfiguration;
    // CTAs in proportion to output slices (plus a per-tile cost: V staged once per
    // tile and the first unit's latency weigh most on projections with few slices),
    // at least one each
    int64_t acc = 0;
    m.cta0[0] = 0;
    for (int i = 0; i < n; ++i) {
        acc += (m.a[i].pool.d_out + kBN - 1) / kBN + kTileCost;
        int c = (int)((acc * G + slices / 2) / slices);
        c = c < m.cta0[i] + 1 ? m.cta0[i] + 1 : c;
        c = c > G - (n - 1 - i) ? G - (n - 1 - i) : c;
        m.cta0[i + 1] = c;
    }
    m.cta0[n] = G;
    if (dev >= 0 && dev < 64 && !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(k_tc_expand_multi, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                      optin - (int)fa.sharedSizeBytes)) != cudaSuccess)
            return e;
        attr_set[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(G);
    cfg.blockDim = dim3(kExpandThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_tc_expand_multi, m);
}

}  // namespace lora

#ifdef LORA_TC_TRACE
extern "C" LORA_API int lora_debug_tc_trace(unsigned long long *host, int n)
{
    return (int)cudaMemcpyFromSymbol(host, lora::g_tc_trace, sizeof(unsigned long long) * (size_t)n);
}
#endif
