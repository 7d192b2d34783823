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
// read, updated and rounded to bf16 once.
//
// Both kernels are persistent (one CTA per SM, 192 threads) and warp
// specialised:
//   warp 0     producer: TMA for the dense operands (x tiles for the shrink, y
//              tiles for the expand; 128-byte swizzle), cp.async for the
//              per-adapter weight tiles (A rows / B rows, placed in the same
//              swizzled K-major layout by hand: adapter offsets live in device
//              memory, so no host-built tensor map can address them);
//   warp 1     one thread issues tcgen05.mma (bf16 x bf16 -> fp32 in TMEM,
//              M = 128) and tracks completion with tcgen05.commit;
//   warps 2-5  epilogue: tcgen05.ld of the accumulator (each warp owns its
//              32-lane quarter of TMEM = 32 rows of the tile).
// Stages hand over through mbarriers; every wait is bounded in time and, if it
// expires, records LORA_ERR_TIMEOUT and winds the CTA down (TMEM is freed).

#include <cuda.h>

#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kTcThreads = 192;
constexpr int kBM = 128;            // rows per tile
constexpr int kBN = 128;            // expand: outputs per unit
constexpr int kBK = 64;             // shrink: d_in per k-block (one 128-byte swizzle atom)
constexpr int kAtom = kBM * 128;    // bytes of a 128-row x 64-column bf16 swizzle atom
constexpr int kShrinkStages = 6;
constexpr int kExpandBStages = 2;
constexpr int kExpandYStages = 3;
constexpr unsigned long long kWaitNs = 2000000000ull;   // 2 s bound on any single wait

// ------------------------------------------------------------------ PTX glue
__device__ __forceinline__ uint32_t smem_u32(const void *p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ unsigned long long now_ns()
{
    unsigned long long t;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void mbar_init(uint64_t *bar, uint32_t count)
{
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t *bar)
{
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t *bar, uint32_t bytes)
{
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)), "r"(bytes) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t *bar, uint32_t parity)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity)
        : "memory");
    return ok != 0;
}

// Bounded wait for the phase with the given parity.  Returns false if the CTA
// is already aborting or the bound expires (then it marks the abort itself).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t *err)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = now_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 255) == 0) {
            if (*abort_flag)
                return false;
            if (now_ns() - t0 > kWaitNs) {
                *abort_flag = 1;
                atomicOr(err, (uint32_t)LORA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// The whole warp waits; all lanes leave together (all succeed or all give up).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *err)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, err));
}

__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%3, %4}], [%2];"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y)
        : "memory");
}

// TMA store of a 2-D box from shared memory (bulk-group completion).
__device__ __forceinline__ void tma_store_2d(const CUtensorMap *map, const void *src, int x, int y)
{
    asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
                 ::"l"(map), "r"(smem_u32(src)), "r"(x), "r"(y)
                 : "memory");
}

__device__ __forceinline__ void bulk_commit() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
// the bulk groups committed by this thread, all but the newest one, have finished reading shared memory
__device__ __forceinline__ void bulk_wait_read_1() { asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_0() { asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory"); }
// ... and have completed
__device__ __forceinline__ void bulk_wait_all() { asm volatile("cp.async.bulk.wait_group 0;" ::: "memory"); }

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t (&w)[4])
{
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr)
                 : "memory");
}

// 16-byte async copy global -> shared; when !pred the destination is zero-filled
// and nothing is read (the source must still be a valid address).
// (No memory clobber: the copy lands asynchronously anyway, and the address
// tables read around it in shared memory must stay free to be scheduled early.)
__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src, bool pred)
{
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src), "r"(pred ? 16 : 0));
}

// Arrive on `bar` once this thread's earlier cp.async copies have landed.
__device__ __forceinline__ void cp_async_arrive(uint64_t *bar)
{
    asm volatile("cp.async.mbarrier.arrive.noinc.shared::cta.b64 [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void fence_async_smem() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tmem_alloc(uint32_t *dst_smem, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(dst_smem)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T, kind::f16 (bf16 inputs, fp32 accumulate).
__device__ __forceinline__ void tc_mma(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                       uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive on `bar` when all tcgen05 operations this thread issued so far complete.
__device__ __forceinline__ void tc_commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
}

// 32 consecutive fp32 columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, float (&v)[32])
{
    uint32_t r[32];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15]),
          "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]),
          "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 32; ++i)
        v[i] = __uint_as_float(r[i]);
}

// Shared-memory matrix descriptor of a K-major operand in 128-byte-swizzled
// atoms (8 rows x 128 bytes; 8-row groups 1024 bytes apart).
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor: bf16 A and B, fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// byte offset of 16-byte chunk c (0..7) of row i inside a 128-byte-swizzle atom
__device__ __forceinline__ uint32_t sw128_off(int i, int c) { return (uint32_t)(i * 128 + ((c ^ (i & 7)) << 4)); }

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

// The adapter stack of one tile: entry i covers ranks [kb[i], kb[i] + r[i]) of
// the stacked axis, reads V columns slot[i] * slot_stride + j and is scaled
// by s[i].  The roles work on different tiles at any moment, so every warp
// keeps its own copy in shared memory.
struct StackSm {
    int n;                                  // entries
    int ktot;                               // stacked rank
    int kpad;                               // stacked rank rounded up to 16 (MMA N or K)
    int a_tma;                              // every entry's A offset is a multiple of d_in
    int r[LORA_MAX_ADS_PER_REQ];
    int kb[LORA_MAX_ADS_PER_REQ];
    int slot[LORA_MAX_ADS_PER_REQ];
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
// e.  Adapters failing validation are left out (and reported when `report`);
// the shrink and the expand leave out the same ones.  The host sends only
// calls whose stacks fit in kKMax ranks; an entry that would not fit is left
// out and reported as a bad segment.
__device__ void warp_build_stack(const TcArgs &p, int item, StackSm &st, bool report)
{
    const int lane = threadIdx.x & 31;
    __syncwarp();                           // this warp's readers of the previous stack are done
    int lo = 0, n = 1;
    if (p.mode == kModeMulti) {
        lo = p.ad_off[item];
        n = min(p.ad_off[item + 1] - lo, p.max_ads);
    }
    int32_t r = 0;
    int64_t ao = 0, bo = 0;
    float sc = 0.f;
    bool ok = false;
    if (lane < n) {
        const int32_t a = p.mode == kModeMulti ? p.ad_id[lo + lane] : p.seg_ad[item];
        ok = adapter_ok(p.pool, a, &r, &ao, &bo);
        if (!ok && report)
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
    const bool fits = ok && incl <= kKMax;
    if (ok && !fits && report)
        atomicOr(p.err, (uint32_t)LORA_ERR_BAD_SEGMENT);
    const unsigned m = __ballot_sync(0xffffffffu, fits);
    const int ktot = (int)__reduce_max_sync(0xffffffffu, fits ? (unsigned)incl : 0u);
    const bool a_tma = __all_sync(0xffffffffu, !fits || (ao % p.pool.d_in) == 0);
    if (fits) {
        const int i = __popc(m & ((1u << lane) - 1u));
        st.r[i] = r;
        st.kb[i] = incl - r;
        st.slot[i] = lane;
        st.s[i] = sc;
        st.aoff[i] = ao;
        st.boff[i] = bo;
    }
    if (lane == 0) {
        st.n = __popc(m);
        st.ktot = ktot;
        st.kpad = (ktot + 15) & ~15;
        st.a_tma = a_tma ? 1 : 0;
    }
    __syncwarp();
}

// ============================================================ shrink kernel
//
// Unit = one tile of <= 128 rows of one item.  D[128 x kpad] = X_tile A_stack^T
// over d_in in 64-column k-blocks; the epilogue writes V rows (fp32).  The A
// rows of a k-block come by TMA in 8-row boxes over the A pool seen as a
// [A_elems / d_in, d_in] matrix (every adapter packed at a multiple of d_in),
// else by cp.async, 16 bytes at a time.
struct ShrinkSmem {
    static constexpr int kA = kKMax * 128;          // up to 128 stacked A rows x 64 columns
    static constexpr int kStage = kAtom + kA;       // x atom + A rows
    static constexpr int kBytes = kShrinkStages * kStage;
};

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_shrink(const __grid_constant__ TcArgs p)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    // 1024-byte alignment for the swizzle atoms
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[kShrinkStages], empty_bar[kShrinkStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ __align__(8) StackSm stk[kTcThreads / 32];
    __shared__ long long arow[kKMax];        // producer, cp.async path: element offset of stacked row j's A row
    __shared__ int vcol[4][kKMax / 4];       // epilogue warp q: V column of stacked columns 4g..4g+3 (-1: none)
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int n_units = p.hdr->n_groups;
    const int G = gridDim.x;
    const int u0 = (int)((int64_t)blockIdx.x * n_units / G), u1 = (int)((int64_t)(blockIdx.x + 1) * n_units / G);
    const int d_in = p.pool.d_in;
    const int n_kb = (d_in + kBK - 1) / kBK;

    if (tid == 0) {
        for (int s = 0; s < kShrinkStages; ++s) {
            mbar_init(&full_bar[s], 33);     // producer lane 0's expect_tx + 32 cp.async arrivals
            mbar_init(&empty_bar[s], 1);     // MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);      // MMA commit
            mbar_init(&acc_empty[b], 4);     // one arrival per epilogue warp
        }
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1)
        tmem_alloc(&tmem_base, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ producer
        StackSm &st = stk[0];
        int it = 0;
        for (int u = u0; u < u1; ++u) {
            const Group gr = p.groups[u];
            warp_build_stack(p, gr.item, st, false);
            const bool use_tma = st.a_tma && p.a_tma;
            const int nbox = st.ktot >> 3;
            int box_row = 0;                 // this lane's 8-row A box: its first row in the pool view
            if (use_tma) {
                if (lane < nbox) {
                    const int e = stack_entry(st, lane * 8);
                    box_row = (int)(st.aoff[e] / d_in) + (lane * 8 - st.kb[e]);
                }
            } else {
                for (int j = lane; j < kKMax; j += 32) {
                    long long o = -1;
                    if (j < st.ktot) {
                        const int e = stack_entry(st, j);
                        o = st.aoff[e] + (long long)(j - st.kb[e]) * d_in;
                    }
                    arow[j] = o;
                }
                __syncwarp();
            }
            const uint32_t tx = (uint32_t)kAtom + (use_tma ? (uint32_t)nbox * 1024u : 0u);
            for (int kb = 0; kb < n_kb; ++kb, ++it) {
                const int s = it % kShrinkStages;
                const uint32_t ph = (it / kShrinkStages) & 1;
                if (!warp_wait(&empty_bar[s], ph ^ 1, &abort_flag, p.err))
                    goto done;
                unsigned char *xs = sm + s * ShrinkSmem::kStage;
                unsigned char *as = xs + kAtom;
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full_bar[s], tx);
                    tma_load_2d(xs, &p.map_x, &full_bar[s], kb * kBK, gr.p0);
                }
                __syncwarp();
                if (use_tma) {
                    if (lane < nbox)
                        tma_load_2d(as + lane * 1024, &p.map_a, &full_bar[s], kb * kBK, box_row);
                } else {
                    // stacked row j, 16-byte chunk c; rows past the stack feed only
                    // accumulator columns that are never stored
                    const int c = lane & 7, col = kb * kBK + c * 8;
                    const bool in = col < d_in;
                    const uint32_t abase = smem_u32(as);
                    for (int j = lane >> 3; j < st.ktot; j += 4)
                        cp_async16(abase + sw128_off(j, c), in ? p.pool.A + arow[j] + col : p.pool.A, in);
                }
                cp_async_arrive(&full_bar[s]);
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        StackSm &st = stk[1];
        int it = 0, t = 0;
        for (int u = u0; u < u1; ++u, ++t) {
            const Group gr = p.groups[u];
            warp_build_stack(p, gr.item, st, false);
            const int kpad = st.kpad;
            const int b = t & 1;
            if (!warp_wait(&acc_empty[b], ((t >> 1) & 1) ^ 1, &abort_flag, p.err))
                goto done;
            tc_fence_after();
            const uint32_t idesc = idesc_bf16(kBM, kpad > 0 ? kpad : 16);
            for (int kb = 0; kb < n_kb; ++kb, ++it) {
                const int s = it % kShrinkStages;
                const uint32_t ph = (it / kShrinkStages) & 1;
                if (!warp_wait(&full_bar[s], ph, &abort_flag, p.err))
                    goto done;
                fence_async_smem();
                tc_fence_after();
                if (lane == 0 && kpad > 0) {
                    const uint32_t xa = smem_u32(sm + s * ShrinkSmem::kStage);
                    const uint32_t aa = xa + kAtom;
#pragma unroll
                    for (int k = 0; k < kBK / 16; ++k)
                        tc_mma(tmem + b * 128, sw128_desc(xa + k * 32), sw128_desc(aa + k * 32), idesc,
                               (kb > 0 || k > 0) ? 1u : 0u);
                }
                __syncwarp();
                if (lane == 0)
                    tc_commit(&empty_bar[s]);
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
            warp_build_stack(p, gr.item, st, warp == 2);
            {
                const int k = lane * 4;
                int c = -1;
                if (k < st.ktot) {
                    const int e = stack_entry(st, k);
                    c = st.slot[e] * p.slot_stride + (k - st.kb[e]);
                }
                vc[lane] = c;
            }
            __syncwarp();
            const int b = t & 1;
            if (!warp_wait(&acc_full[b], (t >> 1) & 1, &abort_flag, p.err))
                goto done;
            tc_fence_after();
            const bool valid = row < gr.cnt;
            float *vrow = p.V + (int64_t)(gr.p0 + (valid ? row : 0)) * p.ldv;
            for (int c0 = 0; c0 < st.kpad; c0 += 32) {
                float v[32];
                tmem_ld32(tmem + b * 128 + ((uint32_t)(q * 32) << 16) + c0, v);
                if (valid) {
#pragma unroll
                    for (int g = 0; g < 8; ++g) {
                        const int col = vc[(c0 >> 2) + g];
                        if (col >= 0)
                            *reinterpret_cast<float4 *>(vrow + col) =
                                make_float4(v[4 * g], v[4 * g + 1], v[4 * g + 2], v[4 * g + 3]);
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
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// ============================================================ expand kernel
//
// Unit = (tile, 128-output slice).  D[128 x 128] = V_tile B_stack[slice]^T over
// the stacked rank (V staged once per tile as bf16 with the scales folded in);
// the epilogue adds D to the y tile (TMA-loaded) in shared memory and a TMA
// store writes the tile back (a ragged tile: plain coalesced stores of its rows).
struct ExpandSmem {
    static constexpr int kV = 2 * kAtom;                 // V: 128 rows x up to 128 ranks
    static constexpr int kB = 2 * kAtom;                 // B: 128 outputs x up to 128 ranks
    static constexpr int kY = kBM * kBN * 2;             // y: 128 rows x 128 outputs (two 64-column atoms)
    static constexpr int kOffB = kV;
    static constexpr int kOffY = kOffB + kExpandBStages * kB;
    static constexpr int kBytes = kOffY + kExpandYStages * kY;
};

__global__ void __launch_bounds__(kTcThreads, 1) k_tc_expand(const __grid_constant__ TcArgs p)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t b_full[kExpandBStages], b_empty[kExpandBStages];
    __shared__ __align__(8) uint64_t y_full[kExpandYStages], y_empty[kExpandYStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ __align__(8) uint64_t v_full, v_empty, ep_bar;
    __shared__ __align__(8) StackSm stk[kTcThreads / 32];
    __shared__ long long cb_off[kKMax / 8];  // producer: B element offset of stacked 8-rank chunk c in output row 0
    __shared__ int cb_r[kKMax / 8];          // its row stride (the adapter's rank); 0 = padding chunk
    __shared__ int vsrc[4][kKMax / 8];       // epilogue warp q: V column of stacked chunk c (-1: zero)
    __shared__ float vsc[4][kKMax / 8];      // and its adapter's scale
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int d_out = p.pool.d_out;
    const int n_ns = (d_out + kBN - 1) / kBN;           // output slices
    const int64_t n_units = (int64_t)p.hdr->n_groups * n_ns;
    const int G = gridDim.x;
    const int64_t u0 = (int64_t)blockIdx.x * n_units / G, u1 = (int64_t)(blockIdx.x + 1) * n_units / G;

    if (tid == 0) {
        for (int s = 0; s < kExpandBStages; ++s) {
            mbar_init(&b_full[s], 32);       // 32 cp.async arrivals
            mbar_init(&b_empty[s], 1);       // MMA commit
        }
        for (int s = 0; s < kExpandYStages; ++s) {
            mbar_init(&y_full[s], 1);        // expect_tx
            mbar_init(&y_empty[s], 1);       // the epilogue thread that stored the tile
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);
            mbar_init(&acc_empty[b], 4);
        }
        mbar_init(&v_full, 4);               // epilogue warps, after staging V
        mbar_init(&v_empty, 1);              // MMA commit after a tile's last unit
        mbar_init(&ep_bar, 4);               // the epilogue warps meet (y tile complete in shared memory)
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1)
        tmem_alloc(&tmem_base, 256);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;

    if (warp == 0) {
        // ------------------------------------------------ producer: y tiles (TMA), B slices (cp.async)
        StackSm &st = stk[0];
        int it = 0;
        int64_t prev_tile = -1;
        int nch = 0, o_l = 0, c_l = 0, dq = 0, dr = 0;
        int p0 = 0;
        for (int64_t u = u0; u < u1; ++u, ++it) {
            const int tile = (int)(u / n_ns), ns = (int)(u - (int64_t)tile * n_ns);
            if (tile != prev_tile) {
                const Group gr = p.groups[tile];
                p0 = gr.p0;
                warp_build_stack(p, gr.item, st, false);
                prev_tile = tile;
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
            const int o0 = ns * kBN;
            const int sy = it % kExpandYStages;
            if (!warp_wait(&y_empty[sy], ((it / kExpandYStages) & 1) ^ 1, &abort_flag, p.err))
                goto done;
            unsigned char *ys = sm + ExpandSmem::kOffY + sy * ExpandSmem::kY;
            if (lane == 0) {
                mbar_arrive_expect_tx(&y_full[sy], ExpandSmem::kY);
                tma_load_2d(ys, &p.map_y, &y_full[sy], o0, p0);
                tma_load_2d(ys + kAtom, &p.map_y, &y_full[sy], o0 + 64, p0);
            }
            const int sb = it % kExpandBStages;
            if (!warp_wait(&b_empty[sb], ((it / kExpandBStages) & 1) ^ 1, &abort_flag, p.err))
                goto done;
            const uint32_t bbase = smem_u32(sm + ExpandSmem::kOffB + sb * ExpandSmem::kB);
            // output o of the slice, 16-byte chunk c of the stacked rank axis (atom c / 8);
            // padding chunks and outputs past d_out are zero-filled
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
            cp_async_arrive(&b_full[sb]);
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        StackSm &st = stk[1];
        int it = 0, vt = 0;
        int64_t prev_tile = -1;
        for (int64_t u = u0; u < u1; ++u, ++it) {
            const int tile = (int)(u / n_ns);
            if (tile != prev_tile) {
                warp_build_stack(p, p.groups[tile].item, st, false);
                prev_tile = tile;
                if (!warp_wait(&v_full, vt & 1, &abort_flag, p.err))
                    goto done;
                ++vt;
            }
            const int b = it & 1;
            if (!warp_wait(&acc_empty[b], ((it >> 1) & 1) ^ 1, &abort_flag, p.err))
                goto done;
            const int sb = it % kExpandBStages;
            if (!warp_wait(&b_full[sb], (it / kExpandBStages) & 1, &abort_flag, p.err))
                goto done;
            fence_async_smem();
            tc_fence_after();
            if (lane == 0) {
                const uint32_t va = smem_u32(sm);
                const uint32_t ba = smem_u32(sm + ExpandSmem::kOffB + sb * ExpandSmem::kB);
                const uint32_t idesc = idesc_bf16(kBM, kBN);
                for (int k = 0; k < st.kpad / 16; ++k) {
                    const uint32_t off = (k >> 2) * kAtom + (k & 3) * 32;
                    tc_mma(tmem + b * 128, sw128_desc(va + off), sw128_desc(ba + off), idesc, k > 0 ? 1u : 0u);
                }
                tc_commit(&b_empty[sb]);
                tc_commit(&acc_full[b]);
                const bool last_of_tile = u + 1 >= u1 || (int)((u + 1) / n_ns) != tile;
                if (last_of_tile)
                    tc_commit(&v_empty);
            }
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue: V staging, y += D, store
        const int q = warp & 3;
        const int row = q * 32 + lane;
        const int et = tid - 64;                // 0..127 over the epilogue warps
        StackSm &st = stk[warp];
        int it = 0, vt = 0, pending = -1;
        uint32_t ep_uses = 0;
        int64_t prev_tile = -1;
        Group gr = {0, 0, 0, 0};
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
                        c = st.slot[e] * p.slot_stride + (k - st.kb[e]);
                        sc = st.s[e];
                    }
                    vsrc[q][lane] = c;
                    vsc[q][lane] = sc;
                }
                __syncwarp();
                // wait until the MMAs of the previous tile stopped reading V
                if (vt > 0 && !warp_wait(&v_empty, (vt - 1) & 1, &abort_flag, p.err))
                    goto done;
                // V[row][stacked k] = bf16(s_e * V_e[row][k - kb_e]), zero outside the tile's rows and the stack
                const bool valid = et < gr.cnt;
                const float *vrow = p.V + (int64_t)(gr.p0 + (valid ? et : 0)) * p.ldv;
                const uint32_t vbase = smem_u32(sm);
                for (int c = 0; c < st.kpad / 8; ++c) {
                    const int col = vsrc[q][c];
                    uint32_t w[4] = {0u, 0u, 0u, 0u};
                    if (valid && col >= 0) {
                        const float sc = vsc[q][c];
                        const float4 a = *reinterpret_cast<const float4 *>(vrow + col);
                        const float4 bq = *reinterpret_cast<const float4 *>(vrow + col + 4);
                        const __nv_bfloat162 h0 = __floats2bfloat162_rn(sc * a.x, sc * a.y);
                        const __nv_bfloat162 h1 = __floats2bfloat162_rn(sc * a.z, sc * a.w);
                        const __nv_bfloat162 h2 = __floats2bfloat162_rn(sc * bq.x, sc * bq.y);
                        const __nv_bfloat162 h3 = __floats2bfloat162_rn(sc * bq.z, sc * bq.w);
                        w[0] = *reinterpret_cast<const uint32_t *>(&h0);
                        w[1] = *reinterpret_cast<const uint32_t *>(&h1);
                        w[2] = *reinterpret_cast<const uint32_t *>(&h2);
                        w[3] = *reinterpret_cast<const uint32_t *>(&h3);
                    }
                    st_shared_v4(vbase + (c >> 3) * kAtom + sw128_off(et, c & 7), w[0], w[1], w[2], w[3]);
                }
                fence_async_smem();
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&v_full);
                ++vt;
            }
            const int b = it & 1;
            const int sy = it % kExpandYStages;
            if (!warp_wait(&acc_full[b], (it >> 1) & 1, &abort_flag, p.err))
                goto done;
            if (!warp_wait(&y_full[sy], (it / kExpandYStages) & 1, &abort_flag, p.err))
                goto done;
            tc_fence_after();
            const int o0 = ns * kBN;
            unsigned char *ys = sm + ExpandSmem::kOffY + sy * ExpandSmem::kY;
            const uint32_t ysa = smem_u32(ys);
#pragma unroll 1
            for (int c0 = 0; c0 < kBN; c0 += 32) {
                float d[32];
                tmem_ld32(tmem + b * 128 + ((uint32_t)(q * 32) << 16) + c0, d);
                if (st.kpad == 0) {   // no valid adapter: no MMA ran, y is stored unchanged
#pragma unroll
                    for (int i = 0; i < 32; ++i)
                        d[i] = 0.f;
                }
                // four 16-byte chunks of this row's y: atom c0 / 64, chunks (c0 % 64) / 8 ..
                const uint32_t atom = ysa + (c0 >> 6) * kAtom;
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                    const uint32_t addr = atom + sw128_off(row, ((c0 & 63) >> 3) + h);
                    uint32_t yw[4];
                    ld_shared_v4(addr, yw);
                    uint32_t ow[4];
#pragma unroll
                    for (int e = 0; e < 4; ++e) {
                        const float2 yf = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162 *>(&yw[e]));
                        const __nv_bfloat162 r2 =
                            __floats2bfloat162_rn(yf.x + d[h * 8 + 2 * e], yf.y + d[h * 8 + 2 * e + 1]);
                        ow[e] = *reinterpret_cast<const uint32_t *>(&r2);
                    }
                    st_shared_v4(addr, ow[0], ow[1], ow[2], ow[3]);
                }
            }
            tc_fence_before();
            fence_async_smem();                 // this thread's y writes, before the TMA store reads them
            __syncwarp();
            if (lane == 0) {
                mbar_arrive(&acc_empty[b]);
                mbar_arrive(&ep_bar);
            }
            if (!warp_wait(&ep_bar, ep_uses & 1, &abort_flag, p.err))
                goto done;
            ++ep_uses;
            if (gr.cnt == kBM) {
                // full tile: one thread stores it; the stage is released once the store has read it
                if (et == 0) {
                    tma_store_2d(&p.map_y, ys, o0, gr.p0);
                    tma_store_2d(&p.map_y, ys + kAtom, o0 + 64, gr.p0);
                    bulk_commit();
                    bulk_wait_read_1();
                    if (pending >= 0)
                        mbar_arrive(&y_empty[pending]);
                    pending = sy;
                }
            } else {
                // ragged tile: the valid rows, 16 bytes per thread, 256 contiguous bytes per row
                for (int idx = et; idx < gr.cnt * 16; idx += 128) {
                    const int r = idx >> 4, ch = idx & 15;
                    const int o = o0 + ch * 8;
                    if (o < d_out) {
                        uint32_t w[4];
                        ld_shared_v4(ysa + (ch >> 3) * kAtom + sw128_off(r, ch & 7), w);
                        *reinterpret_cast<uint4 *>(p.Y + (int64_t)(gr.p0 + r) * p.ldy + o) =
                            make_uint4(w[0], w[1], w[2], w[3]);
                    }
                }
                __syncwarp();
                if (lane == 0)
                    mbar_arrive(&ep_bar);
                if (!warp_wait(&ep_bar, ep_uses & 1, &abort_flag, p.err))
                    goto done;
                ++ep_uses;
                if (et == 0) {
                    bulk_wait_read_0();
                    if (pending >= 0)
                        mbar_arrive(&y_empty[pending]);
                    pending = -1;
                    mbar_arrive(&y_empty[sy]);
                }
            }
        }
    }
done:
    if (tid == 64)
        bulk_wait_all();                        // the last TMA stores have landed
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 256);
    }
}

// -------------------------------------------------------------- host side
typedef CUresult (*EncodeTiledFn)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                  const cuuint64_t *, const cuuint32_t *, const cuuint32_t *, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn()
{
    static EncodeTiledFn fn = [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
            q != cudaDriverEntryPointSuccess)
            p = nullptr;
        return reinterpret_cast<EncodeTiledFn>(p);
    }();
    return fn;
}

// Row-major bf16 matrix [rows, cols] with leading dimension ld: boxes of 64
// columns x 128 rows, 128-byte swizzle, zero fill outside the matrix.
bool encode_rows(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, 128};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

// attr_set: this kernel's per-device "shared-memory opt-in done" flags (one
// array per kernel: the kernels share a type, so they cannot share the flags)
cudaError_t launch_tc(void (*kernel)(TcArgs), bool *attr_set, const TcArgs &a, int smem, int units_hint,
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
    int grid = sm_count();
    if (units_hint > 0 && units_hint < grid)
        grid = units_hint;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kTcThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    return cudaLaunchKernelEx(&cfg, kernel, a);
}

}  // namespace

bool tc_encode_a(TcArgs &a, const void *A, int64_t A_elems, int32_t d_in)
{
    // the A pool as a [A_elems / d_in, d_in] matrix, boxes of 64 columns x 8 rows
    a.a_tma = 0;
    const int64_t rows = A_elems / d_in;
    if (rows < 1 || rows > 0x7fffffffLL)
        return false;
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)d_in, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)d_in * 2};
    const cuuint32_t box[2] = {64, 8};
    const cuuint32_t estr[2] = {1, 1};
    if (fn(&a.map_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(A), dims, strides, box, estr,
           CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
           CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
        return false;
    a.a_tma = 1;
    return true;
}

bool tc_encode_x(TcArgs &a, const void *X, int32_t N, int32_t d_in, int64_t ldx)
{
    return encode_rows(&a.map_x, X, N, d_in, ldx);
}

bool tc_encode_y(TcArgs &a, const void *Y, int32_t N, int32_t d_out, int64_t ldy)
{
    return encode_rows(&a.map_y, Y, N, d_out, ldy);
}

cudaError_t launch_tc_shrink(const TcArgs &a, int max_tiles, cudaStream_t s)
{
    static bool attr_set[64] = {};
    return launch_tc(k_tc_shrink, attr_set, a, ShrinkSmem::kBytes + 1024, max_tiles, s);
}

cudaError_t launch_tc_expand(const TcArgs &a, cudaStream_t s)
{
    static bool attr_set[64] = {};
    return launch_tc(k_tc_expand, attr_set, a, ExpandSmem::kBytes + 1024, 0, s);
}

}  // namespace lora

