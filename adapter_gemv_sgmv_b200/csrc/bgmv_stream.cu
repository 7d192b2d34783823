// Decode BGMV as one persistent launch that streams every touched adapter's
// weights through shared memory with bulk copies.
//
// The operation ("Serving several LoRAs, ControlNet and IP-Adapter", section
// "LoRA: merged or alongside", and exercise 2's answer): y[n] += s B[a] A[a] x[n]
// for a batch whose tokens carry their own adapter ids, the tokens grouped by
// adapter so that each distinct adapter's A and B cross HBM once (the segmented
// gather matrix-vector product of "Punica: multi-tenant LoRA serving",
// contribution 1).
//
// Work layout on B200 (one CTA per SM, 1 producer warp + 8 consumer warps):
// * every CTA rebuilds the grouping in shared memory from the ids: a stable
//   counting sort by adapter gives `perm`; an item is a run of <= 16 tokens of
//   one adapter (one m16 MMA tile);
// * the work is cut into units of near-equal bytes.  A shrink unit is one item's
//   16 rank rows (8 for a rank ending in 8) over one part of d_in, and writes its
//   partial V = X_tile A_rows^T into a plane of the workspace; an expand unit is
//   one item's slice of <= 512 outputs whose B rows weigh <= 16 KB, and adds
//   s (sum of the V planes) B_slice^T to the item's y rows.  Both lists are cut
//   into one contiguous, cost-balanced range per CTA, so mixed ranks (8..128)
//   spread evenly without padding any adapter to the largest rank;
// * the producer warp streams each unit's operands into a ring of shared-memory
//   slots with `cp.async.bulk` (A rows, B slice: one copy per row / slice; x and
//   y rows: one copy per token), completing on the slot's mbarrier.  Adapter
//   weights are immutable inputs, so the first slots' weights are requested
//   before `griddepcontrol.wait`, while the previous kernel on the stream is
//   still running; x and y rows only after it;
// * the consumer warps run warp-level tensor-core MMAs (m16n8k16, bf16 in,
//   fp32 accumulate) on the slots: inside each 32-wide block of the reduction
//   the k order is permuted identically for both operands, so every operand
//   fragment is one 16-byte shared-memory read.  V is summed over its planes in
//   a fixed order and split into bf16 high and low parts, so the expand sees it
//   to ~16 significant bits;
// * a CTA runs its shrink units first, then its expand units.  Each CTA
//   publishes how many shrink units it finished (a per-CTA counter tagged with
//   the call's epoch, in the workspace header); an expand unit waits, with a
//   bounded spin, until the CTAs that own its item's shrink units have passed
//   them.  All CTAs are resident at once (the grid never exceeds what fits), and
//   no CTA waits during its shrink units, so every such wait ends.
//
// Determinism: every V plane element is written by one unit, the planes are
// summed in a fixed order and the warps' partials are reduced in a fixed order.

#include <mutex>

#include "lora_internal.cuh"
#include "tc_ptx.cuh"

namespace lora {
namespace {

#ifdef LORA_STREAM_STAMPS
// Development aid: %globaltimer stamps of each CTA's phases (last call), and a
// per-chunk trace of the first CTAs.
__device__ unsigned long long g_stream_stamps[kMaxStreamCtas * 16];
__device__ unsigned long long g_stream_trace[64 * 256 * 4];
#define STRACE(i, e)                                                                        \
    do {                                                                                    \
        if (blockIdx.x < 64 && (i) < 256)                                                   \
            g_stream_trace[((blockIdx.x * 256) + (i)) * 4 + (e)] = now_ns();                \
    } while (0)
#define SSTAMP(i) g_stream_stamps[blockIdx.x * 16 + (i)] = now_ns()
#define SSTAMP_ADD(i, v) g_stream_stamps[blockIdx.x * 16 + (i)] += (v)
#define SSTAMP_SET(i, v) g_stream_stamps[blockIdx.x * 16 + (i)] = (v)
#else
#define STRACE(i, e) ((void)0)
#define SSTAMP(i) ((void)0)
#define SSTAMP_ADD(i, v) ((void)0)
#define SSTAMP_SET(i, v) ((void)0)
#endif

constexpr int kSCons = 8;                        // consumer warps
constexpr int kSThreads = 32 * (kSCons + 1);     // + one producer warp
constexpr int kSConsThreads = 32 * kSCons;
constexpr int kKC = 512;                         // d_in columns per shrink chunk
// A shrink slot: the 16 A rows as two dense [16][256]-column halves (what two 2-D
// TMA boxes write), then 16 x rows at a padded stride (64 mod 128 bytes).
constexpr int kAHalf = 16 * 256 * 2;             // bytes of one half
constexpr int kXOff = 2 * kAHalf;                // x rows
constexpr int kXRowB = 2 * kKC + 64;
constexpr int kSlotShrink = kXOff + 16 * kXRowB;
constexpr int kSlotExpand = 32768 + 16 * (2 * 512 + 16);
constexpr int kSlot = kSlotShrink > kSlotExpand ? kSlotShrink : kSlotExpand;
constexpr int kEB = 32768;                       // expand: bytes of the B slice part of a slot
constexpr int kOCMax = 512;                      // expand: most outputs per unit
constexpr int kSVS = 160;                        // bf16 row stride of V in shared memory (320 B = 64 mod 128)
constexpr int kUnitsPerCta = 16;                 // shrink units per CTA the d_in split aims at

static_assert(kEB + 16 * (2 * kOCMax + 16) <= kSlot, "expand slot fits");
static_assert(kKC == 512, "a shrink chunk is two 256-column halves");

// byte offset of A element (row j, column c) in a shrink slot
__device__ __forceinline__ uint32_t a_off(int j, int c) { return (uint32_t)((c >> 8) * kAHalf + j * 512 + (c & 255) * 2); }

__device__ __forceinline__ int rank_tiles(int r) { return (r + 15) >> 4; }

// Outputs per expand unit for rank r: a multiple of 16 (the MMA tiles), B slice
// <= 32 KB, at most 512 outputs.
__host__ __device__ __forceinline__ int out_chunk(int r)
{
    const int oc = (kEB / 2 / r) & ~15;
    return oc < kOCMax ? oc : kOCMax;
}

// ------------------------------------------------------------------ device glue
__device__ __forceinline__ void mma16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                         uint32_t b0, uint32_t b1)
{
    asm volatile("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
                 "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
                 : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
                 : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

// One-dimensional bulk copy global -> shared, completing on `bar`; both addresses
// 16-byte aligned, bytes a multiple of 16.
__device__ __forceinline__ void bulk_g2s(uint32_t dst, const void *src, uint32_t bytes, uint64_t *bar,
                                         uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;"
        ::"r"(dst), "l"(src), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
        : "memory");
}

__device__ __forceinline__ void prefetch_l2(const void *p, uint32_t bytes)
{
    asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;" ::"l"(p), "r"(bytes) : "memory");
}

__device__ __forceinline__ uint4 lds128(uint32_t a)
{
    uint4 r;
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w) : "r"(a));
    return r;
}

__device__ __forceinline__ uint2 lds64(uint32_t a)
{
    uint2 r;
    asm volatile("ld.shared.v2.u32 {%0,%1}, [%2];" : "=r"(r.x), "=r"(r.y) : "r"(a));
    return r;
}

__device__ __forceinline__ uint32_t lds32(uint32_t a)
{
    uint32_t r;
    asm volatile("ld.shared.u32 %0, [%1];" : "=r"(r) : "r"(a));
    return r;
}

__device__ __forceinline__ void cons_sync() { asm volatile("bar.sync 1, %0;" ::"n"(kSConsThreads) : "memory"); }

__device__ __forceinline__ unsigned long long ld_acquire_u64(const unsigned long long *p)
{
    unsigned long long v;
    asm volatile("ld.acquire.gpu.global.u64 %0, [%1];" : "=l"(v) : "l"(p) : "memory");
    return v;
}

__device__ __forceinline__ void st_release_u64(unsigned long long *p, unsigned long long v)
{
    asm volatile("st.release.gpu.global.u64 [%0], %1;" ::"l"(p), "l"(v) : "memory");
}

// mbarrier test that suspends the thread (up to `hint_ns`) until the phase
// completes, instead of spinning: waiting warps leave the issue slots to the
// warps doing work.
__device__ __forceinline__ bool mbar_wait_hint(uint64_t *bar, uint32_t parity, uint32_t hint_ns)
{
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\tselp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(smem_u32(bar)), "r"(parity), "r"(hint_ns)
        : "memory");
    return ok != 0;
}

constexpr uint32_t kSuspendNs = 200000;          // longest suspension of one test (0.2 ms)

// A consumer warp hands its slot back.  Relaxed: the warp's reads of the slot have
// completed (their values were used), and nothing else needs ordering here -- a
// release would make the arrive wait for the warp's global stores of y.
__device__ __forceinline__ void slot_release(uint64_t *bar)
{
#ifdef LORA_STREAM_ARRIVE_RELEASE
    mbar_arrive(bar);
#else
    asm volatile("mbarrier.arrive.relaxed.cta.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
#endif
}

// Bounded wait on an mbarrier phase; false once the CTA aborts or `limit_ns`
// passes (then this thread marks the abort and the timeout bit).
__device__ __forceinline__ bool wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *err,
                                           unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = now_ns();
    for (;;) {
        if (mbar_wait_hint(bar, parity, kSuspendNs))
            return true;
        if (*abort_flag)
            return false;
        if (now_ns() - t0 > limit_ns) {
            *abort_flag = 1;
            atomicOr(err, (uint32_t)LORA_ERR_TIMEOUT);
            return false;
        }
    }
}

__device__ __forceinline__ bool warp_wait_phase(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                                uint32_t *err, unsigned long long limit_ns)
{
    return __all_sync(0xffffffffu, wait_phase(bar, parity, abort_flag, err, limit_ns));
}

// ------------------------------------------------------------ shared memory
struct StreamSmem {
    size_t bars, ring, it_tok0, it_cr, it_aoff, it_boff, sp, ep, scp, ecp, perm, first_s, first_e, vh, vl, red,
        total;
    // grouping scratch, inside the ring (dead before the first copy lands)
    size_t t_ids, t_cnt, t_mr, t_ma, t_mb, t_end, t_end_meta;
    int max_items;
};

__host__ __device__ inline size_t al128(size_t x) { return (x + 127) & ~(size_t)127; }

__host__ __device__ inline StreamSmem stream_layout(int N, int n_ad, int G, int ns)
{
    StreamSmem L;
    const int64_t mi = (int64_t)(N < n_ad ? N : n_ad) + N / kFT + 1;
    L.max_items = (int)mi;
    size_t o = 0;
    L.bars = o;
    o = al128(o + 16 * 2 * (size_t)ns);
    L.ring = o;
    o = al128(o + (size_t)kSlot * ns);
    L.it_tok0 = o;
    o = al128(o + 4 * (size_t)mi);
    L.it_cr = o;
    o = al128(o + 4 * (size_t)mi);
    L.it_aoff = o;
    o = al128(o + 8 * (size_t)mi);
    L.it_boff = o;
    o = al128(o + 8 * (size_t)mi);
    L.sp = o;
    o = al128(o + 4 * (size_t)(mi + 1));
    L.ep = o;
    o = al128(o + 4 * (size_t)(mi + 1));
    L.scp = o;
    o = al128(o + 4 * (size_t)(mi + 1));
    L.ecp = o;
    o = al128(o + 4 * (size_t)(mi + 1));
    L.perm = o;
    o = al128(o + 4 * (size_t)N);
    L.first_s = o;
    o = al128(o + 4 * (size_t)(G + 1));
    L.first_e = o;
    o = al128(o + 4 * (size_t)(G + 1));
    L.vh = o;
    o = al128(o + 2 * 16 * (size_t)kSVS);
    L.vl = o;
    o = al128(o + 2 * 16 * (size_t)kSVS);
    L.red = o;
    o = al128(o + 4 * (size_t)kSCons * 256);
    L.total = o;
    // scratch of the grouping, aliased onto the ring
    size_t t = L.ring;
    L.t_ids = t;
    t = al128(t + 4 * (size_t)N);
    L.t_cnt = t;
    t = al128(t + 4 * ((size_t)n_ad + 1));
    L.t_end = t;
    // every adapter's checked rank and offsets, when they fit beside the ids
    L.t_mr = t;
    t = al128(t + 4 * (size_t)n_ad);
    L.t_ma = t;
    t = al128(t + 8 * (size_t)n_ad);
    L.t_mb = t;
    t = al128(t + 8 * (size_t)n_ad);
    L.t_end_meta = t;
    return L;
}

// ------------------------------------------------------------ unit sequences
struct Plan {
    const int32_t *tok0, *cr, *sp, *ep;   // shared memory
    const int64_t *aoff, *boff;
    int n_items, S, KP, d_in, d_out;
};

__device__ __forceinline__ int cr_cnt(int cr) { return cr & 0xff; }
__device__ __forceinline__ int cr_rank(int cr) { return cr >> 8; }

// Last item k with pre[k] <= u (pre is non-decreasing, pre[0] = 0).
__device__ __forceinline__ int item_of(const int32_t *pre, int n, int u)
{
    int lo = 0, hi = n;
    while (hi - lo > 1) {
        const int mid = (lo + hi) >> 1;
        if (pre[mid] <= u)
            lo = mid;
        else
            hi = mid;
    }
    return lo;
}

// One chunk of a CTA's sequence: shrink chunks of its shrink units, then one
// chunk per expand unit.
struct Chunk {
    int expand;      // 0 shrink, 1 expand
    int k;           // item
    int unit;        // global unit index (shrink or expand list)
    // shrink
    int row0, rows;  // rank rows of the unit
    int part;        // d_in part (V plane)
    int k0, kc;      // columns of this chunk
    int first, last; // first / last chunk of the unit
    // expand
    int o0, ocs;     // outputs of the unit
    int new_item;    // first expand chunk of this item in this CTA
};

struct Seq {
    int su, su_end, eu, eu_end;
    int k, c, nch;
    int prev_ek;
};

__device__ __forceinline__ void seq_init(Seq &q, const Plan &P, int s0, int s1, int e0, int e1)
{
    q.su = s0;
    q.su_end = s1;
    q.eu = e0;
    q.eu_end = e1;
    q.k = -1;
    q.c = 0;
    q.nch = 0;
    q.prev_ek = -1;
}

__device__ __forceinline__ int seq_total_chunks(const Plan &P, int s0, int s1, int e0, int e1)
{
    // every shrink unit of this call has the same chunk count, except the last part of d_in
    int n = e1 - e0;
    for (int u = s0; u < s1;) {
        const int k = item_of(P.sp, P.n_items, u);
        const int end = min(s1, P.sp[k + 1]);
        for (; u < end; ++u) {
            const int part = (u - P.sp[k]) % P.S;
            const int k0 = part * P.KP;
            const int k1 = min(P.d_in, k0 + P.KP);
            n += (k1 - k0 + kKC - 1) / kKC;
        }
    }
    return n;
}

// Next chunk; false at the end of the sequence.
__device__ __forceinline__ bool seq_next(Seq &q, const Plan &P, Chunk &ch)
{
    if (q.su < q.su_end) {
        if (q.k < 0 || P.sp[q.k + 1] <= q.su)
            q.k = item_of(P.sp, P.n_items, q.su);
        const int k = q.k;
        const int local = q.su - P.sp[k];
        const int tile = local / P.S, part = local - tile * P.S;
        const int r = cr_rank(P.cr[k]);
        const int k0u = part * P.KP, k1u = min(P.d_in, k0u + P.KP);
        if (q.c == 0)
            q.nch = (k1u - k0u + kKC - 1) / kKC;
        ch.expand = 0;
        ch.k = k;
        ch.unit = q.su;
        ch.row0 = tile * 16;
        ch.rows = min(16, r - tile * 16);
        ch.part = part;
        ch.k0 = k0u + q.c * kKC;
        ch.kc = min(kKC, k1u - ch.k0);
        ch.first = q.c == 0;
        ch.last = q.c == q.nch - 1;
        if (++q.c == q.nch) {
            q.c = 0;
            ++q.su;
        }
        return true;
    }
    if (q.eu < q.eu_end) {
        if (q.k < 0 || P.ep[q.k + 1] <= q.eu || P.ep[q.k] > q.eu)
            q.k = item_of(P.ep, P.n_items, q.eu);
        const int k = q.k;
        const int r = cr_rank(P.cr[k]);
        const int oc = out_chunk(r);
        ch.expand = 1;
        ch.k = k;
        ch.unit = q.eu;
        ch.o0 = (q.eu - P.ep[k]) * oc;
        ch.ocs = min(oc, P.d_out - ch.o0);
        ch.new_item = k != q.prev_ek;
        q.prev_ek = k;
        ++q.eu;
        return true;
    }
    return false;
}

// ------------------------------------------------------------ block helpers
// Exclusive scan of four values per thread over the block (kSThreads threads);
// tmp holds 4 * (warps + 1) ints.
__device__ __forceinline__ int4 block_excl_scan4(int4 v, int *tmp, int4 *total)
{
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    constexpr int W = kSThreads / 32;
    int4 incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        const int a = __shfl_up_sync(0xffffffffu, incl.x, off), b = __shfl_up_sync(0xffffffffu, incl.y, off);
        const int c = __shfl_up_sync(0xffffffffu, incl.z, off), d = __shfl_up_sync(0xffffffffu, incl.w, off);
        if (lane >= off) {
            incl.x += a;
            incl.y += b;
            incl.z += c;
            incl.w += d;
        }
    }
    if (lane == 31) {
        tmp[4 * warp] = incl.x;
        tmp[4 * warp + 1] = incl.y;
        tmp[4 * warp + 2] = incl.z;
        tmp[4 * warp + 3] = incl.w;
    }
    __syncthreads();
    if (threadIdx.x < 4) {
        int run = 0;
        for (int w = 0; w < W; ++w) {
            const int t = tmp[4 * w + threadIdx.x];
            tmp[4 * w + threadIdx.x] = run;
            run += t;
        }
        tmp[4 * W + threadIdx.x] = run;
    }
    __syncthreads();
    const int4 r = make_int4(tmp[4 * warp] + incl.x - v.x, tmp[4 * warp + 1] + incl.y - v.y,
                             tmp[4 * warp + 2] + incl.z - v.z, tmp[4 * warp + 3] + incl.w - v.w);
    *total = make_int4(tmp[4 * W], tmp[4 * W + 1], tmp[4 * W + 2], tmp[4 * W + 3]);
    __syncthreads();
    return r;
}

// First unit of each CTA: CTA c starts at the first unit whose cost position is
// at least C * c / G (units of one item all cost the same).
__device__ void cut_ranges(const int32_t *pre, const int32_t *cpre, int n_items, int G, int32_t *first, int tid,
                           int nthreads)
{
    const long long C = cpre[n_items];
    for (int c = tid; c <= G; c += nthreads) {
        if (c == G || n_items == 0) {
            first[c] = pre[n_items];
            continue;
        }
        const long long pos = C * c / G;
        // last item with cpre[k] <= pos
        int lo = 0, hi = n_items;
        while (hi - lo > 1) {
            const int mid = (lo + hi) >> 1;
            if (cpre[mid] <= pos)
                lo = mid;
            else
                hi = mid;
        }
        const int k = lo;
        const int nu = pre[k + 1] - pre[k];
        const long long ic = cpre[k + 1] - cpre[k];
        int q = 0;
        if (nu > 0 && ic > 0) {
            const long long uc = ic / nu;       // exact: the item's cost is nu * unit cost
            q = (int)((pos - cpre[k] + uc - 1) / uc);
            if (q > nu)
                q = nu;
        }
        first[c] = pre[k] + q;
    }
}

// ------------------------------------------------------------ consumer compute
// Shrink chunk: warp cw takes columns [64 cw, 64 cw + 64) of the chunk.  The
// MMAs run for the whole warp or not at all (warp-uniform conditions only); a
// thread whose 8 columns lie past the chunk's end feeds zeros instead.
__device__ __forceinline__ void shrink_chunk(uint32_t slot, int cw, int g, int qd, int kc, int rows,
                                             float (&acc)[2][2][4])
{
    const uint4 z = make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int kb = 0; kb < 2; ++kb) {
        const int cb = cw * 64 + kb * 32;
        if (cb < kc) {
            const int col = cb + qd * 8;
            const bool in = col < kc;
            const uint4 xa = in ? lds128(slot + kXOff + g * kXRowB + col * 2) : z;
            const uint4 xb = in ? lds128(slot + kXOff + (8 + g) * kXRowB + col * 2) : z;
            const uint4 a0 = in ? lds128(slot + a_off(g, col)) : z;
            // four accumulators (two rank tiles x two k16 halves): independent chains
            mma16816(acc[0][0], xa.x, xb.x, xa.y, xb.y, a0.x, a0.y);
            mma16816(acc[0][1], xa.z, xb.z, xa.w, xb.w, a0.z, a0.w);
            if (rows > 8) {
                const uint4 a1 = in ? lds128(slot + a_off(8 + g, col)) : z;
                mma16816(acc[1][0], xa.x, xb.x, xa.y, xb.y, a1.x, a1.y);
                mma16816(acc[1][1], xa.z, xb.z, xa.w, xb.w, a1.z, a1.w);
            }
        }
    }
}

// Expand chunk: D[16 outputs x 8 tokens] = B_slice[16 x r] V^T per m16n8k16, the
// outputs as the MMA's M so that one MMA covers 256 weights.  Warp cw takes the
// 16-output tiles cw, cw + 8, ...; an item of more than 8 tokens takes a second
// token tile.  Inside each 32-rank block the k order is permuted identically for
// B (rows g, g + 8 of the tile) and V (token g's row), so every fragment is a
// 16-byte shared-memory read (8 bytes for ranks <= 16, one k16 step).  The high
// and low parts of V and the two k16 halves accumulate separately (four
// independent chains) and are summed in fp32 before the one rounding of y.
// vf: V fragments of this item, vf[tt][kb] = {hi, lo} for token tile tt.
template <int NKB>
__device__ __forceinline__ void expand_chunk(uint32_t bslot, uint32_t yslot, int ys, int r, int ocs, int cw, int g,
                                             int qd, const uint4 (&vfh)[2][4], const uint4 (&vfl)[2][4], int cnt,
                                             const int *tok, __nv_bfloat16 *Y, int64_t ldy, int o0, float sc)
{
    const int ntt = cnt > 8 ? 2 : 1;
    const int n_mt = (ocs + 15) >> 4;
    for (int mt = cw; mt < n_mt; mt += kSCons) {
        const int ob = mt * 16;
        const bool r0 = ob + g < ocs, r1 = ob + g + 8 < ocs;
        float acc[2][4][4];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int c = 0; c < 4; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[t][c][e] = 0.f;
#pragma unroll
        for (int kb = 0; kb < NKB; ++kb) {
            const int kc = kb * 32 + qd * 8;
            const bool in = kc < r;
            const uint4 z = make_uint4(0, 0, 0, 0);
            const uint4 b0 = (in && r0) ? lds128(bslot + ((ob + g) * r + kc) * 2) : z;
            const uint4 b1 = (in && r1) ? lds128(bslot + ((ob + g + 8) * r + kc) * 2) : z;
#pragma unroll
            for (int t = 0; t < 2; ++t) {
                if (t < ntt) {
                    const uint4 h = vfh[t][kb], l = vfl[t][kb];
                    mma16816(acc[t][0], b0.x, b1.x, b0.y, b1.y, h.x, h.y);
                    mma16816(acc[t][1], b0.z, b1.z, b0.w, b1.w, h.z, h.w);
                    mma16816(acc[t][2], b0.x, b1.x, b0.y, b1.y, l.x, l.y);
                    mma16816(acc[t][3], b0.z, b1.z, b0.w, b1.w, l.z, l.w);
                }
            }
        }
        // D: (output ob + g, tokens 2qd, 2qd + 1) and (output ob + g + 8, same tokens)
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t < ntt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tt = t * 8 + 2 * qd + (e & 1);
                    const int o = ob + g + (e >> 1) * 8;
                    if (tt < cnt && o < ocs) {
                        const float d = (acc[t][0][e] + acc[t][1][e]) + (acc[t][2][e] + acc[t][3][e]);
                        const uint32_t ya = yslot + tt * ys + o * 2;
                        uint16_t yb;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(yb) : "r"(ya));
                        const float y = __bfloat162float(__ushort_as_bfloat16(yb));
                        Y[(int64_t)tok[tt] * ldy + o0 + o] = __float2bfloat16_rn(fmaf(sc, d, y));
                    }
                }
            }
        }
    }
}

// The same for ranks <= 16: one k16 step, thread quad qd holding ranks 4qd .. 4qd+3.
__device__ __forceinline__ void expand_chunk16(uint32_t bslot, uint32_t yslot, int ys, int r, int ocs, int cw, int g,
                                               int qd, const uint2 (&v16h)[2], const uint2 (&v16l)[2], int cnt,
                                               const int *tok, __nv_bfloat16 *Y, int64_t ldy, int o0, float sc)
{
    const int ntt = cnt > 8 ? 2 : 1;
    const int kc = qd * 4;
    const bool in = kc < r;
    const int n_mt = (ocs + 15) >> 4;
    for (int mt = cw; mt < n_mt; mt += kSCons) {
        const int ob = mt * 16;
        const uint2 z = make_uint2(0, 0);
        const uint2 b0 = (in && ob + g < ocs) ? lds64(bslot + ((ob + g) * r + kc) * 2) : z;
        const uint2 b1 = (in && ob + g + 8 < ocs) ? lds64(bslot + ((ob + g + 8) * r + kc) * 2) : z;
        float acc[2][2][4];
#pragma unroll
        for (int t = 0; t < 2; ++t)
#pragma unroll
            for (int c = 0; c < 2; ++c)
#pragma unroll
                for (int e = 0; e < 4; ++e)
                    acc[t][c][e] = 0.f;
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t < ntt) {
                mma16816(acc[t][0], b0.x, b1.x, b0.y, b1.y, v16h[t].x, v16h[t].y);
                mma16816(acc[t][1], b0.x, b1.x, b0.y, b1.y, v16l[t].x, v16l[t].y);
            }
        }
#pragma unroll
        for (int t = 0; t < 2; ++t) {
            if (t < ntt) {
#pragma unroll
                for (int e = 0; e < 4; ++e) {
                    const int tt = t * 8 + 2 * qd + (e & 1);
                    const int o = ob + g + (e >> 1) * 8;
                    if (tt < cnt && o < ocs) {
                        const float d = acc[t][0][e] + acc[t][1][e];
                        const uint32_t ya = yslot + tt * ys + o * 2;
                        uint16_t yb;
                        asm volatile("ld.shared.u16 %0, [%1];" : "=h"(yb) : "r"(ya));
                        const float y = __bfloat162float(__ushort_as_bfloat16(yb));
                        Y[(int64_t)tok[tt] * ldy + o0 + o] = __float2bfloat16_rn(fmaf(sc, d, y));
                    }
                }
            }
        }
    }
}

// ------------------------------------------------------------ the kernel
__global__ void __launch_bounds__(kSThreads, 1) k_bgmv_stream(const __grid_constant__ StreamBgmvArgs p)
{
    extern __shared__ __align__(128) unsigned char sm[];
    const StreamSmem L = stream_layout(p.N, p.pool.n_adapters, (int)gridDim.x, p.n_slots);
    uint64_t *full = reinterpret_cast<uint64_t *>(sm + L.bars);
    uint64_t *empty = full + p.n_slots;
    const uint32_t ring = smem_u32(sm + L.ring);
    int32_t *it_tok0 = reinterpret_cast<int32_t *>(sm + L.it_tok0);
    int32_t *it_cr = reinterpret_cast<int32_t *>(sm + L.it_cr);
    int64_t *it_aoff = reinterpret_cast<int64_t *>(sm + L.it_aoff);
    int64_t *it_boff = reinterpret_cast<int64_t *>(sm + L.it_boff);
    int32_t *sp = reinterpret_cast<int32_t *>(sm + L.sp);
    int32_t *ep = reinterpret_cast<int32_t *>(sm + L.ep);
    int32_t *scp = reinterpret_cast<int32_t *>(sm + L.scp);
    int32_t *ecp = reinterpret_cast<int32_t *>(sm + L.ecp);
    int32_t *perm = reinterpret_cast<int32_t *>(sm + L.perm);
    int32_t *first_s = reinterpret_cast<int32_t *>(sm + L.first_s);
    int32_t *first_e = reinterpret_cast<int32_t *>(sm + L.first_e);
    __nv_bfloat16 *vh = reinterpret_cast<__nv_bfloat16 *>(sm + L.vh);
    __nv_bfloat16 *vl = reinterpret_cast<__nv_bfloat16 *>(sm + L.vl);
    float *red = reinterpret_cast<float *>(sm + L.red);
    int32_t *t_ids = reinterpret_cast<int32_t *>(sm + L.t_ids);
    int32_t *t_cnt = reinterpret_cast<int32_t *>(sm + L.t_cnt);
    int32_t *t_mr = reinterpret_cast<int32_t *>(sm + L.t_mr);
    int64_t *t_ma = reinterpret_cast<int64_t *>(sm + L.t_ma);
    int64_t *t_mb = reinterpret_cast<int64_t *>(sm + L.t_mb);
    const bool meta_smem = L.t_end_meta <= L.ring + (size_t)kSlot * p.n_slots;

    __shared__ int s_tmp[4 * (kSThreads / 32 + 1)];
    __shared__ int s_bad, s_n_items, s_S, s_cpp, s_abort;
    __shared__ int s_tok[16];

    const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
    const int N = p.N, n_ad = p.pool.n_adapters, d_in = p.pool.d_in, d_out = p.pool.d_out;
    const int G = (int)gridDim.x, cta = (int)blockIdx.x;
    WsHeader *hdr = p.hdr;

    // pool metadata towards L2 while the ids arrive (whole 16-byte lines only)
    if (tid == 0) {
        SSTAMP(0);
        for (int i = 11; i < 16; ++i)
            SSTAMP_SET(i, 0);
        const uint32_t rb = (uint32_t)(n_ad * 4) & ~15u, ob = (uint32_t)(n_ad * 8) & ~15u;
        if (rb)
            prefetch_l2(p.pool.rank, rb);
        if (ob) {
            prefetch_l2(p.pool.A_off, ob);
            prefetch_l2(p.pool.B_off, ob);
        }
        s_bad = 0;
        s_abort = 0;
    }

    // ---- grouping: ids -> per-adapter counts -> stable counting sort (immutable inputs only)
    int U0 = 0;
    for (int a = tid; a <= n_ad; a += kSThreads)
        t_cnt[a] = 0;
    __syncthreads();
    if (meta_smem) {
        // every adapter's metadata, checked, requested together with the ids (one
        // round trip; the lines were prefetched into L2 above)
        for (int a = tid; a < n_ad; a += kSThreads) {
            int32_t r = 0;
            int64_t ao = 0, bo = 0;
            if (!pool_adapter_ok(p.pool, a, &r, &ao, &bo))
                r = 0;
            t_mr[a] = r;
            t_ma[a] = ao;
            t_mb[a] = bo;
        }
    }
    for (int n = tid; n < N; n += kSThreads) {
        int32_t a = p.ids[n];
        if (a < -1 || a >= n_ad) {
            s_bad = 1;
            a = -1;
        }
        t_ids[n] = a;
        if (a >= 0)
            atomicAdd(&t_cnt[a], 1);
    }
    __syncthreads();
    {
        // one scan over adapters: tokens, items (groups of <= 16 tokens) and rank tiles
        // of the items; adapters failing the pool checks get no work (rank 0)
        const int per = (n_ad + kSThreads - 1) / kSThreads;
        const int b = tid * per, e = min(n_ad, b + per);
        int4 loc = make_int4(0, 0, 0, 0);
        for (int a = b; a < e; ++a) {
            const int c = t_cnt[a];
            if (c > 0) {
                int32_t r = 0;
                if (meta_smem) {
                    r = t_mr[a];
                } else {
                    int64_t ao, bo;
                    if (!pool_adapter_ok(p.pool, a, &r, &ao, &bo))
                        r = 0;
                }
                if (r == 0)
                    s_bad = 1;
                const int ng = (c + kFT - 1) / kFT;
                loc.x += c;
                loc.y += ng;
                loc.z += ng * rank_tiles(r);
            }
        }
        int4 tot;
        int4 run = block_excl_scan4(loc, s_tmp, &tot);
        for (int a = b; a < e; ++a) {
            const int c = t_cnt[a];
            const int ng = (c + kFT - 1) / kFT;
            if (ng > 0) {
                int32_t r = 0;
                int64_t ao = 0, bo = 0;
                if (meta_smem) {
                    r = t_mr[a];
                    ao = t_ma[a];
                    bo = t_mb[a];
                } else if (!pool_adapter_ok(p.pool, a, &r, &ao, &bo)) {
                    r = 0;
                }
                for (int gi = 0; gi < ng; ++gi) {
                    it_tok0[run.y + gi] = run.x + gi * kFT;
                    it_cr[run.y + gi] = min(kFT, c - gi * kFT) | (r << 8);
                    it_aoff[run.y + gi] = ao;
                    it_boff[run.y + gi] = bo;
                }
            }
            t_cnt[a] = run.x;      // running position of the stable scatter
            run.x += c;
            run.y += ng;
        }
        if (tid == 0)
            s_n_items = tot.y;
        U0 = tot.z;
        __syncthreads();
    }
    const int n_items = s_n_items;
    if (warp == 0) {
        // stable scatter: tokens in id order within each adapter
        for (int base = 0; base < N; base += 32) {
            const int n = base + lane;
            const int a = n < N ? t_ids[n] : -2;
            const unsigned peers = __match_any_sync(0xffffffffu, a);
            const int leader = __ffs(peers) - 1;
            int pos = 0;
            if (lane == leader && a >= 0) {
                pos = t_cnt[a];
                t_cnt[a] = pos + __popc(peers);
            }
            pos = __shfl_sync(0xffffffffu, pos, leader);
            if (a >= 0)
                perm[pos + __popc(peers & ((1u << lane) - 1u))] = n;
        }
    }
    __syncthreads();

    // ---- units: d_in split, per-item unit counts and costs, CTA ranges
    {
        const int nch = (d_in + kKC - 1) / kKC;
        int S = U0 > 0 ? (kUnitsPerCta * G + U0 - 1) / U0 : 1;
        S = max(1, min(S, min(nch, p.max_parts)));
        const int cpp = (nch + S - 1) / S;
        S = (nch + cpp - 1) / cpp;
        if (tid == 0) {
            s_S = S;
            s_cpp = cpp;
        }
        // per-thread contiguous ranges of items; one scan for the four running sums
        const int per = (n_items + kSThreads - 1) / kSThreads;
        const int b = tid * per, e = min(n_items, b + per);
        int4 loc = make_int4(0, 0, 0, 0);
        for (int k = b; k < e; ++k) {
            const int cr = it_cr[k], r = cr_rank(cr), c = cr_cnt(cr);
            if (r > 0) {
                const int T = rank_tiles(r);
                const int oc = out_chunk(r);
                const int nsu = T * S, neu = (d_out + oc - 1) / oc;
                loc.x += nsu;
                loc.y += neu;
                loc.z += nsu * (r / T + c);
                loc.w += neu * ((r + 2 * c) * (oc / 64));
            }
        }
        int4 tot;
        int4 run = block_excl_scan4(loc, s_tmp, &tot);
        for (int k = b; k < e; ++k) {
            sp[k] = run.x;
            ep[k] = run.y;
            scp[k] = run.z;
            ecp[k] = run.w;
            const int cr = it_cr[k], r = cr_rank(cr), c = cr_cnt(cr);
            if (r > 0) {
                const int T = rank_tiles(r);
                const int oc = out_chunk(r);
                const int nsu = T * S, neu = (d_out + oc - 1) / oc;
                run.x += nsu;
                run.y += neu;
                run.z += nsu * (r / T + c);
                run.w += neu * ((r + 2 * c) * (oc / 64));
            }
        }
        if (tid == 0) {
            sp[n_items] = tot.x;
            ep[n_items] = tot.y;
            scp[n_items] = tot.z;
            ecp[n_items] = tot.w;
        }
        __syncthreads();
        cut_ranges(sp, scp, n_items, G, first_s, tid, kSThreads);
        cut_ranges(ep, ecp, n_items, G, first_e, tid, kSThreads);
        // the grouping scratch in the ring is dead from here on; the ring is next
        // written by the async proxy
        fence_async_smem();
        if (tid == 0) {
            for (int i = 0; i < p.n_slots; ++i) {
                mbar_init(&full[i], 1);
                mbar_init(&empty[i], kSCons);
            }
            asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
        }
        __syncthreads();
    }

    if (tid == 0)
        SSTAMP(1);
    Plan P;
    P.tok0 = it_tok0;
    P.cr = it_cr;
    P.sp = sp;
    P.ep = ep;
    P.aoff = it_aoff;
    P.boff = it_boff;
    P.n_items = n_items;
    P.S = s_S;
    P.KP = s_cpp * kKC;
    P.d_in = d_in;
    P.d_out = d_out;
    const int s0 = first_s[cta], s1 = first_s[cta + 1], e0 = first_e[cta], e1 = first_e[cta + 1];
    const int n_slots = p.n_slots;
    volatile int *abort_flag = &s_abort;

    if (warp == 0) {
        // ================= producer: bulk copies into the ring
        const uint64_t pol_w = policy_evict_first();     // adapter weights: read once
        const uint64_t pol_a = policy_evict_last();      // x rows: re-read by the item's other units
        const int total = p.test_stall ? 0 : seq_total_chunks(P, s0, s1, e0, e1);
        const int pre = min(n_slots, total);
        auto weights = [&](const Chunk &c, int slot) {
            const uint32_t dst = ring + slot * kSlot;
            const int r = cr_rank(P.cr[c.k]), cnt = cr_cnt(P.cr[c.k]);
            if (!c.expand) {
                const int64_t ao = P.aoff[c.k];
                const int halves = c.kc > 256 ? 2 : 1;
                if (p.a_tma && ao % d_in == 0) {
                    // two-dimensional boxes of 16 pool rows x 256 columns (rows past the
                    // adapter's rank and columns past the chunk are read but never used;
                    // past the pool's end they read as zeros)
                    if (lane == 0) {
                        mbar_arrive_expect_tx(&full[slot], (uint32_t)(halves * kAHalf + cnt * c.kc * 2));
                        const int row = (int)(ao / d_in) + c.row0;
                        tma_load_2d_hint(sm + (dst - ring) + L.ring, &p.map_a, &full[slot], c.k0, row, pol_w);
                        if (halves == 2)
                            tma_load_2d_hint(sm + (dst - ring) + L.ring + kAHalf, &p.map_a, &full[slot], c.k0 + 256,
                                             row, pol_w);
                    }
                    __syncwarp();
                } else {
                    // one copy per row and half
                    if (lane == 0)
                        mbar_arrive_expect_tx(&full[slot], (uint32_t)((c.rows + cnt) * c.kc * 2));
                    __syncwarp();
                    if (lane < c.rows) {
                        const __nv_bfloat16 *src = p.pool.A + ao + (int64_t)(c.row0 + lane) * d_in + c.k0;
                        const int n0 = c.kc < 256 ? c.kc : 256;
                        bulk_g2s(dst + lane * 512, src, (uint32_t)(n0 * 2), &full[slot], pol_w);
                        if (c.kc > 256)
                            bulk_g2s(dst + kAHalf + lane * 512, src + 256, (uint32_t)((c.kc - 256) * 2), &full[slot],
                                     pol_w);
                    }
                }
            } else {
                if (lane == 0) {
                    mbar_arrive_expect_tx(&full[slot], (uint32_t)(c.ocs * r * 2 + cnt * c.ocs * 2));
                    bulk_g2s(dst, p.pool.B + P.boff[c.k] + (int64_t)c.o0 * r, (uint32_t)(c.ocs * r * 2),
                             &full[slot], pol_w);
                }
                __syncwarp();
            }
        };
        auto acts = [&](const Chunk &c, int slot) {
            const uint32_t dst = ring + slot * kSlot;
            const int cnt = cr_cnt(P.cr[c.k]);
            const int tok0 = P.tok0[c.k];
            if (!c.expand) {
                if (lane < cnt)
                    bulk_g2s(dst + kXOff + lane * kXRowB, p.X + (int64_t)perm[tok0 + lane] * p.ldx + c.k0,
                             (uint32_t)(c.kc * 2), &full[slot], pol_a);
            } else {
                const int ys = c.ocs * 2 + 16;
                if (lane < cnt)
                    bulk_g2s(dst + kEB + lane * ys, p.Y + (int64_t)perm[tok0 + lane] * p.ldy + c.o0,
                             (uint32_t)(c.ocs * 2), &full[slot], pol_a);
            }
        };
        Seq q;
        seq_init(q, P, s0, s1, e0, e1);
        Chunk ch;
        // the first slots' weights before waiting for the previous kernel
        for (int i = 0; i < pre; ++i) {
            seq_next(q, P, ch);
            weights(ch, i);
        }
        if (lane == 0)
            SSTAMP(2);
        pdl_wait();
        pdl_trigger();
        if (lane == 0) {
            SSTAMP(3);
            SSTAMP_SET(11, total);
        }
        {
            Seq q2;
            seq_init(q2, P, s0, s1, e0, e1);
            for (int i = 0; i < pre; ++i) {
                seq_next(q2, P, ch);
                acts(ch, i);
                if (lane == 0)
                    STRACE(i, 0);
            }
        }
        int issued = pre;
        for (int i = pre; i < total; ++i) {
            const int slot = i % n_slots;
            if (!warp_wait_phase(&empty[slot], ((i / n_slots) - 1) & 1, abort_flag, &hdr->err, p.wait_ns))
                break;
            seq_next(q, P, ch);
            weights(ch, slot);
            acts(ch, slot);
            issued = i + 1;
            if (lane == 0)
                STRACE(i, 0);
        }
        if (lane == 0)
            SSTAMP(4);
        // every copy issued lands before the CTA may exit: wait (bounded) for the
        // last fill of every slot, whether or not the consumers got to it
        for (int i = max(0, issued - n_slots); i < issued; ++i) {
            const int slot = i % n_slots;
            const unsigned long long t0 = now_ns();
            while (!mbar_wait_hint(&full[slot], (i / n_slots) & 1, kSuspendNs)) {
                if (now_ns() - t0 > p.wait_ns) {
                    if (lane == 0)
                        atomicOr(&hdr->err, (uint32_t)LORA_ERR_TIMEOUT);
                    break;
                }
            }
        }
    } else if (p.test_stall) {
        // ================= consumers of a stalled producer: nothing was issued, so
        // the first wait runs out, reports the timeout, and the CTA winds down
        pdl_wait();
        pdl_trigger();
        warp_wait_phase(&full[0], 0, abort_flag, &hdr->err, p.wait_ns);
    } else {
        // ================= consumers
        const int cw = warp - 1, ctid = tid - 32;
        const int g = lane >> 2, qd = lane & 3;
        pdl_wait();
        pdl_trigger();
        const unsigned long long E = (unsigned long long)(*reinterpret_cast<volatile uint32_t *>(&hdr->epoch)) + 1ull;
        if (ctid == 0 && cta == 0 && s_bad)
            atomicOr(&hdr->err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        Seq q;
        seq_init(q, P, s0, s1, e0, e1);
        Chunk ch;
        float acc[2][2][4];
#pragma unroll
        for (int i = 0; i < 2; ++i)
#pragma unroll
            for (int h = 0; h < 2; ++h)
#pragma unroll
                for (int j = 0; j < 4; ++j)
                    acc[i][h][j] = 0.f;
        int done_units = 0;
        int cur_cnt = 0, cur_r = 0;
        uint4 vfh[2][4], vfl[2][4];     // the current item's V fragments: [token tile][32-rank block]
        uint2 v16h[2], v16l[2];         // ... ranks <= 16
        [[maybe_unused]] bool saw_dep = false;
        const float sc = p.scale;
        for (int i = 0; seq_next(q, P, ch); ++i) {
            const int slot = i % n_slots;
            const uint32_t sbase = ring + slot * kSlot;
            if (ch.expand && ch.new_item) {
                // the item's shrink units must be done: wait until every CTA owning
                // one of them has published at least that many finished units
                const int k = ch.k;
                const int u0 = P.sp[k], u1 = P.sp[k + 1];
                cons_sync();    // V buffers of the previous item no longer read
                if (ctid == 0 && u1 > u0 && !*abort_flag) {
                    for (int c = item_of(first_s, G, u0); c < G && first_s[c] < u1; ++c) {
                        const int need = min(u1, first_s[c + 1]) - first_s[c];
                        if (need <= 0)
                            continue;
                        const unsigned long long want = (E << 32) | (unsigned)need;
                        const unsigned long long t0 = now_ns();
                        if (!saw_dep)
                            SSTAMP(7);
                        bool ok = true;
                        for (;;) {
                            const unsigned long long v = ld_acquire_u64(&hdr->progress[c]);
                            if ((v >> 32) == E && v >= want)
                                break;
                            if (*abort_flag || now_ns() - t0 > p.wait_ns) {
                                ok = false;
                                break;
                            }
                            __nanosleep(256);
                        }
                        SSTAMP_ADD(14, now_ns() - t0);
                        if (!ok) {
                            if (!*abort_flag) {
                                *abort_flag = 1;
                                atomicOr(&hdr->err, (uint32_t)LORA_ERR_TIMEOUT);
                            }
                            break;
                        }
                    }
                }
                if (ctid < 16)
                    s_tok[ctid] = ctid < cr_cnt(P.cr[k]) ? perm[P.tok0[k] + ctid] : 0;
                cons_sync();
                // V = sum of the planes (fixed order), as bf16 high + low parts, zero padded
                cur_cnt = cr_cnt(P.cr[k]);
                cur_r = cr_rank(P.cr[k]);
                constexpr int rp = kMaxRank;             // all columns written: zeros past the rank
                const bool live = !*abort_flag;
                for (int e = ctid; live && e < 16 * rp; e += kSConsThreads) {
                    const int t = e / rp, j = e - t * rp;
                    float s = 0.f;
                    if (t < cur_cnt && j < cur_r) {
                        // L2 reads (not L1: other CTAs wrote the planes during this launch),
                        // independent, so they are in flight together
                        const float *v = p.V + (int64_t)s_tok[t] * p.ldv + j;
                        float part[4] = {0.f, 0.f, 0.f, 0.f};
                        int pl = 0;
                        for (; pl + 4 <= P.S; pl += 4) {
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                part[u] = __ldcg(v + (int64_t)(pl + u) * p.plane);
#pragma unroll
                            for (int u = 0; u < 4; ++u)
                                s += part[u];
                        }
                        for (; pl < P.S; ++pl)
                            s += __ldcg(v + (int64_t)pl * p.plane);
                    }
                    const __nv_bfloat16 h = __float2bfloat16_rn(s);
                    vh[t * kSVS + j] = h;
                    vl[t * kSVS + j] = __float2bfloat16_rn(s - __bfloat162float(h));
                }
                cons_sync();
                // this item's V fragments stay in registers for all its expand chunks
                {
                    const uint32_t uvh = smem_u32(vh), uvl = smem_u32(vl);
#pragma unroll
                    for (int t = 0; t < 2; ++t) {
                        const int row = t * 8 + g;          // token of this lane's B fragment
                        v16h[t] = lds64(uvh + (row * kSVS + qd * 4) * 2);
                        v16l[t] = lds64(uvl + (row * kSVS + qd * 4) * 2);
#pragma unroll
                        for (int kb = 0; kb < 4; ++kb) {
                            const int kc = kb * 32 + qd * 8;
                            vfh[t][kb] = lds128(uvh + (row * kSVS + kc) * 2);
                            vfl[t][kb] = lds128(uvl + (row * kSVS + kc) * 2);
                        }
                    }
                }
                if (ctid == 0 && !saw_dep) {
                    SSTAMP(8);
                    saw_dep = true;
                }
            }
            // after a failed wait the warps keep walking the sequence without work, so
            // every consumer thread reaches the same named barriers
#ifdef LORA_STREAM_STAMPS
            const unsigned long long tw = now_ns();
#endif
            const bool have = warp_wait_phase(&full[slot], (i / n_slots) & 1, abort_flag, &hdr->err, p.wait_ns);
            if (ctid == 0) {
                SSTAMP_ADD(15, now_ns() - tw);
                STRACE(i, 1);
                if (i == 0)
                    SSTAMP(5);
            }
            if (!have) {
                // nothing to compute
            } else if (!ch.expand) {
                shrink_chunk(sbase, cw, g, qd, ch.kc, ch.rows, acc);
            } else {
                const int ys = ch.ocs * 2 + 16;
#define LORA_EXP(NKB)                                                                                          \
    expand_chunk<NKB>(sbase, sbase + kEB, ys, cur_r, ch.ocs, cw, g, qd, vfh, vfl, cur_cnt, s_tok, p.Y, p.ldy, ch.o0, \
                      sc)
                if (cur_r <= 16)
                    expand_chunk16(sbase, sbase + kEB, ys, cur_r, ch.ocs, cw, g, qd, v16h, v16l, cur_cnt, s_tok, p.Y,
                                   p.ldy, ch.o0, sc);
                else if (cur_r <= 32)
                    LORA_EXP(1);
                else if (cur_r <= 64)
                    LORA_EXP(2);
                else if (cur_r <= 96)
                    LORA_EXP(3);
                else
                    LORA_EXP(4);
#undef LORA_EXP
            }
            __syncwarp();
            if (lane == 0)
                slot_release(&empty[slot]);
            if (ctid == 0)
                STRACE(i, 2);
            if (!ch.expand && ch.last) {
                // reduce the warps' partials (fixed order) and write this unit's V plane rows
                const int k = ch.k;
                float *rw = red + cw * 256;
#pragma unroll
                for (int nt = 0; nt < 2; ++nt) {
                    const int j = nt * 8 + 2 * qd;
                    rw[g * 16 + j] = acc[nt][0][0] + acc[nt][1][0];
                    rw[g * 16 + j + 1] = acc[nt][0][1] + acc[nt][1][1];
                    rw[(g + 8) * 16 + j] = acc[nt][0][2] + acc[nt][1][2];
                    rw[(g + 8) * 16 + j + 1] = acc[nt][0][3] + acc[nt][1][3];
                }
                cons_sync();
                const bool live = !*abort_flag;
                {
                    const int t = ctid >> 4, j = ctid & 15;
                    if (live && t < cr_cnt(P.cr[k]) && j < ch.rows) {
                        float s = 0.f;
#pragma unroll
                        for (int w = 0; w < kSCons; ++w)
                            s += red[w * 256 + t * 16 + j];
                        const int tok = perm[P.tok0[k] + t];
                        p.V[(int64_t)ch.part * p.plane + (int64_t)tok * p.ldv + ch.row0 + j] = s;
                    }
                }
                cons_sync();
                ++done_units;
                // the barrier orders every thread's V writes before this release
                if (ctid == 0 && live) {
                    st_release_u64(&hdr->progress[cta], (E << 32) | (unsigned)done_units);
                    SSTAMP(6);
                    SSTAMP_SET(12, done_units);
                    STRACE(i, 3);
                }
#pragma unroll
                for (int x = 0; x < 2; ++x)
#pragma unroll
                    for (int h = 0; h < 2; ++h)
#pragma unroll
                        for (int y = 0; y < 4; ++y)
                            acc[x][h][y] = 0.f;
            }
        }
    }

    // ---- end of the call: the last CTA out advances the workspace's epoch
    __syncthreads();
    if (tid == 0) {
        SSTAMP(10);
        __threadfence();
        const unsigned old = atomicAdd(&hdr->done, 1u);
        if (old == (unsigned)G - 1u) {
            hdr->done = 0u;
            __threadfence();
            *reinterpret_cast<volatile uint32_t *>(&hdr->epoch) = hdr->epoch + 1u;
        }
    }
}

struct StreamOcc {
    int dev = -1;
    size_t smem = 0;
    int blocks = 0;
};

int stream_blocks_per_sm(int dev, size_t smem)
{
    static StreamOcc cache[16];
    static std::mutex mu;
    std::lock_guard<std::mutex> lock(mu);
    for (auto &c : cache)
        if (c.dev == dev && c.smem == smem)
            return c.blocks;
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k_bgmv_stream, kSThreads, smem) != cudaSuccess)
        n = 0;
    for (auto &c : cache)
        if (c.dev < 0) {
            c.dev = dev;
            c.smem = smem;
            c.blocks = n;
            break;
        }
    return n;
}

}  // namespace

int stream_grid(int32_t N, int32_t n_adapters, int *n_slots_out, size_t *smem_out)
{
    if (N < 1 || N > kStreamMaxTokens || n_adapters < 1)
        return 0;
    const int G = sm_count() < kMaxStreamCtas ? sm_count() : kMaxStreamCtas;
    const size_t cap = kStreamMaxSmem;
    int ns = 0;
    for (int s = kStreamMaxSlots; s >= kStreamMinSlots; --s) {
        const StreamSmem L = stream_layout(N, n_adapters, G, s);
        if (L.total <= cap && L.t_end <= L.ring + (size_t)kSlot * s) {
            ns = s;
            break;
        }
    }
    if (!ns)
        return 0;
    if (n_slots_out)
        *n_slots_out = ns;
    if (smem_out)
        *smem_out = stream_layout(N, n_adapters, G, ns).total;
    return G;
}

bool stream_bgmv_supported(int32_t N, int32_t n_adapters) { return stream_grid(N, n_adapters, nullptr, nullptr) > 0; }

cudaError_t launch_bgmv_stream(const StreamBgmvArgs &a_in, cudaStream_t s, bool pdl)
{
    StreamBgmvArgs a = a_in;
    size_t smem = 0;
    int ns = 0;
    int G = stream_grid(a.N, a.pool.n_adapters, &ns, &smem);
    if (G <= 0)
        return cudaErrorNotSupported;
    a.n_slots = ns;
    // the A pool as a 2-D tensor for the shrink's row boxes (rows of d_in >= 256 columns)
    a.a_tma = 0;
    const int64_t a_rows = a.pool.d_in > 0 ? a.pool.A_elems / a.pool.d_in : 0;
    if (a.pool.d_in >= 256 && a_rows >= 16 && a_rows <= 0x7fffffffLL) {
        EncodeTiledFn fn = encode_fn();
        if (fn) {
            const cuuint64_t dims[2] = {(cuuint64_t)a.pool.d_in, (cuuint64_t)a_rows};
            const cuuint64_t strides[1] = {(cuuint64_t)a.pool.d_in * 2};
            const cuuint32_t box[2] = {256, 16};
            const cuuint32_t estr[2] = {1, 1};
            a.a_tma = fn(&a.map_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<__nv_bfloat16 *>(a.pool.A), dims,
                         strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
                         CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
        }
    }
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    static bool attr_set[64] = {};
    static std::mutex mu;
    {
        std::lock_guard<std::mutex> lock(mu);
        if (dev < 0 || dev >= 64 || !attr_set[dev]) {
            e = cudaFuncSetAttribute(k_bgmv_stream, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kStreamMaxSmem);
            if (e != cudaSuccess)
                return e;
            if (dev >= 0 && dev < 64)
                attr_set[dev] = true;
        }
    }
    // every CTA must be resident at once (expand units wait on other CTAs' shrink units)
    const int per_sm = stream_blocks_per_sm(dev, smem);
    if (per_sm < 1)
        return cudaErrorNotSupported;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3((unsigned)G);
    cfg.blockDim = dim3(kSThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_bgmv_stream, a);
}

}  // namespace lora

#ifdef LORA_STREAM_STAMPS
extern "C" LORA_API int lora_debug_stream_stamps(unsigned long long *host, int n)
{
    return (int)cudaMemcpyFromSymbol(host, lora::g_stream_stamps, sizeof(unsigned long long) * (size_t)n);
}
extern "C" LORA_API int lora_debug_stream_trace(unsigned long long *host, int n)
{
    return (int)cudaMemcpyFromSymbol(host, lora::g_stream_trace, sizeof(unsigned long long) * (size_t)n);
}
#endif
