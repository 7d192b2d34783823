// A projection and its LoRA delta in one tensor-core pass ("Serving several
// LoRAs, ControlNet and IP-Adapter", section "LoRA: merged or alongside": served
// unmerged, an adapted layer computes x W^T plus the low-rank x A^T B^T, scaled):
//
//     Y[n] = W x[n] + s B[a] (A[a] x[n])       (a = the row's segment adapter; -1: none)
//
// Unit = (pair of tiles of <= 128 rows, each inside one segment; slice of 256
// outputs).  Two TMEM accumulators D0, D1 [128 x 256] take X_tile W_slice^T over
// d_in in 64-column k-blocks, both tiles against the same W box (so W crosses
// from L2 once per 256 rows), and then, as further k-blocks, each tile's
// (s V)_tile B[a]_slice^T: the tcgen05 shrink has already written s V = s A[a] x as
// two bf16 parts (high and low), each contracted against the same B columns, so
// the delta joins the base product in fp32 and y is rounded to bf16 once.  Y is
// written, never read.
//
// One persistent CTA per SM, 320 threads, warp specialised:
//   warp 0     producer: TMA boxes into a three-stage ring of 64 KB stages -- two
//              128 x 64 x boxes and a 256 x 64 W box per base k-block; the s V part
//              box and two 128-row boxes of the adapter's B columns per LoRA k-block;
//   warp 1     one thread issues tcgen05.mma (M = 128, N = 256, K = 16) and commits;
//   warps 2-9  epilogue: four warps per tile (one per TMEM lane quarter), 256
//              columns each -- tcgen05.ld, round to bf16, 16-byte stores.
// The two accumulators fill all 512 TMEM columns, so a unit's epilogue runs while
// the producer refills the ring for the next unit.  Units go out in blocks of all
// tile pairs against 8 output slices, and the CTAs take consecutive units, so the
// units in flight at one time share a few MB of X and W in L2 (the W slices stay
// there for the whole block).
//
// The LoRA k-blocks read B through the pool views of ranks 16, 32, 64 and 128
// when the adapter's offset is a multiple of its rank, and gather it with 16-byte
// cp.async copies into the same swizzled layout otherwise (any rank that is a
// multiple of 8); a segment whose adapter fails the pool checks gets the base
// product only and sets LORA_ERR_BAD_ADAPTER.  Every wait is bounded as in the
// other tcgen05 kernels.

#include "lora_internal.cuh"
#include "tc_ptx.cuh"

namespace lora {
namespace {

constexpr int kLinThreads = 320;            // producer, MMA, 8 epilogue warps
constexpr int kLinEpiWarps = 8;
constexpr int kLN = 256;                    // outputs per unit (MMA N)
constexpr int kLStage = 2 * kAtom + kLN * 128;   // two x atoms (a pair of tiles) + W box: 64 KB
constexpr int kLStages = 3;
constexpr int kLNsBlock = 8;                // output slices per block of the unit order

struct LinUnit {
    int pair, ns;
};

// Unit u in the blocked order: block k holds every tile pair against slices
// 8k .. 8k + 7 (fewer in the last block), pair-major inside the block.
__device__ __forceinline__ LinUnit lin_unit(int64_t u, int n_pairs, int n_ns)
{
    const int64_t per_blk = (int64_t)n_pairs * kLNsBlock;
    const int blk = (int)(u / per_blk);
    const int64_t rem = u - blk * per_blk;
    const int nsb = min(kLNsBlock, n_ns - blk * kLNsBlock);
    LinUnit x;
    x.pair = (int)(rem / nsb);
    x.ns = blk * kLNsBlock + (int)(rem - (int64_t)x.pair * nsb);
    return x;
}

struct LinAd {
    int r;          // rank, 0: no LoRA k-blocks
    int brow;       // TMA: row of output 0 in the B view of rank r
    int m;          // TMA: that view's index; -1: B rows gathered with cp.async
    int64_t boff;   // gather: element offset of the adapter's B
};

// The segment's adapter as the LoRA k-blocks use it: B through the pool's view of
// its rank when there is one (ranks 16, 32, 64, 128, offset a multiple of the
// rank), else gathered row by row.
__device__ LinAd lin_adapter(const LinArgs &p, int item, bool report)
{
    LinAd d = {0, 0, 0, 0};
    const int32_t a = p.seg_ad[item];
    if (a == -1)
        return d;
    int32_t r = 0;
    int64_t ao = 0, bo = 0;
    if (!pool_adapter_ok(p.pool, a, &r, &ao, &bo)) {
        if (report)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        return d;
    }
    const int m = b_map(r);
    d.r = r;
    d.boff = bo;
    if (m >= 0 && ((p.b_tma >> m) & 1) && (bo % r) == 0 && bo / r <= 0x7fffffffLL) {
        d.brow = (int)(bo / r);
        d.m = m;
    } else {
        d.m = -1;
    }
    return d;
}

__device__ __forceinline__ int lora_kblocks(const LinAd &d) { return d.r ? 2 * ((d.r + 63) >> 6) : 0; }

// The two tiles of pair `pair` (the second may be absent) and their adapters.
struct LinPair {
    Group g[2];
    bool has1;
    LinAd ad[2];
    int nl[2];          // LoRA k-blocks of each tile
};

__device__ __forceinline__ LinPair lin_pair(const LinArgs &p, int pair, int n_tiles, bool report)
{
    LinPair x;
    x.g[0] = p.groups[2 * pair];
    x.has1 = 2 * pair + 1 < n_tiles;
    x.g[1] = x.has1 ? p.groups[2 * pair + 1] : x.g[0];
    x.ad[0] = lin_adapter(p, x.g[0].item, report);
    x.ad[1] = x.has1 ? lin_adapter(p, x.g[1].item, report) : LinAd{0, 0, 0, 0};
    x.nl[0] = lora_kblocks(x.ad[0]);
    x.nl[1] = lora_kblocks(x.ad[1]);
    return x;
}

__global__ void __launch_bounds__(kLinThreads, 1) k_tc_linear(const __grid_constant__ LinArgs p)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[kLStages], empty_bar[kLStages];
    __shared__ __align__(8) uint64_t acc_full, acc_empty, mma_drain;
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int n_kb = (p.d_in + kBK - 1) / kBK;
    const int n_ns = (p.d_out + kLN - 1) / kLN;

    if (tid == 0) {
        for (int s = 0; s < kLStages; ++s) {
            mbar_init(&full_bar[s], 33);         // producer lane 0's expect_tx + 32 cp.async arrivals
            mbar_init(&empty_bar[s], 1);         // MMA commit
        }
        mbar_init(&acc_full, 1);                 // MMA commit
        mbar_init(&acc_empty, kLinEpiWarps);
        mbar_init(&mma_drain, 1);                // the MMA issuer's last commit before TMEM is freed
        abort_flag = 0;
        asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    }
    if (warp == 1)
        tmem_alloc(&tmem_base, 2 * kLN);
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = tmem_base;
    pdl_wait();                                   // tiles (plan) and s V (shrink) are complete
    pdl_trigger();
    const int n_tiles = p.hdr->n_groups;
    const int n_pairs = (n_tiles + 1) / 2;
    const int64_t n_units = (int64_t)n_pairs * n_ns;
    int issued = 0;                               // producer: stage fills issued

    if (warp == 0) {
        // ------------------------------------------------ producer
        int it = 0;
        if (p.test_stall)
            goto done;
        const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
        for (int64_t u = blockIdx.x; u < n_units; u += G) {
            const LinUnit un = lin_unit(u, n_pairs, n_ns);
            const LinPair pr = lin_pair(p, un.pair, n_tiles, lane == 0 && un.ns == 0);
            const int n_all = n_kb + pr.nl[0] + pr.nl[1];
            const int o0 = un.ns * kLN;
            for (int kb = 0; kb < n_all; ++kb, ++it) {
                const int s = it % kLStages;
                const uint32_t ph = (it / kLStages) & 1;
                if (!warp_wait(&empty_bar[s], ph ^ 1, &abort_flag, p.err, p.wait_ns))
                    goto done;
                if (lane == 0) {
                    unsigned char *xs = sm + s * kLStage;
                    unsigned char *wsm = xs + 2 * kAtom;
                    if (kb < n_kb) {
                        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)((pr.has1 ? 2 : 1) * kAtom + kLN * 128));
                        tma_load_2d_hint(xs, &p.map_x, &full_bar[s], kb * kBK, pr.g[0].p0, pol_x);
                        if (pr.has1)
                            tma_load_2d_hint(xs + kAtom, &p.map_x, &full_bar[s], kb * kBK, pr.g[1].p0, pol_x);
                        tma_load_2d_hint(wsm, &p.map_w, &full_bar[s], kb * kBK, o0, pol_w);
                    } else {
                        // LoRA k-blocks of tile 0, then of tile 1; k-block j of a tile: part
                        // j % 2 (high, low) of rank columns 64 (j / 2) ..
                        int j = kb - n_kb;
                        const int ti = j < pr.nl[0] ? 0 : 1;
                        if (ti)
                            j -= pr.nl[0];
                        const LinAd ad = ti ? pr.ad[1] : pr.ad[0];
                        const int part = j & 1, c = j >> 1;
                        const int w = ad.r < 64 ? ad.r : 64;
                        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(kAtom + (ad.m >= 0 ? 2 * 128 * w * 2 : 0)));
                        tma_load_2d_hint(xs, &p.map_v, &full_bar[s], part * p.kv + c * 64,
                                         ti ? pr.g[1].p0 : pr.g[0].p0, pol_x);
                        if (ad.m >= 0) {
                            tma_load_2d_hint(wsm, &p.map_b[ad.m], &full_bar[s], c * 64, ad.brow + o0, pol_w);
                            tma_load_2d_hint(wsm + 128 * w * 2, &p.map_b[ad.m], &full_bar[s], c * 64,
                                             ad.brow + o0 + 128, pol_w);
                        }
                    }
                }
                __syncwarp();
                if (kb >= n_kb) {
                    // a LoRA k-block whose adapter has no B view: all lanes gather its
                    // 256 output rows x 64 rank columns (16-byte chunks, 128-byte swizzle,
                    // the layout of the rank >= 64 views); ranks past r and outputs past
                    // d_out are zero-filled
                    int j = kb - n_kb;
                    const int ti = j < pr.nl[0] ? 0 : 1;
                    if (ti)
                        j -= pr.nl[0];
                    const LinAd ad = ti ? pr.ad[1] : pr.ad[0];
                    if (ad.m < 0) {
                        const int rc0 = (j >> 1) * 64;
                        const uint32_t wbase = smem_u32(sm + s * kLStage + 2 * kAtom);
                        for (int idx = lane; idx < kLN * 8; idx += 32) {
                            const int o = idx >> 3, cc = idx & 7;
                            const int col = rc0 + cc * 8;
                            const bool ok = o0 + o < p.d_out && col < ad.r;
                            const __nv_bfloat16 *src = ok ? p.pool.B + ad.boff + (int64_t)(o0 + o) * ad.r + col
                                                          : p.pool.B;
                            cp_async16(wbase + (o >> 7) * kAtom + sw128_off(o & 127, cc), src, ok);
                        }
                    }
                }
                cp_async_arrive(&full_bar[s]);
                issued = it + 1;
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        int it = 0, t = 0;
        const uint32_t idesc = idesc_bf16(kBM, kLN);
        for (int64_t u = blockIdx.x; u < n_units; u += G, ++t) {
            const LinUnit un = lin_unit(u, n_pairs, n_ns);
            const LinPair pr = lin_pair(p, un.pair, n_tiles, false);
            const int n_all = n_kb + pr.nl[0] + pr.nl[1];
            if (!warp_wait(&acc_empty, (t & 1) ^ 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            tc_fence_after();
            for (int kb = 0; kb < n_all; ++kb, ++it) {
                const int s = it % kLStages;
                const uint32_t ph = (it / kLStages) & 1;
                if (!warp_wait(&full_bar[s], ph, &abort_flag, p.err, p.wait_ns))
                    goto done;
                if (kb >= n_kb)
                    fence_async_smem();             // B may have been written by cp.async (generic proxy)
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t xa = smem_u32(sm + s * kLStage), wa = xa + 2 * kAtom;
                    if (kb < n_kb) {
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            tc_mma(tmem, sw128_desc(xa + k * 32), sw128_desc(wa + k * 32), idesc,
                                   (kb > 0 || k > 0) ? 1u : 0u);
                        if (pr.has1) {
#pragma unroll
                            for (int k = 0; k < kBK / 16; ++k)
                                tc_mma(tmem + kLN, sw128_desc(xa + kAtom + k * 32), sw128_desc(wa + k * 32), idesc,
                                       (kb > 0 || k > 0) ? 1u : 0u);
                        }
                    } else {
                        int j = kb - n_kb;
                        const int ti = j < pr.nl[0] ? 0 : 1;
                        if (ti)
                            j -= pr.nl[0];
                        const LinAd ad = ti ? pr.ad[1] : pr.ad[0];
                        const int r = ad.r;
                        const int left = r - (j >> 1) * 64;          // ranks in this k-block
                        const int steps = ((left < 64 ? left : 64) + 15) >> 4;
                        for (int k = 0; k < steps; ++k) {
                            // B columns in the view's swizzle: 128-byte rows from rank 64 up
                            // (and for every gathered block), 64-byte rows at rank 32,
                            // 32-byte rows at rank 16
                            const uint64_t bdesc = (r >= 64 || ad.m < 0) ? sw128_desc(wa + k * 32)
                                                 : (r == 32 ? sw64_desc(wa + k * 32) : sw32_desc(wa));
                            tc_mma(tmem + ti * kLN, sw128_desc(xa + k * 32), bdesc, idesc, 1u);
                        }
                    }
                    tc_commit(&empty_bar[s]);
                }
                __syncwarp();
            }
            if (lane == 0)
                tc_commit(&acc_full);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue: D -> y rows
        const int e = warp - 2;                  // 0..7
        const int q = warp & 3;                  // TMEM lane quarter this warp may read
        const int ti = e >> 2;                   // tile of the pair (its accumulator)
        const int row = q * 32 + lane;
        int t = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += G, ++t) {
            const LinUnit un = lin_unit(u, n_pairs, n_ns);
            const int tile = 2 * un.pair + ti;
            if (!warp_wait(&acc_full, t & 1, &abort_flag, p.err, p.wait_ns))
                goto done;
            tc_fence_after();
            if (tile < n_tiles) {
                const Group gr = p.groups[tile];
                const bool valid = row < gr.cnt;
                __nv_bfloat16 *yrow = p.Y + (int64_t)(gr.p0 + (valid ? row : 0)) * p.ldy;
                const int o0 = un.ns * kLN;
#pragma unroll 1
                for (int c0 = 0; c0 < kLN; c0 += 32) {
                    float v[32];
                    tmem_ld32(tmem + ti * kLN + ((uint32_t)(q * 32) << 16) + c0, v);
                    if (valid) {
#pragma unroll
                        for (int g = 0; g < 4; ++g) {
                            const int o = o0 + c0 + 8 * g;
                            if (o < p.d_out) {
                                uint32_t w4[4];
#pragma unroll
                                for (int jj = 0; jj < 4; ++jj) {
                                    const __nv_bfloat162 hv =
                                        __floats2bfloat162_rn(v[8 * g + 2 * jj], v[8 * g + 2 * jj + 1]);
                                    w4[jj] = *reinterpret_cast<const uint32_t *>(&hv);
                                }
                                *reinterpret_cast<uint4 *>(yrow + o) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
                            }
                        }
                    }
                }
            }
            tc_fence_before();
            __syncwarp();
            if (lane == 0)
                mbar_arrive(&acc_empty);
        }
    }
done:
    // nothing may land in shared memory or TMEM after this CTA lets go of them
    if (warp == 0)
        drain_fills(full_bar, kLStages, issued, p.err, p.wait_ns);
    if (warp == 1 && lane == 0)
        drain_mma(&mma_drain, 0, p.err, p.wait_ns);
    __syncthreads();
    if (warp == 1) {
        tc_fence_after();
        tmem_dealloc(tmem, 2 * kLN);
    }
}

}  // namespace

bool lin_encode(LinArgs &a, const void *X, int64_t ldx, int32_t N, const void *W, int64_t ldw, const void *Vb,
                int64_t ldvb, const void *B, int64_t B_elems, int32_t d_in, int32_t d_out)
{
    if (!encode_box(&a.map_x, X, N, d_in, ldx, 128))
        return false;
    if (!encode_box(&a.map_w, W, d_out, d_in, ldw, kLN))
        return false;
    if (!encode_box(&a.map_v, Vb, N, 2 * (int64_t)a.kv, ldvb, 128))
        return false;
    a.b_tma = encode_b_views(a.map_b, B, B_elems);
    a.d_in = d_in;
    a.d_out = d_out;
    return true;
}

cudaError_t launch_tc_linear(const LinArgs &a_in, int max_units, cudaStream_t s)
{
    LinArgs a = a_in;
    a.wait_ns = wait_bound_ns();
    a.test_stall = test_stall_mode();
    static bool attr_set[64] = {};
    const int smem = kLStages * kLStage + 1024;
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        if ((e = cudaFuncSetAttribute(k_tc_linear, cudaFuncAttributeMaxDynamicSharedMemorySize, smem)) != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    int grid = sm_count();
    if (max_units > 0 && max_units < grid)
        grid = max_units;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(grid);
    cfg.blockDim = dim3(kLinThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_tc_linear, a);
}

}  // namespace lora
