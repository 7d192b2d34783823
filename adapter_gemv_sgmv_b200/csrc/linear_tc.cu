// A projection and its LoRA delta in one tensor-core pass ("Serving several
// LoRAs, ControlNet and IP-Adapter", section "LoRA: merged or alongside": served
// unmerged, an adapted layer computes x W^T plus the low-rank x A^T B^T, scaled):
//
//     Y[n] = W x[n] + s B[a] (A[a] x[n])       (a = the row's segment adapter; -1: none)
//
// Unit = (tile of <= 128 rows of one segment, slice of 256 outputs).  One TMEM
// accumulator D[128 x 256] takes X_tile W_slice^T over d_in in 64-column k-blocks
// and then, as further k-blocks, (s V)_tile B[a]_slice^T: the tcgen05 shrink has
// already written s V = s A[a] x as two bf16 parts (high and low), each contracted
// against the same B columns, so the delta joins the base product in fp32 and y is
// rounded to bf16 once.  Y is written, never read.
//
// One persistent CTA per SM, 320 threads, warp specialised:
//   warp 0     producer: TMA boxes into a four-stage ring of 48 KB stages -- a
//              128 x 64 x box and a 256 x 64 W box per base k-block; the s V part box
//              and two 128-row boxes of the adapter's B columns per LoRA k-block;
//   warp 1     one thread issues tcgen05.mma (M = 128, N = 256, K = 16) and commits;
//   warps 2-9  epilogue: two warps per TMEM lane quarter, 128 columns each --
//              tcgen05.ld, round to bf16, 16-byte stores.
// Two 256-column accumulators let one unit's epilogue overlap the next unit's main
// loop.  Units go out in blocks of all tiles against 8 output slices, and the CTAs
// take consecutive units, so the units in flight at one time share a few MB of X
// and W in L2 (the W slices stay there for the whole block).
//
// The LoRA k-blocks read B through the pool views of ranks 16, 32, 64 and 128
// (adapter offsets multiples of the rank); a segment whose adapter is outside
// those (or fails the pool checks) gets the base product only and sets
// LORA_ERR_BAD_ADAPTER.  Every wait is bounded as in the other tcgen05 kernels.

#include "lora_internal.cuh"
#include "tc_ptx.cuh"

namespace lora {
namespace {

constexpr int kLinThreads = 320;            // producer, MMA, 8 epilogue warps
constexpr int kLinEpiWarps = 8;
constexpr int kLN = 256;                    // outputs per unit (MMA N)
constexpr int kLStage = kAtom + kLN * 128;  // x (or s V) atom + W (or B) box: 48 KB
constexpr int kLStages = 4;
constexpr int kLNsBlock = 8;                // output slices per block of the unit order

struct LinUnit {
    int tile, ns;
};

// Unit u in the blocked order: block k holds every tile against slices
// 8k .. 8k + 7 (fewer in the last block), tile-major inside the block.
__device__ __forceinline__ LinUnit lin_unit(int64_t u, int n_tiles, int n_ns)
{
    const int64_t per_blk = (int64_t)n_tiles * kLNsBlock;
    const int blk = (int)(u / per_blk);
    const int64_t rem = u - blk * per_blk;
    const int nsb = min(kLNsBlock, n_ns - blk * kLNsBlock);
    LinUnit x;
    x.tile = (int)(rem / nsb);
    x.ns = blk * kLNsBlock + (int)(rem - (int64_t)x.tile * nsb);
    return x;
}

struct LinAd {
    int r;      // rank, 0: no LoRA k-blocks
    int brow;   // row of output 0 in the B view of rank r
    int m;      // that view's index
};

// The segment's adapter as the LoRA k-blocks use it.
__device__ LinAd lin_adapter(const LinArgs &p, int item, bool report)
{
    LinAd d = {0, 0, 0};
    const int32_t a = p.seg_ad[item];
    if (a == -1)
        return d;
    int32_t r = 0;
    int64_t ao = 0, bo = 0;
    bool ok = pool_adapter_ok(p.pool, a, &r, &ao, &bo);
    const int m = ok ? b_map(r) : -1;
    ok = ok && m >= 0 && ((p.b_tma >> m) & 1) && (bo % r) == 0;
    if (!ok) {
        if (report)
            atomicOr(p.err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        return d;
    }
    d.r = r;
    d.brow = (int)(bo / r);
    d.m = m;
    return d;
}

__device__ __forceinline__ int lora_kblocks(const LinAd &d) { return d.r ? 2 * ((d.r + 63) >> 6) : 0; }

__global__ void __launch_bounds__(kLinThreads, 1) k_tc_linear(const __grid_constant__ LinArgs p)
{
    extern __shared__ __align__(1024) unsigned char sm_dyn[];
    unsigned char *sm = reinterpret_cast<unsigned char *>((reinterpret_cast<uintptr_t>(sm_dyn) + 1023) & ~(uintptr_t)1023);
    __shared__ __align__(8) uint64_t full_bar[kLStages], empty_bar[kLStages];
    __shared__ __align__(8) uint64_t acc_full[2], acc_empty[2];
    __shared__ uint32_t tmem_base;
    __shared__ int abort_flag;

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int G = gridDim.x;
    const int n_kb = (p.d_in + kBK - 1) / kBK;
    const int n_ns = (p.d_out + kLN - 1) / kLN;

    if (tid == 0) {
        for (int s = 0; s < kLStages; ++s) {
            mbar_init(&full_bar[s], 1);          // producer's expect_tx
            mbar_init(&empty_bar[s], 1);         // MMA commit
        }
        for (int b = 0; b < 2; ++b) {
            mbar_init(&acc_full[b], 1);          // MMA commit
            mbar_init(&acc_empty[b], kLinEpiWarps);
        }
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
    const int64_t n_units = (int64_t)n_tiles * n_ns;

    if (warp == 0) {
        // ------------------------------------------------ producer
        int it = 0;
        const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
        for (int64_t u = blockIdx.x; u < n_units; u += G) {
            const LinUnit t = lin_unit(u, n_tiles, n_ns);
            const Group gr = p.groups[t.tile];
            const LinAd ad = lin_adapter(p, gr.item, lane == 0 && t.ns == 0);
            const int n_all = n_kb + lora_kblocks(ad);
            const int o0 = t.ns * kLN;
            const int w = ad.r < 64 ? ad.r : 64;          // B columns per LoRA k-block
            for (int kb = 0; kb < n_all; ++kb, ++it) {
                const int s = it % kLStages;
                const uint32_t ph = (it / kLStages) & 1;
                if (!warp_wait(&empty_bar[s], ph ^ 1, &abort_flag, p.err))
                    goto done;
                if (lane == 0) {
                    unsigned char *xs = sm + s * kLStage;
                    unsigned char *wsm = xs + kAtom;
                    if (kb < n_kb) {
                        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)kLStage);
                        tma_load_2d_hint(xs, &p.map_x, &full_bar[s], kb * kBK, gr.p0, pol_x);
                        tma_load_2d_hint(wsm, &p.map_w, &full_bar[s], kb * kBK, o0, pol_w);
                    } else {
                        // LoRA k-block j: part j % 2 (high, low) of rank columns 64 (j / 2) ..
                        const int j = kb - n_kb, part = j & 1, c = j >> 1;
                        mbar_arrive_expect_tx(&full_bar[s], (uint32_t)(kAtom + 2 * 128 * w * 2));
                        tma_load_2d_hint(xs, &p.map_v, &full_bar[s], part * p.kv + c * 64, gr.p0, pol_x);
                        tma_load_2d_hint(wsm, &p.map_b[ad.m], &full_bar[s], c * 64, ad.brow + o0, pol_w);
                        tma_load_2d_hint(wsm + 128 * w * 2, &p.map_b[ad.m], &full_bar[s], c * 64,
                                         ad.brow + o0 + 128, pol_w);
                    }
                }
                __syncwarp();
            }
        }
    } else if (warp == 1) {
        // ------------------------------------------------ MMA issuer
        int it = 0, t = 0;
        const uint32_t idesc = idesc_bf16(kBM, kLN);
        for (int64_t u = blockIdx.x; u < n_units; u += G, ++t) {
            const LinUnit un = lin_unit(u, n_tiles, n_ns);
            const LinAd ad = lin_adapter(p, p.groups[un.tile].item, false);
            const int n_all = n_kb + lora_kblocks(ad);
            const int steps = (ad.r < 64 ? ad.r : 64) >> 4;   // k16 steps of a LoRA k-block
            const int b = t & 1;
            if (!warp_wait(&acc_empty[b], ((t >> 1) & 1) ^ 1, &abort_flag, p.err))
                goto done;
            tc_fence_after();
            for (int kb = 0; kb < n_all; ++kb, ++it) {
                const int s = it % kLStages;
                const uint32_t ph = (it / kLStages) & 1;
                if (!warp_wait(&full_bar[s], ph, &abort_flag, p.err))
                    goto done;
                tc_fence_after();
                if (lane == 0) {
                    const uint32_t xa = smem_u32(sm + s * kLStage), wa = xa + kAtom;
                    if (kb < n_kb) {
#pragma unroll
                        for (int k = 0; k < kBK / 16; ++k)
                            tc_mma(tmem + b * kLN, sw128_desc(xa + k * 32), sw128_desc(wa + k * 32), idesc,
                                   (kb > 0 || k > 0) ? 1u : 0u);
                    } else {
                        for (int k = 0; k < steps; ++k) {
                            // B columns in the view's swizzle: 128-byte rows from rank 64 up,
                            // 64-byte rows at rank 32, 32-byte rows at rank 16
                            const uint64_t bdesc = ad.r >= 64 ? sw128_desc(wa + k * 32)
                                                 : (ad.r == 32 ? sw64_desc(wa + k * 32) : sw32_desc(wa));
                            tc_mma(tmem + b * kLN, sw128_desc(xa + k * 32), bdesc, idesc, 1u);
                        }
                    }
                    tc_commit(&empty_bar[s]);
                }
                __syncwarp();
            }
            if (lane == 0)
                tc_commit(&acc_full[b]);
            __syncwarp();
        }
    } else {
        // ------------------------------------------------ epilogue: D -> y rows
        const int e = warp - 2;                  // 0..7
        const int q = warp & 3;                  // TMEM lane quarter this warp may read
        const int h = e >> 2;                    // 128-column half of the slice
        const int row = q * 32 + lane;
        int t = 0;
        for (int64_t u = blockIdx.x; u < n_units; u += G, ++t) {
            const LinUnit un = lin_unit(u, n_tiles, n_ns);
            const Group gr = p.groups[un.tile];
            const int b = t & 1;
            if (!warp_wait(&acc_full[b], (t >> 1) & 1, &abort_flag, p.err))
                goto done;
            tc_fence_after();
            const bool valid = row < gr.cnt;
            __nv_bfloat16 *yrow = p.Y + (int64_t)(gr.p0 + (valid ? row : 0)) * p.ldy;
            const int o0 = un.ns * kLN + h * 128;
#pragma unroll 1
            for (int c0 = 0; c0 < 128; c0 += 32) {
                float v[32];
                tmem_ld32(tmem + b * kLN + ((uint32_t)(q * 32) << 16) + h * 128 + c0, v);
                if (valid) {
#pragma unroll
                    for (int g = 0; g < 4; ++g) {
                        const int o = o0 + c0 + 8 * g;
                        if (o < p.d_out) {
                            uint32_t w4[4];
#pragma unroll
                            for (int j = 0; j < 4; ++j) {
                                const __nv_bfloat162 hv = __floats2bfloat162_rn(v[8 * g + 2 * j], v[8 * g + 2 * j + 1]);
                                w4[j] = *reinterpret_cast<const uint32_t *>(&hv);
                            }
                            *reinterpret_cast<uint4 *>(yrow + o) = make_uint4(w4[0], w4[1], w4[2], w4[3]);
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

cudaError_t launch_tc_linear(const LinArgs &a, int max_units, cudaStream_t s)
{
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
