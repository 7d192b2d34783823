// Device and host helpers shared by the tcgen05 kernels: mbarriers with
// bounded waits, TMA loads with L2 hints, TMEM allocation, tcgen05 MMA issue,
// commit and load, shared-memory matrix descriptors, programmatic dependent
// launch, and tensor-map encoding.  Everything sits in an unnamed namespace, so
// each kernel file keeps its own copy.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora_sgmv.h"

namespace lora {
namespace {

// B-pool TMA views: map_b[m] sees the pool as [B_elems / r, r] for r = 16 << m, so
// adapter a's output o is row B_off[a] / r + o when B_off[a] is a multiple of r
__host__ __device__ constexpr int b_map(int r) { return r == 16 ? 0 : (r == 32 ? 1 : (r == 64 ? 2 : (r == 128 ? 3 : -1))); }
constexpr int kBM = 128;            // rows per tile
constexpr int kBK = 64;             // d_in per k-block (one 128-byte swizzle atom)
constexpr int kAtom = kBM * 128;    // bytes of a 128-row x 64-column bf16 swizzle atom

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
// is already aborting or `limit_ns` passes (then it marks the abort itself).
__device__ __forceinline__ bool mbar_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag,
                                          uint32_t *err, unsigned long long limit_ns)
{
    if (mbar_try_wait(bar, parity))
        return true;
    const unsigned long long t0 = now_ns();
    for (uint32_t i = 1;; ++i) {
        if (mbar_try_wait(bar, parity))
            return true;
        if ((i & 63) == 0) {
            if (*abort_flag)
                return false;
            if (now_ns() - t0 > limit_ns) {
                *abort_flag = 1;
                atomicOr(err, (uint32_t)LORA_ERR_TIMEOUT);
                return false;
            }
        }
    }
}

// The whole warp waits; all lanes leave together (all succeed or all give up).
__device__ __forceinline__ bool warp_wait(uint64_t *bar, uint32_t parity, volatile int *abort_flag, uint32_t *err,
                                          unsigned long long limit_ns)
{
    return __all_sync(0xffffffffu, mbar_wait(bar, parity, abort_flag, err, limit_ns));
}

// Before a CTA that gave up may exit: every fill of a ring of `n_stages` barriers
// issued so far (fills 0 .. issued-1, fill i on barrier i % n_stages) must have
// landed, whether or not a consumer got to it.  Bounded like every wait.
__device__ __forceinline__ void drain_fills(uint64_t *bars, int n_stages, int issued, uint32_t *err,
                                            unsigned long long limit_ns)
{
    for (int i = issued > n_stages ? issued - n_stages : 0; i < issued; ++i) {
        const unsigned long long t0 = now_ns();
        while (!mbar_try_wait(&bars[i % n_stages], (uint32_t)((i / n_stages) & 1))) {
            if (now_ns() - t0 > limit_ns) {
                atomicOr(err, (uint32_t)LORA_ERR_TIMEOUT);
                break;
            }
        }
    }
}

// Before TMEM is freed: every tcgen05.mma this thread issued has completed
// (a commit to `bar`, a fresh phase of a barrier of count 1).  Bounded.
__device__ __forceinline__ void drain_mma(uint64_t *bar, uint32_t parity, uint32_t *err, unsigned long long limit_ns)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_u32(bar))
                 : "memory");
    const unsigned long long t0 = now_ns();
    while (!mbar_try_wait(bar, parity)) {
        if (now_ns() - t0 > limit_ns) {
            atomicOr(err, (uint32_t)LORA_ERR_TIMEOUT);
            break;
        }
    }
}

__device__ __forceinline__ void st_shared_v4(uint32_t addr, uint32_t a, uint32_t b, uint32_t c, uint32_t d)
{
    asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};" ::"r"(addr), "r"(a), "r"(b), "r"(c), "r"(d) : "memory");
}

__device__ __forceinline__ void ld_shared_v4(uint32_t addr, uint32_t (&w)[4])
{
    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];" : "=r"(w[0]), "=r"(w[1]), "=r"(w[2]), "=r"(w[3]) : "r"(addr)
                 : "memory");
}

// TMA load of a 2-D box into shared memory, completing on `bar`, with an L2
// eviction-priority hint (a createpolicy value).
__device__ __forceinline__ void tma_load_2d_hint(void *dst, const CUtensorMap *map, uint64_t *bar, int x, int y,
                                                 uint64_t policy)
{
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint"
        " [%0], [%1, {%3, %4}], [%2], %5;"
        ::"r"(smem_u32(dst)), "l"(map), "r"(smem_u32(bar)), "r"(x), "r"(y), "l"(policy)
        : "memory");
}

// L2 policies: streamed data (x, y) leaves L2 first, adapter weights (re-read by
// every tile of a segment) last.
__device__ __forceinline__ uint64_t policy_evict_first()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ uint64_t policy_evict_last()
{
    uint64_t pol;
    asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
    return pol;
}

__device__ __forceinline__ void st_global_v4_hint(void *ptr, uint32_t a, uint32_t b, uint32_t c, uint32_t d,
                                                  uint64_t policy)
{
    asm volatile("st.global.L1::no_allocate.L2::cache_hint.v4.b32 [%0], {%1,%2,%3,%4}, %5;" ::"l"(ptr), "r"(a),
                 "r"(b), "r"(c), "r"(d), "l"(policy)
                 : "memory");
}

// Programmatic dependent launch: wait until the previous kernel on the stream has
// completed (its writes visible), then let the next one start its prologue.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

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

// The same for the 64- and 32-byte swizzles (8-row groups 512 / 256 bytes apart).
__device__ __forceinline__ uint64_t sw64_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(512 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)4 << 61);
}

__device__ __forceinline__ uint64_t sw32_desc(uint32_t saddr)
{
    return (uint64_t)((saddr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) | ((uint64_t)(256 >> 4) << 32) |
           ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}

// Instruction descriptor: bf16 A and B, fp32 D, both K-major, M x N.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N)
{
    return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// byte offset of 16-byte chunk c (0..7) of row i inside a 128-byte-swizzle atom
__device__ __forceinline__ uint32_t sw128_off(int i, int c) { return (uint32_t)(i * 128 + ((c ^ (i & 7)) << 4)); }

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
// columns x box_rows rows, 128-byte swizzle, zero fill outside the matrix.
bool encode_box(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld, int box_rows)
{
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return false;
    const cuuint64_t dims[2] = {(cuuint64_t)cols, (cuuint64_t)rows};
    const cuuint64_t strides[1] = {(cuuint64_t)ld * 2};
    const cuuint32_t box[2] = {64, (cuuint32_t)box_rows};
    const cuuint32_t estr[2] = {1, 1};
    return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(base), dims, strides, box, estr,
              CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool encode_rows(CUtensorMap *m, const void *base, int64_t rows, int64_t cols, int64_t ld)
{
    return encode_box(m, base, rows, cols, ld, 128);
}

// The B pool seen as [B_elems / r, r] for r = 16, 32, 64, 128 (maps[m], r = 16 << m):
// boxes of 128 rows (outputs) x min(r, 64) columns, swizzled to the row width.
// Returns the bit mask of the views that could be encoded.
int encode_b_views(CUtensorMap *maps, const void *B, int64_t B_elems)
{
    int mask = 0;
    EncodeTiledFn fn = encode_fn();
    if (!fn)
        return 0;
    for (int m = 0; m < 4; ++m) {
        const int r = 16 << m;
        const int64_t rows = B_elems / r;
        if (rows < 1 || rows > 0x7fffffffLL)
            continue;
        const cuuint64_t dims[2] = {(cuuint64_t)r, (cuuint64_t)rows};
        const cuuint64_t strides[1] = {(cuuint64_t)r * 2};
        const cuuint32_t box[2] = {(cuuint32_t)(r < 64 ? r : 64), 128};
        const cuuint32_t estr[2] = {1, 1};
        const CUtensorMapSwizzle sw = r == 16 ? CU_TENSOR_MAP_SWIZZLE_32B
                                    : (r == 32 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B);
        if (fn(&maps[m], CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(B), dims, strides, box, estr,
               CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS)
            mask |= 1 << m;
    }
    return mask;
}

int sm_count()
{
    int dev = 0, n = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess)
        return 148;
    return n;
}

}  // namespace
}  // namespace lora
