// lora_apply_multi_static: lora_apply_multi for callers that cannot allocate
// device memory.
//
// Some callers may not call cudaMalloc at all: code running inside a region
// that is being captured into a CUDA graph where allocation is forbidden, a
// host that runs under a device-memory budget owned by another allocator, or
// a plugin whose host framework gives it only the input and output buffers.
// They cannot provide the workspace lora_apply_multi needs.  This variant runs
// the same three kernels (plan, shrink, expand) but takes its scratch from a
// fixed array compiled into the library instead of from the caller.

#include <mutex>

#include "lora_internal.cuh"

using namespace lora;

namespace {

// The scratch every call of lora_apply_multi_static shares: its work-group list,
// error word and fp32 rank-r intermediate.  Every GPU that loads the library
// holds these bytes until the process exits.
constexpr size_t kStaticScratchBytes = LORA_STATIC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_static_scratch[kStaticScratchBytes];

// The array's device address, looked up once per device.  In host code the name
// g_static_scratch is only a host-side stand-in; a kernel handed it would fault
// or read the wrong memory.
std::mutex g_setup_mu;
void *g_scratch_ptr[64] = {};

cudaError_t scratch_for_current_device(void **out)
{
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64)
        return cudaErrorInvalidDevice;
    std::lock_guard<std::mutex> lock(g_setup_mu);
    if (!g_scratch_ptr[dev]) {
        void *p = nullptr;
        e = cudaGetSymbolAddress(&p, g_static_scratch);
        if (e != cudaSuccess)
            return e;
        g_scratch_ptr[dev] = p;
    }
    *out = g_scratch_ptr[dev];
    return cudaSuccess;
}

size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

}  // namespace

extern "C" lora_status lora_apply_multi_static(const void *X, int64_t ldx, void *Y, int64_t ldy,
                                               const lora_pool *p, const int32_t *req_off,
                                               const int32_t *ad_off, const int32_t *ad_id,
                                               const float *ad_scale, int32_t n_req, int32_t N,
                                               int32_t max_ads_per_req, uint32_t *err_out, void *stream)
{
    // argument checks: the same rules as lora_apply_multi
    if (!p || !p->A || !p->B || !p->A_off || !p->B_off || !p->rank || p->A_elems < 0 || p->B_elems < 0)
        return LORA_ERR_INVALID_ARG;
    if (p->n_adapters < 1 || p->n_adapters > LORA_MAX_ADAPTERS || p->d_in <= 0 || p->d_out <= 0 ||
        (p->d_in & 7) || (p->d_out & 7) || p->max_rank < 8 || p->max_rank > LORA_MAX_RANK || (p->max_rank & 7) ||
        ((uintptr_t)p->A & 15) || ((uintptr_t)p->B & 15))
        return LORA_ERR_UNSUPPORTED;
    if (N < 0 || n_req < 0 || !req_off || !ad_off || (n_req > 0 && (!ad_id || !ad_scale)))
        return LORA_ERR_INVALID_ARG;
    if (max_ads_per_req < 1 || max_ads_per_req > LORA_MAX_ADS_PER_REQ)
        return LORA_ERR_UNSUPPORTED;
    if ((N > 0 && (!X || !Y)) || ldx < p->d_in || ldy < p->d_out)
        return LORA_ERR_INVALID_ARG;
    if ((ldx & 7) || (ldy & 7) || ((uintptr_t)X & 15) || ((uintptr_t)Y & 15))
        return LORA_ERR_UNSUPPORTED;

    // the scratch this call needs, laid out like lora_apply_multi's workspace
    const int32_t max_groups = (int32_t)((int64_t)N / kGroup + n_req + 1);
    const size_t off_groups = align256(sizeof(WsHeader));
    const size_t off_V = align256(off_groups + (size_t)max_groups * sizeof(Group));
    const size_t need = align256(off_V + (size_t)N * max_ads_per_req * p->max_rank * sizeof(float));
    if (need > kStaticScratchBytes)
        return LORA_ERR_WORKSPACE;   // beyond the fixed scratch: use lora_apply_multi with a workspace

    cudaStream_t s = (cudaStream_t)stream;
    void *base = nullptr;
    if (scratch_for_current_device(&base) != cudaSuccess)
        return LORA_ERR_CUDA;
    char *ws = static_cast<char *>(base);
    WsHeader *hdr = reinterpret_cast<WsHeader *>(ws);
    Group *groups = reinterpret_cast<Group *>(ws + off_groups);
    float *V = reinterpret_cast<float *>(ws + off_V);

    // the previous call's contents stay in the array: only the header (error
    // word, counters) must start at zero; groups and V are written before read
    if (cudaMemsetAsync(hdr, 0, sizeof(WsHeader), s) != cudaSuccess)
        return LORA_ERR_CUDA;
    if (N > 0 && n_req > 0) {
        PoolDev pd;
        pd.A = static_cast<const __nv_bfloat16 *>(p->A);
        pd.B = static_cast<const __nv_bfloat16 *>(p->B);
        pd.A_off = p->A_off;
        pd.B_off = p->B_off;
        pd.rank = p->rank;
        pd.A_elems = p->A_elems;
        pd.B_elems = p->B_elems;
        pd.n_adapters = p->n_adapters;
        pd.max_rank = p->max_rank;
        pd.d_in = p->d_in;
        pd.d_out = p->d_out;
        const int32_t ldv = max_ads_per_req * p->max_rank;

        PlanArgs pa = {};
        pa.mode = kModeMulti;
        pa.N = N;
        pa.item_off = req_off;
        pa.n_items = n_req;
        pa.ad_off = ad_off;
        pa.max_ads = max_ads_per_req;
        pa.groups = groups;
        pa.max_groups = max_groups;
        pa.group = kGroup;
        pa.hdr = hdr;
        if (launch_plan(pa, s) != cudaSuccess)
            return LORA_ERR_CUDA;

        ShrinkArgs sa = {};
        sa.X = static_cast<const __nv_bfloat16 *>(X);
        sa.ldx = ldx;
        sa.perm = nullptr;
        sa.groups = groups;
        sa.hdr = hdr;
        sa.mode = kModeMulti;
        sa.ad_off = ad_off;
        sa.ad_id = ad_id;
        sa.pool = pd;
        sa.kc = p->d_in;
        sa.V = V;
        sa.ldv = ldv;
        sa.chunk_stride = 0;
        sa.slot_stride = p->max_rank;
        sa.err = &hdr->err;
        if (launch_shrink(sa, max_groups, 1, max_ads_per_req, s) != cudaSuccess)
            return LORA_ERR_CUDA;

        ExpandArgs ea = {};
        ea.Y = static_cast<__nv_bfloat16 *>(Y);
        ea.ldy = ldy;
        ea.perm = nullptr;
        ea.groups = groups;
        ea.hdr = hdr;
        ea.mode = kModeMulti;
        ea.ad_off = ad_off;
        ea.ad_id = ad_id;
        ea.ad_scale = ad_scale;
        ea.scale = 1.0f;
        ea.pool = pd;
        ea.V = V;
        ea.ldv = ldv;
        ea.chunk_stride = 0;
        ea.n_chunks = 1;
        ea.slot_stride = p->max_rank;
        ea.max_ads = max_ads_per_req;
        ea.err = &hdr->err;
        if (launch_expand(ea, max_groups, s) != cudaSuccess)
            return LORA_ERR_CUDA;
    }
    if (err_out && cudaMemcpyAsync(err_out, &hdr->err, sizeof(uint32_t), cudaMemcpyDeviceToDevice, s) != cudaSuccess)
        return LORA_ERR_CUDA;
    return LORA_OK;
}
