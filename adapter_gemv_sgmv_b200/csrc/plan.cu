// Grouping of a batch by adapter and construction of the work-group list.
//
// "Serving several LoRAs, ControlNet and IP-Adapter", exercise 2's answer: a
// stable counting sort of the tokens by adapter id, one kernel over all the
// resulting runs, and the results scattered back to token order.  For an
// unsorted decode batch the sort is histogram -> exclusive scan -> stable
// scatter.  Prefill segments and multi-adapter
// requests arrive already grouped; the plan kernel only validates their
// offsets.  In every mode it then cuts each item (segment / request) into
// work groups of at most `group` tokens.
//
// One CTA of 1024 threads does everything: the decode batches this serves
// hold hundreds to a few thousand tokens, and one CTA keeps the histogram in
// shared memory and needs no grid-wide synchronisation.

#include "lora_internal.cuh"

namespace lora {
namespace {

constexpr int kPlanThreads = 1024;

// Exclusive scan over i in [0, L) of f(i) with every thread of the block.
// Calls out(i, prefix, f(i)) in order of i within each thread's contiguous
// slice; returns the total.  f must be pure while the scan runs except for
// what out() itself changes at index i after f(i) was read.
template <class T, class F, class O>
__device__ T block_scan(int L, F f, O out, T *sm /* 33 entries */)
{
    const int nt = blockDim.x;
    const int per = (L + nt - 1) / nt;
    const int b = threadIdx.x * per;
    const int e = min(L, b + per);
    T local = 0;
    for (int i = b; i < e; ++i)
        local += f(i);
    const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
    T incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
        T v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off)
            incl += v;
    }
    if (lane == 31)
        sm[w] = incl;
    __syncthreads();
    if (w == 0) {
        const int nw = nt >> 5;
        T v = lane < nw ? sm[lane] : T(0);
        T iv = v;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
            T u = __shfl_up_sync(0xffffffffu, iv, off);
            if (lane >= off)
                iv += u;
        }
        if (lane < nw)
            sm[lane] = iv - v;
        if (lane == nw - 1)
            sm[32] = iv;
    }
    __syncthreads();
    T run = sm[w] + incl - local;
    for (int i = b; i < e; ++i) {
        T v = f(i);
        out(i, run, v);
        run += v;
    }
    T total = sm[32];
    __syncthreads();
    return total;
}

__global__ void __launch_bounds__(kPlanThreads) k_plan(PlanArgs p)
{
    extern __shared__ int32_t hist[];   // [n_adapters] (route mode only)
    __shared__ long long sm_scan[33];
    __shared__ int32_t sm_flag;
    // programmatic dependent launch: the previous kernel on the stream (which may
    // produce this call's inputs or still read the workspace) completes first
    asm volatile("griddepcontrol.wait;" ::: "memory");
    asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
    const int tid = threadIdx.x;
    const int32_t N = p.N;
    const int32_t *item_off = p.item_off;
    int32_t n_items = p.n_items;

    if (tid == 0)
        sm_flag = 0;
    __syncthreads();

    if (p.mode == kModeRoute) {
        const int32_t n_ad = p.n_adapters;
        for (int a = tid; a < n_ad; a += blockDim.x)
            hist[a] = 0;
        __syncthreads();
        for (int n = tid; n < N; n += blockDim.x) {
            const int32_t a = p.ids[n];
            if (a >= 0 && a < n_ad)
                atomicAdd(&hist[a], 1);
            else if (a != -1)
                sm_flag = 1;
        }
        __syncthreads();
        if (tid == 0 && sm_flag)
            atomicOr(&p.hdr->err, (uint32_t)LORA_ERR_BAD_ADAPTER);
        // one scan gives both the start of each adapter's run (high word) and
        // the index of its segment among the adapters present (low word)
        int32_t *seg_off = p.seg_off;
        int32_t *seg_ad = p.seg_ad;
        long long tot = block_scan<long long>(
            n_ad,
            [&](int a) { return ((long long)hist[a] << 32) | (long long)(hist[a] > 0); },
            [&](int a, long long pre, long long v) {
                const int32_t start = (int32_t)(pre >> 32);
                if (v != 0) {
                    const int32_t k = (int32_t)(pre & 0xffffffffll);
                    seg_ad[k] = a;
                    seg_off[k] = start;
                }
                hist[a] = start;   // becomes the scatter cursor
            },
            sm_scan);
        const int32_t n_seg = (int32_t)(tot & 0xffffffffll);
        const int32_t n_valid = (int32_t)(tot >> 32);
        if (tid == 0) {
            seg_off[n_seg] = n_valid;
            p.hdr->n_seg = n_seg;
            if (p.n_seg_out)
                *p.n_seg_out = n_seg;
        }
        // stable scatter: one warp walks the tokens in order, 32 at a time;
        // equal ids inside a step are ranked by lane, and the cursor of each
        // id advances once per step by its multiplicity.
        if (tid < 32) {
            const int lane = tid;
            for (int base = 0; base < N; base += 32) {
                const int n = base + lane;
                const int32_t a = n < N ? p.ids[n] : -1;
                const bool valid = n < N && a >= 0 && a < n_ad;
                const int32_t key = valid ? a : -1;
                const unsigned peers = __match_any_sync(0xffffffffu, key);
                if (valid) {
                    const int r = __popc(peers & ((1u << lane) - 1u));
                    p.perm[hist[a] + r] = n;
                }
                __syncwarp();
                if (valid && (peers >> lane) == 1u)
                    hist[a] += __popc(peers);
                __syncwarp();
            }
        }
        __syncthreads();
        item_off = seg_off;
        n_items = n_seg;
    } else {
        // caller's segments / requests: non-decreasing, within [0, N]
        for (int k = tid; k < n_items; k += blockDim.x) {
            const int32_t lo = item_off[k], hi = item_off[k + 1];
            if (lo < 0 || hi < lo || hi > N)
                sm_flag = 1;
            if (p.mode == kModeMulti) {
                const int32_t c = p.ad_off[k + 1] - p.ad_off[k];
                if (c < 0 || c > p.max_ads || p.ad_off[k] < 0)
                    sm_flag = 1;
            }
        }
        __syncthreads();
        if (sm_flag) {
            if (tid == 0) {
                atomicOr(&p.hdr->err, (uint32_t)LORA_ERR_BAD_SEGMENT);
                p.hdr->n_groups = 0;
            }
            return;
        }
    }

    // cut every item into groups of at most p.group tokens
    Group *groups = p.groups;
    const int32_t max_groups = p.max_groups;
    const int32_t G = p.group;
    long long total = block_scan<long long>(
        n_items,
        [&](int k) { return (long long)((item_off[k + 1] - item_off[k] + G - 1) / G); },
        [&](int k, long long pre, long long v) {
            const int32_t lo = item_off[k], hi = item_off[k + 1];
            for (int32_t i = 0; i < (int32_t)v; ++i) {
                const long long g = pre + i;
                if (g < max_groups) {
                    Group gr;
                    gr.p0 = lo + i * G;
                    gr.cnt = min(G, hi - gr.p0);
                    gr.item = k;
                    gr.pad = 0;
                    groups[g] = gr;
                }
            }
        },
        sm_scan);
    if (tid == 0) {
        if (total > max_groups) {
            atomicOr(&p.hdr->err, (uint32_t)LORA_ERR_BAD_SEGMENT);
            total = max_groups;
        }
        p.hdr->n_groups = (int32_t)total;
    }
}

}  // namespace

size_t plan_smem_bytes(int32_t mode, int32_t n_adapters)
{
    return mode == kModeRoute ? (size_t)n_adapters * sizeof(int32_t) : 0;
}

cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s)
{
    const size_t smem = plan_smem_bytes(a.mode, a.n_adapters);
    // the opt-in shared-memory limit is a per-device function attribute;
    // setting it twice is harmless, so racing first calls are fine
    static bool attr_set[64] = {};
    int dev = 0;
    cudaError_t e = cudaGetDevice(&dev);
    if (e != cudaSuccess)
        return e;
    if (dev < 0 || dev >= 64 || !attr_set[dev]) {
        e = cudaFuncSetAttribute(k_plan, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                 (int)(LORA_MAX_ADAPTERS * sizeof(int32_t)));
        if (e != cudaSuccess)
            return e;
        if (dev >= 0 && dev < 64)
            attr_set[dev] = true;
    }
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(1);
    cfg.blockDim = dim3(kPlanThreads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = s;
    cfg.attrs = attr;
    cfg.numAttrs = pdl_enabled() ? 1 : 0;
    return cudaLaunchKernelEx(&cfg, k_plan, a);
}

}  // namespace lora
