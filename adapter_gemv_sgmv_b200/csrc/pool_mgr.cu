// Resident adapter pool with on-demand loads ("Serving several LoRAs, ControlNet and
// IP-Adapter", section "Placement": the LoRAs in use stay resident on the GPU; the
// rest wait in host memory and are brought in when a batch needs them).
//
// The caller owns the pool's device storage (a lora_pool of n_slots fixed-size
// slots); the manager keeps the host side -- the registry of host copies by key and
// the slot policy (SlotCache: keys of a batch stay or come in, least recently used
// slots not needed by the batch make room) -- and issues the host -> device copies
// and the rank updates on the caller's stream, so kernels later on that stream see
// the batch's adapters in place.

#include <algorithm>
#include <mutex>
#include <unordered_map>
#include <unordered_set>
#include <vector>

#include "lora_internal.cuh"
#include "slot_cache.h"

using namespace lora;

namespace {

__global__ void k_pm_init(int64_t *A_off, int64_t *B_off, int32_t *rank, int32_t n_slots, int64_t a_slot,
                          int64_t b_slot)
{
    for (int s = blockIdx.x * blockDim.x + threadIdx.x; s < n_slots; s += gridDim.x * blockDim.x) {
        A_off[s] = (int64_t)s * a_slot;
        B_off[s] = (int64_t)s * b_slot;
        rank[s] = 0;              // empty: the kernels reject it as an adapter
    }
}

// slot's rank, written in stream order after its copies (the value travels as an argument)
__global__ void k_pm_set_rank(int32_t *rank, int32_t slot, int32_t r) { rank[slot] = r; }

struct HostAdapter {
    const void *A;
    const void *B;
    int32_t rank;
};

}  // namespace

struct lora_pool_mgr;
static bool copy_in(lora_pool_mgr *m, const std::vector<std::pair<int, int64_t>> &loads, cudaStream_t st);

struct lora_pool_mgr {
    std::mutex mu;
    lora_pool pool;               // the caller's device storage
    int64_t a_slot, b_slot;       // elements per slot
    SlotCache cache;
    std::unordered_map<int64_t, HostAdapter> reg;
    std::vector<int32_t> slot_rank;
    CoOccurrence co;              // requests' adapter sets seen so far
    int32_t top_k = 0;            // partners of each acquired key preloaded (0: off)
    int32_t preloaded = 0;        // adapters the last acquire preloaded

    explicit lora_pool_mgr(const lora_pool &p)
        : pool(p), a_slot((int64_t)p.max_rank * p.d_in), b_slot((int64_t)p.d_out * p.max_rank),
          cache(p.n_adapters), slot_rank(p.n_adapters, 0) {}
};

// Copies (slot, key) pairs in on `st`: A, B, then the slot's rank.  On a failed
// copy the failing key and every later one are rolled back (not resident).
static bool copy_in(lora_pool_mgr *m, const std::vector<std::pair<int, int64_t>> &loads, cudaStream_t st)
{
    char *A = static_cast<char *>(const_cast<void *>(m->pool.A));
    char *B = static_cast<char *>(const_cast<void *>(m->pool.B));
    for (size_t i = 0; i < loads.size(); ++i) {
        const int slot = loads[i].first;
        const HostAdapter &h = m->reg[loads[i].second];
        const size_t a_bytes = (size_t)h.rank * m->pool.d_in * 2, b_bytes = (size_t)m->pool.d_out * h.rank * 2;
        cudaError_t e = cudaMemcpyAsync(A + (size_t)slot * m->a_slot * 2, h.A, a_bytes, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess)
            e = cudaMemcpyAsync(B + (size_t)slot * m->b_slot * 2, h.B, b_bytes, cudaMemcpyHostToDevice, st);
        if (e == cudaSuccess) {
            k_pm_set_rank<<<1, 1, 0, st>>>(const_cast<int32_t *>(m->pool.rank), slot, h.rank);
            e = cudaGetLastError();
        }
        if (e != cudaSuccess) {
            m->cache.rollback(loads, i);
            return false;
        }
        m->slot_rank[slot] = h.rank;
    }
    return true;
}

extern "C" {

lora_status lora_pm_create(const lora_pool *storage, void *stream, lora_pool_mgr **out)
{
    if (!out)
        return LORA_ERR_INVALID_ARG;
    *out = nullptr;
    if (!storage || !storage->A || !storage->B || !storage->A_off || !storage->B_off || !storage->rank)
        return LORA_ERR_INVALID_ARG;
    const lora_pool &p = *storage;
    if (p.n_adapters < 1 || p.n_adapters > LORA_MAX_ADAPTERS || p.d_in <= 0 || p.d_out <= 0 || (p.d_in & 7) ||
        (p.d_out & 7) || p.max_rank < 8 || p.max_rank > LORA_MAX_RANK || (p.max_rank & 7) ||
        ((uintptr_t)p.A & 15) || ((uintptr_t)p.B & 15))
        return LORA_ERR_UNSUPPORTED;
    const int64_t a_need = (int64_t)p.n_adapters * p.max_rank * p.d_in;
    const int64_t b_need = (int64_t)p.n_adapters * p.d_out * p.max_rank;
    if (p.A_elems < a_need || p.B_elems < b_need)
        return LORA_ERR_INVALID_ARG;
    lora_pool_mgr *m = new lora_pool_mgr(p);
    const int blocks = (p.n_adapters + 255) / 256;
    k_pm_init<<<blocks, 256, 0, (cudaStream_t)stream>>>(const_cast<int64_t *>(p.A_off),
                                                        const_cast<int64_t *>(p.B_off),
                                                        const_cast<int32_t *>(p.rank), p.n_adapters, m->a_slot,
                                                        m->b_slot);
    if (cudaGetLastError() != cudaSuccess) {
        delete m;
        return LORA_ERR_CUDA;
    }
    *out = m;
    return LORA_OK;
}

void lora_pm_destroy(lora_pool_mgr *m) { delete m; }

lora_status lora_pm_register(lora_pool_mgr *m, int64_t key, const void *A_host, const void *B_host, int32_t rank)
{
    if (!m || key < 0 || !A_host || !B_host)
        return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(m->mu);
    if (rank < 8 || rank > m->pool.max_rank || (rank & 7))
        return LORA_ERR_UNSUPPORTED;
    m->reg[key] = HostAdapter{A_host, B_host, rank};
    m->cache.drop(key);           // a new host copy: the next batch that needs it reloads it
    return LORA_OK;
}

lora_status lora_pm_acquire(lora_pool_mgr *m, const int64_t *keys, int32_t n, int32_t *slots, int32_t *n_loaded,
                            void *stream)
{
    if (!m || n < 0 || (n > 0 && !keys))
        return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(m->mu);
    for (int32_t i = 0; i < n; ++i)
        if (m->reg.find(keys[i]) == m->reg.end())
            return LORA_ERR_INVALID_ARG;   // unregistered key: nothing changes
    std::vector<int> s(n > 0 ? n : 1);
    std::vector<std::pair<int, int64_t>> loads;
    if (!m->cache.assign(keys, n, s.data(), &loads))
        return LORA_ERR_UNSUPPORTED;       // more distinct keys than slots: nothing changes
    cudaStream_t st = (cudaStream_t)stream;
    if (!copy_in(m, loads, st))
        return LORA_ERR_CUDA;
    m->preloaded = 0;
    if (m->top_k > 0) {
        // the top-k co-occurring partners of the batch's keys, registered and not in
        // the batch, in order of first appearance, come in while slots allow
        std::vector<int64_t> want, partners;
        std::unordered_set<int64_t> in_batch(keys, keys + n);
        for (int32_t i = 0; i < n; ++i) {
            if (i > 0 && std::find(keys, keys + i, keys[i]) != keys + i)
                continue;
            m->co.top(keys[i], m->top_k, &partners);
            for (int64_t p : partners)
                if (!in_batch.count(p) && m->reg.count(p) && std::find(want.begin(), want.end(), p) == want.end())
                    want.push_back(p);
        }
        std::vector<std::pair<int, int64_t>> pre;
        m->cache.preload(want.data(), (int)want.size(), &pre);
        if (!copy_in(m, pre, st))
            return LORA_ERR_CUDA;
        m->preloaded = (int32_t)pre.size();
    }
    if (slots)
        for (int32_t i = 0; i < n; ++i)
            slots[i] = s[i];
    if (n_loaded)
        *n_loaded = (int32_t)loads.size();
    return LORA_OK;
}

lora_status lora_pm_observe(lora_pool_mgr *m, const int64_t *keys, int32_t n)
{
    if (!m || n < 0 || (n > 0 && !keys))
        return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(m->mu);
    m->co.observe(keys, n);
    return LORA_OK;
}

lora_status lora_pm_set_preload(lora_pool_mgr *m, int32_t top_k)
{
    if (!m || top_k < 0)
        return LORA_ERR_INVALID_ARG;
    std::lock_guard<std::mutex> lock(m->mu);
    m->top_k = top_k;
    return LORA_OK;
}

int32_t lora_pm_preloaded(lora_pool_mgr *m)
{
    if (!m)
        return -1;
    std::lock_guard<std::mutex> lock(m->mu);
    return m->preloaded;
}

}  // extern "C"
