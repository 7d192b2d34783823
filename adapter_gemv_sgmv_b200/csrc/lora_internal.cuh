// Internal declarations shared by the kernel files and the C-ABI layer.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include "lora_sgmv.h"

namespace lora {

constexpr int kMaxRank = LORA_MAX_RANK;
constexpr int kGroup = 8;            // tokens per work group in the CUDA-core kernels
constexpr int kThreads = 128;        // threads per CTA of the CUDA-core kernels
constexpr int kStageK = 1024;        // d_in elements of X staged in shared memory at a time
constexpr int kExpandPerThread = 8;  // consecutive outputs per thread in the expand
constexpr int kExpandTile = kThreads * kExpandPerThread;
constexpr int kBgmvChunk = 512;      // split of d_in across CTAs in the decode shrink

constexpr unsigned long long kWaitBoundNs = 2000000000ull;   // bound of any single wait in a kernel (2 s)

// Head of every workspace (256 bytes).
struct WsHeader {
    uint32_t err;       // device error bits (lora_status values), sticky until lora_get_error
    int32_t n_seg;      // distinct adapters found by the grouping
    int32_t n_groups;   // work groups written by the plan kernel
    uint32_t sched[2];  // decode kernel: next item position handed out, clusters finished
                        // (both back to zero when the launch ends)
    int32_t pad[59];
};
static_assert(sizeof(WsHeader) == 256, "header is 256 bytes");

// A run of at most kGroup tokens that share one item (segment or request).
// Tokens are positions p0 .. p0+cnt-1: row indices, or indices into perm.
struct Group {
    int32_t p0, cnt, item, pad;
};

enum Mode : int32_t { kModeRoute = 0, kModeSgmv = 1, kModeMulti = 2, kModeProj = 3 };

// ---------------------------------------------------------------- plan kernel
struct PlanArgs {
    int32_t mode;
    int32_t N;
    // route (decode): unsorted ids
    const int32_t *ids;
    int32_t n_adapters;
    int32_t *perm;       // out [N]
    int32_t *seg_off;    // out [min(N, n_adapters) + 1]
    int32_t *seg_ad;     // out [min(N, n_adapters)]
    int32_t *n_seg_out;  // optional out
    // sgmv: caller's segments; multi: caller's requests
    const int32_t *item_off;  // [n_items + 1]
    int32_t n_items;
    const int32_t *ad_off;    // multi only: adapter list bounds
    int32_t max_ads;
    // groups
    Group *groups;
    int32_t max_groups;
    int32_t group;            // tokens per group (kGroup for the CUDA-core kernels, 128 for tcgen05)
    WsHeader *hdr;
};

// ----------------------------------------------------------- CUDA-core kernels
// Device view of one projection's adapter pool.
struct PoolDev {
    const __nv_bfloat16 *A;
    const __nv_bfloat16 *B;
    const int64_t *A_off;
    const int64_t *B_off;
    const int32_t *rank;
    int64_t A_elems, B_elems;
    int32_t n_adapters, max_rank, d_in, d_out;
};

// Adapter a of pool P passes the device checks: id in range, rank a multiple of 8
// in [8, max_rank], A and B offsets non-negative multiples of 8 whose matrices end
// inside the pool.
__device__ __forceinline__ bool pool_adapter_ok(const PoolDev &P, int32_t a, int32_t *r_out, int64_t *aoff,
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

struct ShrinkArgs {
    const __nv_bfloat16 *X;
    int64_t ldx;
    const int32_t *perm;   // nullable
    const Group *groups;
    const WsHeader *hdr;
    int32_t mode;
    const int32_t *seg_ad;   // route / sgmv: adapter of an item
    const int32_t *ad_off;   // multi
    const int32_t *ad_id;    // multi
    PoolDev pool;
    int32_t kc;
    float *V;
    int64_t ldv;           // elements between positions
    int64_t chunk_stride;  // elements between split-K partial planes
    int32_t slot_stride;   // elements between stacked adapters of one row
    uint32_t *err;
};

struct ExpandArgs {
    __nv_bfloat16 *Y;
    int64_t ldy;
    const int32_t *perm;
    const Group *groups;
    const WsHeader *hdr;
    int32_t mode;
    const int32_t *seg_ad;
    const int32_t *ad_off;
    const int32_t *ad_id;
    const float *ad_scale;
    float scale;
    PoolDev pool;
    const float *V;
    int64_t ldv;
    int64_t chunk_stride;
    int32_t n_chunks;
    int32_t slot_stride;
    int32_t max_ads;
    uint32_t *err;
};

// --------------------------------------------------- fused decode (one launch)
constexpr int kFT = 16;             // tokens per (adapter, group) item = MMA tile rows
constexpr int kFThreads = 128;      // threads per CTA
constexpr int kFWarps = kFThreads / 32;
constexpr int kFC = 8;              // CTAs per cluster: d_in / d_out split in kFC chunks
constexpr int kVS = 160;            // bf16 row stride of the staged rank-r vectors (bank-conflict-free)
constexpr int kFMaxTokens = 8192;   // ids staged in shared memory
constexpr int kFMaxAdapters = 8192; // per-adapter group offsets in shared memory
constexpr int kFMaxChunk = 1 << 20; // d_in chunk per CTA (nothing of it is staged)
constexpr size_t kFMaxSmem = 200 * 1024;

constexpr int kFItemTable = 1024;   // most items whose adapter the grouping writes into a table

struct FusedSmem {
    size_t ids, cnt, items, order, vpart, vsum, bst, yst, total;
    int n_tab;       // entries of the item -> adapter table and of the item order (int16)
    int vs;          // bf16 row stride of the staged rank-r vectors
    bool staged;     // this CTA's B chunk and the item's y rows are copied to shared memory
};

__host__ __device__ inline size_t fused_align16(size_t x) { return (x + 15) & ~(size_t)15; }

// Shared memory of the fused decode kernel.  The rank-dependent parts are sized
// by the pool's max_rank; when a CTA's B chunk (Wo x max_rank) and the y rows of
// an item (kFT x Wo) fit 16 KB each, both are staged with cp.async while the
// shrink and the cluster exchange run.
__host__ __device__ inline FusedSmem fused_smem_layout(int32_t N, int32_t n_adapters, int32_t max_rank, int32_t Wo)
{
    FusedSmem L;
    const int mr = max_rank > kMaxRank ? kMaxRank : max_rank;
    L.vs = mr <= 32 ? 40 : kVS;                       // 80-byte rows: 16-byte reads conflict-free
    size_t off = 0;
    L.ids = off;
    off = fused_align16(off + 4 * (size_t)N);
    L.cnt = off;
    off = fused_align16(off + 4 * ((size_t)n_adapters + 1));
    // items: at most min(N, n_adapters) adapters plus one more 16-token group per 16 tokens
    const int64_t max_items = (int64_t)(N < n_adapters ? N : n_adapters) + N / kFT + 1;
    L.n_tab = (int)(max_items < kFItemTable ? max_items : kFItemTable);
    L.items = off;
    off = fused_align16(off + 2 * (size_t)L.n_tab);
    L.order = off;
    off = fused_align16(off + 2 * (size_t)L.n_tab);
    L.vpart = off;
    off = fused_align16(off + 4 * (size_t)mr * kFT);
    L.vsum = off;
    off = fused_align16(off + 2 * 2 * (size_t)kFT * L.vs);   // bf16 hi and lo
    L.staged = Wo > 0 && (int64_t)Wo * mr <= 8192 && (int64_t)kFT * Wo <= 8192 &&
               off + 2 * 16384 + 32 <= kFMaxSmem;
    L.bst = off;
    if (L.staged)
        off = fused_align16(off + 2 * (size_t)Wo * mr);
    L.yst = off;
    if (L.staged)
        off = fused_align16(off + 2 * (size_t)kFT * Wo);
    L.total = off;
    return L;
}

// Chunk of a dimension d per CTA of a cluster, rounded up to 8 elements.
__host__ __device__ inline int32_t fused_chunk(int32_t d)
{
    const int32_t w = (d + kFC - 1) / kFC;
    return (w + 7) & ~7;
}

struct FusedBgmvArgs {
    const __nv_bfloat16 *X;
    int64_t ldx;
    __nv_bfloat16 *Y;
    int64_t ldy;
    const int32_t *ids;
    int32_t N;
    PoolDev pool;
    float scale;
    int32_t Wk, Wo;
    uint32_t *err;
    uint32_t *sched;     // the workspace header's item counter pair
};

size_t fused_smem_bytes(int32_t N, int32_t n_adapters, int32_t max_rank, int32_t Wo);
bool fused_bgmv_supported(int32_t N, int32_t n_adapters, int32_t d_in);
cudaError_t launch_bgmv_fused(const FusedBgmvArgs &a, cudaStream_t s, bool pdl);
bool pdl_enabled();

// Testing hook (lora_test_stall): while set, the kernels with a load pipeline issue
// no loads, and every wait inside a kernel is bounded by wait_bound_ns().
int test_stall_mode();
unsigned long long wait_bound_ns();

// ------------------------------------------------------------ tcgen05 kernels
constexpr int kTcGroup = 128;       // rows per tensor-core tile
constexpr int kKMax = 128;          // stacked rank a tile may carry (expand; shrink of one pool)
constexpr int kKMaxShrink = 256;    // stacked rank of a shrink tile (projections sharing X)
constexpr int kMaxProj = LORA_MAX_PROJ;

struct TcArgs {
    CUtensorMap map_x;       // X [N, d_in], boxes 64 x 128, 128-byte swizzle (shrink)
    CUtensorMap map_y;       // Y [N, d_out], same boxes (expand)
    CUtensorMap map_a[3 * kMaxProj];   // A pool p as [A_elems / d_in, d_in], boxes of 64 columns x 64 / 32 / 8 rows: map_a[3p + m]
    int32_t a_tma;           // bit p: map_a[3p .. 3p + 2] valid (shrink)
    CUtensorMap map_b[4];    // B pool as [B_elems / r, r], r = 16 << m, boxes of min(r, 64) x 128 rows
    int32_t b_tma;           // bit m: map_b[m] valid (expand)
    int32_t e_natoms;        // expand: 16 KB atoms per V / B stage (1 or 2; set by the launcher)
    int32_t e_ystages;       // expand: y stages (set by the launcher)
    int32_t s_stages;        // shrink: pipeline stages (set by the launcher)
    int32_t s_stage;         // shrink: bytes per stage (set by the launcher)
    int32_t s_acc;           // shrink: TMEM columns per accumulator, 128 or 256 (set by the launcher)
    int32_t mode;            // kModeSgmv or kModeMulti
    const Group *groups;     // tiles of <= kTcGroup rows, one item each
    const WsHeader *hdr;
    const int32_t *seg_ad;
    const int32_t *ad_off;
    const int32_t *ad_id;
    const float *ad_scale;
    int32_t max_ads;
    float scale;
    PoolDev pool;            // kModeProj: proj[0]
    int32_t n_proj;          // kModeProj: a segment's stack is its adapter in proj[0 .. n_proj)
    PoolDev proj[kMaxProj];
    int32_t proj_vcol[kMaxProj];   // V column of projection p's rank 0
    float *V;                // fp32 intermediate, row stride ldv, stacked adapters slot_stride apart
    int64_t ldv;
    int32_t slot_stride;
    __nv_bfloat16 *Vb;       // shrink, if set (instead of V): scale * v as bf16 high part at Vb[n][c]
    int64_t ldvb;            //   and low part at Vb[n][vb_lo + c]
    int32_t vb_lo;
    int32_t allow_none;      // an item adapter of -1 means no adapter (not reported)
    __nv_bfloat16 *Y;
    int64_t ldy;
    uint32_t *err;
    unsigned long long wait_ns;   // bound of every wait (set by the launcher)
    int32_t test_stall;           // the producer issues nothing (set by the launcher)
};

bool tc_encode_x(TcArgs &a, const void *X, int32_t N, int32_t d_in, int64_t ldx);
bool tc_encode_y(TcArgs &a, const void *Y, int32_t N, int32_t d_out, int64_t ldy);
// optional: without it the shrink gathers A rows with cp.async
bool tc_encode_a(TcArgs &a, const void *A, int64_t A_elems, int32_t d_in, int pool_index = 0);
// optional: without it the expand gathers B rows with cp.async
bool tc_encode_b(TcArgs &a, const void *B, int64_t B_elems);
// kk: the largest stacked rank of any item (<= kKMaxShrink)
cudaError_t launch_tc_shrink(const TcArgs &a, int max_tiles, int kk, cudaStream_t s);
// kk: the largest stacked rank of any item (max_rank, or max_ads * max_rank)
cudaError_t launch_tc_expand(const TcArgs &a, int kk, cudaStream_t s);
// n expands over the same tiles in one launch (kk: the largest stacked rank of any)
cudaError_t launch_tc_expand_multi(const TcArgs *a, int n, int kk, cudaStream_t s);
bool tc_enabled();

// ------------------------------------------- projection + LoRA delta (tcgen05)
struct LinArgs {
    CUtensorMap map_x;       // X [N, d_in], boxes 64 x 128, 128-byte swizzle
    CUtensorMap map_w;       // W [d_out, d_in], boxes 64 x 256
    CUtensorMap map_v;       // s V as bf16 parts [N, 2 kv] (high, then low from column kv), boxes 64 x 128
    CUtensorMap map_b[4];    // B pool as [B_elems / r, r], r = 16 << m, boxes of min(r, 64) x 128 rows
    int32_t b_tma;           // bit m: map_b[m] valid
    int32_t kv;              // column of the low parts (max_rank rounded up to 64)
    const Group *groups;     // tiles of <= 128 rows, one segment each
    const WsHeader *hdr;
    const int32_t *seg_ad;   // -1: no adapter
    PoolDev pool;
    __nv_bfloat16 *Y;
    int64_t ldy;
    int32_t d_in, d_out;
    uint32_t *err;
    unsigned long long wait_ns;   // bound of every wait (set by the launcher)
    int32_t test_stall;           // the producer issues nothing (set by the launcher)
};

// Fills the tensor maps, d_in and d_out (kv must be set first); false if a map
// cannot be encoded (alignment, sizes).
bool lin_encode(LinArgs &a, const void *X, int64_t ldx, int32_t N, const void *W, int64_t ldw, const void *Vb,
                int64_t ldvb, const void *B, int64_t B_elems, int32_t d_in, int32_t d_out);
cudaError_t launch_tc_linear(const LinArgs &a, int max_units, cudaStream_t s);

// Workspace bytes of lora_merge (0 for unsupported sizes).
size_t merge_workspace_size(int32_t d_in, int32_t d_out, int32_t max_rank);

// Launchers (return the CUDA error of the launch).
cudaError_t launch_plan(const PlanArgs &a, cudaStream_t s);
cudaError_t launch_shrink(const ShrinkArgs &a, int grid_groups, int n_chunks, int max_ads, cudaStream_t s);
cudaError_t launch_expand(const ExpandArgs &a, int grid_groups, cudaStream_t s);

// Shared memory the plan kernel needs for a route over n_adapters.
size_t plan_smem_bytes(int32_t mode, int32_t n_adapters);

}  // namespace lora
