/*
 * CPU oracle for the unmerged multi-LoRA delta -- TEST INFRASTRUCTURE ONLY.
 *
 * Only the tests, the smoke check and the benchmark's CPU-baseline leg use
 * this file.  It shares nothing with the CUDA library: no header, no helper,
 * no table.  It is deliberately plain and slow: fp64 loops, one OpenMP
 * parallel-for over output rows, no blocking, no reordering of the sums.
 *
 * What is computed (source: "Serving several LoRAs, ControlNet and
 * IP-Adapter", section "LoRA: merged or alongside"):
 *   a LoRA adds W' = W + B A to a weight, A is r x d and B is d x r; computed
 *   alongside ("unmerged"), each layer adds x A^T B^T to x W^T.  Per token row
 *   x[n] (a d_in vector) and adapter a of rank r_a:
 *       v_j   = sum_i A[a][j][i] * x[n][i]          j < r_a   (shrink)
 *       d[o]  = s * sum_j B[a][o][j] * v_j          o < d_out (expand)
 *   The per-adapter weight s is a runtime scalar (same page: the LoRA's weight
 *   can change every denoising step, "swap a scalar each step").
 * Grouping (same page, exercise 2's answer): a mixed batch is grouped by LoRA
 * index, each group computes its own x A^T B^T, and the results go back in the
 * original order -- so the result of a token depends only on its own row and
 * its own adapter(s), which is what every function here computes directly.
 * Stacking several LoRAs on one request (same page, table row "Stacking
 * several LoRAs") adds their deltas.
 *
 * Storage: X, A, B arrive as bf16 bit patterns (uint16) and are widened to
 * double exactly; every sum is accumulated in double; outputs are double.
 * Pool layout: adapter a's A is [rank[a], d_in] row-major at element offset
 * A_off[a]; its B is [d_out, rank[a]] row-major at B_off[a].
 *
 * Return value of every entry point: 0 on success, a negative code when an
 * adapter id, offset or rank in the metadata is out of range (nothing is
 * written for that row; the remaining rows are still computed).
 */
#include <stdint.h>
#include <string.h>

#define ORC_OK 0
#define ORC_BAD_ID (-1)
#define ORC_BAD_SEGMENT (-2)
#define ORC_BAD_RANK (-3)

static double widen_bf16(uint16_t h)
{
    uint32_t u = ((uint32_t)h) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/* One token row through one adapter: d_row[o] += s * B_a (A_a x). */
static int one_adapter(const uint16_t *x, const uint16_t *A, const int64_t *A_off,
                       const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                       int32_t n_adapters, int32_t d_in, int32_t d_out, int32_t a,
                       double s, double *v /* scratch [128] */, double *d_row)
{
    if (a < 0 || a >= n_adapters)
        return ORC_BAD_ID;
    int32_t r = rank[a];
    if (r <= 0 || r > 128)
        return ORC_BAD_RANK;
    const uint16_t *Aa = A + A_off[a];
    const uint16_t *Ba = B + B_off[a];
    for (int32_t j = 0; j < r; ++j) {
        double acc = 0.0;
        for (int32_t i = 0; i < d_in; ++i)
            acc += widen_bf16(Aa[(int64_t)j * d_in + i]) * widen_bf16(x[i]);
        v[j] = acc;
    }
    for (int32_t o = 0; o < d_out; ++o) {
        double acc = 0.0;
        for (int32_t j = 0; j < r; ++j)
            acc += widen_bf16(Ba[(int64_t)o * r + j]) * v[j];
        d_row[o] += s * acc;
    }
    return ORC_OK;
}

/*
 * BGMV (one token per request): token n uses adapter ids[n]; ids[n] == -1
 * means "no adapter" (zero delta).  D[k][:] receives the delta of token
 * rows[k] (all tokens in order when rows == NULL, n_rows = N).
 */
int oracle_bgmv_delta(const uint16_t *X, int64_t ldx,
                      const uint16_t *A, const int64_t *A_off,
                      const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                      int32_t n_adapters, int32_t d_in, int32_t d_out,
                      const int32_t *ids, int32_t N, double scale,
                      const int32_t *rows, int32_t n_rows, double *D)
{
    int status = ORC_OK;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        double v[128];
        double *d_row = D + (int64_t)k * d_out;
        for (int32_t o = 0; o < d_out; ++o)
            d_row[o] = 0.0;
        if (n < 0 || n >= N) {
#pragma omp atomic write
            status = ORC_BAD_SEGMENT;
            continue;
        }
        int32_t a = ids[n];
        if (a == -1)
            continue;
        int rc = one_adapter(X + (int64_t)n * ldx, A, A_off, B, B_off, rank, n_adapters,
                             d_in, d_out, a, scale, v, d_row);
        if (rc != ORC_OK) {
#pragma omp atomic write
            status = rc;
        }
    }
    return status;
}

/* Find the segment k with seg_off[k] <= n < seg_off[k+1]; -1 if none. */
static int32_t segment_of(const int32_t *seg_off, int32_t n_seg, int32_t n)
{
    for (int32_t k = 0; k < n_seg; ++k)
        if (seg_off[k] <= n && n < seg_off[k + 1])
            return k;
    return -1;
}

static int check_segments(const int32_t *seg_off, int32_t n_seg, int32_t N)
{
    if (seg_off[0] < 0)
        return ORC_BAD_SEGMENT;
    for (int32_t k = 0; k < n_seg; ++k)
        if (seg_off[k + 1] < seg_off[k])
            return ORC_BAD_SEGMENT;
    if (seg_off[n_seg] > N)
        return ORC_BAD_SEGMENT;
    return ORC_OK;
}

/*
 * SGMV shrink: rows seg_off[k]..seg_off[k+1]-1 use adapter seg_ad[k];
 * V[k'][j] = sum_i A[a][j][i] x[n][i] for j < rank[a], for token n = rows[k']
 * (all N rows when rows == NULL).  Entries j >= rank[a], and rows outside every
 * segment, are left as they were.
 */
int oracle_sgmv_shrink(const uint16_t *X, int64_t ldx,
                       const uint16_t *A, const int64_t *A_off, const int32_t *rank,
                       int32_t n_adapters, int32_t d_in,
                       const int32_t *seg_off, const int32_t *seg_ad, int32_t n_seg, int32_t N,
                       const int32_t *rows, int32_t n_rows, double *V, int64_t ldv)
{
    int status = check_segments(seg_off, n_seg, N);
    if (status != ORC_OK)
        return status;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        int32_t sg = segment_of(seg_off, n_seg, n);
        if (sg < 0)
            continue;
        int32_t a = seg_ad[sg];
        if (a < 0 || a >= n_adapters || rank[a] <= 0 || rank[a] > 128) {
#pragma omp atomic write
            status = ORC_BAD_ID;
            continue;
        }
        const uint16_t *Aa = A + A_off[a];
        const uint16_t *x = X + (int64_t)n * ldx;
        for (int32_t j = 0; j < rank[a]; ++j) {
            double acc = 0.0;
            for (int32_t i = 0; i < d_in; ++i)
                acc += widen_bf16(Aa[(int64_t)j * d_in + i]) * widen_bf16(x[i]);
            V[(int64_t)k * ldv + j] = acc;
        }
    }
    return status;
}

/*
 * SGMV expand: D[k'][o] = scale * sum_{j<rank[a]} B[a][o][j] * V[n][j] for
 * token n = rows[k'] in a segment with adapter a; zero for rows outside every
 * segment.  V is the fp32 intermediate the CUDA expand also receives.
 */
int oracle_sgmv_expand(const float *V, int64_t ldv,
                       const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                       int32_t n_adapters, int32_t d_out,
                       const int32_t *seg_off, const int32_t *seg_ad, int32_t n_seg, int32_t N,
                       double scale, const int32_t *rows, int32_t n_rows, double *D)
{
    int status = check_segments(seg_off, n_seg, N);
    if (status != ORC_OK)
        return status;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        double *d_row = D + (int64_t)k * d_out;
        for (int32_t o = 0; o < d_out; ++o)
            d_row[o] = 0.0;
        int32_t sg = segment_of(seg_off, n_seg, n);
        if (sg < 0)
            continue;
        int32_t a = seg_ad[sg];
        if (a < 0 || a >= n_adapters || rank[a] <= 0 || rank[a] > 128) {
#pragma omp atomic write
            status = ORC_BAD_ID;
            continue;
        }
        const uint16_t *Ba = B + B_off[a];
        int32_t r = rank[a];
        for (int32_t o = 0; o < d_out; ++o) {
            double acc = 0.0;
            for (int32_t j = 0; j < r; ++j)
                acc += widen_bf16(Ba[(int64_t)o * r + j]) * (double)V[(int64_t)n * ldv + j];
            d_row[o] = scale * acc;
        }
    }
    return status;
}

/* Full SGMV delta (shrink and expand with the intermediate kept in double). */
int oracle_sgmv_delta(const uint16_t *X, int64_t ldx,
                      const uint16_t *A, const int64_t *A_off,
                      const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                      int32_t n_adapters, int32_t d_in, int32_t d_out,
                      const int32_t *seg_off, const int32_t *seg_ad, int32_t n_seg, int32_t N,
                      double scale, const int32_t *rows, int32_t n_rows, double *D)
{
    int status = check_segments(seg_off, n_seg, N);
    if (status != ORC_OK)
        return status;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        double v[128];
        double *d_row = D + (int64_t)k * d_out;
        for (int32_t o = 0; o < d_out; ++o)
            d_row[o] = 0.0;
        int32_t sg = segment_of(seg_off, n_seg, n);
        if (sg < 0)
            continue;
        int rc = one_adapter(X + (int64_t)n * ldx, A, A_off, B, B_off, rank, n_adapters,
                             d_in, d_out, seg_ad[sg], scale, v, d_row);
        if (rc != ORC_OK) {
#pragma omp atomic write
            status = rc;
        }
    }
    return status;
}

/*
 * Multi-adapter requests: request q covers rows req_off[q]..req_off[q+1]-1 and
 * stacks adapters ad_id[p] with weights ad_scale[p], p in ad_off[q]..ad_off[q+1]-1;
 * their deltas are summed.  Rows outside every request get a zero delta.
 */
int oracle_apply_multi(const uint16_t *X, int64_t ldx,
                       const uint16_t *A, const int64_t *A_off,
                       const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                       int32_t n_adapters, int32_t d_in, int32_t d_out,
                       const int32_t *req_off, const int32_t *ad_off, const int32_t *ad_id,
                       const float *ad_scale, int32_t n_req, int32_t N,
                       const int32_t *rows, int32_t n_rows, double *D)
{
    int status = check_segments(req_off, n_req, N);
    if (status != ORC_OK)
        return status;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        double v[128];
        double *d_row = D + (int64_t)k * d_out;
        for (int32_t o = 0; o < d_out; ++o)
            d_row[o] = 0.0;
        int32_t q = segment_of(req_off, n_req, n);
        if (q < 0)
            continue;
        for (int32_t p = ad_off[q]; p < ad_off[q + 1]; ++p) {
            int rc = one_adapter(X + (int64_t)n * ldx, A, A_off, B, B_off, rank, n_adapters,
                                 d_in, d_out, ad_id[p], (double)ad_scale[p], v, d_row);
            if (rc != ORC_OK) {
#pragma omp atomic write
                status = rc;
            }
        }
    }
    return status;
}

/*
 * Grouping of an unsorted id array by adapter (the "group the batch by LoRA
 * index" step): a stable counting sort.  Tokens with id -1 are left out.
 * Outputs: perm[0..n_valid) = token indices, grouped by adapter in ascending
 * id order and in original order within a group; seg_ad[0..n_seg) = the
 * distinct adapters present, ascending; seg_off[0..n_seg] = group bounds in
 * perm; *n_seg_out.  counts must hold n_adapters int32 of scratch.
 */
int oracle_route(const int32_t *ids, int32_t N, int32_t n_adapters,
                 int32_t *counts, int32_t *perm, int32_t *seg_off, int32_t *seg_ad,
                 int32_t *n_seg_out)
{
    for (int32_t a = 0; a < n_adapters; ++a)
        counts[a] = 0;
    for (int32_t n = 0; n < N; ++n) {
        if (ids[n] == -1)
            continue;
        if (ids[n] < -1 || ids[n] >= n_adapters)
            return ORC_BAD_ID;
        counts[ids[n]] += 1;
    }
    int32_t n_seg = 0, pos = 0;
    seg_off[0] = 0;
    for (int32_t a = 0; a < n_adapters; ++a) {
        if (counts[a] == 0)
            continue;
        seg_ad[n_seg] = a;
        /* place this adapter's tokens in original order */
        for (int32_t n = 0; n < N; ++n)
            if (ids[n] == a)
                perm[pos++] = n;
        seg_off[++n_seg] = pos;
    }
    *n_seg_out = n_seg;
    return ORC_OK;
}

/*
 * Merge (same page, section "LoRA: merged or alongside": a merged LoRA is
 * W' = W + B A folded into the weight; switching adapters merges one and
 * unmerges the other, i.e. adds and subtracts s * B A).  For adapter a and the
 * base weight W [d_out, d_in] (bf16 bit patterns, row stride ldw):
 *     Wm[k][i] = W[o][i] + s * sum_j B[a][o][j] * A[a][j][i],   o = rows[k]
 * in double, without rounding (all rows in order when rows == NULL, n_rows =
 * d_out).  Unmerging is the same call with -s.
 */
int oracle_merge(const uint16_t *W, int64_t ldw,
                 const uint16_t *A, const int64_t *A_off,
                 const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                 int32_t n_adapters, int32_t d_in, int32_t d_out, int32_t a, double scale,
                 const int32_t *rows, int32_t n_rows, double *Wm)
{
    if (a < 0 || a >= n_adapters)
        return ORC_BAD_ID;
    int32_t r = rank[a];
    if (r <= 0 || r > 128)
        return ORC_BAD_RANK;
    if (rows == NULL)
        n_rows = d_out;
    const uint16_t *Aa = A + A_off[a];
    const uint16_t *Ba = B + B_off[a];
    int status = ORC_OK;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t o = rows ? rows[k] : k;
        double *w_row = Wm + (int64_t)k * d_in;
        if (o < 0 || o >= d_out) {
#pragma omp atomic write
            status = ORC_BAD_SEGMENT;
            continue;
        }
        for (int32_t i = 0; i < d_in; ++i) {
            double acc = 0.0;
            for (int32_t j = 0; j < r; ++j)
                acc += widen_bf16(Ba[(int64_t)o * r + j]) * widen_bf16(Aa[(int64_t)j * d_in + i]);
            w_row[i] = widen_bf16(W[(int64_t)o * ldw + i]) + scale * acc;
        }
    }
    return status;
}

/*
 * A projection with its LoRA delta, computed unmerged (same page, section
 * "LoRA: merged or alongside": the unmerged layer adds x A^T B^T to x W^T).
 * For token n = rows[k] in segment g with adapter a = seg_ad[g]:
 *     Y[k][o] = sum_i W[o][i] * x[n][i] + s * sum_j B[a][o][j] * v_j,
 *     v_j     = sum_i A[a][j][i] * x[n][i],
 * and seg_ad[g] == -1 means no adapter (the first sum alone).  W is
 * [d_out, d_in] (bf16 bit patterns, row stride ldw).  Rows outside every
 * segment get zeros (the library leaves them untouched).
 */
int oracle_linear_sgmv(const uint16_t *X, int64_t ldx, const uint16_t *W, int64_t ldw,
                       const uint16_t *A, const int64_t *A_off,
                       const uint16_t *B, const int64_t *B_off, const int32_t *rank,
                       int32_t n_adapters, int32_t d_in, int32_t d_out,
                       const int32_t *seg_off, const int32_t *seg_ad, int32_t n_seg, int32_t N,
                       double scale, const int32_t *rows, int32_t n_rows, double *Y)
{
    int status = check_segments(seg_off, n_seg, N);
    if (status != ORC_OK)
        return status;
    if (rows == NULL)
        n_rows = N;
#pragma omp parallel for schedule(dynamic, 1)
    for (int32_t k = 0; k < n_rows; ++k) {
        int32_t n = rows ? rows[k] : k;
        const uint16_t *x = X + (int64_t)n * ldx;
        double v[128];
        double *y_row = Y + (int64_t)k * d_out;
        for (int32_t o = 0; o < d_out; ++o)
            y_row[o] = 0.0;
        int32_t sg = segment_of(seg_off, n_seg, n);
        if (sg < 0)
            continue;
        for (int32_t o = 0; o < d_out; ++o) {
            double acc = 0.0;
            for (int32_t i = 0; i < d_in; ++i)
                acc += widen_bf16(W[(int64_t)o * ldw + i]) * widen_bf16(x[i]);
            y_row[o] = acc;
        }
        if (seg_ad[sg] == -1)
            continue;
        int rc = one_adapter(x, A, A_off, B, B_off, rank, n_adapters, d_in, d_out, seg_ad[sg], scale, v, y_row);
        if (rc != ORC_OK) {
#pragma omp atomic write
            status = rc;
        }
    }
    return status;
}
