/*
 * mg_oracle.c -- the oracle for paged KV store + decode/extend attention.
 *
 * TEST INFRASTRUCTURE.  Only tests/, __graft_entry__.smoke() and the
 * cpu_baseline leg of bench.py may load or call this code.  The product path
 * (the CUDA library and its Python binding) never does, and shares no code,
 * header, table or helper with it.
 *
 * What it computes, and where that is defined (page title, then section):
 *
 *  [E]  "手写 mini-sglang 阶段一 · Engine 与采样器" (Stage 1, Engine and sampler)
 *       - §初始化的顺序 (initialisation order): the KV pool holds one K and one V
 *         tensor per layer of shape [pages+1, page_size, kv_heads, head_dim]; the
 *         page table is int32 [max_running_req+1, align32(max_seq_len)] and each
 *         row stores the KV location of every token of one request.
 *       - §手工驱动引擎 (driving the engine by hand): a request's new tokens sit at
 *         positions arange(cached_len, device_len); their K/V go to
 *         out_loc = page_table[table_idx, cached_len:device_len]; the tokens of
 *         all requests are concatenated in request order.
 *  [T]  "Mini-SGLang" tag page, Engine post, §一 (GPU inference is not only
 *       matrix multiplication): per layer the order is QKV -> RoPE -> write KV
 *       cache -> attention, so attention sees the tokens just written.
 *       KV Cache post, §一 (why a KV cache): at step t the query attends to the
 *       keys/values of positions 0..t.
 *  [S]  "mini-sglang from Scratch Stage 4 · Faster and bigger", §What each chapter
 *       adds: attention works on the paged pool in place and keeps the score
 *       matrix out of memory (the kernels' concern; the oracle may store one
 *       row of scores, which is the plain definition).
 *
 * Readings taken where the pages are silent: page_size is 1, so the pool is
 * [num_slots, kv_heads, head_dim] and a page-table entry is a slot; q head h uses KV head h / g with g = Hq / Hkv
 * (consecutive q heads share a KV head); scores are scale * <q, k>; softmax is
 * exp(x - max) / sum; decode is the one-new-token case (cached_len = L - 1).
 *
 * Arithmetic: every bf16 input is widened exactly to double; all sums run in
 * double, in increasing key / dimension order.  No blocking, fusion or
 * reordering.  Compile without -ffast-math.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>
#ifdef _OPENMP
#include <omp.h>
#endif

/* Error codes returned by the oracle entry points. */
enum {
    ORACLE_OK = 0,
    ORACLE_BAD_ARGUMENT = 1,
    ORACLE_SLOT_OUT_OF_RANGE = 2,
    ORACLE_ROW_OUT_OF_RANGE = 3,
    ORACLE_LENGTH_OUT_OF_RANGE = 4,
    ORACLE_NO_MEMORY = 5
};

/* bf16 is the top half of an IEEE binary32; widening it is exact. */
static double bf16_bits_to_double(uint16_t bits) {
    uint32_t u = ((uint32_t)bits) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

/*
 * KV store ([E] §手工驱动引擎; [T] Engine post §一):
 *   for every new token t and KV head h:  k_pool[out_loc[t]][h][:] = k[t][h][:],
 *   and the same for v.  A pure copy of the bf16 bit patterns.
 */
int oracle_store_kv(const uint16_t *k, const uint16_t *v, const int32_t *out_loc,
                    int64_t num_tokens, uint16_t *k_pool, uint16_t *v_pool,
                    int64_t num_slots, int64_t num_kv_heads, int64_t head_dim) {
    if (num_tokens < 0 || num_slots <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return ORACLE_BAD_ARGUMENT;
    const int64_t row = num_kv_heads * head_dim; /* elements per token */
    for (int64_t t = 0; t < num_tokens; ++t) {
        int64_t slot = out_loc[t];
        if (slot < 0 || slot >= num_slots) return ORACLE_SLOT_OUT_OF_RANGE;
        for (int64_t h = 0; h < num_kv_heads; ++h) {
            for (int64_t d = 0; d < head_dim; ++d) {
                k_pool[slot * row + h * head_dim + d] = k[t * row + h * head_dim + d];
                v_pool[slot * row + h * head_dim + d] = v[t * row + h * head_dim + d];
            }
        }
    }
    return ORACLE_OK;
}

/*
 * Attention of one query vector over the keys at positions 0..last of one
 * page-table row, for one KV head:
 *   x_j = scale * sum_d q[d] * K[row[j]][kvh][d]
 *   w_j = exp(x_j - max_j x_j)
 *   o[d] = sum_j w_j * V[row[j]][kvh][d] / sum_j w_j
 * `x` is caller-provided scratch of at least last+1 doubles.
 */
static int attend_one_query(const uint16_t *q_vec, const uint16_t *k_pool,
                            const uint16_t *v_pool, int64_t num_slots,
                            const int32_t *pt_row, int64_t last, int64_t kvh,
                            int64_t num_kv_heads, int64_t head_dim, double scale,
                            double *x, double *o) {
    const int64_t row = num_kv_heads * head_dim;
    double x_max = -INFINITY;
    for (int64_t j = 0; j <= last; ++j) {
        int64_t slot = pt_row[j];
        if (slot < 0 || slot >= num_slots) return ORACLE_SLOT_OUT_OF_RANGE;
        const uint16_t *k_vec = k_pool + slot * row + kvh * head_dim;
        double dot = 0.0;
        for (int64_t d = 0; d < head_dim; ++d)
            dot += bf16_bits_to_double(q_vec[d]) * bf16_bits_to_double(k_vec[d]);
        x[j] = scale * dot;
        if (x[j] > x_max) x_max = x[j];
    }
    double denom = 0.0;
    for (int64_t d = 0; d < head_dim; ++d) o[d] = 0.0;
    for (int64_t j = 0; j <= last; ++j) {
        double w = exp(x[j] - x_max);
        denom += w;
        const uint16_t *v_vec = v_pool + (int64_t)pt_row[j] * row + kvh * head_dim;
        for (int64_t d = 0; d < head_dim; ++d) o[d] += w * bf16_bits_to_double(v_vec[d]);
    }
    for (int64_t d = 0; d < head_dim; ++d) o[d] /= denom;
    return ORACLE_OK;
}

/*
 * Decode attention ([T] KV Cache post §一; [E] §手工驱动引擎 with one new token):
 * request r has context length L = seq_len[r] (the new token included, already
 * stored), its page-table row is page_table[table_idx[r]], and its single query
 * (q[r], position L-1) attends to positions 0..L-1.
 *   q      [B, Hq, D] bf16 bits          out [B, Hq, D] double
 *   pool   [num_slots, Hkv, D] bf16 bits page_table [pt_rows, pt_stride] int32
 * req_mask (may be NULL): compute only requests with req_mask[r] != 0; the
 * other rows of `out` are left untouched.
 */
int oracle_decode(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                  int64_t num_slots, const int32_t *page_table, int64_t pt_rows,
                  int64_t pt_stride, const int32_t *table_idx, const int32_t *seq_len,
                  int64_t batch, int64_t num_q_heads, int64_t num_kv_heads,
                  int64_t head_dim, double scale, const uint8_t *req_mask,
                  int num_threads, double *out) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_q_heads % num_kv_heads != 0 || num_slots <= 0 || pt_rows <= 0 || pt_stride <= 0)
        return ORACLE_BAD_ARGUMENT;
    for (int64_t r = 0; r < batch; ++r) {
        if (req_mask && !req_mask[r]) continue;
        if (table_idx[r] < 0 || table_idx[r] >= pt_rows) return ORACLE_ROW_OUT_OF_RANGE;
        if (seq_len[r] < 1 || seq_len[r] > pt_stride) return ORACLE_LENGTH_OUT_OF_RANGE;
    }
    const int64_t group = num_q_heads / num_kv_heads;
    const int64_t units = batch * num_q_heads;
    int err = ORACLE_OK;
#ifdef _OPENMP
    if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(max : err)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t r = u / num_q_heads, h = u % num_q_heads;
        if (req_mask && !req_mask[r]) continue;
        const int64_t L = seq_len[r];
        double *x = (double *)malloc(sizeof(double) * (size_t)L);
        if (!x) { err = ORACLE_NO_MEMORY; continue; }
        int e = attend_one_query(q + (r * num_q_heads + h) * head_dim, k_pool, v_pool,
                                 num_slots, page_table + (int64_t)table_idx[r] * pt_stride,
                                 L - 1, h / group, num_kv_heads, head_dim, scale, x,
                                 out + (r * num_q_heads + h) * head_dim);
        free(x);
        if (e != ORACLE_OK) err = e;
    }
    return err;
}

/*
 * Extend (chunked-prefill) attention ([E] §手工驱动引擎; [T] Scheduler post on
 * chunked prefill): request r has c = cached_len[r] tokens already in the pool
 * and n = seq_len[r] - c new ones (stored before attention).  Its new tokens'
 * queries are rows q_offset[r] .. q_offset[r]+n-1 of q, in request order; new
 * token i sits at position c+i and attends to positions 0..c+i (causal).
 *   q [total_q, Hq, D] bf16 bits   out [total_q, Hq, D] double
 *   q_offset [B+1]: q_offset[0] = 0, q_offset[r+1] - q_offset[r] = n_r.
 */
int oracle_extend(const uint16_t *q, const uint16_t *k_pool, const uint16_t *v_pool,
                  int64_t num_slots, const int32_t *page_table, int64_t pt_rows,
                  int64_t pt_stride, const int32_t *table_idx, const int32_t *cached_len,
                  const int32_t *seq_len, const int32_t *q_offset, int64_t batch,
                  int64_t total_q, int64_t num_q_heads, int64_t num_kv_heads,
                  int64_t head_dim, double scale, const uint8_t *req_mask,
                  int num_threads, double *out) {
    if (batch < 0 || num_q_heads <= 0 || num_kv_heads <= 0 || head_dim <= 0 ||
        num_q_heads % num_kv_heads != 0 || num_slots <= 0 || pt_rows <= 0 || pt_stride <= 0)
        return ORACLE_BAD_ARGUMENT;
    if (q_offset[0] != 0 || q_offset[batch] != total_q) return ORACLE_BAD_ARGUMENT;
    for (int64_t r = 0; r < batch; ++r) {
        if (q_offset[r + 1] - q_offset[r] != (int64_t)seq_len[r] - cached_len[r])
            return ORACLE_BAD_ARGUMENT;
        if (req_mask && !req_mask[r]) continue;
        if (table_idx[r] < 0 || table_idx[r] >= pt_rows) return ORACLE_ROW_OUT_OF_RANGE;
        if (cached_len[r] < 0 || seq_len[r] < cached_len[r] || seq_len[r] > pt_stride)
            return ORACLE_LENGTH_OUT_OF_RANGE;
    }
    const int64_t group = num_q_heads / num_kv_heads;
    int err = ORACLE_OK;
    const int64_t units = batch * num_q_heads;
#ifdef _OPENMP
    if (num_threads <= 0) num_threads = omp_get_max_threads();
#pragma omp parallel for schedule(dynamic, 1) num_threads(num_threads) reduction(max : err)
#endif
    for (int64_t u = 0; u < units; ++u) {
        const int64_t r = u / num_q_heads, h = u % num_q_heads;
        if (req_mask && !req_mask[r]) continue;
        const int64_t c = cached_len[r], n = (int64_t)seq_len[r] - c;
        if (n == 0) continue;
        double *x = (double *)malloc(sizeof(double) * (size_t)(c + n));
        if (!x) { err = ORACLE_NO_MEMORY; continue; }
        const int32_t *pt_row = page_table + (int64_t)table_idx[r] * pt_stride;
        for (int64_t i = 0; i < n; ++i) {
            const int64_t t = q_offset[r] + i;
            int e = attend_one_query(q + (t * num_q_heads + h) * head_dim, k_pool, v_pool,
                                     num_slots, pt_row, c + i, h / group, num_kv_heads,
                                     head_dim, scale, x, out + (t * num_q_heads + h) * head_dim);
            if (e != ORACLE_OK) { err = e; break; }
        }
        free(x);
    }
    return err;
}
