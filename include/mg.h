/*
 * mg.h -- C ABI of the B200 (sm_100a) paged KV attention library (libmg.so).
 *
 * Three operations make up the per-layer attention hot path of the
 * mini-sglang engine.  Each layer of its forward pass runs the QKV
 * projection, RoPE, the KV-cache write, attention and o_proj, in that order
 * (Mini-SGLang tag page, Engine post, §一); this library covers the KV-cache
 * write and attention:
 *
 *   mg_store_kv     write the new tokens' K/V into pool slots at out_loc;
 *   mg_decode_attn  one query token per request against its paged history
 *                   (balanced split-KV kernel + merge kernel);
 *   mg_store_decode_attn  the two above fused into one decode launch;
 *   mg_decode_attn_shared_prefix  decode reading a shared prefix once per group;
 *   mg_store_decode_attn_shared_prefix  the store fused into that decode;
 *   mg_mixed_attn   extend semantics for mixed batches: one-token requests by
 *                   the decode kernel, prompt chunks by the extend kernel;
 *   mg_extend_attn  a chunk of new tokens per request (chunked prefill),
 *                   causal over cached_len + i, on tcgen05 tensor cores.
 *
 * Data structures ("手写 mini-sglang 阶段一 · Engine 与采样器" (Stage 1, Engine and
 * sampler), §初始化的顺序 and §手工驱动引擎):
 *   - KV pool, per layer, K and V separately: [num_slots, num_kv_heads, head_dim]
 *     bf16, row-major.  This is the engine's [pages, page_size, heads, dim]
 *     pool flattened with page_size 1, so a page-table entry is a slot.
 *   - page_table: int32 [page_table_rows, page_table_stride], row-major.  Row
 *     table_idx[r] holds the slot of every token of request r, position 0 first.
 *   - a request has cached_len tokens already in the pool and seq_len tokens
 *     after this step (seq_len is the engine's device_len); its new tokens sit
 *     at positions cached_len .. seq_len-1.
 *   - q head h reads KV head h / (num_q_heads / num_kv_heads) (grouped-query
 *     attention with consecutive q heads sharing a KV head).
 *
 * Conventions for every entry point:
 *   - Pointers named as tensors are DEVICE pointers (the current CUDA device);
 *     bf16 data is passed as void*.  Every tensor is dense and row-major, and
 *     every bf16 tensor must start on a 16-byte boundary.
 *   - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *     enqueued on it (mg_mixed_attn's split also forks onto a stream of the
 *     library's and joins back); no entry point synchronises the host,
 *     allocates device memory or keeps state between calls (save the wait
 *     limit of mg_set_extend_wait_limit and that one stream per device), so
 *     calls can be captured in a CUDA graph (mg_read_device_error excepted,
 *     which synchronises).
 *   - The caller owns every buffer.  Inputs are read-only except the pools
 *     in mg_store_kv; outputs are written in full for every real (request,
 *     head) row.
 *   - The kernels are launched with programmatic dependent launch, so one
 *     may start while the previous kernel on the stream finishes.  Before it
 *     waits for that kernel, a kernel of this library reads only the request
 *     metadata (page_table, table_idx, seq_len, cached_len, q_offset,
 *     group_first, prefix_len), which none of its kernels writes: the pools,
 *     q, the new K/V rows, the workspace and the outputs are touched only
 *     after the wait.  A kernel of the caller's that ends with a programmatic
 *     launch trigger must therefore have written that metadata before its
 *     trigger (a kernel without a trigger completes before ours start).
 *   - The softmax scale must be finite and > 0 (else MG_ERR_INVALID_ARGUMENT):
 *     the kernels take row maxima of the unscaled scores and scale them after,
 *     which needs a positive scale.  (scale = 0, whose result is the plain
 *     mean of the V rows, is therefore not accepted.)
 *   - page_table_rows is passed with the page table so that the kernels can
 *     check table_idx against it; decode's num_partitions picks or forces the
 *     number of workers of its plan (mg_decode_plan).  Extend needs no
 *     workspace, so it takes none.
 *   - Errors found on the host (null pointer, bad size, unsupported shape,
 *     misalignment, workspace too small) return a status BEFORE anything is
 *     launched.  A failed launch returns MG_ERR_CUDA.  Metadata that can only
 *     be checked on the device (a slot outside the pool, a page-table row
 *     outside the table, a length beyond the page-table width or the
 *     max_seq_len hint) never makes a kernel read or write out of bounds: the
 *     offending token or request is skipped, a bit is set in a device error
 *     word, and mg_read_device_error reports it.
 */
#ifndef MG_H
#define MG_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum mg_status {
    MG_OK = 0,
    MG_ERR_INVALID_ARGUMENT = 1,    /* null pointer, negative or zero size, bad hint */
    MG_ERR_UNSUPPORTED_SHAPE = 2,   /* head_dim != 128, Hq % Hkv != 0, group > 16 */
    MG_ERR_MISALIGNED = 3,          /* a bf16 tensor not on a 16-byte boundary */
    MG_ERR_WORKSPACE_TOO_SMALL = 4, /* decode workspace below mg_decode_workspace_bytes */
    MG_ERR_CUDA = 5,                /* a CUDA runtime call or launch failed */
    MG_ERR_DEVICE_CHECK = 6,        /* device-side metadata check failed (see bits) */
    MG_ERR_DEVICE_TIMEOUT = 7       /* a bounded device wait gave up (see bits) */
} mg_status;

/* Bits of the device error word (mg_read_device_error). */
#define MG_DEVERR_SLOT_RANGE 0x1u    /* a slot (out_loc or page-table entry) outside [0, num_slots) */
#define MG_DEVERR_ROW_RANGE 0x2u     /* table_idx outside [0, page_table_rows) */
#define MG_DEVERR_LENGTH 0x4u        /* seq_len / cached_len / q_offset inconsistent or beyond hints */
#define MG_DEVERR_WAIT_TIMEOUT 0x8u  /* a pipeline wait ran past its time limit (mg_set_extend_wait_limit) */
#define MG_DEVERR_INTERNAL 0x10u     /* a launch invariant failed on the device (a library fault, not
                                        the caller's metadata): extend's shared memory not 1024-byte
                                        aligned; the kernel refused to run */

/* Human-readable name of a status. Never NULL. */
const char *mg_status_string(mg_status status);

/* ABI version: bumped on any incompatible change of a signature below. */
int32_t mg_abi_version(void);

/*
 * mg_store_kv -- KV write (the engine's KV-cache write step; one of the small
 * steps whose launch and memory cost the engine's own kernels target,
 * "mini-sglang from Scratch Stage 4 · Faster and bigger", §What each chapter
 * adds).
 *
 *   k_cache[out_loc[t], h, :] = k[t, h, :]   and   v_cache[out_loc[t], h, :] = v[t, h, :]
 *   for t < num_tokens, h < num_kv_heads.  A bit copy.
 *
 *   k, v          [num_tokens, num_kv_heads, head_dim] bf16 (the new tokens,
 *                 concatenated in request order)
 *   out_loc       [num_tokens] int32 slots = page_table[table_idx[r], cached_len:seq_len]
 *   k_cache/v_cache [num_slots, num_kv_heads, head_dim] bf16, updated in place
 * num_tokens == 0 is a no-op.  Slots must be distinct except for a dummy slot
 * that padded requests share (which write lands there is unspecified).  A slot
 * outside [0, num_slots) is skipped and sets MG_DEVERR_SLOT_RANGE.
 * head_dim * num_kv_heads * 2 must be a multiple of 16 bytes.
 */
mg_status mg_store_kv(const void *k, const void *v, const int32_t *out_loc, int32_t num_tokens,
                      void *k_cache, void *v_cache, int64_t num_slots, int32_t num_kv_heads,
                      int32_t head_dim, void *stream);

/*
 * mg_decode_plan -- the host-side plan of mg_decode_attn (the role FlashInfer's
 * "plan" step plays, Stage 4 page, §Checkpoint).  The decode work is cut into
 * units of 16 keys of one (request, kv head) pair; `workers` warps share the
 * units equally and in order, so a pair may be split across workers, whose
 * partial results a merge kernel combines.  num_partitions == 0 picks one
 * worker per warp of the decode grid on the current device (SMs x 2 CTAs x
 * 4 warps); > 0 forces that many workers.
 * slots_out = batch * num_kv_heads + workers partial slots.
 * The plan depends only on these arguments (never on the lengths), so a
 * captured launch stays valid for any batch with lengths <= max_seq_len.
 */
mg_status mg_decode_plan(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len,
                         int32_t num_partitions, int32_t *workers_out, int64_t *slots_out);

/* Bytes of workspace mg_decode_attn needs for this plan (0 on bad arguments). */
size_t mg_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t max_seq_len, int32_t num_partitions);

/*
 * mg_decode_attn -- paged decode attention, one query token per request
 * (Mini-SGLang tag page, KV Cache post §一: at step t the query attends to
 * positions 0..t; Stage 1 page §手工驱动引擎 for the metadata).
 *
 *   for request r with L = seq_len[r], row = page_table[table_idx[r]], q head h,
 *   kv head kh = h / (Hq / Hkv):
 *     x_j = scale * <q[r, h, :], k_cache[row[j], kh, :]>,  j = 0 .. L-1
 *     out[r, h, :] = sum_j softmax(x)_j * v_cache[row[j], kh, :]
 *   The new token (position L-1) must already be stored (mg_store_kv).
 *
 *   q, out        [batch, num_q_heads, head_dim] bf16 (out rounded from fp32, RNE)
 *   page_table    [page_table_rows, page_table_stride] int32
 *   table_idx, seq_len  [batch] int32, 1 <= seq_len[r] <= min(max_seq_len, stride)
 *   max_seq_len   host-side upper bound of seq_len
 *   scale         softmax scale, finite and > 0 (else MG_ERR_INVALID_ARGUMENT)
 *   num_partitions 0 = automatic plan; > 0 forces the number of workers
 *   workspace     device buffer of >= mg_decode_workspace_bytes(...) bytes,
 *                 16-byte aligned.  Contents on entry do not matter; it holds
 *                 the per-request unit prefix and the partial results.
 * Launches two kernels on `stream` (workers, then merge).
 * Supported: head_dim == 128, num_q_heads % num_kv_heads == 0, group <= 16,
 * batch <= 131072.
 */
mg_status mg_decode_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                         const int32_t *page_table, int32_t page_table_rows,
                         int32_t page_table_stride, const int32_t *table_idx,
                         const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                         int32_t num_partitions, void *out, void *workspace, size_t workspace_bytes,
                         void *stream);

/*
 * mg_store_decode_attn -- mg_store_kv of the step's new tokens followed by
 * mg_decode_attn, in one launch of the decode kernel (plus the merge kernel)
 * instead of two.  The engine runs exactly this pair in every layer of a
 * decode step (Mini-SGLang tag page, Engine post §一: write KV cache ->
 * attention); fusing it removes a launch and a pool round trip per layer
 * ("mini-sglang from Scratch Stage 4 · Faster and bigger", §What each chapter
 * adds: a step as small as the KV write costs more in launch than in work).
 *
 *   k_new, v_new  [batch, num_kv_heads, head_dim] bf16: request r's new token
 *   out_loc       [batch] int32, out_loc[r] = page_table[table_idx[r]][seq_len[r]-1]
 *   k_cache, v_cache  updated in place exactly as mg_store_kv would
 * Every other argument and the output are those of mg_decode_attn.  The new
 * token's K/V enter attention from k_new / v_new directly; its pool slot is
 * written by the one worker that owns that (request, kv head) tile.  An
 * out_loc[r] that differs from the page-table entry of position seq_len-1 sets
 * MG_DEVERR_LENGTH (the store and the attention would disagree); one outside
 * the pool sets MG_DEVERR_SLOT_RANGE and is not written.
 */
mg_status mg_store_decode_attn(const void *q, const void *k_new, const void *v_new, const int32_t *out_loc,
                               void *k_cache, void *v_cache, int64_t num_slots, const int32_t *page_table,
                               int32_t page_table_rows, int32_t page_table_stride, const int32_t *table_idx,
                               const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                               int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                               int32_t num_partitions, void *out, void *workspace, size_t workspace_bytes,
                               void *stream);

/*
 * mg_decode_attn_shared_prefix -- mg_decode_attn for a batch in which groups
 * of requests share the beginning of their history, as a radix prefix cache
 * hands out (Mini-SGLang tag page, KV Cache post: paged KV with prefix reuse,
 * RadixPrefixCache): the shared tokens are stored once in the pool and every
 * member's page-table row begins with the same slots.  The result is exactly
 * mg_decode_attn's; the shared prefix's K/V rows are read from HBM once per
 * group and KV head, for all the group's q heads, instead of once per request.
 *
 *   requests group_first[G] .. group_first[G+1]-1 form group G (consecutive
 *   in the batch; group_first[0] = 0, group_first[num_groups] = batch, non-
 *   decreasing), and share the first P = prefix_len[G] page-table entries:
 *     page_table[table_idx[r]][j] == page_table[table_idx[group_first[G]]][j]
 *     for every member r and j < P   (the caller's guarantee; not checked)
 *   For each group and KV head, one pass over keys [0, P) of the first
 *   member's row serves the q heads of all members; each request then
 *   attends to its own keys [P, seq_len[r]); the merge kernel combines the
 *   two log-sum-exp partials of every (request, q head).
 *
 *   group_first   [num_groups + 1] int32;  prefix_len [num_groups] int32
 *   A group needs 0 <= P <= seq_len[r] - 1 for every member (the new token is
 *   the request's own) and at most 16 / (num_q_heads / num_kv_heads) members;
 *   P = 0 or a single member is allowed (no sharing).  A group that breaks
 *   these rules sets MG_DEVERR_LENGTH and its members are served as plain
 *   requests (the result stays exact).
 *   workspace     >= mg_decode_shared_prefix_workspace_bytes(...) bytes
 * Every other argument is mg_decode_attn's.  Two kernels on `stream`.
 */
size_t mg_decode_shared_prefix_workspace_bytes(int32_t batch, int32_t num_groups, int32_t num_q_heads,
                                               int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                               int32_t num_partitions);
mg_status mg_decode_attn_shared_prefix(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                                       const int32_t *page_table, int32_t page_table_rows,
                                       int32_t page_table_stride, const int32_t *table_idx,
                                       const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                                       const int32_t *group_first, const int32_t *prefix_len,
                                       int32_t num_groups, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, float scale, int32_t num_partitions, void *out,
                                       void *workspace, size_t workspace_bytes, void *stream);

/*
 * mg_store_decode_attn_shared_prefix -- mg_store_kv of the step's new tokens
 * followed by mg_decode_attn_shared_prefix, in one launch of the decode kernel
 * (plus the merge kernel), as mg_store_decode_attn does for mg_decode_attn.
 * k_new, v_new and out_loc are mg_store_decode_attn's; every other argument
 * and the output are mg_decode_attn_shared_prefix's.  A request's new token
 * (position seq_len-1) lies after its group's prefix, so it is always read
 * and stored by the worker that owns the last tile of the request's own keys.
 * The same checks of out_loc set the same error bits.
 */
mg_status mg_store_decode_attn_shared_prefix(const void *q, const void *k_new, const void *v_new,
                                             const int32_t *out_loc, void *k_cache, void *v_cache,
                                             int64_t num_slots, const int32_t *page_table,
                                             int32_t page_table_rows, int32_t page_table_stride,
                                             const int32_t *table_idx, const int32_t *seq_len, int32_t batch,
                                             int32_t max_seq_len, const int32_t *group_first,
                                             const int32_t *prefix_len, int32_t num_groups,
                                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                             float scale, int32_t num_partitions, void *out, void *workspace,
                                             size_t workspace_bytes, void *stream);

/*
 * mg_extend_attn -- chunked-prefill ("extend") attention over the paged pool
 * (Stage 1 page §手工驱动引擎: positions = arange(cached_len, device_len), new
 * tokens concatenated in request order; Mini-SGLang tag page, Scheduler post:
 * chunked prefill).  The chunk's K/V must already be stored (mg_store_kv).
 *
 *   for request r: c = cached_len[r], n = seq_len[r] - c, new token i < n is
 *   query row t = q_offset[r] + i, at position c + i, and attends to the keys at
 *   positions 0 .. c + i of its page-table row:
 *     out[t, h, :] = sum_{j <= c+i} softmax_j(scale * <q[t, h], k[row[j], kh]>) v[row[j], kh]
 *
 *   q, out        [total_q, num_q_heads, head_dim] bf16
 *   cached_len, seq_len [batch] int32; q_offset [batch + 1] int32 prefix sums of
 *                 n (q_offset[0] = 0, q_offset[batch] = total_q)
 *   max_q_len     host bound of n;  max_seq_len  host bound of seq_len
 *   scale         softmax scale, finite and > 0 (else MG_ERR_INVALID_ARGUMENT)
 * Requests with n == 0 are allowed and produce no rows.  Same shape limits as
 * decode; needs no workspace.
 */
mg_status mg_extend_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                         const int32_t *page_table, int32_t page_table_rows,
                         int32_t page_table_stride, const int32_t *table_idx,
                         const int32_t *cached_len, const int32_t *seq_len,
                         const int32_t *q_offset, int32_t batch, int32_t total_q,
                         int32_t max_q_len, int32_t max_seq_len, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, float scale, void *out,
                         void *stream);

/*
 * mg_mixed_attn -- mg_extend_attn for the mixed batches a chunked-prefill
 * scheduler forms (Mini-SGLang tag page, Scheduler post: continuous batching
 * with chunked prefill), where most requests are decoding (one new token) and
 * a few carry a prompt chunk.  Same arguments, metadata and result as
 * mg_extend_attn, plus a workspace.  Requests with exactly one new token go
 * through the split-KV decode kernel and its merge (query and output row
 * q_offset[r]; all keys 0 .. seq_len-1, the causal limit of a token at
 * position seq_len-1), every other request through the extend kernel, which
 * leaves the one-token requests alone: one call, three kernels, each request
 * served by the kernel built for its shape.
 *   num_partitions  the decode kernel's plan (mg_decode_plan)
 *   extend_ctas     0: the kernels run one after the other on `stream`.  > 0:
 *                   the extend kernel runs on that many SMs at the same time
 *                   as the decode kernel runs on the rest (capped at the SM
 *                   count - 1; the decode plan then has 8 workers per
 *                   remaining SM, or num_partitions if fewer): the decode
 *                   kernel is bound by HBM and the extend kernel by its
 *                   softmax and tensor cores, so they overlap.  The extend
 *                   kernel then runs on a stream the library creates once per
 *                   device and context, forked from and joined back to
 *                   `stream` with two events created and released by the
 *                   call (graph capture follows the fork and the join).  A
 *                   good split gives each kernel the SMs that make them finish
 *                   together; `mixed_extend_ctas` in the Python binding
 *                   estimates it from the batch's lengths.  < 0: invalid.
 *   workspace       >= mg_mixed_workspace_bytes(...) bytes (the decode plan's)
 * Metadata errors are flagged as in mg_decode_attn / mg_extend_attn.
 */
size_t mg_mixed_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_seq_len, int32_t num_partitions);
mg_status mg_mixed_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                        const int32_t *page_table, int32_t page_table_rows, int32_t page_table_stride,
                        const int32_t *table_idx, const int32_t *cached_len, const int32_t *seq_len,
                        const int32_t *q_offset, int32_t batch, int32_t total_q, int32_t max_q_len,
                        int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        float scale, int32_t num_partitions, int32_t extend_ctas, void *out, void *workspace,
                        size_t workspace_bytes, void *stream);

/*
 * mg_decode_attn_static_workspace -- mg_decode_attn for callers that cannot
 * pass device scratch memory.  (The pages have no counterpart: this is a
 * deployment convenience of this library, not a step of the method.)
 *
 * Who needs it: callers whose device memory is all owned by another allocator
 * (a serving engine's pre-sized pool, a framework's caching allocator), so an
 * extra cudaMalloc would fail or fragment it; plug-ins that are given only
 * their inputs and outputs; step loops that must not pay an allocation, which
 * can synchronise the device, in the middle of a step.
 *
 * Same arguments and result as mg_decode_attn, without workspace and
 * workspace_bytes.  The workspace is a fixed array of
 * MG_DECODE_STATIC_WORKSPACE_BYTES in device global memory inside this library;
 * every device that loads the library holds it until the process exits.
 *   - Limit: a plan needing more than MG_DECODE_STATIC_WORKSPACE_BYTES (see
 *     mg_decode_workspace_bytes) returns MG_ERR_WORKSPACE_TOO_SMALL before any
 *     launch; use mg_decode_attn with your own workspace instead.
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on each device looks up the array's device address (with
 *     that device current) and caches it; make that first call before any
 *     stream capture.  The cache is keyed on the CUDA context, so after
 *     cudaDeviceReset the next call (again before any capture) looks the
 *     address up anew in the new context.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Nothing in it needs to start at zero (every value is written before it is
 *     read within a call), but calls that overlap on the GPU (e.g. on two
 *     streams, or from two host threads) race on it and corrupt each other:
 *     serialise them.
 */
#define MG_DECODE_STATIC_WORKSPACE_BYTES (16u << 20)
mg_status mg_decode_attn_static_workspace(const void *q, const void *k_cache, const void *v_cache,
                                          int64_t num_slots, const int32_t *page_table,
                                          int32_t page_table_rows, int32_t page_table_stride,
                                          const int32_t *table_idx, const int32_t *seq_len, int32_t batch,
                                          int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads,
                                          int32_t head_dim, float scale, int32_t num_partitions, void *out,
                                          void *stream);

/*
 * mg_set_extend_wait_limit -- the time bound of mg_extend_attn's pipeline
 * waits, and a fault-injection hook to test what happens when one runs out.
 * (The pages have no counterpart; their engine bounds its distributed setup
 * with a timeout, Stage 1 page §配置, distributed_timeout.)
 *
 * Inside the extend kernel the load warps, the MMA issuer and the softmax
 * warps hand tiles to one another through shared-memory barriers.  Every wait
 * on one gives up after limit_ns nanoseconds: the CTA then records
 * MG_DEVERR_WAIT_TIMEOUT, raises an abort flag that releases every other
 * wait, lets the copies and MMAs it already issued land, frees its tensor
 * memory and returns, so the CUDA context stays usable and
 * mg_read_device_error reports MG_ERR_DEVICE_TIMEOUT.  In normal operation
 * every wait is satisfied within microseconds by the same CTA.
 *
 *   limit_ns      0 restores the default, 2 000 000 000 (2 s)
 *   inject_stall  != 0: later extend launches withhold one hand-off (the
 *                 first score tile of the first Q tile is computed but never
 *                 signalled), so the waits on it run out -- a fault injected
 *                 on purpose, for tests; 0 = normal operation (the default)
 * Process-wide setting, read when mg_extend_attn launches (a launch captured
 * in a CUDA graph keeps the values it was captured with).  The one piece of
 * state the library keeps between calls.  Always MG_OK.
 */
mg_status mg_set_extend_wait_limit(uint64_t limit_ns, int32_t inject_stall);

/*
 * mg_read_device_error -- synchronise `stream`, return the device error word
 * accumulated since the last call on this device (bits MG_DEVERR_*) in
 * *bits_out (may be NULL), and clear it.  Returns MG_OK when no bit was set,
 * MG_ERR_DEVICE_TIMEOUT if MG_DEVERR_WAIT_TIMEOUT is set, else
 * MG_ERR_DEVICE_CHECK.  Not capturable (it synchronises).
 */
mg_status mg_read_device_error(void *stream, uint32_t *bits_out);

#ifdef __cplusplus
}
#endif

#endif /* MG_H */
