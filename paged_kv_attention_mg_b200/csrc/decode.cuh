// decode.cuh -- balanced split-KV paged decode attention + merge.
//
// What it computes: for request r (context length L = seq_len[r], page-table
// row page_table[table_idx[r]]) and q head h, the single query attends to the
// keys at positions 0..L-1 (Mini-SGLang tag page, KV Cache post §一; the new
// token is stored first, Engine post §一).  The score matrix is never written
// to memory; K/V rows are read straight from the pool through the page table
// ("mini-sglang from Scratch Stage 4 · Faster and bigger", §What each chapter
// adds).
//
// Work decomposition (B200 design, not the pages'):
//   * the work is a sequence of units, one unit = 16 consecutive keys of one
//     (request, kv head) pair, ordered request-major, then kv head, then key.
//     Every warp of the grid is an independent worker that takes an equal,
//     contiguous share of the units (floor(w T / W) .. floor((w+1) T / W)), so
//     all workers finish together whatever the length mix (no tail of long
//     splits).  A worker's share covers one or a few "segments" (its part of a
//     pair).  Two CTAs of 4 warps per SM by default, so each SM sub-partition
//     holds two workers (with one 7-warp CTA the worker alone on its
//     sub-partition ran ahead of the others and the call ended with the slowest).
//   * two prefetch distances per worker: the page-table entries of tile
//     k + IDX_AHEAD are copied (4-byte cp.async) into a per-warp index ring, and
//     tile k + STAGES - 1 is gathered (16-byte cp.async, two 256-byte rows per
//     warp instruction) into the warp's STAGES-deep shared-memory ring in the
//     128-byte-swizzled layout ldmatrix reads without bank conflicts.
//   * transposed warp-level bf16 tensor-core products (m16n8k16, fp32
//     accumulate): S^T = K Q^T and O^T += V^T P^T with keys / head dims in M and
//     the GQA heads in N, so each K/V row is read from HBM once for all g heads
//     and a g <= 8 group takes 8 QK^T MMAs per 16-key tile, plus 16 for P V,
//     whose P enters as a bf16 high part and a bf16 residual (P to ~2^-17, so
//     the fp32 row sum of the weights is the normaliser); online softmax in
//     the exp2 domain with quad shuffles, O kept in registers.
//   * shared-prefix mode (CASCADE): the units run over virtual requests, first
//     one per group (the group's common prefix keys, its members' q rows
//     stacked, up to 16 rows = two n-tiles), then one per request (its keys
//     after the prefix); the merge combines a request's own partials with its
//     group's.  The groups' ranges and checked prefixes are copied into shared
//     memory once per CTA.  Mixed-batch mode (row_map): only the one-token
//     requests count units, each writing the output row q_offset[r].
//   * fused store (mg_store_decode_attn, mg_store_decode_attn_shared_prefix):
//     the new token (position L-1) is read from k_new / v_new instead of the
//     pool, and the worker that owns that tile (in shared-prefix mode, the last
//     tile of the request's own keys) writes it to its pool slot from shared
//     memory once the tile has landed.
//   * a segment that is a whole pair writes bf16 output directly; otherwise it
//     writes (O / l, m + log2 l) partials to slot (pair + worker), a slot that
//     is unique because along the unit sequence either the pair or the worker
//     advances at every segment boundary.  The merge kernel combines a pair's
//     partials: lse = log2 sum_s 2^lse_s,  o = sum_s 2^(lse_s - lse) o_s.
//   * no CTA-wide barrier after the prologue: the warps of a CTA only share
//     the scan that locates their first unit.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace mg {
namespace decode {

constexpr int kKeys = 16;          // keys per unit / pipeline tile
#ifndef MG_DECODE_WARPS
#define MG_DECODE_WARPS 4  // workers per CTA (build-time tunable)
#endif
constexpr int kWarps = MG_DECODE_WARPS;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;          // MMA M: GQA group padded to 16
constexpr int kRowBytes = kHeadDim * 2;
constexpr int kTileBytes = 2 * kKeys * kRowBytes;  // K + V rows of one tile: 8 KB
constexpr int kMaxBatch = 131072;                  // requests per call

#ifndef MG_DECODE_STAGES
#define MG_DECODE_STAGES 3  // per-worker ring depth (build-time tunable)
#endif
#ifndef MG_DECODE_MIN_BLOCKS
#define MG_DECODE_MIN_BLOCKS 2  // resident CTAs per SM (the shared memory is sized for it)
#endif
#ifndef MG_DECODE_SPLIT_P
// 1: P enters the PV product as bf16 hi + lo parts (two products), so the
// weights carry ~2^-17 relative error instead of bf16's 2^-9; decode is bound
// by HBM, not by its tensor-core products, so the second product is cheap
#define MG_DECODE_SPLIT_P 1
#endif
#ifndef MG_DECODE_IDX_AHEAD
#define MG_DECODE_IDX_AHEAD 12  // tiles of page-table entries fetched ahead of compute
#endif
constexpr int kStages = MG_DECODE_STAGES;
constexpr int kScanChunk = 4 * kThreads;  // requests per scan step
constexpr int kMaxScanChunks = (kMaxBatch + kScanChunk - 1) / kScanChunk;
constexpr int kIdxAhead = MG_DECODE_IDX_AHEAD;
constexpr int kDescRing = 16;  // per-warp ring of tile descriptors / index rows
static_assert(kDescRing >= kIdxAhead + 1, "descriptor ring too small");
static_assert(kIdxAhead >= kStages, "page-table entries must lead the K/V loads");
constexpr int kRingBytes = kWarps * kStages * kTileBytes;
constexpr int kSmemBytes = kRingBytes + 1024;  // + alignment slack (128-byte swizzle atoms)
constexpr int kHalfRows = kKeys * 128;          // one 64-column half of a 16-row tile: 2 KB

struct Params {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *page_table;
    const int32_t *table_idx;
    const int32_t *seq_len;
    __nv_bfloat16 *out;
    int64_t *prefix;  // [B + 1] units before request r (written by CTA 0 for the merge)
    // fused KV store (store + decode in one launch), else null: the new token
    // of request r is row r of k_new / v_new [B, Hkv, 128], destined for
    // pool slot out_loc[r], which must be the page-table entry of position L-1
    const __nv_bfloat16 *k_new;
    const __nv_bfloat16 *v_new;
    const int32_t *out_loc;
    __nv_bfloat16 *k_store;  // the pools, writable
    __nv_bfloat16 *v_store;
    float *part_lse;  // [slots, rows_per_slot]
    float *part_o;    // [slots, rows_per_slot, 128]
    // shared-prefix (cascade) mode, else num_groups == 0: requests
    // group_first[G] .. group_first[G+1]-1 share the first prefix_len[G]
    // page-table entries, whose K/V rows are read once for all their q heads
    const int32_t *group_first;  // [num_groups + 1]
    const int32_t *prefix_len;   // [num_groups]
    int32_t num_groups;
    int32_t max_members;    // members one shared prefix serves (16 / group)
    int32_t rows_per_slot;  // partial rows per workspace slot: group, or 16 in cascade mode
    int32_t num_vreqs;      // virtual requests: batch (+ num_groups in cascade mode)
    // mixed-batch mode, else null: q and out rows of request r are row row_map[r]
    // ([batch + 1] prefix sums of new tokens, the extend layout) and only
    // requests with exactly one new token are served
    const int32_t *row_map;
    int32_t total_rows;
    int64_t num_slots;
    int32_t pt_rows, pt_stride;
    int32_t batch, num_q_heads, num_kv_heads, group;
    int32_t num_workers, max_seq_len;
    float scale_log2;  // softmax scale * log2(e)
};

// byte offset of 16-byte chunk c (0..15) of row `row` in a [16 rows x 256 B]
// tile stored as two 64-column halves with the 128-byte XOR swizzle
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)((c >> 3) * kHalfRows + row * 128 + (((c & 7) ^ (row & 7)) << 4));
}

// Units of request r (0 for a request whose metadata is invalid).
__device__ __forceinline__ int64_t request_units(const Params &p, int r, int &L, int &row, unsigned &bad) {
    row = __ldg(p.table_idx + r);
    L = __ldg(p.seq_len + r);
    if (p.row_map) {  // mixed batch: requests with other than one new token are not ours
        const int q0 = __ldg(p.row_map + r), q1 = __ldg(p.row_map + r + 1);
        if (q1 - q0 != 1) return 0;
        if (q0 < 0 || q0 >= p.total_rows) { bad |= MG_DEVERR_LENGTH; return 0; }
    }
    if (row < 0 || row >= p.pt_rows) { bad |= MG_DEVERR_ROW_RANGE; return 0; }
    if (L < 1 || L > p.pt_stride || L > p.max_seq_len) { bad |= MG_DEVERR_LENGTH; return 0; }
    return (int64_t)((L + kKeys - 1) / kKeys) * p.num_kv_heads;
}

// q / out row of request r (its own index, or its row of a mixed batch)
__device__ __forceinline__ int64_t row_of(const Params &p, int r) {
    return p.row_map ? (int64_t)__ldg(p.row_map + r) : (int64_t)r;
}

// ---- shared-prefix (cascade) mode: virtual requests.
// A virtual request is a key range [k0, k1) of one page-table row attended by
// the q heads of requests r0 .. r0 + m - 1.  Virtual requests 0 .. G-1 are the
// groups' shared prefixes (keys [0, P) of the first member's row, all members'
// q heads, m <= max_members); G .. G+B-1 are the requests, each over the keys
// after its group's prefix.  A group that is malformed (members outside the
// batch, too many members, or a prefix not shorter than every member's
// length) is flagged and its members are served as plain requests.
struct VReq {
    int row, k0, k1, r0, m;
    bool grouped;  // a request whose prefix is served by its group's virtual request
};

// The shared prefix length of group grp if the group is well formed and has
// one (else 0).
__device__ __forceinline__ int group_prefix(const Params &p, int grp, unsigned &bad) {
    const int P = __ldg(p.prefix_len + grp);
    if (P == 0) return 0;
    const int f0 = __ldg(p.group_first + grp), f1 = __ldg(p.group_first + grp + 1);
    bool ok = P > 0 && f0 >= 0 && f1 <= p.batch && f1 > f0 && f1 - f0 <= p.max_members;
    if (ok) {
        const int row0 = __ldg(p.table_idx + f0);
        ok = row0 >= 0 && row0 < p.pt_rows;
        for (int r = f0; ok && r < f1; ++r) {
            const int L = __ldg(p.seq_len + r);
            ok = L >= 1 && L <= p.pt_stride && L <= p.max_seq_len && P <= L - 1;
        }
    }
    if (!ok) { bad |= MG_DEVERR_LENGTH; return 0; }
    return P;
}

// The group whose member range holds request r, or -1 (group_first is
// non-decreasing in a well-formed call; anything else leaves r ungrouped).
__device__ __forceinline__ int group_of(const Params &p, int r) {
    int lo = 0, hi = p.num_groups - 1;
    while (lo < hi) {  // last group with group_first <= r
        const int mid = (lo + hi + 1) >> 1;
        if (__ldg(p.group_first + mid) <= r) lo = mid; else hi = mid - 1;
    }
    if (p.num_groups <= 0) return -1;
    return (__ldg(p.group_first + lo) <= r && r < __ldg(p.group_first + lo + 1)) ? lo : -1;
}

// Every group's member range and checked prefix length (0 when it has none
// or is malformed), copied to shared memory once per CTA when there are at
// most kGroupCache groups, so that a virtual request's description costs one
// round of metadata loads instead of a chain of them.
constexpr int kGroupCache = kThreads;
struct GroupCache {
    int first[kGroupCache + 1];
    int prefix[kGroupCache];
};

// group_of over the cached group_first
__device__ __forceinline__ int group_of_cached(const GroupCache &gc, int num_groups, int r) {
    if (num_groups <= 0) return -1;
    int lo = 0, hi = num_groups - 1;
    while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (gc.first[mid] <= r) lo = mid; else hi = mid - 1;
    }
    return (gc.first[lo] <= r && r < gc.first[lo + 1]) ? lo : -1;
}

// Units of virtual request v (cascade mode), and its description; gc, when
// given, holds the groups' ranges and prefixes.
__device__ __forceinline__ int64_t vreq_units(const Params &p, int v, VReq &vr, unsigned &bad,
                                              const GroupCache *gc = nullptr) {
    vr.m = 1;
    vr.grouped = false;
    vr.k0 = 0;
    if (v < p.num_groups) {
        const int P = gc ? gc->prefix[v] : group_prefix(p, v, bad);
        if (P == 0) { vr.k1 = 0; return 0; }
        vr.r0 = gc ? gc->first[v] : __ldg(p.group_first + v);
        vr.m = (gc ? gc->first[v + 1] : __ldg(p.group_first + v + 1)) - vr.r0;
        vr.row = __ldg(p.table_idx + vr.r0);
        vr.k1 = P;
        return (int64_t)((P + kKeys - 1) / kKeys) * p.num_kv_heads;
    }
    const int r = v - p.num_groups;
    int L;
    const int64_t u = request_units(p, r, L, vr.row, bad);
    vr.r0 = r;
    vr.k1 = L;
    if (u == 0) return 0;
    const int grp = gc ? group_of_cached(*gc, p.num_groups, r) : group_of(p, r);
    if (grp >= 0) {
        unsigned ignore = 0;  // flagged where the group's own virtual request is resolved
        const int P = gc ? gc->prefix[grp] : group_prefix(p, grp, ignore);
        if (P > 0) {
            vr.k0 = P;
            vr.grouped = true;
        }
    }
    return (int64_t)((L - vr.k0 + kKeys - 1) / kKeys) * p.num_kv_heads;
}

// First unit of worker w out of W over `total` units (the host guarantees
// total * W < 2^62, so the product fits 64 bits).
__device__ __forceinline__ int64_t worker_begin(int64_t total, int w, int W) {
    return total * (int64_t)w / (int64_t)W;
}

// Block-wide exclusive scan of one int64 per thread; returns the block total.
__device__ __forceinline__ int64_t block_scan_excl(int64_t v, int64_t &excl, int64_t *sh) {
    const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
    int64_t x = v;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
        const int64_t y = __shfl_up_sync(0xffffffffu, x, o);
        if (lane >= o) x += y;
    }
    if (lane == 31) sh[warp] = x;
    __syncthreads();
    int64_t before = 0, total = 0;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        const int64_t t = sh[w];
        if (w < warp) before += t;
        total += t;
    }
    __syncthreads();
    excl = before + x - v;
    return total;
}

// The walk along a worker's units: pair (r, kvh), tile t of the pair.  In
// cascade mode r is a virtual request, whose keys start at k0 and whose q
// rows belong to requests r0 .. r0 + m - 1.
struct Cursor {
    int r, kvh, t, tiles, L, row;
    int next_L, next_row;  // metadata of request r + 1, loaded ahead of the boundary
    int k0, r0, m;         // cascade mode (else 0, r, 1)
    bool grouped;
};

// What the pipeline stages need to know about one tile.
struct TileDesc {
    int r, kvh, t, tiles, L, row;
    unsigned valid;  // bit i: key i has an accepted slot (set when the tile is issued)
    int store_slot;  // fused store: out_loc[r] when this is the pair's last tile
    int k0, r0, m;   // first key of the pair's range, first request and count of its q rows
    int grouped;
};

__device__ __forceinline__ bool metadata_ok(const Params &p, int L, int row) {
    return row >= 0 && row < p.pt_rows && L >= 1 && L <= p.pt_stride && L <= p.max_seq_len;
}

__device__ __forceinline__ void cursor_prefetch_next(const Params &p, Cursor &c) {
    if (c.r + 1 < p.batch) {
        c.next_L = __ldg(p.seq_len + c.r + 1);  // consumed only at the next request boundary
        c.next_row = __ldg(p.table_idx + c.r + 1);
    }
}

// Position the cursor on the first request >= c.r that owns units.
template <bool CASCADE>
__device__ __forceinline__ void cursor_load_request(const Params &p, Cursor &c, const GroupCache *gc = nullptr) {
    for (;;) {
        unsigned bad = 0;
        int64_t u;
        if constexpr (CASCADE) {
            VReq vr;
            u = vreq_units(p, c.r, vr, bad, gc);
            c.row = vr.row; c.L = vr.k1; c.k0 = vr.k0; c.r0 = vr.r0; c.m = vr.m; c.grouped = vr.grouped;
        } else {
            u = request_units(p, c.r, c.L, c.row, bad);
            c.k0 = 0; c.r0 = c.r; c.m = 1; c.grouped = false;
        }
        if (u > 0) {
            c.tiles = (c.L - c.k0 + kKeys - 1) / kKeys;
            if constexpr (!CASCADE) cursor_prefetch_next(p, c);
            return;
        }
        ++c.r;  // zero-unit (rejected) request: it owns no units, skip it
        if (c.r >= p.num_vreqs) { c.tiles = 1; c.L = 0; c.k0 = 0; return; }
    }
}

template <bool CASCADE>
__device__ __forceinline__ void cursor_advance(const Params &p, Cursor &c, const GroupCache *gc = nullptr) {
    if (++c.t < c.tiles) return;
    c.t = 0;
    if (++c.kvh < p.num_kv_heads) return;
    c.kvh = 0;
    ++c.r;
    if (c.r >= p.num_vreqs) return;
    if constexpr (CASCADE) {
        cursor_load_request<true>(p, c, gc);
        return;
    }
    if (!p.row_map && metadata_ok(p, c.next_L, c.next_row)) {  // the common case: no stall at the boundary
        c.L = c.next_L;
        c.row = c.next_row;
        c.tiles = (c.L + kKeys - 1) / kKeys;
        cursor_prefetch_next(p, c);
    } else {
        cursor_load_request<false>(p, c);
    }
}

// Units of virtual request v (a request, outside cascade mode).
template <bool CASCADE>
__device__ __forceinline__ int64_t units_of(const Params &p, int v, unsigned &bad, const GroupCache *gc = nullptr) {
    if constexpr (CASCADE) {
        VReq vr;
        return vreq_units(p, v, vr, bad, gc);
    } else {
        int L, row;
        return request_units(p, v, L, row, bad);
    }
}

// NT: n-tiles of 8 q rows (1 for g <= 8, 2 for g <= 16 or cascade mode).
// FUSED: the KV store of the step's new tokens happens in the same launch.
// CASCADE: shared-prefix mode (virtual requests, partial outputs merged).
template <int NT, bool FUSED, bool CASCADE = false>
__global__ void __launch_bounds__(kThreads, MG_DECODE_MIN_BLOCKS)
    decode_kernel(const Params p) {
    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
    __shared__ __align__(16) int idx_ring[kWarps][kDescRing][kKeys];
    __shared__ __align__(16) TileDesc desc_ring[kWarps][kDescRing];
    __shared__ float sh_lse[kWarps][16];
    __shared__ int64_t sh_bound[kWarps + 1];
    __shared__ int64_t sh_scan[kWarps];
    __shared__ int64_t sh_chunk_excl[kMaxScanChunks + 1];
    __shared__ int sh_start_r[kWarps];
    __shared__ int64_t sh_start_prefix[kWarps];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = p.num_workers;
    const int w = blockIdx.x * kWarps + warp;
    const int nchunks = (p.num_vreqs + kScanChunk - 1) / kScanChunk;

    // ---- pass 1: units per scan chunk (and the total T).  It reads request
    // metadata only, which no kernel of this library writes, so it runs before
    // the wait on the previous kernel (e.g. the KV store, or the previous
    // layer's merge) and overlaps that kernel's tail.
    unsigned bad = 0;
    // shared-prefix mode: the groups' ranges and prefixes, checked once
    __shared__ GroupCache sh_gc;
    const GroupCache *gc = nullptr;
    if constexpr (CASCADE) {
        if (p.num_groups <= kGroupCache) {  // uniform
            for (int gi = tid; gi <= p.num_groups; gi += kThreads) {
                sh_gc.first[gi] = __ldg(p.group_first + gi);
                if (gi < p.num_groups) sh_gc.prefix[gi] = group_prefix(p, gi, bad);
            }
            __syncthreads();
            gc = &sh_gc;
        }
    }
    int64_t running = 0;
    int64_t u1[4], excl1 = 0;  // the first chunk's units and prefix, reused by pass 2 when it is the only one
    for (int ch = 0; ch < nchunks; ++ch) {
        int64_t v = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ch * kScanChunk + tid * 4 + i;
            u1[i] = r < p.num_vreqs ? units_of<CASCADE>(p, r, bad, gc) : 0;
            v += u1[i];
        }
        int64_t excl;
        const int64_t tot = block_scan_excl(v, excl, sh_scan);
        if (ch == 0) excl1 = excl;
        if (tid == 0) sh_chunk_excl[ch] = running;
        running += tot;
    }
    const int64_t T = running;
    if (tid == 0) sh_chunk_excl[nchunks] = T;
    if (blockIdx.x == 0 && bad) atomicOr(&g_mg_device_error, bad);
    __syncthreads();

    // ---- pass 2: locate the request holding each worker's first unit (CTA 0
    // scans every chunk and also publishes the per-request prefix for the
    // merge, so it waits first: the workspace may still be read by the
    // previous call's merge; every other warp waits in its main loop, before
    // its first pool, workspace or output access)
    if (blockIdx.x == 0) griddep_wait();
    if (tid <= kWarps) sh_bound[tid] = worker_begin(T, blockIdx.x * kWarps + tid, W);
    __syncthreads();
    {
        const int64_t b0 = sh_bound[0], b3 = sh_bound[kWarps - 1];
        for (int ch = 0; ch < nchunks; ++ch) {
            const int64_t lo = sh_chunk_excl[ch], hi = sh_chunk_excl[ch + 1];
            const bool needed = blockIdx.x == 0 || (hi > b0 && lo <= b3);
            if (!needed) continue;  // uniform across the CTA
            int64_t u[4], v = 0;
            const int r0 = ch * kScanChunk + tid * 4;
            int64_t excl;
            if (nchunks == 1) {  // (uniform) pass 1 scanned this chunk already
#pragma unroll
                for (int i = 0; i < 4; ++i) u[i] = u1[i];
                excl = excl1;
            } else {
#pragma unroll
                for (int i = 0; i < 4; ++i) {
                    unsigned dummy = 0;
                    u[i] = r0 + i < p.num_vreqs ? units_of<CASCADE>(p, r0 + i, dummy, gc) : 0;
                    v += u[i];
                }
                block_scan_excl(v, excl, sh_scan);
            }
            int64_t pre = lo + excl;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + i;
                if (r < p.num_vreqs) {
                    if (blockIdx.x == 0) p.prefix[r] = pre;
#pragma unroll
                    for (int k = 0; k < kWarps; ++k) {
                        const int64_t bk = sh_bound[k];
                        if (u[i] > 0 && bk >= pre && bk < pre + u[i]) {
                            sh_start_r[k] = r;
                            sh_start_prefix[k] = pre;
                        }
                    }
                }
                pre += u[i];
            }
        }
        if (blockIdx.x == 0 && tid == 0) p.prefix[p.num_vreqs] = T;
    }
    __syncthreads();

    // the merge kernel may launch now and wait on us (triggered after the scans
    // rather than at the start: merge CTAs resident beside the scans measured
    // slower on the shared-prefix workload)
    griddep_launch_dependents();

    // ---- this warp's share
    const int64_t ub = sh_bound[warp], ue = sh_bound[warp + 1];
    if (w >= W || ub >= ue) return;
    const int n_units = (int)(ue - ub);

    const int g = p.group;
    const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * kStages * kTileBytes);
    const int64_t head_stride = (int64_t)p.num_kv_heads * kHeadDim;

    Cursor cur;  // position of the next tile whose page-table entries are fetched
    cur.r = sh_start_r[warp];
    cursor_load_request<CASCADE>(p, cur, gc);
    {
        const int64_t off = ub - sh_start_prefix[warp];
        cur.kvh = (int)(off / cur.tiles);
        cur.t = (int)(off - (int64_t)cur.kvh * cur.tiles);
    }
    int (*my_idx)[kKeys] = idx_ring[warp];
    TileDesc *my_desc = desc_ring[warp];

    // Fetch stage: record tile j's descriptor and start copying its 16
    // page-table entries into the index ring (one cp.async group per tile).
    auto fetch = [&](int j) {
        if (j < n_units) {
            const int e = j % kDescRing;
            if (lane == 0) {
                TileDesc d;
                d.r = cur.r; d.kvh = cur.kvh; d.t = cur.t; d.tiles = cur.tiles; d.L = cur.L; d.row = cur.row;
                d.valid = 0; d.store_slot = -1;
                if constexpr (CASCADE) { d.k0 = cur.k0; d.r0 = cur.r0; d.m = cur.m; d.grouped = cur.grouped; }
                my_desc[e] = d;
                // the pair's last tile holds the new token (in shared-prefix mode: of
                // a request's own keys; a group's prefix holds none)
                if (FUSED && cur.t == cur.tiles - 1 && (!CASCADE || cur.r >= p.num_groups))
                    cp_async_4(smem_u32(&my_desc[e].store_slot), p.out_loc + (CASCADE ? cur.r0 : cur.r));
            }
            const int key = cur.k0 + cur.t * kKeys + lane;
            if (lane < kKeys) {
                if (key < cur.L)
                    cp_async_4(smem_u32(&my_idx[e][lane]), p.page_table + (int64_t)cur.row * p.pt_stride + key);
                else
                    my_idx[e][lane] = -1;
            }
            cursor_advance<CASCADE>(p, cur, gc);
        }
    };
    // this lane's shared-memory offsets within a stage for its 16 copies of a
    // tile (lanes 0-15 and 16-31 move one row each per copy: K rows first, then
    // V): the same for every tile, so computed once
    uint32_t soff[16];
#pragma unroll
    for (int it = 0; it < 16; ++it) {
        const int rr = it * 2 + (lane >> 4);
        soff[it] = (rr >= kKeys ? 2 * kHalfRows : 0) + swz(rr & (kKeys - 1), lane & 15);
    }
    const uint32_t row_bytes = (uint32_t)(head_stride * (int64_t)sizeof(__nv_bfloat16));  // one slot's K (or V) row
    // Issue stage: read tile j's entries, check them, gather its 16 K and 16 V
    // rows into the tile's shared-memory stage.
    auto issue = [&](int j) {
        const int e = j % kDescRing, stage = j % kStages;
        const TileDesc d = my_desc[e];
        int slot = -1;
        if (lane < kKeys && (CASCADE ? d.k0 : 0) + d.t * kKeys + lane < d.L) {
            slot = my_idx[e][lane];
            if (slot < 0 || (int64_t)slot >= p.num_slots) {
                atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
                slot = -1;
            }
        }
        const unsigned valid = __ballot_sync(0xffffffffu, slot >= 0) & 0xFFFFu;
        if (lane == 0) my_desc[e].valid = valid;
        // fused store: the new token (position L-1) is read from k_new / v_new,
        // the pool slot is written only after this tile lands.  Its row comes
        // from k_new / v_new whatever its page-table entry holds, so the store
        // writes it even when that entry was rejected (the key is then masked
        // out of the attention, as any rejected key is): its copy is given a
        // non-negative stand-in slot here, once, rather than a test per row below
        const int new_key = (FUSED && d.t == d.tiles - 1 && (!CASCADE || d.r >= p.num_groups))
                                ? d.L - 1 - (CASCADE ? d.k0 : 0) - d.t * kKeys
                                : -1;
        if (FUSED && lane == new_key && slot < 0) slot = 0;
        // 16-byte cp.async: each warp instruction moves two whole 256-byte rows
        // (lanes 0-15 and 16-31); 32 rows per tile (16 K then 16 V)
        const uint32_t base = ring + (uint32_t)(stage * kTileBytes);
        const int ch = lane & 15;
        const size_t head_off = ((size_t)d.kvh * kHeadDim + ch * 8) * sizeof(__nv_bfloat16);
        const char *kb = reinterpret_cast<const char *>(p.k_cache) + head_off;
        const char *vb = reinterpret_cast<const char *>(p.v_cache) + head_off;
        if (FUSED && new_key >= 0) {  // the pair's last tile, which holds the new token
            const int64_t new_off = ((int64_t)(CASCADE ? d.r0 : d.r) * p.num_kv_heads + d.kvh) * kHeadDim + ch * 8;
#pragma unroll
            for (int it = 0; it < 16; ++it) {
                const int key = (it * 2 + (lane >> 4)) & (kKeys - 1);
                const bool is_v = it >= kKeys / 2;
                const int sl = __shfl_sync(0xffffffffu, slot, key);
                const void *src = (is_v ? vb : kb) + (uint64_t)(uint32_t)max(sl, 0) * row_bytes;
                if (key == new_key) src = (is_v ? p.v_new : p.k_new) + new_off;
                cp_async_16(base + soff[it], src, sl < 0 ? 0u : 16u);
            }
        } else {
#pragma unroll
            for (int it = 0; it < 16; ++it) {
                const int key = (it * 2 + (lane >> 4)) & (kKeys - 1);
                const int sl = __shfl_sync(0xffffffffu, slot, key);
                cp_async_16(base + soff[it], (it >= kKeys / 2 ? vb : kb) + (uint64_t)(uint32_t)max(sl, 0) * row_bytes,
                            sl < 0 ? 0u : 16u);
            }
        }
    };

    constexpr int kPre = kIdxAhead;  // page-table fetch runs this many tiles ahead of compute

    // Transposed tile products: S^T[key, head] = K Q^T and O^T[dim, head] +=
    // V^T P^T, keys / dims in the MMA M dimension and the GQA heads in N (8 per
    // n-tile), so a g <= 8 group needs 16 m16n8k16 MMAs per 16-key tile.
    // Fragment ownership: lane l holds heads nt*8 + 2(l%4) + {0,1} of the keys
    // (or dims) l/4 and l/4 + 8.
    float o[NT][8][4];
    float mh[NT][2], lh[NT][2];  // running max / partial sum of this lane's two heads per n-tile
    uint32_t qb[NT][8][2];       // Q^T as B fragments
    const int quad = lane & 3;
    int seg_first_t = 0;
    int k = -kPre;

    // One software pipeline, one cp.async group per iteration k: fetch the
    // page-table entries of tile k + IDX_AHEAD; copy tile k + STAGES - 1 into
    // its shared-memory stage (its entries arrived: their group is
    // IDX_AHEAD - STAGES + 1 iterations old; the stage was freed when tile
    // k - 1 finished); compute tile k.
    for (; k < n_units; ++k) {
        fetch(k + kPre);
        const int j = k + kStages - 1;
        cp_async_wait<kIdxAhead - kStages>();
        __syncwarp();
        // the page-table fetches before the first K/V gather read metadata
        // only, so they run ahead of the wait on the previous kernel
        if (k == 1 - kStages && blockIdx.x != 0) griddep_wait();
        if (j >= 0 && j < n_units) issue(j);
        cp_async_commit();
        if (k < 0) continue;
        const TileDesc c = my_desc[k % kDescRing];
        // n-tiles this tile's query rows need: a grouped shared prefix can fill
        // two, a request's own keys (g <= 8 rows) one
        const int ntu = NT == 1 ? 1 : ((CASCADE ? c.m * g : g) > 8 ? 2 : 1);
        // the tile's work, compiled once per n-tile count so each path keeps
        // its two n-tiles' products interleaved (or has no second one at all)
        auto tile = [&](auto ntu_c) {
            constexpr int NTU = decltype(ntu_c)::value;
            const bool first = k == 0 || c.t == 0;
            const bool last = k == n_units - 1 || c.t == c.tiles - 1;
            if (first) {
                // new segment: this pair's q as B fragments (head l/4 of each n-tile), reset the state
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    const int hl = nt * 8 + (lane >> 2);
                    bool hv;
                    const __nv_bfloat16 *qh;
                    if constexpr (CASCADE) {  // row hl: head hl % g of member hl / g
                        const int member = hl / g;
                        hv = member < c.m;
                        qh = p.q + ((int64_t)(c.r0 + member) * p.num_q_heads + (int64_t)c.kvh * g + (hl - member * g)) *
                                       kHeadDim + quad * 2;
                    } else {
                        hv = hl < g;
                        qh = p.q + (row_of(p, c.r) * p.num_q_heads + (int64_t)c.kvh * g + hl) * kHeadDim + quad * 2;
                    }
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        if (nt >= NTU) break;
                        qb[nt][kk][0] = hv ? __ldg(reinterpret_cast<const uint32_t *>(qh + kk * 16)) : 0u;
                        qb[nt][kk][1] = hv ? __ldg(reinterpret_cast<const uint32_t *>(qh + kk * 16 + 8)) : 0u;
                    }
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) o[nt][dt][0] = o[nt][dt][1] = o[nt][dt][2] = o[nt][dt][3] = 0.f;
                    mh[nt][0] = mh[nt][1] = -INFINITY;
                    lh[nt][0] = lh[nt][1] = 0.f;
                }
                seg_first_t = c.t;
            }
            cp_async_wait<kStages - 1>();  // tile k landed
            __syncwarp();

            const uint32_t kt = ring + (uint32_t)((k % kStages) * kTileBytes);
            const uint32_t vt = kt + 2 * kHalfRows;

            // ---- S^T = K Q^T: two accumulators (even / odd k-steps) halve the MMA chain
            float sa[NT][4], sb[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt)
#pragma unroll
                for (int e = 0; e < 4; ++e) sa[nt][e] = sb[nt][e] = 0.f;
            {
                const int mi = lane >> 3;
                const int key = (mi & 1) * 8 + (lane & 7);
#pragma unroll
                for (int kk = 0; kk < 8; ++kk) {
                    uint32_t a[4];
                    ldmatrix_x4(kt + swz(key, 2 * kk + (mi >> 1)), a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (nt >= NTU) break;
                        if (kk & 1) mma_bf16_16816(sb[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
                        else mma_bf16_16816(sa[nt], a, qb[nt][kk][0], qb[nt][kk][1]);
                    }
                }
            }
            // keys past the end, or whose slot was rejected (zero-filled), are masked
            const bool v0 = (c.valid >> (lane >> 2)) & 1u, v1 = (c.valid >> ((lane >> 2) + 8)) & 1u;
            bool changed = false;
            float sc[NT][4];
#pragma unroll
            for (int nt = 0; nt < NT; ++nt) {
                if (nt >= NTU) break;
                sc[nt][0] = v0 ? (sa[nt][0] + sb[nt][0]) * p.scale_log2 : -INFINITY;  // key l/4,   head even
                sc[nt][1] = v0 ? (sa[nt][1] + sb[nt][1]) * p.scale_log2 : -INFINITY;  // key l/4,   head odd
                sc[nt][2] = v1 ? (sa[nt][2] + sb[nt][2]) * p.scale_log2 : -INFINITY;  // key l/4+8, head even
                sc[nt][3] = v1 ? (sa[nt][3] + sb[nt][3]) * p.scale_log2 : -INFINITY;  // key l/4+8, head odd
                float x0 = fmaxf(sc[nt][0], sc[nt][2]), x1 = fmaxf(sc[nt][1], sc[nt][3]);
#pragma unroll
                for (int off = 4; off < 32; off <<= 1) {
                    x0 = fmaxf(x0, __shfl_xor_sync(0xffffffffu, x0, off));
                    x1 = fmaxf(x1, __shfl_xor_sync(0xffffffffu, x1, off));
                }
                const float n0 = fmaxf(mh[nt][0], x0), n1 = fmaxf(mh[nt][1], x1);
                changed |= (n0 != mh[nt][0]) || (n1 != mh[nt][1]);
                sa[nt][0] = n0;  // reuse: new maxima
                sa[nt][1] = n1;
            }
            if (__any_sync(0xffffffffu, changed)) {
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt >= NTU) break;
                    const float n0 = sa[nt][0], n1 = sa[nt][1];
                    const float c0 = mh[nt][0] == -INFINITY ? 0.f : fast_exp2(mh[nt][0] - (n0 == -INFINITY ? 0.f : n0));
                    const float c1 = mh[nt][1] == -INFINITY ? 0.f : fast_exp2(mh[nt][1] - (n1 == -INFINITY ? 0.f : n1));
                    lh[nt][0] *= c0;
                    lh[nt][1] *= c1;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        o[nt][dt][0] *= c0;
                        o[nt][dt][1] *= c1;
                        o[nt][dt][2] *= c0;
                        o[nt][dt][3] *= c1;
                    }
                    mh[nt][0] = n0;
                    mh[nt][1] = n1;
                }
            }
            // ---- P^T (bf16) as B fragments: lane l needs keys 2(l%4), +1 (and +8)
            // of head l/4, which sit in lanes 8(l%4) + l/8 and that + 4
            uint32_t pb[NT][2];
    #if MG_DECODE_SPLIT_P
            uint32_t pl[NT][2];  // the bf16 residuals p - hi
    #endif
            {
                const int s0 = 8 * quad + (lane >> 3);
                const uint32_t sel = ((lane >> 2) & 1) ? 0x7632u : 0x5410u;
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt >= NTU) break;
                    const float mu0 = mh[nt][0] == -INFINITY ? 0.f : mh[nt][0];
                    const float mu1 = mh[nt][1] == -INFINITY ? 0.f : mh[nt][1];
                    const float p0 = fast_exp2(sc[nt][0] - mu0), p1 = fast_exp2(sc[nt][1] - mu1);
                    const float p2 = fast_exp2(sc[nt][2] - mu0), p3 = fast_exp2(sc[nt][3] - mu1);
                    const uint32_t X = pack_bf16x2(p0, p1), Y = pack_bf16x2(p2, p3);
    #if MG_DECODE_SPLIT_P
                    // hi + lo carries P to ~2^-17 relative, so the fp32 weights are the normaliser
                    lh[nt][0] += p0 + p2;
                    lh[nt][1] += p1 + p3;
                    const uint32_t XL = pack_bf16x2(p0 - bf16x2_lo(X), p1 - bf16x2_hi(X));
                    const uint32_t YL = pack_bf16x2(p2 - bf16x2_lo(Y), p3 - bf16x2_hi(Y));
                    const uint32_t la = __shfl_sync(0xffffffffu, XL, s0), lb = __shfl_sync(0xffffffffu, XL, s0 + 4);
                    const uint32_t lc = __shfl_sync(0xffffffffu, YL, s0), ld = __shfl_sync(0xffffffffu, YL, s0 + 4);
                    pl[nt][0] = __byte_perm(la, lb, sel);
                    pl[nt][1] = __byte_perm(lc, ld, sel);
    #else
                    // the normaliser sums the same bf16-rounded weights the PV product uses
                    lh[nt][0] += bf16x2_lo(X) + bf16x2_lo(Y);
                    lh[nt][1] += bf16x2_hi(X) + bf16x2_hi(Y);
    #endif
                    const uint32_t xa = __shfl_sync(0xffffffffu, X, s0), xb = __shfl_sync(0xffffffffu, X, s0 + 4);
                    const uint32_t ya = __shfl_sync(0xffffffffu, Y, s0), yb = __shfl_sync(0xffffffffu, Y, s0 + 4);
                    pb[nt][0] = __byte_perm(xa, xb, sel);
                    pb[nt][1] = __byte_perm(ya, yb, sel);
                }
            }
            // ---- O^T += V^T P^T (hi, then lo parts of P)
            {
                const int mi = lane >> 3;
                const int key = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
                for (int dt = 0; dt < 8; ++dt) {
                    uint32_t a[4];
                    ldmatrix_x4_trans(vt + swz(key, 2 * dt + (mi & 1)), a[0], a[1], a[2], a[3]);
#pragma unroll
                    for (int nt = 0; nt < NT; ++nt) {
                        if (nt >= NTU) break;
                        mma_bf16_16816(o[nt][dt], a, pb[nt][0], pb[nt][1]);
    #if MG_DECODE_SPLIT_P
                        mma_bf16_16816(o[nt][dt], a, pl[nt][0], pl[nt][1]);
    #endif
                    }
                }
            }
            if (FUSED && c.t == c.tiles - 1 && (!CASCADE || c.r >= p.num_groups)) {
                // fused store: lanes 0-15 copy the new token's K row, lanes 16-31 its V row,
                // 16 bytes each, from the landed stage into pool slot out_loc[r]
                const int nk = c.L - 1 - (CASCADE ? c.k0 : 0) - c.t * kKeys;
                const int ss = c.store_slot;
                const int pt_slot = my_idx[k % kDescRing][nk];
                if (ss < 0 || (int64_t)ss >= p.num_slots) {
                    if (lane == 0) atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
                } else {
                    if (lane == 0 && ss != pt_slot) atomicOr(&g_mg_device_error, MG_DEVERR_LENGTH);
                    const int ch = lane & 15;
                    const bool is_v = lane >= 16;
                    uint4 v;
                    asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
                                 : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
                                 : "r"(kt + (is_v ? 2 * kHalfRows : 0) + swz(nk, ch)));
                    __nv_bfloat16 *dst = (is_v ? p.v_store : p.k_store) + (int64_t)ss * head_stride +
                                         (int64_t)c.kvh * kHeadDim + ch * 8;
                    *reinterpret_cast<uint4 *>(dst) = v;
                }
            }
            __syncwarp();  // every lane is done reading this stage

            if (last) {
                // ---- finish the segment through the (now idle) stage as fp32 scratch
                // [heads][dims + 4]: whole pair -> bf16 out, else a partial
                float *scr = reinterpret_cast<float *>(smem + (size_t)(warp * kStages + k % kStages) * kTileBytes);
                constexpr int kPitch = NT == 1 ? kHeadDim + 4 : kHeadDim;  // pad when there is room
                static_assert(NT * 8 * kPitch * 4 <= kTileBytes, "scratch must fit in one stage");
                float *lse_scr = sh_lse[warp];
#pragma unroll
                for (int nt = 0; nt < NT; ++nt) {
                    if (nt >= NTU) break;
                    float l0 = lh[nt][0], l1 = lh[nt][1];
#pragma unroll
                    for (int off = 4; off < 32; off <<= 1) {
                        l0 += __shfl_xor_sync(0xffffffffu, l0, off);
                        l1 += __shfl_xor_sync(0xffffffffu, l1, off);
                    }
                    const float i0 = l0 > 0.f ? 1.f / l0 : 0.f, i1 = l1 > 0.f ? 1.f / l1 : 0.f;
                    const int h0 = nt * 8 + 2 * quad;
#pragma unroll
                    for (int dt = 0; dt < 8; ++dt) {
                        const int d0 = dt * 16 + (lane >> 2);
                        scr[h0 * kPitch + d0] = o[nt][dt][0] * i0;
                        scr[(h0 + 1) * kPitch + d0] = o[nt][dt][1] * i1;
                        scr[h0 * kPitch + d0 + 8] = o[nt][dt][2] * i0;
                        scr[(h0 + 1) * kPitch + d0 + 8] = o[nt][dt][3] * i1;
                    }
                    if (lane < 4) {  // log2-sum-exp of heads h0, h0 + 1
                        lse_scr[h0] = l0 > 0.f ? mh[nt][0] + __log2f(l0) : -INFINITY;
                        lse_scr[h0 + 1] = l1 > 0.f ? mh[nt][1] + __log2f(l1) : -INFINITY;
                    }
                }
                __syncwarp();
                // a whole pair of a plain request writes the output; anything else
                // (part of a pair, a shared prefix, a request whose prefix is
                // shared) writes partials for the merge kernel
                bool whole = seg_first_t == 0 && c.t == c.tiles - 1;
                if constexpr (CASCADE) whole = whole && !c.grouped && c.r >= p.num_groups;
                const int rows = CASCADE ? c.m * g : g;
                const int64_t rs = CASCADE ? p.rows_per_slot : g;
                const int64_t head0 = (CASCADE ? (int64_t)c.r0 : row_of(p, c.r)) * p.num_q_heads + (int64_t)c.kvh * g;
                const int64_t slot = (int64_t)c.r * p.num_kv_heads + c.kvh + w;
                for (int h = 0; h < rows; ++h) {
                    const float4 v = *reinterpret_cast<const float4 *>(scr + h * kPitch + lane * 4);
                    if (whole) {
                        uint2 packed;
                        packed.x = pack_bf16x2(v.x, v.y);
                        packed.y = pack_bf16x2(v.z, v.w);
                        *reinterpret_cast<uint2 *>(p.out + (head0 + h) * kHeadDim + lane * 4) = packed;
                    } else {
                        *reinterpret_cast<float4 *>(p.part_o + (slot * rs + h) * kHeadDim + lane * 4) = v;
                    }
                }
                if (!whole && lane < rows) p.part_lse[slot * rs + lane] = lse_scr[lane];
                __syncwarp();  // scratch reads done before the stage is refilled
            }
        };
        if constexpr (NT == 1 || !CASCADE) tile(std::integral_constant<int, NT>{});
        else if (ntu == 1) tile(std::integral_constant<int, 1>{});
        else tile(std::integral_constant<int, 2>{});
    }
    cp_async_wait<0>();  // page-table copies still in flight
}

// One warp per (request, q head): combine the partials of a pair that more
// than one worker touched.
#ifndef MG_DECODE_MERGE_BATCH
#define MG_DECODE_MERGE_BATCH 8
#endif
constexpr int kMergeBatch = MG_DECODE_MERGE_BATCH;  // partial segments loaded per round
constexpr int kMergeScanMax = 64;  // requests a merge warp counts units over itself (two per lane)
__global__ void __launch_bounds__(128) decode_merge_kernel(const Params p) {
    const int wg = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    griddep_launch_dependents();
    if (wg >= p.batch * p.num_q_heads) return;
    const int r = wg / p.num_q_heads, h = wg - r * p.num_q_heads;
    const int g = p.group;
    const int kvh = h / g, j = h - kvh * g;
    const int vs = p.num_groups + r;  // the request's own virtual request
    // Before the wait, from request metadata only (which no kernel of this
    // library writes), so it overlaps the decode kernel: with few requests and
    // no shared prefixes, the unit offsets of this request's pair are counted
    // here exactly as the decode kernel counts them; otherwise they come from
    // the table the decode kernel publishes.
    const bool own_scan = p.num_groups == 0 && p.num_vreqs <= kMergeScanMax;
    int64_t T = 0, pr0 = 0, pr1 = 0;
    if (own_scan) {
        int64_t tot = 0, before = 0, mine = 0;
        for (int v = lane; v < p.num_vreqs; v += 32) {
            int L, row;
            unsigned bad = 0;
            const int64_t u = request_units(p, v, L, row, bad);
            tot += u;
            before += v < vs ? u : 0;
            mine += v == vs ? u : 0;
        }
#pragma unroll
        for (int o = 16; o > 0; o >>= 1) {
            tot += __shfl_xor_sync(0xffffffffu, tot, o);
            before += __shfl_xor_sync(0xffffffffu, before, o);
            mine += __shfl_xor_sync(0xffffffffu, mine, o);
        }
        T = tot;
        pr0 = before;
        pr1 = before + mine;
    }
    int grp = -1;  // cascade: the group whose shared prefix this request reads
    if (p.num_groups > 0) {
        grp = group_of(p, r);
        unsigned ignore = 0;
        if (grp >= 0 && group_prefix(p, grp, ignore) == 0) grp = -1;
    }
    griddep_wait();  // the decode kernel's partials (and its unit table)
    if (!own_scan) {
        T = p.prefix[p.num_vreqs];
        pr0 = p.prefix[vs];
        pr1 = p.prefix[vs + 1];
    }
    const int W = p.num_workers;
    const int64_t rs = p.rows_per_slot;
    auto worker_of = [&](int64_t u) -> int {  // the worker whose share holds unit u
        const int64_t wv = ((u + 1) * (int64_t)W - 1) / T;
        return (int)(wv < W - 1 ? wv : W - 1);
    };
    // the workers [wf, wl] that held the pair of kv head kvh of a virtual
    // request whose units start at unit pr (units_v of them)
    auto pair_workers = [&](int64_t pr, int64_t units_v, int &wf, int &wl) -> bool {
        if (units_v <= 0) return false;  // rejected (flagged by the decode kernel)
        const int64_t tiles = units_v / p.num_kv_heads;
        const int64_t u0 = pr + kvh * tiles;
        wf = worker_of(u0);
        wl = worker_of(u0 + tiles - 1);
        return true;
    };
    int wf, wl;
    if (T <= 0 || !pair_workers(pr0, pr1 - pr0, wf, wl)) return;
    int wfp = 0, wlp = -1;
    if (grp >= 0 && !pair_workers(p.prefix[grp], p.prefix[grp + 1] - p.prefix[grp], wfp, wlp)) grp = -1;
    if (grp < 0 && wf == wl) return;  // one worker held the whole pair and wrote the output
    // with at least as many units as workers every share is non-empty; else
    // skip the workers that got no units (and wrote no partial)
    const bool sparse = T < W;
    // online combine, kMergeBatch segments per round so their loads are in flight together
    float mx = -INFINITY, wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    auto combine = [&](int64_t pair, int w_first, int w_last, int row) {
        for (int w0 = w_first; w0 <= w_last; w0 += kMergeBatch) {
            float ls[kMergeBatch];
            float4 v[kMergeBatch];
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i) {
                const int wk = w0 + i;
                const bool use = wk <= w_last && (!sparse || worker_begin(T, wk, W) != worker_begin(T, wk + 1, W));
                const int64_t s = pair + wk;
                ls[i] = use ? p.part_lse[s * rs + row] : -INFINITY;
                v[i] = use ? reinterpret_cast<const float4 *>(p.part_o + (s * rs + row) * kHeadDim)[lane]
                           : make_float4(0.f, 0.f, 0.f, 0.f);
            }
#pragma unroll
            for (int i = 0; i < kMergeBatch; ++i) {
                if (ls[i] == -INFINITY) continue;
                const float mn = fmaxf(mx, ls[i]);
                const float c = mx == -INFINITY ? 0.f : fast_exp2(mx - mn);
                const float wt = fast_exp2(ls[i] - mn);
                wsum = wsum * c + wt;
                acc.x = acc.x * c + wt * v[i].x;
                acc.y = acc.y * c + wt * v[i].y;
                acc.z = acc.z * c + wt * v[i].z;
                acc.w = acc.w * c + wt * v[i].w;
                mx = mn;
            }
        }
    };
    combine((int64_t)vs * p.num_kv_heads + kvh, wf, wl, j);
    if (grp >= 0)  // the shared prefix's partials: this request's row of its group's q rows
        combine((int64_t)grp * p.num_kv_heads + kvh, wfp, wlp, (r - __ldg(p.group_first + grp)) * g + j);
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(p.out + (row_of(p, r) * p.num_q_heads + h) * kHeadDim + lane * 4) = packed;
}

}  // namespace decode
}  // namespace mg
