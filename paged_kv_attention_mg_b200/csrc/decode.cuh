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
//     pair).
//   * per tile a worker gathers the 16 K and 16 V rows (256 B each) with
//     16-byte cp.async into its own STAGES-deep ring, one full row per 16
//     lanes, XOR-swizzled so ldmatrix is conflict-free; page-table entries of
//     the next tile are prefetched one step ahead.
//   * the GQA group is the M dimension of warp-level bf16 tensor-core MMAs
//     (m16n8k16, fp32 accumulate, g <= 16 rows, zero padded), so each K/V row
//     is read from HBM once for all g heads: S = Q K^T, online softmax in the
//     exp2 domain with quad shuffles, O += P V, O kept in registers.
//   * a segment that is a whole pair writes bf16 output directly; otherwise it
//     writes (O / l, m + log2 l) partials to slot (pair + worker), a slot that
//     is unique because along the unit sequence either the pair or the worker
//     advances at every segment boundary.  The merge kernel combines a pair's
//     partials: lse = log2 sum_s 2^lse_s,  o = sum_s 2^(lse_s - lse) o_s.
//   * no CTA-wide barrier after the prologue: the 4 warps of a CTA only share
//     the scan that locates their first unit.
#pragma once

#include "common.cuh"

namespace mg {
namespace decode {

constexpr int kKeys = 16;          // keys per unit / pipeline tile
constexpr int kWarps = 4;          // workers per CTA
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;          // MMA M: GQA group padded to 16
constexpr int kRowBytes = kHeadDim * 2;
constexpr int kTileBytes = 2 * kKeys * kRowBytes;  // K + V rows of one tile: 8 KB
constexpr int kScanChunk = 4 * kThreads;           // requests per scan step
constexpr int kMaxScanChunks = 256;                // requests <= 131072

#ifndef MG_DECODE_STAGES
#define MG_DECODE_STAGES 2  // per-worker cp.async ring depth (build-time tunable)
#endif
#ifndef MG_DECODE_MIN_BLOCKS
#define MG_DECODE_MIN_BLOCKS 3  // resident CTAs per SM the register budget is sized for
#endif
constexpr int kStages = MG_DECODE_STAGES;
constexpr int kSmemBytes = kWarps * kStages * kTileBytes;

struct Params {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *page_table;
    const int32_t *table_idx;
    const int32_t *seq_len;
    __nv_bfloat16 *out;
    int64_t *prefix;  // [B + 1] units before request r (written by CTA 0 for the merge)
    float *part_lse;  // [slots, group]
    float *part_o;    // [slots, group, 128]
    int64_t num_slots;
    int32_t pt_rows, pt_stride;
    int32_t batch, num_q_heads, num_kv_heads, group;
    int32_t num_workers, max_seq_len;
    float scale_log2;  // softmax scale * log2(e)
};

__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)(row * kRowBytes + ((c ^ (row & 7)) << 4));
}

// Units of request r (0 for a request whose metadata is invalid).
__device__ __forceinline__ int64_t request_units(const Params &p, int r, int &L, int &row, unsigned &bad) {
    row = __ldg(p.table_idx + r);
    L = __ldg(p.seq_len + r);
    if (row < 0 || row >= p.pt_rows) { bad |= MG_DEVERR_ROW_RANGE; return 0; }
    if (L < 1 || L > p.pt_stride || L > p.max_seq_len) { bad |= MG_DEVERR_LENGTH; return 0; }
    return (int64_t)((L + kKeys - 1) / kKeys) * p.num_kv_heads;
}

__device__ __forceinline__ int64_t worker_begin(int64_t total, int w, int W) {
    return (int64_t)(((__int128)total * w) / W);
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

// The walk along a worker's units: pair (r, kvh), tile t of the pair.
struct Cursor {
    int r, kvh, t, tiles, L, row;
    unsigned valid;  // bit i: key i of the tile has an accepted slot (set when issued)
};

__device__ __forceinline__ void cursor_load_request(const Params &p, Cursor &c) {
    for (;;) {
        unsigned bad = 0;
        const int64_t u = request_units(p, c.r, c.L, c.row, bad);
        if (u > 0) {
            c.tiles = (c.L + kKeys - 1) / kKeys;
            return;
        }
        ++c.r;  // zero-unit (rejected) request: it owns no units, skip it
        if (c.r >= p.batch) { c.tiles = 1; c.L = 0; return; }
    }
}

__device__ __forceinline__ void cursor_advance(const Params &p, Cursor &c) {
    if (++c.t < c.tiles) return;
    c.t = 0;
    if (++c.kvh < p.num_kv_heads) return;
    c.kvh = 0;
    ++c.r;
    if (c.r < p.batch) cursor_load_request(p, c);
}

__global__ void __launch_bounds__(kThreads, MG_DECODE_MIN_BLOCKS) decode_kernel(const Params p) {
    extern __shared__ __align__(128) uint8_t smem[];
    __shared__ int64_t sh_scan[kWarps];
    __shared__ int64_t sh_chunk_excl[kMaxScanChunks + 1];
    __shared__ int sh_start_r[kWarps];
    __shared__ int64_t sh_start_prefix[kWarps];

    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    const int W = p.num_workers;
    const int w = blockIdx.x * kWarps + warp;
    const int nchunks = (p.batch + kScanChunk - 1) / kScanChunk;

    // ---- pass 1: units per scan chunk (and the total T)
    unsigned bad = 0;
    int64_t running = 0;
    for (int ch = 0; ch < nchunks; ++ch) {
        int64_t v = 0;
#pragma unroll
        for (int i = 0; i < 4; ++i) {
            const int r = ch * kScanChunk + tid * 4 + i;
            int L, row;
            if (r < p.batch) v += request_units(p, r, L, row, bad);
        }
        int64_t excl;
        const int64_t tot = block_scan_excl(v, excl, sh_scan);
        if (tid == 0) sh_chunk_excl[ch] = running;
        running += tot;
    }
    const int64_t T = running;
    if (tid == 0) sh_chunk_excl[nchunks] = T;
    if (blockIdx.x == 0 && bad) atomicOr(&g_mg_device_error, bad);
    __syncthreads();

    // ---- pass 2: locate the request holding each worker's first unit (CTA 0
    // scans every chunk and also publishes the per-request prefix for the merge)
    {
        const int64_t b0 = worker_begin(T, blockIdx.x * kWarps, W);
        const int64_t b3 = worker_begin(T, blockIdx.x * kWarps + kWarps - 1, W);
        for (int ch = 0; ch < nchunks; ++ch) {
            const int64_t lo = sh_chunk_excl[ch], hi = sh_chunk_excl[ch + 1];
            const bool needed = blockIdx.x == 0 || (hi > b0 && lo <= b3);
            if (!needed) continue;  // uniform across the CTA
            int64_t u[4], v = 0;
            int r0 = ch * kScanChunk + tid * 4;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                int L, row;
                unsigned dummy = 0;
                u[i] = r0 + i < p.batch ? request_units(p, r0 + i, L, row, dummy) : 0;
                v += u[i];
            }
            int64_t excl;
            block_scan_excl(v, excl, sh_scan);
            int64_t pre = lo + excl;
#pragma unroll
            for (int i = 0; i < 4; ++i) {
                const int r = r0 + i;
                if (r < p.batch) {
                    if (blockIdx.x == 0) p.prefix[r] = pre;
#pragma unroll
                    for (int k = 0; k < kWarps; ++k) {
                        const int64_t bk = worker_begin(T, blockIdx.x * kWarps + k, W);
                        if (u[i] > 0 && bk >= pre && bk < pre + u[i]) {
                            sh_start_r[k] = r;
                            sh_start_prefix[k] = pre;
                        }
                    }
                }
                pre += u[i];
            }
        }
        if (blockIdx.x == 0 && tid == 0) p.prefix[p.batch] = T;
    }
    __syncthreads();

    // ---- this warp's share
    const int64_t ub = worker_begin(T, w, W), ue = worker_begin(T, w + 1, W);
    if (w >= W || ub >= ue) return;
    const int n_units = (int)(ue - ub);

    const int64_t head_stride = (int64_t)p.num_kv_heads * kHeadDim;
    const int g = p.group;
    const uint32_t ring = smem_u32(smem) + (uint32_t)(warp * kStages * kTileBytes);

    Cursor cur;  // position of the tile being prefetched
    cur.r = sh_start_r[warp];
    cursor_load_request(p, cur);
    {
        const int64_t off = ub - sh_start_prefix[warp];
        cur.kvh = (int)(off / cur.tiles);
        cur.t = (int)(off - (int64_t)cur.kvh * cur.tiles);
    }

    // per-tile descriptors travel with the pipeline in registers
    Cursor dq[kStages + 1];
    int idx_next = -1;  // lanes 0..15: slot of key lane of the next tile to issue

    auto fetch_idx = [&](const Cursor &c) -> int {
        const int key = c.t * kKeys + lane;
        int s = -1;
        if (lane < kKeys && key < c.L) {
            s = __ldg(p.page_table + (int64_t)c.row * p.pt_stride + key);
            if (s < 0 || (int64_t)s >= p.num_slots) {
                atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
                s = -1;
            }
        }
        return s;
    };
    auto issue = [&](Cursor &c, int slot_reg, int stage) {
        c.valid = __ballot_sync(0xffffffffu, slot_reg >= 0) & 0xFFFFu;
        const uint32_t base = ring + (uint32_t)(stage * kTileBytes);
        const int ch = lane & 15;
#pragma unroll
        for (int it = 0; it < 16; ++it) {
            const int rr = it * 2 + (lane >> 4);  // 0..31: K rows 0-15, V rows 16-31
            const int key = rr & (kKeys - 1);
            const bool is_v = rr >= kKeys;
            const int slot = __shfl_sync(0xffffffffu, slot_reg, key);
            const __nv_bfloat16 *src = (is_v ? p.v_cache : p.k_cache) +
                                       (int64_t)(slot < 0 ? 0 : slot) * head_stride +
                                       (int64_t)c.kvh * kHeadDim + ch * 8;
            cp_async_16(base + (is_v ? kKeys * kRowBytes : 0) + swz(key, ch), src, slot < 0 ? 0u : 16u);
        }
    };

    // prologue: tiles 0 .. STAGES-2 in flight, indices of tile STAGES-1 in registers
    {
        int idx0 = fetch_idx(cur);
#pragma unroll
        for (int s = 0; s < kStages - 1; ++s) {
            if (s < n_units) {
                issue(cur, idx0, s);
                dq[s] = cur;
                cursor_advance(p, cur);
                if (s + 1 < n_units) idx0 = fetch_idx(cur);
            }
            cp_async_commit();
        }
        idx_next = idx0;
    }

    float o[16][4];
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lane/4 and lane/4+8
    uint32_t qf[8][4];
    const int ra = lane >> 2, rb = ra + 8;
    int seg_first_t = 0;

    for (int k = 0; k < n_units; ++k) {
        // issue tile k + STAGES - 1, prefetch the indices of the tile after it
        {
            const int j = k + kStages - 1;
            if (j < n_units) {
                issue(cur, idx_next, j % kStages);
                dq[j % (kStages + 1)] = cur;
                cursor_advance(p, cur);
                if (j + 1 < n_units) idx_next = fetch_idx(cur);
            }
            cp_async_commit();
        }
        const Cursor c = dq[k % (kStages + 1)];
        const bool first = k == 0 || c.t == 0;
        const bool last = k == n_units - 1 || c.t == c.tiles - 1;
        if (first) {
            // new segment: load this pair's q as MMA A fragments, reset the state
            const int h0 = c.kvh * g;
            const int cq = (lane & 3) * 2;
            const __nv_bfloat16 *qa = p.q + ((int64_t)c.r * p.num_q_heads + h0 + ra) * kHeadDim;
            const __nv_bfloat16 *qb = p.q + ((int64_t)c.r * p.num_q_heads + h0 + rb) * kHeadDim;
            const bool va = ra < g, vb = rb < g;
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                const int c0 = kk * 16 + cq;
                qf[kk][0] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + c0)) : 0u;
                qf[kk][1] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + c0)) : 0u;
                qf[kk][2] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + c0 + 8)) : 0u;
                qf[kk][3] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + c0 + 8)) : 0u;
            }
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) o[jj][0] = o[jj][1] = o[jj][2] = o[jj][3] = 0.f;
            m0 = m1 = -INFINITY;
            l0 = l1 = 0.f;
            seg_first_t = c.t;
        }
        cp_async_wait<kStages - 1>();
        __syncwarp();

        const uint32_t kt = ring + (uint32_t)((k % kStages) * kTileBytes);
        const uint32_t vt = kt + kKeys * kRowBytes;

        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int mi = lane >> 3;
            const int key = (mi >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kt + swz(key, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                mma_bf16_16816(sc[0], qf[kk], b0, b1);
                mma_bf16_16816(sc[1], qf[kk], b2, b3);
            }
        }
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int e = 0; e < 2; ++e) {
                const int key = nt * 8 + (lane & 3) * 2 + e;
                // keys past the end, or whose slot was rejected (zero-filled), are masked
                const bool ok = (c.valid >> key) & 1u;
                const float s0 = ok ? sc[nt][e] * p.scale_log2 : -INFINITY;
                const float s1 = ok ? sc[nt][e + 2] * p.scale_log2 : -INFINITY;
                sc[nt][e] = s0;
                sc[nt][e + 2] = s1;
                mx0 = fmaxf(mx0, s0);
                mx1 = fmaxf(mx1, s1);
            }
        }
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 1));
        mx0 = fmaxf(mx0, __shfl_xor_sync(0xffffffffu, mx0, 2));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 1));
        mx1 = fmaxf(mx1, __shfl_xor_sync(0xffffffffu, mx1, 2));
        const float mn0 = fmaxf(m0, mx0), mn1 = fmaxf(m1, mx1);
        const float mu0 = mn0 == -INFINITY ? 0.f : mn0;
        const float mu1 = mn1 == -INFINITY ? 0.f : mn1;
        if (mn0 != m0 || mn1 != m1) {
            const float corr0 = fast_exp2(m0 - mu0), corr1 = fast_exp2(m1 - mu1);
            l0 *= corr0;
            l1 *= corr1;
#pragma unroll
            for (int jj = 0; jj < 16; ++jj) {
                o[jj][0] *= corr0;
                o[jj][1] *= corr0;
                o[jj][2] *= corr1;
                o[jj][3] *= corr1;
            }
            m0 = mn0;
            m1 = mn1;
        }
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sc[nt][0] = fast_exp2(sc[nt][0] - mu0);
            sc[nt][1] = fast_exp2(sc[nt][1] - mu0);
            sc[nt][2] = fast_exp2(sc[nt][2] - mu1);
            sc[nt][3] = fast_exp2(sc[nt][3] - mu1);
            l0 += sc[nt][0] + sc[nt][1];
            l1 += sc[nt][2] + sc[nt][3];
        }
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
        pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
        pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
        pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
        {
            const int mi = lane >> 3;
            const int key = (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vt + swz(key, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
                mma_bf16_16816(o[2 * dp], pa, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
        __syncwarp();  // every lane is done with this stage before it is refilled

        if (last) {
            // ---- finish the segment: whole pair -> bf16 out, else a partial
            float la = l0 + __shfl_xor_sync(0xffffffffu, l0, 1);
            la += __shfl_xor_sync(0xffffffffu, la, 2);
            float lb = l1 + __shfl_xor_sync(0xffffffffu, l1, 1);
            lb += __shfl_xor_sync(0xffffffffu, lb, 2);
            const float ia = la > 0.f ? 1.f / la : 0.f, ib = lb > 0.f ? 1.f / lb : 0.f;
            const bool whole = seg_first_t == 0 && c.t == c.tiles - 1;
            const int64_t head0 = (int64_t)c.r * p.num_q_heads + (int64_t)c.kvh * g;
            const int64_t slot = (int64_t)c.r * p.num_kv_heads + c.kvh + w;
            const int dcol = (lane & 3) * 2;
            if (whole) {
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    if (ra < g)
                        *reinterpret_cast<uint32_t *>(p.out + (head0 + ra) * kHeadDim + jj * 8 + dcol) =
                            pack_bf16x2(o[jj][0] * ia, o[jj][1] * ia);
                    if (rb < g)
                        *reinterpret_cast<uint32_t *>(p.out + (head0 + rb) * kHeadDim + jj * 8 + dcol) =
                            pack_bf16x2(o[jj][2] * ib, o[jj][3] * ib);
                }
            } else {
                float *po = p.part_o + slot * g * kHeadDim;
#pragma unroll
                for (int jj = 0; jj < 16; ++jj) {
                    if (ra < g)
                        *reinterpret_cast<float2 *>(po + ra * kHeadDim + jj * 8 + dcol) =
                            make_float2(o[jj][0] * ia, o[jj][1] * ia);
                    if (rb < g)
                        *reinterpret_cast<float2 *>(po + rb * kHeadDim + jj * 8 + dcol) =
                            make_float2(o[jj][2] * ib, o[jj][3] * ib);
                }
                if ((lane & 3) == 0) {
                    if (ra < g) p.part_lse[slot * g + ra] = la > 0.f ? m0 + __log2f(la) : -INFINITY;
                    if (rb < g) p.part_lse[slot * g + rb] = lb > 0.f ? m1 + __log2f(lb) : -INFINITY;
                }
            }
        }
    }
    cp_async_wait<0>();
}

// One warp per (request, q head): combine the partials of a pair that more
// than one worker touched.
__global__ void __launch_bounds__(128) decode_merge_kernel(const Params p) {
    const int wg = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wg >= p.batch * p.num_q_heads) return;
    const int r = wg / p.num_q_heads, h = wg - r * p.num_q_heads;
    const int g = p.group;
    const int kvh = h / g, j = h - kvh * g;
    const int64_t T = p.prefix[p.batch];
    const int64_t pr = p.prefix[r], units_r = p.prefix[r + 1] - pr;
    if (units_r <= 0 || T <= 0) return;  // rejected request (flagged by the decode kernel)
    const int64_t tiles = units_r / p.num_kv_heads;
    const int64_t u0 = pr + kvh * tiles, u1 = u0 + tiles;  // this pair's units
    const int W = p.num_workers;
    auto worker_of = [&](int64_t u) -> int {
        const int64_t wv = (int64_t)((((__int128)(u + 1)) * W - 1) / T);
        return (int)(wv < W - 1 ? wv : W - 1);
    };
    const int wf = worker_of(u0), wl = worker_of(u1 - 1);
    if (wf == wl) return;  // one worker held the whole pair and wrote the output
    const int64_t pair = (int64_t)r * p.num_kv_heads + kvh;
    float mx = -INFINITY;
    for (int wk = wf + lane; wk <= wl; wk += 32) {
        if (worker_begin(T, wk, W) == worker_begin(T, wk + 1, W)) continue;
        mx = fmaxf(mx, p.part_lse[(pair + wk) * g + j]);
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int wk = wf; wk <= wl; ++wk) {
        if (worker_begin(T, wk, W) == worker_begin(T, wk + 1, W)) continue;
        const int64_t s = pair + wk;
        const float ls = p.part_lse[s * g + j];
        const float wt = ls == -INFINITY ? 0.f : fast_exp2(ls - mx);
        const float4 v = reinterpret_cast<const float4 *>(p.part_o + (s * g + j) * kHeadDim)[lane];
        wsum += wt;
        acc.x += wt * v.x;
        acc.y += wt * v.y;
        acc.z += wt * v.z;
        acc.w += wt * v.w;
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(p.out + ((int64_t)r * p.num_q_heads + h) * kHeadDim + lane * 4) = packed;
}

}  // namespace decode
}  // namespace mg
