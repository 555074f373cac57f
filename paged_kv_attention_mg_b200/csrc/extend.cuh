// extend.cuh -- chunked-prefill ("extend") attention on tcgen05 tensor cores.
//
// What it computes ("手写 mini-sglang 阶段一 · Engine 与采样器", §手工驱动引擎;
// Mini-SGLang tag page, Scheduler post, chunked prefill): request r has
// c = cached_len[r] tokens in the pool and n = seq_len[r] - c new ones, already
// stored; new token i (query row q_offset[r] + i, position c + i) attends to the
// keys at positions 0 .. c + i of its page-table row.
//
// Work decomposition (B200 design):
//   * a work item is (request, kv head, q block); a q block is two 128-row Q
//     tiles, a row being (token, head) with the g heads that share the KV head
//     adjacent, so one K/V tile feeds 2 x 128 query rows (GQA packing).  An
//     item costs one pass over its keys, ceil((c + last token + 1) / 128) KV
//     tiles of 128 keys.
//   * persistent CTAs, one per SM.  Every CTA computes the same work list
//     (items sorted by cost, heaviest first, when at most kMaxSortGroups
//     (request, q block) groups hold tokens: a block-wide scan over the
//     requests compacts them, one warp sorts them in registers) and takes its
//     items in snake order (k, 2G-1-k, 2G+k, ...),
//     so the heavy items start first and the loads even out.  Across a CTA's
//     items the pipelines never drain: K/V rings, barrier phases and TMEM run
//     on, the next item's Q tiles load while the current item finishes, and an
//     item's epilogue overlaps the next item's first Q K^T.
//   * 16 warps in four warpgroups, register budgets moved by setmaxnreg
//     (warpgroups 0 and 3: 72 registers a thread; 1 and 2: 184):
//       - warps 0-3 load V tiles, warps 13-15 load K tiles (decoupled rings, so
//         K can run ahead of V): 16-byte cp.async straight from the paged pool
//         into the 128-byte swizzled UMMA layout, each warp instruction moving
//         two 256-byte rows; each lane holds the page-table entries of the keys
//         it is responsible for in registers, fetched a tile ahead; the tile's
//         full barrier is armed by cp.async.mbarrier.arrive.noinc, so it
//         completes when the copies land and the loaders never wait for them.
//       - warp 12, one thread: tcgen05.mma (M=128, N=128, K=16, bf16 in, fp32
//         accumulate in TMEM).  S_t = Q_t K^T lands in TMEM; P_t (bf16) is
//         written back over S_t and consumed straight from TMEM as the A
//         operand of O_t += P_t V.  Issue order S0, S1, then per KV tile
//         P0 V, S0', P1 V, S1': while one Q tile's softmax runs, the tensor
//         core works on the other's.
//       - warpgroups 1 / 2: softmax of Q tile 0 / 1, one TMEM lane (= query
//         row) per thread: causal mask key <= c + i, online softmax in the
//         exp2 domain (exponentials on MUFU; 32-key chunks past every row's
//         causal edge skipped), O rescaled in TMEM only when the running max
//         grows by more than 2^8 (exact: P and the row sum use the same stale
//         max and the same bf16-rounded P), epilogue O / l -> bf16 -> global.
//         Each also
//         loads its next item's Q tile by TMA as soon as its last score tile
//         has landed (the tile's last reader is that Q K^T).
// TMEM: S0 [0,128)  S1 [128,256)  O0 [256,384)  O1 [384,512) columns.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace mg {
namespace extend {

constexpr int kM = 128;                     // query rows per Q tile
constexpr int kN = 128;                     // keys per KV tile
constexpr int kQTiles = 2;
// Ring depths and loader warps: V gets the deeper ring and the larger loader
// group because a V tile is needed only ~one softmax after its K tile but its
// slot frees later (after both Q tiles' P V); measured with K 3 / V 2, the MMA
// issuer waited for V tiles while K tiles sat ready for over 10k cycles.
constexpr int kKStages = 2;                 // K ring
constexpr int kVStages = 3;                 // V ring
constexpr int kThreads = 512;
constexpr int kKLoadWarp0 = 13, kKLoaders = 3;   // K loaders: warps 13-15
constexpr int kMmaWarp = 12;
constexpr int kVLoadWarp0 = 0, kVLoaders = 4;    // V loaders: warps 0-3
constexpr int kPairs = kN / 2;              // row pairs per tile (one warp instruction moves a pair)
constexpr int kRegsLoad = 72;               // registers a thread in warpgroups 0 and 3
constexpr int kRegsSoftmax = 184;           // registers a thread in warpgroups 1 and 2
static_assert(2 * 128 * kRegsLoad + 2 * 128 * kRegsSoftmax == 65536 && 65536 / kThreads == 128,
              "the register split must add up to what the block is launched with");
constexpr int kHalfBytes = 128 * 128;       // 128 rows x 128 B (64 bf16): one swizzle column
constexpr int kTileBytes = 2 * kHalfBytes;  // 128 rows x 256 B
constexpr int kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int t) { return (uint32_t)t * 128u; }
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + (uint32_t)t * 128u; }
constexpr float kRescaleThreshold = 8.0f;   // log2 units
// The work list is sorted by cost when at most kMaxSortGroups groups hold
// tokens (a group: the Hkv items of one (request, q block), which cost the
// same); one warp sorts the group keys in registers.  A CTA keeps at most
// kMaxItemsPerCta items of a sorted list: the host sizes the grid for that
// when every group may hold tokens, otherwise the kernel checks it and walks
// the unsorted enumeration instead.
constexpr int kSortPerLane = 8;
constexpr int kMaxSortGroups = 32 * kSortPerLane;
constexpr int kMaxItemsPerCta = 32;
constexpr int kMaxCost = 0xFFFF;            // cost key clamp (KV tiles)
#ifndef MG_EXTEND_EMU_PAIRS
#define MG_EXTEND_EMU_PAIRS 0  // of every 16 pairs of exponentials, this many on the FMA pipe
#endif
constexpr int kEmuPairs = MG_EXTEND_EMU_PAIRS;
static_assert(kEmuPairs >= 0 && kEmuPairs <= 16, "pairs per chunk of 16");

// shared memory map.  The kernel has no static shared memory, so its dynamic
// shared memory starts on a 1024-byte boundary (checked at run time), as the
// 128-byte swizzle atoms require; every tile region below keeps that alignment.
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
constexpr int kOffV = kOffK + kKStages * kTileBytes;
constexpr int kOffBar = kOffV + kVStages * kTileBytes;
// mbarriers, by index (8 bytes each from kOffBar)
constexpr int kBarDrain = 0;
constexpr int kBarQFull = kBarDrain + 1;          // + Q tile
constexpr int kBarKFull = kBarQFull + kQTiles;    // + K stage
constexpr int kBarKEmpty = kBarKFull + kKStages;
constexpr int kBarVFull = kBarKEmpty + kKStages;  // + V stage
constexpr int kBarVEmpty = kBarVFull + kVStages;
constexpr int kBarSFull = kBarVEmpty + kVStages;  // + Q tile
constexpr int kBarPFull = kBarSFull + kQTiles;
constexpr int kBarODone = kBarPFull + kQTiles;
constexpr int kBarOFree = kBarODone + kQTiles;
constexpr int kNumBars = kBarOFree + kQTiles;
constexpr int kOffItems = kOffBar + kNumBars * 8;
constexpr int kOffMisc = kOffItems + kMaxItemsPerCta * 4;
constexpr int kSmemBytes = kOffMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "extend shared memory over the per-CTA limit");
static_assert(kMaxSortGroups * 4 + (kThreads / 32 + 1) * 4 <= kKStages * kTileBytes,
              "the group scan and the sort run in the K ring before any load");

struct Params {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *page_table;
    const int32_t *table_idx;
    const int32_t *cached_len;
    const int32_t *seq_len;
    const int32_t *q_offset;
    __nv_bfloat16 *out;
    int64_t num_slots;
    int32_t pt_rows, pt_stride;
    int32_t batch, total_q, max_q_len, max_seq_len;
    int32_t num_q_heads, num_kv_heads, group;
    int32_t tokens_per_qtile;  // floor(128 / group)
    int32_t num_qblocks;       // ceil(max_q_len / (2 * tokens_per_qtile))
    int32_t num_items;         // num_qblocks * batch * num_kv_heads
    int32_t sorted;            // num_qblocks * batch < 2^16: try the sorted list (group ids fit a key)
    float scale_log2;
    int32_t skip_single;       // mixed batches: requests with one new token are served by decode
    uint64_t wait_limit_ns;    // bound of every pipeline wait
    int32_t inject_stall;      // test hook: withhold the first score tile's hand-off
};

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 version bits, as
// its two 32-bit words.  The low word holds the start address (bits 0-13, in
// 16-byte units) and the leading byte offset; the high word the stride byte
// offset, the version bit (46) and the swizzle mode (61-63), fixed per operand
// kind.  A k step or a stage moves only the address field, by a constant: the
// issuer adds it to the low word (the field cannot carry: shared addresses
// stay below 2^18 bytes).
__device__ __forceinline__ uint32_t sw128_lo(uint32_t saddr, uint32_t lbo) {
    return ((saddr & 0x3FFFFu) >> 4) | (((lbo >> 4) & 0x3FFFu) << 16);
}
__host__ __device__ constexpr uint32_t sw128_hi(uint32_t sbo) {
    return ((sbo >> 4) & 0x3FFFu) | (1u << 14) | (2u << 29);
}

// Instruction descriptor, kind::f16: bf16 x bf16 -> f32, M = 128, N = 128.
__host__ __device__ constexpr uint32_t idesc_bf16(bool b_mn_major) {
    return (1u << 4)                         // D format f32
           | (1u << 7)                       // A bf16
           | (1u << 10)                      // B bf16
           | ((b_mn_major ? 1u : 0u) << 16)  // B major
           | ((uint32_t)(kN >> 3) << 17)     // N / 8
           | ((uint32_t)(kM >> 4) << 24);    // M / 16
}

// shared-memory address of mbarrier `index`
__device__ __forceinline__ uint32_t bar_at(uint32_t sbase, int index) {
    return sbase + (uint32_t)(kOffBar + index * 8);
}

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    return now;
}

// Waits with a time bound (limit_ns, timed from the wait's first check of the
// clock); on timeout records the error, raises the CTA abort flag and returns
// false.  Once the flag is up every later wait returns false at once, so all
// roles drain to the final barrier.  A phase that has already completed (the
// common case for the issuer's K and V waits) returns at the first,
// non-blocking test.
__device__ __forceinline__ bool wait_or_abort_thread(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                     uint64_t limit_ns) {
    if (mbar_test_wait(bar, parity)) return true;
    if (*abort_flag) return false;
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 1023u) == 1023u) {
            const uint64_t now = global_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > limit_ns || *abort_flag) {
                *abort_flag = 1;
                atomicOr(&g_mg_device_error, MG_DEVERR_WAIT_TIMEOUT);
                return false;
            }
        }
    }
}

// A bounded wait that ignores the abort flag: used after an abort to let work
// already in flight (issued MMAs, a TMA load) land before the CTA frees TMEM
// and exits.  Returns false if the bound ran out.
__device__ __forceinline__ bool wait_bounded(uint32_t bar, uint32_t parity, uint64_t limit_ns) {
    uint64_t t0 = 0;
    for (uint32_t it = 0;; ++it) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((it & 1023u) == 1023u) {
            const uint64_t now = global_ns();
            if (t0 == 0) t0 = now;
            else if (now - t0 > limit_ns) return false;
        }
    }
}

// Warp-uniform form for roles where all 32 lanes wait together: the warp
// proceeds only if every lane did (tcgen05.ld/st and __syncwarp need the whole
// warp converged).  The single-thread MMA issuer uses wait_or_abort_thread.
__device__ __forceinline__ bool wait_or_abort(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                              uint64_t limit_ns) {
    const bool ok = wait_or_abort_thread(bar, parity, abort_flag, limit_ns);
    return __all_sync(0xffffffffu, ok);
}

// ---------------------------------------------------------------- exp2 on the FMA pipe
// 2^x for x <= 8 from fused multiply-adds and integer adds, for a share of the
// softmax exponentials, so that the MUFU unit (16 results per clock per SM,
// as many as the tensor core finishes (query, key) pairs at head_dim 128) is
// not the only unit computing them.  Method: Cody-Waite range reduction
// x = n + f with n = round(x) (by adding 1.5 * 2^23, which leaves round(x)
// in the low mantissa bits) and f in [-1/2, 1/2]; 2^f by a degree-3
// polynomial whose coefficients were fitted here to minimise the relative
// error on that interval (7.5e-5, far below half a bf16 ulp, 2^-9); then n
// added to the exponent field.  x is clamped at -126 first, so the exponent
// never underflows past zero (such weights are below 2^-126 of the row max,
// zero in bf16 after the sum).
__device__ __forceinline__ float2 exp2_fma2(float2 x) {
    constexpr float kRound = 12582912.0f;  // 1.5 * 2^23
    x.x = fmaxf(x.x, -126.0f);
    x.y = fmaxf(x.y, -126.0f);
    const float2 round2 = make_float2(kRound, kRound);
    const float2 t = fadd2(x, round2);
    const float2 f = fsub2(x, fsub2(t, round2));
    float2 p = ffma2(make_float2(0.05517132208f, 0.05517132208f), f,
                     make_float2(0.24261054396f, 0.24261054396f));
    p = ffma2(p, f, make_float2(0.69326096773f, 0.69326096773f));
    p = ffma2(p, f, make_float2(0.99992811680f, 0.99992811680f));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}

// ---------------------------------------------------------------- work items
// Item id enumeration (also the tie order of the sorted list): the q block
// with the latest tokens first, then request, then kv head.
struct Item {
    int r, kvh, row, c, n, qo, tok0, kv_len, n_kv;
    bool q1;  // the second Q tile holds tokens
};

// Request r's metadata into it (row, c, n, qo): 1, or -1 when it is
// inconsistent (no item of the request runs).
__device__ __forceinline__ int request_info(const Params &p, int r, Item &it) {
    it.r = r;
    it.row = __ldg(p.table_idx + it.r);
    it.c = __ldg(p.cached_len + it.r);
    const int L = __ldg(p.seq_len + it.r);
    it.qo = __ldg(p.q_offset + it.r);
    it.n = L - it.c;
    if (it.row < 0 || it.row >= p.pt_rows || it.c < 0 || it.n < 0 || L > p.pt_stride || L > p.max_seq_len ||
        it.n > p.max_q_len || it.qo < 0 || it.qo + it.n > p.total_q || __ldg(p.q_offset + it.r + 1) - it.qo != it.n)
        return -1;
    return 1;
}

// 1: the item has work; 0: its q block holds no token of the request;
// -1: the request's metadata is inconsistent (no item of it runs).
__device__ __forceinline__ int item_info(const Params &p, int id, Item &it) {
    const int per_qb = p.batch * p.num_kv_heads;
    const int qb = p.num_qblocks - 1 - id / per_qb;
    const int rest = id - (id / per_qb) * per_qb;
    if (request_info(p, rest / p.num_kv_heads, it) < 0) return -1;
    it.kvh = rest - it.r * p.num_kv_heads;
    const int tpq = p.tokens_per_qtile;
    it.tok0 = qb * kQTiles * tpq;
    if (it.tok0 >= it.n || (p.skip_single && it.n == 1)) return 0;
    const int last_tok = min(it.tok0 + kQTiles * tpq, it.n) - 1;
    it.kv_len = it.c + last_tok + 1;
    it.n_kv = (it.kv_len + kN - 1) / kN;
    it.q1 = it.tok0 + tpq < it.n;
    return 1;
}

// error bits of a request whose item_info returned -1
__device__ __forceinline__ unsigned item_error(const Params &p, const Item &it) {
    return (it.row < 0 || it.row >= p.pt_rows) ? (unsigned)MG_DEVERR_ROW_RANGE : (unsigned)MG_DEVERR_LENGTH;
}

// The position in the work list of this CTA's k-th item: snake order over the
// G CTAs (k, 2G-1-k, 2G+k, ...).
__device__ __forceinline__ int snake_position(int k) {
    const int G = gridDim.x, c = blockIdx.x;
    const int round = k >> 1;
    return round * 2 * G + ((k & 1) ? 2 * G - 1 - c : c);
}

// Walks this CTA's items: sorted mode reads the CTA's list, otherwise the
// item ids at the snake positions of the enumeration (skipping empty ones).
struct ItemCursor {
    int k;  // next index into the CTA's sequence
};
// With `flag` set, an item whose request metadata is inconsistent is flagged
// (unsorted mode: each CTA flags the items at its own positions; sorted mode
// flags them while the list is built).
__device__ __forceinline__ bool next_item(const Params &p, ItemCursor &cur, const int *list, int list_len,
                                          bool sorted, Item &it, bool flag = false) {
    for (;;) {
        int id;
        if (sorted) {
            if (cur.k >= list_len) return false;
            id = list[cur.k++];
        } else {
            id = snake_position(cur.k++);
            if (id >= p.num_items) return false;
        }
        const int st = item_info(p, id, it);
        if (st == 1) return true;
        if (st < 0 && flag && !sorted) atomicOr(&g_mg_device_error, item_error(p, it));
    }
}

// ---------------------------------------------------------------- loaders
// One loader group (NW warps) copies the K (or V) rows of every tile of the
// CTA's items into its ring.  Warp u of the group owns the row pairs
// p = u, u + NW, ... of a tile (keys 2p, 2p+1); its key list index i is pair
// i / 2, key 2p + (i & 1), and lane l holds the page-table entries (slots) of
// list indices l and l + 32, fetched one tile ahead.
template <int NW, int STAGES>
__device__ __forceinline__ void load_rows(const Params &p, uint32_t ring_base, uint32_t full0, uint32_t empty0,
                                          const __nv_bfloat16 *pool, int u, int lane, const int *list, int list_len,
                                          bool sorted, volatile int *abort_flag, uint64_t lim, bool flag_errors) {
    constexpr int kMaxPairs = (kPairs + NW - 1) / NW;
    const int npairs = (kPairs - u + NW - 1) / NW;
    const uint32_t row_bytes = (uint32_t)p.num_kv_heads * kHeadDim * 2;  // one slot's K (or V) row
    auto key_of = [&](int i) { return 2 * (u + NW * (i >> 1)) + (i & 1); };
    // slots of (item, tile j) for list indices lane and lane + 32 (-1: none)
    auto fetch = [&](int row, int kv_len, int j, int &sa, int &sb) {
        const int32_t *pt = p.page_table + (int64_t)row * p.pt_stride;
        sa = sb = -1;
        const int ka = j * kN + key_of(lane), kb = j * kN + key_of(lane + 32);
        if (lane < 2 * npairs && ka < kv_len) sa = __ldg(pt + ka);
        if (lane + 32 < 2 * npairs && kb < kv_len) sb = __ldg(pt + kb);
    };
    // a slot outside the pool: flagged, and its row zero-filled (and masked by
    // the causal limit or never read: a rejected key of a visible position
    // reads as zeros, as in the other kernels' bounds checks)
    auto check = [&](int &s, bool present) {
        if (present && (s < 0 || (int64_t)s >= p.num_slots)) {
            if (flag_errors) atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
            s = -1;
        }
    };
    ItemCursor cur{0};
    const bool flag_items = flag_errors && u == 0 && lane == 0;
    int row, kvh, kv_len, n_kv;  // the current item, as the copies need it
    {
        Item it;
        if (!next_item(p, cur, list, list_len, sorted, it, flag_items)) return;
        row = it.row; kvh = it.kvh; kv_len = it.kv_len; n_kv = it.n_kv;
    }
    int j = 0;
    int sa, sb;
    fetch(row, kv_len, 0, sa, sb);
    const int c = lane & 15, half = c >> 3, cc = c & 7;
    // the shared-memory offset of each of this lane's copies within a stage: the
    // same for every tile, so it is computed once
    uint32_t doff[kMaxPairs];
#pragma unroll
    for (int m = 0; m < kMaxPairs; ++m) {
        const int key = key_of(2 * m + (lane >> 4));
        doff[m] = (uint32_t)(half * kHalfBytes + key * 128 + ((cc ^ (key & 7)) << 4));
    }
    for (int seq = 0;; ++seq) {
        // tile (it, j): wait for its ring stage
        const int stage = seq % STAGES;
        if (seq >= STAGES && !wait_or_abort(empty0 + stage * 8, ((seq / STAGES) - 1) & 1, abort_flag, lim)) break;
        check(sa, lane < 2 * npairs && j * kN + key_of(lane) < kv_len);
        check(sb, lane + 32 < 2 * npairs && j * kN + key_of(lane + 32) < kv_len);
        const uint32_t tile = ring_base + (uint32_t)(stage * kTileBytes);
        const char *base = reinterpret_cast<const char *>(pool + (int64_t)kvh * kHeadDim + c * 8);
#pragma unroll
        for (int m = 0; m < kMaxPairs; ++m) {
            if (m < npairs) {
                const int i = 2 * m + (lane >> 4);  // list index this half-warp copies
                const int slot = m < 16 ? __shfl_sync(0xffffffffu, sa, i & 31) : __shfl_sync(0xffffffffu, sb, i & 31);
                // one wide multiply-add: base + slot * row bytes (a slot row is at most 4 KB)
                const char *src = base + (uint64_t)(uint32_t)max(slot, 0) * row_bytes;
                cp_async_16(tile + doff[m], src, slot < 0 ? 0u : 16u);
            }
        }
        cp_async_arrive_noinc(full0 + stage * 8);
        // advance to the next tile and fetch its page-table entries now, so they
        // arrive while this warp waits for the next stage
        if (++j == n_kv) {
            Item it;
            if (!next_item(p, cur, list, list_len, sorted, it, flag_items)) break;
            row = it.row; kvh = it.kvh; kv_len = it.kv_len; n_kv = it.n_kv;
            j = 0;
        }
        fetch(row, kv_len, j, sa, sb);
    }
    cp_async_commit();
    cp_async_wait<0>();  // nothing in flight into shared memory at teardown
}

// ---------------------------------------------------------------- the sort
// One warp sorts the 32 * R keys at `keys` (shared memory) in descending order:
// a bitonic network over elements e = lane * R + r, partners within a lane
// compared by register, partners across lanes by shuffle.
template <int R, int J>
__device__ __forceinline__ void sort_local_stage(uint32_t (&kr)[R], int lane, int k) {
#pragma unroll
    for (int r = 0; r < R; ++r) {
        if ((r & J) == 0) {
            const int e = lane * R + r;
            const bool desc = (e & k) == 0;
            const uint32_t a = kr[r], b = kr[r | J];
            const bool swap = desc ? a < b : a > b;
            kr[r] = swap ? b : a;
            kr[r | J] = swap ? a : b;
        }
    }
}
template <int R>
__device__ __forceinline__ void warp_sort_desc(uint32_t *keys, int lane) {
    uint32_t kr[R];
#pragma unroll
    for (int r = 0; r < R; ++r) kr[r] = keys[lane * R + r];
    for (int k = 2; k <= 32 * R; k <<= 1) {
        for (int j = k >> 1; j >= R; j >>= 1) {
            const int lane_mask = j / R;
#pragma unroll
            for (int r = 0; r < R; ++r) {
                const int e = lane * R + r;
                const uint32_t other = __shfl_xor_sync(0xffffffffu, kr[r], lane_mask);
                const bool lower = (e & j) == 0, desc = (e & k) == 0;
                kr[r] = lower == desc ? max(kr[r], other) : min(kr[r], other);
            }
        }
        if constexpr (R >= 8) {
            if (k >= 8) sort_local_stage<R, 4>(kr, lane, k);
        }
        if (k >= 4) sort_local_stage<R, 2>(kr, lane, k);
        sort_local_stage<R, 1>(kr, lane, k);
    }
    __syncwarp();
#pragma unroll
    for (int r = 0; r < R; ++r) keys[lane * R + r] = kr[r];
}

// ---------------------------------------------------------------- the kernel

__global__ void __launch_bounds__(kThreads, 1)
    extend_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment: refuse, never fault
        if (threadIdx.x == 0) atomicOr(&g_mg_device_error, MG_DEVERR_INTERNAL);
        return;
    }
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + kOffMisc + 4);
    int *sh_count = reinterpret_cast<int *>(smem + kOffMisc + 8);
    int *items = reinterpret_cast<int *>(smem + kOffItems);
    const uint64_t lim = p.wait_limit_ns;  // nanoseconds
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
    griddep_launch_dependents();

    // ---- the work list.  Sorted mode: every CTA sorts the same group keys
    // (cost descending, enumeration order for ties; a group is the Hkv items of
    // one (request, q block), which cost the same) and keeps the item ids at its
    // snake positions of the expanded list.  The keys live in the K ring, which
    // no load has touched yet.
    bool sorted = false;
    int groups = 0;  // groups that hold tokens
    if (p.sorted) {
        uint32_t *keys = reinterpret_cast<uint32_t *>(smem + kOffK);
        int *scan = reinterpret_cast<int *>(smem + kOffK + kMaxSortGroups * 4);  // kThreads / 32 + 1 ints
        if (tid < kMaxSortGroups) keys[tid] = 0;
        // each thread counts the groups of its requests that hold tokens ...
        int mine = 0;
        for (int r = tid; r < p.batch; r += kThreads) {
            Item it;
            const int st = request_info(p, r, it);
            if (st < 0 && blockIdx.x == 0) atomicOr(&g_mg_device_error, item_error(p, it));
            if (st >= 0 && !(p.skip_single && it.n == 1)) mine += (it.n + kQTiles * p.tokens_per_qtile - 1) /
                                                                 (kQTiles * p.tokens_per_qtile);
        }
        // ... a block-wide exclusive scan places them ...
        int incl = mine;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
            const int y = __shfl_up_sync(0xffffffffu, incl, o);
            if (lane >= o) incl += y;
        }
        if (lane == 31) scan[warp] = incl;
        __syncthreads();
        if (tid == 0) {
            int run = 0;
            for (int w = 0; w < kThreads / 32; ++w) {
                const int x = scan[w];
                scan[w] = run;
                run += x;
            }
            scan[kThreads / 32] = run;
        }
        __syncthreads();
        groups = scan[kThreads / 32];
        // ... and, if the sorted list fits, writes their keys (cost descending,
        // enumeration order for ties; the key's low half is 0xFFFF - group id)
        sorted = groups <= kMaxSortGroups &&
                 (int64_t)groups * p.num_kv_heads <= (int64_t)kMaxItemsPerCta * gridDim.x;
        if (sorted && mine > 0) {
            int at = scan[warp] + incl - mine;
            for (int r = tid; r < p.batch; r += kThreads) {
                Item it;
                if (request_info(p, r, it) < 0 || (p.skip_single && it.n == 1)) continue;
                const int span = kQTiles * p.tokens_per_qtile;
                for (int qb = 0; qb * span < it.n; ++qb) {
                    const int kv_len = it.c + min((qb + 1) * span, it.n);
                    const int n_kv = (kv_len + kN - 1) / kN;
                    const int gid = (p.num_qblocks - 1 - qb) * p.batch + r;
                    keys[at++] = ((uint32_t)min(n_kv, kMaxCost) << 16) | (uint32_t)(0xFFFF - gid);
                }
            }
        }
        __syncthreads();
        if (sorted && warp == 0) {
            if (groups <= 32 * 4) warp_sort_desc<4>(keys, lane);
            else warp_sort_desc<kSortPerLane>(keys, lane);
            __syncwarp();
            if (lane == 0) {
                int cnt = 0;
                for (int k = 0; cnt < kMaxItemsPerCta; ++k) {
                    const int pos = snake_position(k);
                    const int grp = pos / p.num_kv_heads;
                    if (grp >= kMaxSortGroups || keys[grp] == 0) break;
                    items[cnt++] = (0xFFFF - (int)(keys[grp] & 0xFFFFu)) * p.num_kv_heads + (pos - grp * p.num_kv_heads);
                }
                *sh_count = cnt;
            }
        }
    }
    if (!sorted && tid == 0) *sh_count = 0;

    if (tid == 0) {
        *abort_flag = 0;
        mbar_init(bar_at(sbase, kBarDrain), 1);
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(bar_at(sbase, kBarQFull + t), 1);
            mbar_init(bar_at(sbase, kBarSFull + t), 1);
            mbar_init(bar_at(sbase, kBarPFull + t), 128);
            mbar_init(bar_at(sbase, kBarODone + t), 1);
            mbar_init(bar_at(sbase, kBarOFree + t), 128);
        }
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(bar_at(sbase, kBarKFull + s), kKLoaders * 32);  // one arrival per lane of the K loaders
            mbar_init(bar_at(sbase, kBarKEmpty + s), 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(bar_at(sbase, kBarVFull + s), kVLoaders * 32);
            mbar_init(bar_at(sbase, kBarVEmpty + s), 1);
        }
        fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {  // TMEM allocation is warp-wide
        tmem_alloc(smem_u32(tmem_holder), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();  // also: the sort scratch in the K ring is dead from here on
    tc_fence_after();
    // The work list above reads request metadata only, which no kernel of this
    // library writes, so it was built while the previous kernel (e.g. the KV
    // store) may still run; the pool, q and out are touched only from here on.
    griddep_wait();
    const uint32_t tmem = *tmem_holder;
    const int list_len = *sh_count;
    const int g = p.group, tpq = p.tokens_per_qtile;

    // setmaxnreg is issued once per warpgroup role, at the top of its branch
    if (warp >= 4 && warp < 12) {
        setmaxnreg_inc<kRegsSoftmax>();
        // =============================================================== softmax
        const int t = (warp - 4) >> 2;  // Q tile
        const int wq = warp & 3;        // TMEM lane quarter this warp may access
        const int qrow = wq * 32 + lane;
        const int tok_local = qrow / g, head_local = qrow - tok_local * g;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + col_s(t);
        const uint32_t tO = tmem + lane_addr + col_o(t);
        const bool elected = (warp & 3) == 0 && lane == 0;  // issues this Q tile's TMA loads
        const uint32_t qbytes = (uint32_t)(2 * 128 * g * tpq);
        const uint32_t b_q = bar_at(sbase, kBarQFull + t), b_s = bar_at(sbase, kBarSFull + t);
        const uint32_t b_p = bar_at(sbase, kBarPFull + t), b_o = bar_at(sbase, kBarODone + t);
        const uint32_t b_free = bar_at(sbase, kBarOFree + t);
        auto load_q = [&](const Item &it) {
            mbar_arrive_expect_tx(b_q, qbytes);
            for (int h = 0; h < 2; ++h)
                tma_load_3d(sbase + kOffQ + t * kTileBytes + h * kHalfBytes, &tm_q, b_q, h * 64, it.kvh * g,
                            it.qo + it.tok0 + t * tpq);
        };
        // the items that use this Q tile: all of them for tile 0, those whose
        // second tile holds tokens for tile 1
        auto next_active = [&](ItemCursor &c, Item &out) {
            while (next_item(p, c, items, list_len, sorted, out))
                if (t == 0 || out.q1) return true;
            return false;
        };
        ItemCursor cur{0}, ahead{0};
        Item it, nx;
        int cnt = 0;       // KV tiles this Q tile has processed (phase of s_full / p_full / o_done)
        int q_issued = 0;  // Q loads issued for this Q tile (phase of q_full)
        bool ok = true;
        if (elected) {  // the first item's Q tile
            prefetch_tmap(&tm_q);
            if (next_active(ahead, nx)) {
                load_q(nx);
                ++q_issued;
            }
        }
        __syncwarp();
        while (ok && next_active(cur, it)) {
            const int i = it.tok0 + t * tpq + tok_local;  // new-token index within the request
            const bool valid = tok_local < tpq && i < it.n;
            const int last_key = valid ? it.c + i : it.kv_len - 1;  // last visible key position
            const int n_kv = it.n_kv;
            const int64_t out_row = (int64_t)(it.qo + i) * p.num_q_heads + it.kvh * g + head_local;
            // a warp whose 32 rows are all padding (a ragged last Q tile, a
            // one-token request) computes nothing: its rows of P and O are never
            // read back, it only passes the hand-offs on
            const bool live = __any_sync(0xffffffffu, valid);
            float m_run = -INFINITY, l_run = 0.f;
            for (int j = 0; j < n_kv; ++j) {
                if (!(ok = wait_or_abort(b_s, (cnt + j) & 1, abort_flag, lim))) break;
                tc_fence_after();
                if (j == n_kv - 1 && elected && next_active(ahead, nx)) {
                    // the last Q K^T of this item has completed: Q tile t is free for
                    // the next item that uses it
                    load_q(nx);
                    ++q_issued;
                }
                __syncwarp();  // the TMEM loads below are warp-collective
                if (!live) {
                    tc_fence_before();
                    mbar_arrive(b_p);
                    continue;
                }
                uint32_t sv[128];
                const int key0 = j * kN;
                const int nvis = min(max(last_key - key0 + 1, 0), kN);  // visible keys in this tile
                // Row max of the raw scores (scale > 0, so scaling commutes with the
                // max); a tile every key of which is visible to the whole warp skips
                // the mask, and takes the max of its first 64 columns while the other
                // 64 are still being read from TMEM.
                const bool full = __all_sync(0xffffffffu, nvis == kN);
                float mx;
                if (full) {
                    // the four 32-column chunks of S come from TMEM one behind the
                    // other, each chunk's max taken while the next one loads, in
                    // eight independent chains (the max is a latency chain otherwise)
                    float mc[8];
#pragma unroll
                    for (int c = 0; c < 8; ++c) mc[c] = -INFINITY;
                    tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                    tmem_ld_wait();
                    reg_barrier<32>(&sv[0]);
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        if (cb < 3)
                            tmem_ld_32x32b_x32(tS + 32 * (cb + 1), *reinterpret_cast<uint32_t(*)[32]>(&sv[32 * (cb + 1)]));
#pragma unroll
                        for (int c = 0; c < 8; ++c)
                            mc[c] = fmax3(mc[c], fmaxf(__uint_as_float(sv[32 * cb + 4 * c]), __uint_as_float(sv[32 * cb + 4 * c + 1])),
                                          fmaxf(__uint_as_float(sv[32 * cb + 4 * c + 2]), __uint_as_float(sv[32 * cb + 4 * c + 3])));
                        if (cb < 3) {
                            tmem_ld_wait();
                            reg_barrier<32>(&sv[32 * (cb + 1)]);
                        }
                    }
                    mx = fmaxf(fmaxf(fmaxf(mc[0], mc[1]), fmaxf(mc[2], mc[3])),
                               fmaxf(fmaxf(mc[4], mc[5]), fmaxf(mc[6], mc[7])));
                } else {
                    tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
                    tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
                    tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
                    tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
                    tmem_ld_wait();
                    reg_barrier<128>(&sv[0]);
                    mx = -INFINITY;
#pragma unroll
                    for (int e = 0; e < 128; ++e) {
                        const float x = e < nvis ? __uint_as_float(sv[e]) : -INFINITY;
                        sv[e] = __float_as_uint(x);
                        mx = fmaxf(mx, x);
                    }
                }
                const float m_new = fmaxf(m_run, mx * p.scale_log2);
                const bool need = m_new > m_run + kRescaleThreshold;  // also true for the first tile
                const bool warp_need = __any_sync(0xffffffffu, need);
                float corr = 1.f;
                if (warp_need) {
                    const float m_tgt = need ? m_new : m_run;
                    corr = m_run == -INFINITY ? 0.f : fast_exp2(m_run - m_tgt);
                    m_run = m_tgt;
                    l_run *= corr;
                }
                // P = 2^(s * scale_log2 - m), one fused multiply-add per pair of keys;
                // the first kEmuPairs pairs of every 16 on the FMA pipe, the rest on MUFU
                const float mu = m_run == -INFINITY ? 0.f : m_run;
                const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
                const float2 nmu2 = make_float2(-mu, -mu);
                float rs[8];  // eight row-sum chains: two per column block
#pragma unroll
                for (int c = 0; c < 8; ++c) rs[c] = 0.f;
                // 32-key chunks past every row's last visible key (the causal edge of a
                // diagonal tile) hold no weight for any row of the warp: their P is
                // stored as zeros without computing it
                const int live_chunks = full ? 4 : (int)__reduce_max_sync(0xffffffffu, (unsigned)(nvis + 31) / 32u);
#pragma unroll
                for (int cb = 0; cb < 4; ++cb) {  // masked keys hold -inf and give exactly 0
                    uint32_t pk[16];
                    if (cb >= live_chunks) {
#pragma unroll
                        for (int e = 0; e < 16; ++e) pk[e] = 0u;
                        tmem_st_32x32b_x16(tS + cb * 16, pk);
                        continue;
                    }
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = ffma2(make_float2(__uint_as_float(sv[cb * 32 + 2 * e]),
                                                           __uint_as_float(sv[cb * 32 + 2 * e + 1])),
                                               sc2, nmu2);
                        if (e < kEmuPairs) {
                            const float2 ex = exp2_fma2(x);
                            pk[e] = pack_bf16x2(ex.x, ex.y);
                        } else {
                            pk[e] = pack_bf16x2(fast_exp2(x.x), fast_exp2(x.y));
                        }
                        // the row sum adds the same bf16-rounded P the PV product reads
                        add_bf16x2_f32(rs[2 * cb], rs[2 * cb + 1], pk[e]);
                    }
                    tmem_st_32x32b_x16(tS + cb * 16, pk);
                }
                l_run += ((rs[0] + rs[1]) + (rs[2] + rs[3])) + ((rs[4] + rs[5]) + (rs[6] + rs[7]));
                if (warp_need && j > 0) {
                    // O holds the sum up to tile j-1; rescale it once that PV is done
                    if (!(ok = wait_or_abort(b_o, (cnt + j - 1) & 1, abort_flag, lim))) break;
                    tc_fence_after();
#pragma unroll
                    for (int cb = 0; cb < 4; ++cb) {
                        uint32_t ov[32];
                        tmem_ld_32x32b_x32(tO + cb * 32, ov);
                        tmem_ld_wait();
                        uint32_t lo[16], hi[16];
#pragma unroll
                        for (int e = 0; e < 16; ++e) {
                            lo[e] = __float_as_uint(__uint_as_float(ov[e]) * corr);
                            hi[e] = __float_as_uint(__uint_as_float(ov[16 + e]) * corr);
                        }
                        tmem_st_32x32b_x16(tO + cb * 32, lo);
                        tmem_st_32x32b_x16(tO + cb * 32 + 16, hi);
                    }
                }
                tmem_st_wait();
                tc_fence_before();
                mbar_arrive(b_p);
            }
            if (!ok) break;
            // ---- epilogue: O / l -> bf16 -> out, then O is free for the next item
            if (!(ok = wait_or_abort(b_o, (cnt + n_kv - 1) & 1, abort_flag, lim))) break;
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *dst = p.out + out_row * kHeadDim;
#pragma unroll
            for (int cb = 0; cb < 4 && live; ++cb) {
                uint32_t ov[32];
                tmem_ld_32x32b_x32(tO + cb * 32, ov);
                tmem_ld_wait();
                if (valid) {
                    uint4 *d4 = reinterpret_cast<uint4 *>(dst + cb * 32);
#pragma unroll
                    for (int v = 0; v < 4; ++v) {
                        uint4 w;
                        w.x = pack_bf16x2(__uint_as_float(ov[8 * v + 0]) * inv, __uint_as_float(ov[8 * v + 1]) * inv);
                        w.y = pack_bf16x2(__uint_as_float(ov[8 * v + 2]) * inv, __uint_as_float(ov[8 * v + 3]) * inv);
                        w.z = pack_bf16x2(__uint_as_float(ov[8 * v + 4]) * inv, __uint_as_float(ov[8 * v + 5]) * inv);
                        w.w = pack_bf16x2(__uint_as_float(ov[8 * v + 6]) * inv, __uint_as_float(ov[8 * v + 7]) * inv);
                        d4[v] = w;
                    }
                }
            }
            tc_fence_before();
            mbar_arrive(b_free);
            cnt += n_kv;
        }
        // a Q load issued for an item that never ran (after an abort) must land
        // before the CTA exits; after a normal run it has long completed
        if (elected && q_issued > 0) wait_bounded(b_q, (q_issued - 1) & 1, lim);
    } else {
        setmaxnreg_dec<kRegsLoad>();
        if (warp == kMmaWarp) {
            // =============================================================== MMA issue
            if (lane == 0) {
                constexpr uint32_t idesc_qk = idesc_bf16(false);
                constexpr uint32_t idesc_pv = idesc_bf16(true);
                constexpr uint32_t kHiK = sw128_hi(1024), kHiV = sw128_hi(1024);
                // Fully unrolled: per MMA, the two address words are the stage's
                // base plus a constant.  The bases pass through an empty asm so
                // the compiler cannot precompute every stage's and step's words
                // outside the item loop (they would not fit in 72 registers).
                auto issue_s = [&](int t, int stage, bool signal) {
                    uint32_t qa = sw128_lo(sbase + kOffQ + t * kTileBytes, 16);
                    uint32_t ka = sw128_lo(sbase + kOffK + stage * kTileBytes, 16);
                    opaque_u32(qa);
                    opaque_u32(ka);
                    const uint32_t d = tmem + col_s(t);
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (uint32_t)((kk >> 2) * kHalfBytes + (kk & 3) * 32) >> 4;
                        umma_ss_words(d, qa + off, kHiK, ka + off, kHiK, idesc_qk, kk > 0 ? 1u : 0u);
                    }
                    if (signal) umma_commit(bar_at(sbase, kBarSFull + t));
                };
                auto issue_pv = [&](int t, int stage, bool accumulate) {
                    uint32_t vb = sw128_lo(sbase + kOffV + stage * kTileBytes, kHalfBytes);
                    opaque_u32(vb);
                    const uint32_t d = tmem + col_o(t), a = tmem + col_s(t);
                    umma_ts_words(d, a, vb, kHiV, idesc_pv, accumulate ? 1u : 0u);
#pragma unroll
                    for (int kk = 1; kk < 8; ++kk)
                        umma_ts_words(d, a + kk * 8, vb + (uint32_t)(kk * 2048 >> 4), kHiV, idesc_pv, 1u);
                    umma_commit(bar_at(sbase, kBarODone + t));
                };
                ItemCursor cur{0};
                Item it;
                int cnt[kQTiles] = {0, 0};      // KV tiles processed per Q tile
                int items_t[kQTiles] = {0, 0};  // items processed per Q tile (phase of q_full / o_free)
                int kseq = 0, vseq = 0;
                bool ok = true, first = true;
                while (ok && next_item(p, cur, items, list_len, sorted, it)) {
                    const bool q1 = it.q1;
                    ok = wait_or_abort_thread(bar_at(sbase, kBarQFull), items_t[0] & 1, abort_flag, lim) &&
                         (!q1 || wait_or_abort_thread(bar_at(sbase, kBarQFull + 1), items_t[1] & 1, abort_flag, lim)) &&
                         wait_or_abort_thread(bar_at(sbase, kBarKFull + kseq % kKStages), (kseq / kKStages) & 1,
                                              abort_flag, lim);
                    if (!ok) break;
                    fence_proxy_async_smem();
                    tc_fence_after();
                    {
                        const int ks = kseq % kKStages;
                        // the fault-injection hook withholds the first item's first
                        // hand-off to Q tile 0's softmax, which then waits for a tile
                        // that is never signalled ready
                        issue_s(0, ks, !(first && p.inject_stall));
                        if (q1) issue_s(1, ks, true);
                        umma_commit(bar_at(sbase, kBarKEmpty + ks));
                        ++kseq;
                    }
                    first = false;
                    for (int j = 0; j < it.n_kv; ++j) {
                        const int vs = vseq % kVStages;
                        if (!(ok = wait_or_abort_thread(bar_at(sbase, kBarVFull + vs), (vseq / kVStages) & 1,
                                                        abort_flag, lim)))
                            break;
                        fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor core reads
                        if (!(ok = wait_or_abort_thread(bar_at(sbase, kBarPFull), (cnt[0] + j) & 1, abort_flag, lim)))
                            break;
                        // O_0 holds the previous item's result until its epilogue has read it
                        if (j == 0 && items_t[0] > 0 &&
                            !(ok = wait_or_abort_thread(bar_at(sbase, kBarOFree), (items_t[0] - 1) & 1, abort_flag,
                                                        lim)))
                            break;
                        tc_fence_after();
                        issue_pv(0, vs, j > 0);
                        const bool more = j + 1 < it.n_kv;
                        const int ks = kseq % kKStages;
                        if (more) {
                            if (!(ok = wait_or_abort_thread(bar_at(sbase, kBarKFull + ks), (kseq / kKStages) & 1,
                                                            abort_flag, lim)))
                                break;
                            fence_proxy_async_smem();
                            tc_fence_after();
                            issue_s(0, ks, true);
                        }
                        if (q1) {
                            if (!(ok = wait_or_abort_thread(bar_at(sbase, kBarPFull + 1), (cnt[1] + j) & 1, abort_flag,
                                                            lim)))
                                break;
                            if (j == 0 && items_t[1] > 0 &&
                                !(ok = wait_or_abort_thread(bar_at(sbase, kBarOFree + 1), (items_t[1] - 1) & 1,
                                                            abort_flag, lim)))
                                break;
                            tc_fence_after();
                            issue_pv(1, vs, j > 0);
                        }
                        umma_commit(bar_at(sbase, kBarVEmpty + vs));
                        ++vseq;
                        if (more) {
                            if (q1) issue_s(1, ks, true);
                            umma_commit(bar_at(sbase, kBarKEmpty + ks));
                            ++kseq;
                        }
                    }
                    cnt[0] += it.n_kv;
                    ++items_t[0];
                    if (q1) {
                        cnt[1] += it.n_kv;
                        ++items_t[1];
                    }
                }
                // before TMEM is freed, every MMA this thread issued must have
                // completed, also after an abort: one commit tracks them all, and
                // its wait ignores the abort flag (after a normal run it returns
                // at once: the softmax warps already waited for the last P V)
                umma_commit(bar_at(sbase, kBarDrain));
                wait_bounded(bar_at(sbase, kBarDrain), 0, lim);
            }
            __syncwarp();
        } else if (warp >= kKLoadWarp0 && warp < kKLoadWarp0 + kKLoaders) {
            // =============================================================== K loads
            load_rows<kKLoaders, kKStages>(p, sbase + kOffK, bar_at(sbase, kBarKFull), bar_at(sbase, kBarKEmpty),
                                           p.k_cache, warp - kKLoadWarp0, lane, items, list_len, sorted, abort_flag,
                                           lim, true);
        } else {
            // =============================================================== V loads
            load_rows<kVLoaders, kVStages>(p, sbase + kOffV, bar_at(sbase, kBarVFull), bar_at(sbase, kBarVEmpty),
                                           p.v_cache, warp - kVLoadWarp0, lane, items, list_len, sorted, abort_flag,
                                           lim, false);
        }
    }

    // ---- teardown: everyone meets here, even after an abort
    tc_fence_before();
    __syncthreads();
    if (warp == kMmaWarp) {
        tc_fence_after();
        tmem_dealloc(tmem, kTmemCols);
    }
}

// ---------------------------------------------------------------- host side

inline cudaError_t set_attributes() {
    return cudaFuncSetAttribute(extend_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kSmemBytes);
}

inline mg_status launch(Params &p, int sms, cudaStream_t stream) {
    EncodeTiledFn enc = encode_fn();
    if (!enc) return MG_ERR_CUDA;
    const int g = p.group;
    p.tokens_per_qtile = kM / g;
    CUtensorMap tq;
    {
        cuuint64_t dims[3] = {(cuuint64_t)kHeadDim, (cuuint64_t)p.num_q_heads, (cuuint64_t)p.total_q};
        cuuint64_t strides[2] = {(cuuint64_t)kHeadDim * 2, (cuuint64_t)p.num_q_heads * kHeadDim * 2};
        cuuint32_t box[3] = {64, (cuuint32_t)g, (cuuint32_t)p.tokens_per_qtile};
        cuuint32_t es[3] = {1, 1, 1};
        if (enc(&tq, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<__nv_bfloat16 *>(p.q), dims, strides, box, es,
                CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_128B,
                CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) != CUDA_SUCCESS)
            return MG_ERR_CUDA;
    }
    const int64_t tokens_per_item = kQTiles * p.tokens_per_qtile;
    const int64_t nqb = (p.max_q_len + tokens_per_item - 1) / tokens_per_item;
    const int64_t items = nqb * p.batch * p.num_kv_heads;
    if (items <= 0) return MG_OK;
    if (items >= (int64_t)1 << 30) return MG_ERR_UNSUPPORTED_SHAPE;
    p.num_qblocks = (int32_t)nqb;
    p.num_items = (int32_t)items;
    // the kernel sorts the groups that hold tokens when there are at most
    // kMaxSortGroups of them; group ids must fit the key's low 16 bits
    p.sorted = nqb * p.batch < 0xFFFF ? 1 : 0;
    // one CTA per SM; when every group may hold tokens and the list is sure to
    // be sorted, no CTA may need more than kMaxItemsPerCta items
    int64_t grid = items < sms ? items : sms;
    if (nqb * p.batch <= kMaxSortGroups) {
        const int64_t min_grid = (items + kMaxItemsPerCta - 1) / kMaxItemsPerCta;
        if (grid < min_grid) grid = min_grid;
    }
    return launch_pdl(extend_kernel, dim3((unsigned)grid), dim3(kThreads), kSmemBytes, stream, tq, p);
}

}  // namespace extend
}  // namespace mg
