// extend.cuh -- chunked-prefill ("extend") attention on tcgen05 tensor cores.
//
// What it computes ("手写 mini-sglang 阶段一 · Engine 与采样器", §手工驱动引擎;
// Mini-SGLang tag page, Scheduler post, chunked prefill): request r has
// c = cached_len[r] tokens in the pool and n = seq_len[r] - c new ones, already
// stored; new token i (query row q_offset[r] + i, position c + i) attends to the
// keys at positions 0 .. c + i of its page-table row.
//
// Work decomposition (B200 design; 16 warps in four warpgroups with their
// register budgets moved by setmaxnreg: warpgroups 0 and 3 load and issue
// MMAs on 72 registers a thread, warpgroups 1 and 2 run the softmax on 184):
//   * one CTA per (q block, kv head, request).  A q block is two 128-row Q
//     tiles; a row is (token, head) with the g heads that share the KV head
//     adjacent, so one K/V tile feeds 2 x 128 query rows (GQA packing).
//   * seven load warps (0-3, 13-15): the Q tiles with 3-D TMA, the K and V
//     tiles (128 keys each) with 16-byte cp.async straight from the paged pool
//     into the 128-byte swizzled layout, behind mbarriers.  A warp keeps about
//     one 512-byte cp.async in flight per 70 cycles whatever the SM does, so
//     the copy rate grows with the number of issuing warps; every load warp
//     owns every seventh pair of rows of each tile.
//   * warp 12, one thread: issues tcgen05.mma (M=128, N=128, K=16, bf16 in,
//     fp32 accumulate in TMEM).  S_t = Q_t K^T lands in TMEM; P_t (bf16) is
//     written back over S_t and consumed straight from TMEM as the A operand
//     of O_t += P_t V.  The MMAs of the two Q tiles interleave, each issued
//     once its inputs are ready.  (Since P_t overwrites S_t, S_t of the next
//     KV tile waits for P_t V; measured, both Q tiles' softmaxes then wait on
//     the same KV tile, so the softmax and the tensor core mostly alternate
//     instead of overlapping: the kernel's present bound.)
//   * warpgroups 1 / 2: softmax for Q tile 0 / 1, one TMEM lane (= one query
//     row) per thread: causal mask key <= c + i, online softmax in the exp2
//     domain, O rescaled in TMEM only when the running max grows by more than
//     2^8 (exact: the same stale max is used for P and for the row sum),
//     epilogue O / l -> bf16 -> global.
// TMEM: S0 [0,128)  S1 [128,256)  O0 [256,384)  O1 [384,512) columns.
#pragma once

#include <cuda.h>

#include "common.cuh"

namespace mg {
namespace extend {

constexpr int kM = 128;                     // query rows per Q tile
constexpr int kN = 128;                     // keys per KV tile
constexpr int kQTiles = 2;
constexpr int kKStages = 3;                 // K ring: S of a tile needs K before P V needs V
constexpr int kVStages = 2;                 // V ring
constexpr int kIdxAhead = 3;                // tiles of page-table entries in flight ahead of the K issue
constexpr int kIdxRing = 4;                 // >= kIdxAhead + 1
constexpr int kThreads = 512;               // 16 warps: 7 load, 1 MMA, 8 softmax
constexpr int kLoaders = 7;                 // load warps 0-3 and 13-15
constexpr int kMmaWarp = 12;
constexpr int kPairs = kN / 2;              // row pairs per tile (one warp instruction moves a pair)
constexpr int kMaxPairsPerLoader = (kPairs + kLoaders - 1) / kLoaders;
constexpr int kRegsLoad = 72;               // registers a thread in warpgroups 0 and 3
constexpr int kRegsSoftmax = 184;           // registers a thread in warpgroups 1 and 2
static_assert(2 * 128 * kRegsLoad + 2 * 128 * kRegsSoftmax == 65536 && 65536 / kThreads == 128,
              "the register split must add up to what the block is launched with");
static_assert(2 * kMaxPairsPerLoader <= 32, "a load warp fetches one page-table entry per lane");
constexpr int kHalfBytes = 128 * 128;       // 128 rows x 128 B (64 bf16): one swizzle column
constexpr int kTileBytes = 2 * kHalfBytes;  // 128 rows x 256 B
constexpr int kTmemCols = 512;
__device__ __forceinline__ uint32_t col_s(int t) { return (uint32_t)t * 128u; }
__device__ __forceinline__ uint32_t col_o(int t) { return 256u + (uint32_t)t * 128u; }
constexpr float kRescaleThreshold = 8.0f;   // log2 units

// shared memory map.  The kernel has no static shared memory, so its dynamic
// shared memory starts on a 1024-byte boundary (checked at run time), as the
// 128-byte swizzle atoms require; every region below keeps that alignment.
constexpr int kOffQ = 0;
constexpr int kOffK = kOffQ + kQTiles * kTileBytes;
constexpr int kOffV = kOffK + kKStages * kTileBytes;
constexpr int kOffIdx = kOffV + kVStages * kTileBytes;
constexpr int kOffBar = kOffIdx + kIdxRing * kN * 4;
constexpr int kNumBars = 2 + 2 * kKStages + 2 * kVStages + 3 * kQTiles;  // + the abort drain
constexpr int kOffMisc = kOffBar + kNumBars * 8;
constexpr int kSmemBytes = kOffMisc + 16;
static_assert(kSmemBytes <= 227 * 1024, "extend shared memory over the per-CTA limit");

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
    float scale_log2;
    uint64_t wait_limit_ns;    // bound of every pipeline wait
    int32_t inject_stall;      // test hook: withhold the first score tile's hand-off
};

// UMMA shared-memory descriptor, 128-byte swizzle, sm_100 version bits.
__device__ __forceinline__ uint64_t sw128_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr & 0x3FFFFu) >> 4);
    d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;  // descriptor version (Blackwell)
    d |= (uint64_t)2 << 61;  // SWIZZLE_128B
    return d;
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

struct Sync {
    uint32_t q_full, drain;
    uint32_t k_full[kKStages], k_empty[kKStages], v_full[kVStages], v_empty[kVStages];
    uint32_t s_full[kQTiles], p_full[kQTiles], o_done[kQTiles];
};

__device__ __forceinline__ uint64_t global_ns() {
    uint64_t now;
    asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(now));
    return now;
}

// Waits with a time bound (limit_ns, timed from the wait's first check of the
// clock); on timeout records the error, raises the CTA abort flag and returns
// false.  Once the flag is up every later wait returns false at once, so all
// roles drain to the final barrier.
__device__ __forceinline__ bool wait_or_abort_thread(uint32_t bar, uint32_t parity, volatile int *abort_flag,
                                                     uint64_t limit_ns) {
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

__global__ void __launch_bounds__(kThreads, 1)
    extend_kernel(const __grid_constant__ CUtensorMap tm_q, const Params p) {
    extern __shared__ __align__(1024) uint8_t smem[];
    const uint32_t sbase = smem_u32(smem);
    if (sbase & 1023u) {  // the swizzled layouts need 1024-byte alignment: refuse, never fault
        if (threadIdx.x == 0) atomicOr(&g_mg_device_error, MG_DEVERR_INTERNAL);
        return;
    }
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + kOffMisc);
    const uint64_t lim = p.wait_limit_ns;  // nanoseconds
    uint32_t *tmem_holder = reinterpret_cast<uint32_t *>(smem + kOffMisc + 4);

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int r = blockIdx.z, kvh = blockIdx.y;
    griddep_launch_dependents();
    griddep_wait();  // inputs written by the previous kernel (e.g. the KV store)
    const int qb = gridDim.x - 1 - blockIdx.x;  // heaviest (latest) q blocks first

    // ---- request metadata (uniform across the CTA; exit before any barrier)
    const int row = __ldg(p.table_idx + r);
    const int c = __ldg(p.cached_len + r);
    const int L = __ldg(p.seq_len + r);
    const int qo = __ldg(p.q_offset + r);
    const int n = L - c;
    {
        unsigned bad = 0;
        if (row < 0 || row >= p.pt_rows) bad |= MG_DEVERR_ROW_RANGE;
        if (c < 0 || n < 0 || L > p.pt_stride || L > p.max_seq_len || n > p.max_q_len || qo < 0 ||
            qo + n > p.total_q || __ldg(p.q_offset + r + 1) - qo != n)
            bad |= MG_DEVERR_LENGTH;
        if (bad) {
            if (threadIdx.x == 0 && blockIdx.x == 0 && kvh == 0) atomicOr(&g_mg_device_error, bad);
            return;
        }
    }
    const int tpq = p.tokens_per_qtile;
    const int g = p.group;
    const int tok0 = qb * kQTiles * tpq;
    if (tok0 >= n) return;
    const int last_tok = min(tok0 + kQTiles * tpq, n) - 1;
    const int kv_len = c + last_tok + 1;  // keys this CTA needs: positions [0, kv_len)
    const int n_kv = (kv_len + kN - 1) / kN;
    const bool has_q1 = tok0 + tpq < n;

    Sync sy;
    {
        uint32_t b = sbase + kOffBar;
        sy.q_full = b; b += 8;
        sy.drain = b; b += 8;
        for (int s = 0; s < kKStages; ++s) { sy.k_full[s] = b; b += 8; }
        for (int s = 0; s < kKStages; ++s) { sy.k_empty[s] = b; b += 8; }
        for (int s = 0; s < kVStages; ++s) { sy.v_full[s] = b; b += 8; }
        for (int s = 0; s < kVStages; ++s) { sy.v_empty[s] = b; b += 8; }
        for (int t = 0; t < kQTiles; ++t) { sy.s_full[t] = b; b += 8; }
        for (int t = 0; t < kQTiles; ++t) { sy.p_full[t] = b; b += 8; }
        for (int t = 0; t < kQTiles; ++t) { sy.o_done[t] = b; b += 8; }
    }
    if (threadIdx.x == 0) {
        *abort_flag = 0;
        mbar_init(sy.q_full, 1);
        mbar_init(sy.drain, 1);
        for (int s = 0; s < kKStages; ++s) {
            mbar_init(sy.k_full[s], kLoaders * 32);  // one arrival per lane of the load warps
            mbar_init(sy.k_empty[s], 1);
        }
        for (int s = 0; s < kVStages; ++s) {
            mbar_init(sy.v_full[s], kLoaders * 32);
            mbar_init(sy.v_empty[s], 1);
        }
        for (int t = 0; t < kQTiles; ++t) {
            mbar_init(sy.s_full[t], 1);
            mbar_init(sy.p_full[t], 128);
            mbar_init(sy.o_done[t], 1);
        }
        fence_mbarrier_init();
    }
    if (warp == kMmaWarp) {  // TMEM allocation is warp-wide
        tmem_alloc(smem_u32(tmem_holder), kTmemCols);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_holder;

    // setmaxnreg is issued once per warpgroup role, at the top of its branch
    if (warp >= 4 && warp < 12) {
        setmaxnreg_inc<kRegsSoftmax>();
        // =============================================================== softmax
        const int t = (warp - 4) >> 2;  // Q tile
        const int wq = warp & 3;        // TMEM lane quarter this warp may access
        const int qrow = wq * 32 + lane;
        const int tok_local = qrow / g, head_local = qrow - tok_local * g;
        const int i = tok0 + t * tpq + tok_local;  // new-token index within the request
        const bool valid = tok_local < tpq && i < n;
        const int last_key = valid ? c + i : kv_len - 1;  // last visible key position
        const bool active = t == 0 || has_q1;
        const uint32_t lane_addr = (uint32_t)(wq * 32) << 16;
        const uint32_t tS = tmem + lane_addr + col_s(t);
        const uint32_t tO = tmem + lane_addr + col_o(t);
        float m_run = -INFINITY, l_run = 0.f;
        bool ok = active;
        for (int j = 0; ok && j < n_kv; ++j) {
            if (!(ok = wait_or_abort(sy.s_full[t], j & 1, abort_flag, lim))) break;
            tc_fence_after();
            uint32_t sv[128];
            tmem_ld_32x32b_x32(tS + 0, *reinterpret_cast<uint32_t(*)[32]>(&sv[0]));
            tmem_ld_32x32b_x32(tS + 32, *reinterpret_cast<uint32_t(*)[32]>(&sv[32]));
            tmem_ld_32x32b_x32(tS + 64, *reinterpret_cast<uint32_t(*)[32]>(&sv[64]));
            tmem_ld_32x32b_x32(tS + 96, *reinterpret_cast<uint32_t(*)[32]>(&sv[96]));
            tmem_ld_wait();
            const int key0 = j * kN;
            const int nvis = min(max(last_key - key0 + 1, 0), kN);  // visible keys in this tile
            // Row max of the raw scores (scale > 0, so scaling commutes with the
            // max); a tile every key of which is visible to the whole warp skips
            // the mask.
            const bool full = __all_sync(0xffffffffu, nvis == kN);
            float mx;
            if (full) {
                float m0 = -INFINITY, m1 = -INFINITY;
#pragma unroll
                for (int e = 0; e < 128; e += 4) {
                    m0 = fmax3(m0, __uint_as_float(sv[e]), __uint_as_float(sv[e + 1]));
                    m1 = fmax3(m1, __uint_as_float(sv[e + 2]), __uint_as_float(sv[e + 3]));
                }
                mx = fmaxf(m0, m1);
            } else {
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
            // P = 2^(s * scale_log2 - m), one fused multiply-add per pair of keys
            const float mu = m_run == -INFINITY ? 0.f : m_run;
            const float2 sc2 = make_float2(p.scale_log2, p.scale_log2);
            const float2 nmu2 = make_float2(-mu, -mu);
            float2 rs2 = make_float2(0.f, 0.f);
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {  // masked keys hold -inf and give exactly 0
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e) {
                    const float2 x = ffma2(make_float2(__uint_as_float(sv[cb * 32 + 2 * e]),
                                                       __uint_as_float(sv[cb * 32 + 2 * e + 1])),
                                           sc2, nmu2);
                    pk[e] = pack_bf16x2(fast_exp2(x.x), fast_exp2(x.y));
                    // the row sum adds the same bf16-rounded P the PV product reads
                    rs2 = fadd2(rs2, make_float2(bf16x2_lo(pk[e]), bf16x2_hi(pk[e])));
                }
                tmem_st_32x32b_x16(tS + cb * 16, pk);
            }
            l_run += rs2.x + rs2.y;
            if (warp_need && j > 0) {
                // O holds the sum up to tile j-1; rescale it once that PV is done
                if (!(ok = wait_or_abort(sy.o_done[t], (j - 1) & 1, abort_flag, lim))) break;
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
            mbar_arrive(sy.p_full[t]);
        }
        // ---- epilogue: O / l -> bf16 -> out
        if (ok && wait_or_abort(sy.o_done[t], (n_kv - 1) & 1, abort_flag, lim)) {
            tc_fence_after();
            const float inv = l_run > 0.f ? 1.f / l_run : 0.f;
            __nv_bfloat16 *dst = p.out + ((int64_t)(qo + i) * p.num_q_heads + kvh * g + head_local) * kHeadDim;
#pragma unroll
            for (int cb = 0; cb < 4; ++cb) {
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
        }
    } else {
        setmaxnreg_dec<kRegsLoad>();
        if (warp == kMmaWarp) {
            // =============================================================== MMA issue
            if (lane == 0) {
                constexpr uint32_t idesc_qk = idesc_bf16(false);
                constexpr uint32_t idesc_pv = idesc_bf16(true);
                auto issue_s = [&](int t, int j, bool signal) {
                    const uint32_t qa = sbase + kOffQ + t * kTileBytes;
                    const uint32_t ka = sbase + kOffK + (j % kKStages) * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk) {
                        const uint32_t off = (kk >> 2) * kHalfBytes + (kk & 3) * 32;
                        umma_ss(tmem + col_s(t), sw128_desc(qa + off, 16, 1024), sw128_desc(ka + off, 16, 1024),
                                idesc_qk, kk > 0);
                    }
                    if (signal) umma_commit(sy.s_full[t]);
                };
                auto issue_pv = [&](int t, int j) {
                    const uint32_t va = sbase + kOffV + (j % kVStages) * kTileBytes;
#pragma unroll
                    for (int kk = 0; kk < 8; ++kk)
                        umma_ts(tmem + col_o(t), tmem + col_s(t) + kk * 8,
                                sw128_desc(va + kk * 2048, kHalfBytes, 1024), idesc_pv, (j > 0 || kk > 0));
                    umma_commit(sy.o_done[t]);
                };
                bool ok = wait_or_abort_thread(sy.q_full, 0, abort_flag, lim) && wait_or_abort_thread(sy.k_full[0], 0, abort_flag, lim);
                if (ok) {
                    fence_proxy_async_smem();
                    tc_fence_after();
                    // the fault-injection hook withholds Q tile 0's first hand-off, so its
                    // softmax warps wait for a tile that is never signalled ready
                    issue_s(0, 0, p.inject_stall == 0);
                    if (has_q1) issue_s(1, 0, true);
                    umma_commit(sy.k_empty[0]);
                }
                for (int j = 0; ok && j < n_kv; ++j) {
                    const int sv = j % kVStages;
                    if (!(ok = wait_or_abort_thread(sy.v_full[sv], (j / kVStages) & 1, abort_flag, lim))) break;
                    fence_proxy_async_smem();  // cp.async (generic proxy) writes -> tensor core reads
                    if (!(ok = wait_or_abort_thread(sy.p_full[0], j & 1, abort_flag, lim))) break;
                    tc_fence_after();
                    issue_pv(0, j);
                    const bool more = j + 1 < n_kv;
                    if (more) {
                        const int sk = (j + 1) % kKStages;
                        if (!(ok = wait_or_abort_thread(sy.k_full[sk], ((j + 1) / kKStages) & 1, abort_flag, lim))) break;
                        fence_proxy_async_smem();
                        tc_fence_after();
                        issue_s(0, j + 1, true);
                    }
                    if (has_q1) {
                        if (!(ok = wait_or_abort_thread(sy.p_full[1], j & 1, abort_flag, lim))) break;
                        tc_fence_after();
                        issue_pv(1, j);
                    }
                    umma_commit(sy.v_empty[sv]);
                    if (more) {
                        if (has_q1) issue_s(1, j + 1, true);
                        umma_commit(sy.k_empty[(j + 1) % kKStages]);
                    }
                }
                // before TMEM is freed, every MMA this thread issued must have
                // completed, also after an abort: one commit tracks them all, and
                // its wait ignores the abort flag (after a normal run it returns
                // at once: the softmax warps already waited for the last P V)
                umma_commit(sy.drain);
                wait_bounded(sy.drain, 0, lim);
            }
            __syncwarp();
        } else {
            // =============================================================== loads
            const int li = warp < 4 ? warp : warp - 9;  // load warp index 0 .. kLoaders - 1
            if (li == 0 && lane == 0) {
                prefetch_tmap(&tm_q);
                const uint32_t qbytes = (uint32_t)(kQTiles * 2 * 128 * g * tpq);
                mbar_arrive_expect_tx(sy.q_full, qbytes);
                for (int t = 0; t < kQTiles; ++t)
                    for (int h = 0; h < 2; ++h)
                        tma_load_3d(sbase + kOffQ + t * kTileBytes + h * kHalfBytes, &tm_q, sy.q_full, h * 64,
                                    kvh * g, qo + tok0 + t * tpq);
            }
            const int32_t *pt = p.page_table + (int64_t)row * p.pt_stride;
            const int64_t head_stride = (int64_t)p.num_kv_heads * kHeadDim;
            int *idx_ring = reinterpret_cast<int *>(smem + kOffIdx);
            // this warp's row pairs of every tile: li, li + kLoaders, ... (< kPairs)
            const int npairs = (kPairs - li + kLoaders - 1) / kLoaders;
            // lane l < 2 * npairs owns the page-table entry of key 2 (li + kLoaders (l / 2)) + l % 2
            const bool has_key = lane < 2 * npairs;
            const int my_key = 2 * (li + kLoaders * (lane >> 1)) + (lane & 1);
            // Iteration j copies this warp's K rows of tile j and V rows of tile
            // j - 1 (K leads V by one tile); each lane then arms the tile's full
            // barrier with cp.async.mbarrier.arrive.noinc, so the barrier
            // completes when every load lane's copies have landed, without the
            // load warps waiting for them.  The page-table entries of tile
            // j + kIdxAhead ride in the iteration's commit group, the only group
            // the warp waits for.
            auto fetch_idx = [&](int j) {
                if (j < n_kv && has_key) {
                    const int key = j * kN + my_key;
                    int *dst = idx_ring + (j % kIdxRing) * kN + my_key;
                    if (key < kv_len) cp_async_4(smem_u32(dst), pt + key);
                    else *dst = -1;
                }
            };
            // This warp's row pairs of K or V into a tile stored as two 64-column
            // halves with the 128-byte swizzle; each warp instruction moves one pair.
            auto copy_rows = [&](int j, const __nv_bfloat16 *pool, uint32_t tile_base) {
                const int *ids = idx_ring + (j % kIdxRing) * kN;
                const int c = lane & 15, half = c >> 3, cc = c & 7;
#pragma unroll
                for (int m = 0; m < kMaxPairsPerLoader; ++m) {
                    if (m < npairs) {
                        const int key = 2 * (li + kLoaders * m) + (lane >> 4);
                        int slot = j * kN + key < kv_len ? ids[key] : -1;
                        if (slot >= 0 && (int64_t)slot >= p.num_slots) slot = -1;  // flagged by check_rows
                        const __nv_bfloat16 *src = pool + (int64_t)(slot < 0 ? 0 : slot) * head_stride +
                                                   (int64_t)kvh * kHeadDim + c * 8;
                        const uint32_t dst = tile_base + half * kHalfBytes + key * 128 + ((cc ^ (key & 7)) << 4);
                        cp_async_16(dst, src, slot < 0 ? 0u : 16u);
                    }
                }
            };
            auto check_rows = [&](int j) {  // record rejected page-table entries (they were zero-filled)
                if (has_key && j * kN + my_key < kv_len) {
                    const int slot = idx_ring[(j % kIdxRing) * kN + my_key];
                    if (slot < 0 || (int64_t)slot >= p.num_slots) atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
                }
            };
#pragma unroll
            for (int j = 0; j < kIdxAhead; ++j) {
                fetch_idx(j);
                cp_async_commit();
            }
            for (int j = 0; j <= n_kv; ++j) {
                if (j < n_kv) {
                    const int s = j % kKStages;
                    if (j >= kKStages && !wait_or_abort(sy.k_empty[s], ((j / kKStages) - 1) & 1, abort_flag, lim)) break;
                }
                if (j >= 1) {
                    const int jv = j - 1, s = jv % kVStages;
                    if (jv >= kVStages && !wait_or_abort(sy.v_empty[s], ((jv / kVStages) - 1) & 1, abort_flag, lim)) break;
                }
                cp_async_wait<kIdxAhead - 1>();  // entries of tile j (kIdxAhead groups old) landed
                __syncwarp();
                if (j < n_kv) {
                    check_rows(j);
                    copy_rows(j, p.k_cache, sbase + kOffK + (j % kKStages) * kTileBytes);
                    cp_async_arrive_noinc(sy.k_full[j % kKStages]);
                }
                if (j >= 1) {
                    copy_rows(j - 1, p.v_cache, sbase + kOffV + ((j - 1) % kVStages) * kTileBytes);
                    cp_async_arrive_noinc(sy.v_full[(j - 1) % kVStages]);
                }
                // only now reuse the ring slot of tile j - 1 (every lane has read its
                // entries for the V rows just issued)
                __syncwarp();
                fetch_idx(j + kIdxAhead);
                cp_async_commit();
            }
            cp_async_wait<0>();  // nothing in flight into shared memory at teardown
            // the Q tiles' TMA load completes on q_full; after an abort nobody may
            // have waited for it, and it must land before the CTA exits
            if (li == 0 && lane == 0) wait_bounded(sy.q_full, 0, lim);
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

inline mg_status launch(Params &p, cudaStream_t stream) {
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
    const int tokens_per_cta = kQTiles * p.tokens_per_qtile;
    const int nqb = (p.max_q_len + tokens_per_cta - 1) / tokens_per_cta;
    if (nqb > 0x7fffffff || p.batch > 65535 || p.num_kv_heads > 65535) return MG_ERR_INVALID_ARGUMENT;
    dim3 grid((unsigned)nqb, (unsigned)p.num_kv_heads, (unsigned)p.batch);
    return launch_pdl(extend_kernel, grid, dim3(kThreads), kSmemBytes, stream, tq, p);
}

}  // namespace extend
}  // namespace mg
