// decode.cuh -- split-KV paged decode attention + merge.
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
//   * one CTA per (kv head, split, request); a split is `chunk` consecutive
//     positions of one request.  The CTA serves the whole GQA group: the g q
//     heads that share this KV head form the M=16 rows of warp-level bf16
//     tensor-core MMAs (g <= 16, zero padded), so each K/V row is read from
//     HBM exactly once per step.
//   * the split's page-table entries are prefetched into shared memory once;
//     K and V rows (256 B each) are gathered with 16-byte cp.async into a
//     STAGES-deep ring of 64-key tiles, XOR-swizzled so ldmatrix is
//     bank-conflict free.
//   * each of the 4 warps takes 16 keys of every tile: S = Q K^T (mma.sync
//     m16n8k16), online softmax in the exp2 domain with quad-shuffle max/sum,
//     O += P V.  At the end the 4 warps' (m, l, O) are merged through shared
//     memory.
//   * a request that fits in one split writes bf16 output directly; otherwise
//     each split writes (O / l, log2-sum-exp) partials in fp32 and the merge
//     kernel combines them:  lse = log2 sum_s 2^lse_s,  o = sum_s 2^(lse_s - lse) o_s.
#pragma once

#include "common.cuh"

namespace mg {
namespace decode {

constexpr int kTile = 64;          // keys per pipeline stage
constexpr int kWarps = 4;
constexpr int kThreads = kWarps * 32;
constexpr int kRows = 16;          // MMA M: GQA group padded to 16
constexpr int kMaxChunk = 2048;    // keys per split (page-table prefetch capacity)
constexpr int kRowBytes = kHeadDim * 2;
constexpr int kStageBytes = 2 * kTile * kRowBytes;  // K tile + V tile

template <int STAGES>
struct Smem {
    static constexpr int kStages = STAGES;
    static constexpr int kRingBytes = STAGES * kStageBytes;
    static constexpr int kIdxOffset = kRingBytes;
    static constexpr int kBytes = kRingBytes + kMaxChunk * 4;
    static_assert(kRingBytes >= kWarps * kRows * kHeadDim * 4, "merge scratch must fit in the ring");
};

struct Params {
    const __nv_bfloat16 *q;
    const __nv_bfloat16 *k_cache;
    const __nv_bfloat16 *v_cache;
    const int32_t *page_table;
    const int32_t *table_idx;
    const int32_t *seq_len;
    __nv_bfloat16 *out;
    float *part_o;    // [B, Hq, num_splits, 128]
    float *part_lse;  // [B, Hq, num_splits]
    int64_t num_slots;
    int32_t pt_rows, pt_stride;
    int32_t batch, num_q_heads, num_kv_heads, group;
    int32_t chunk, num_splits, max_seq_len;
    float scale_log2;  // softmax scale * log2(e)
};

// byte offset of 16-byte chunk `c` of row `row` inside a [rows x 256 B] tile
__device__ __forceinline__ uint32_t swz(int row, int c) {
    return (uint32_t)(row * kRowBytes + ((c ^ (row & 7)) << 4));
}

// Returns the request's length, or 0 if its metadata is invalid (flagged).
__device__ __forceinline__ int checked_length(const Params &p, int r, int &row) {
    row = __ldg(p.table_idx + r);
    const int L = __ldg(p.seq_len + r);
    if (row < 0 || row >= p.pt_rows) return -1;
    if (L < 1 || L > p.pt_stride || L > p.max_seq_len) return -2;
    return L;
}

#ifndef MG_DECODE_MIN_BLOCKS
#define MG_DECODE_MIN_BLOCKS 2  // resident CTAs per SM the register budget is sized for
#endif

template <int STAGES>
__global__ void __launch_bounds__(kThreads, MG_DECODE_MIN_BLOCKS) decode_split_kernel(const Params p) {
    using S = Smem<STAGES>;
    extern __shared__ __align__(1024) uint8_t smem[];
    int32_t *idx = reinterpret_cast<int32_t *>(smem + S::kIdxOffset);
    __shared__ float red_m[kWarps][kRows];
    __shared__ float red_l[kWarps][kRows];

    const int kvh = blockIdx.x, split = blockIdx.y, r = blockIdx.z;
    const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

    int row;
    const int L = checked_length(p, r, row);
    if (L <= 0) {
        if (tid == 0 && split == 0 && kvh == 0)
            atomicOr(&g_mg_device_error, L == -1 ? MG_DEVERR_ROW_RANGE : MG_DEVERR_LENGTH);
        return;
    }
    const int start = split * p.chunk;
    if (start >= L) return;
    const int n = min(L - start, p.chunk);
    const int nsplit_r = (L + p.chunk - 1) / p.chunk;

    // ---- prefetch this split's page-table entries
    const int32_t *pt = p.page_table + (int64_t)row * p.pt_stride + start;
    for (int i = tid; i < n; i += kThreads) {
        int s = __ldg(pt + i);
        if (s < 0 || (int64_t)s >= p.num_slots) {
            atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
            s = -1;
        }
        idx[i] = s;
    }

    // ---- Q as MMA A fragments: rows = the g heads of this KV head (zero padded)
    uint32_t qf[8][4];
    {
        const int h0 = kvh * p.group;
        const int ra = lane >> 2, rb = ra + 8, cq = (lane & 3) * 2;
        const __nv_bfloat16 *qa = p.q + ((int64_t)r * p.num_q_heads + h0 + ra) * kHeadDim;
        const __nv_bfloat16 *qb = p.q + ((int64_t)r * p.num_q_heads + h0 + rb) * kHeadDim;
        const bool va = ra < p.group, vb = rb < p.group;
#pragma unroll
        for (int kk = 0; kk < 8; ++kk) {
            const int c0 = kk * 16 + cq;
            qf[kk][0] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + c0)) : 0u;
            qf[kk][1] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + c0)) : 0u;
            qf[kk][2] = va ? __ldg(reinterpret_cast<const uint32_t *>(qa + c0 + 8)) : 0u;
            qf[kk][3] = vb ? __ldg(reinterpret_cast<const uint32_t *>(qb + c0 + 8)) : 0u;
        }
    }
    __syncthreads();  // idx visible

    const uint32_t ring = smem_u32(smem);
    const int ntiles = (n + kTile - 1) / kTile;
    const int64_t head_stride = (int64_t)p.num_kv_heads * kHeadDim;

    // Each warp instruction copies two full 256-byte rows (lanes 0-15 / 16-31);
    // 128 rows per stage (64 K + 64 V) -> 16 instructions per warp.
    auto issue = [&](int tile) {
        const uint32_t base = ring + (uint32_t)((tile % STAGES) * kStageBytes);
        const int key0 = tile * kTile;
        const int c = lane & 15;
#pragma unroll
        for (int it = 0; it < 16; ++it) {
            const int rr = it * 8 + warp * 2 + (lane >> 4);  // 0..127
            const int key = rr & (kTile - 1);
            const bool is_v = rr >= kTile;
            const int pos = key0 + key;
            const int slot = pos < n ? idx[pos] : -1;
            const __nv_bfloat16 *src = (is_v ? p.v_cache : p.k_cache) +
                                       (int64_t)(slot < 0 ? 0 : slot) * head_stride +
                                       (int64_t)kvh * kHeadDim + c * 8;
            cp_async_16(base + (is_v ? kTile * kRowBytes : 0) + swz(key, c), src, slot < 0 ? 0u : 16u);
        }
    };

#pragma unroll
    for (int s = 0; s < STAGES - 1; ++s) {
        if (s < ntiles) issue(s);
        cp_async_commit();
    }

    float o[16][4];
#pragma unroll
    for (int j = 0; j < 16; ++j) o[j][0] = o[j][1] = o[j][2] = o[j][3] = 0.f;
    float m0 = -INFINITY, m1 = -INFINITY, l0 = 0.f, l1 = 0.f;  // rows lane/4 and lane/4+8

    for (int tile = 0; tile < ntiles; ++tile) {
        cp_async_wait<STAGES - 2>();
        __syncthreads();  // tile landed for all threads; slot of tile-1 is free
        {
            const int nt = tile + STAGES - 1;
            if (nt < ntiles) issue(nt);
            cp_async_commit();
        }
        const int kbase = tile * kTile + warp * 16;  // first key of this warp
        if (kbase >= n) continue;
        const uint32_t kt = ring + (uint32_t)((tile % STAGES) * kStageBytes);
        const uint32_t vt = kt + kTile * kRowBytes;

        // S = Q K^T for this warp's 16 keys (two n8 tiles)
        float sc[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
        {
            const int mi = lane >> 3;
            const int key = warp * 16 + (mi >> 1) * 8 + (lane & 7);
#pragma unroll
            for (int kk = 0; kk < 8; ++kk) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4(kt + swz(key, 2 * kk + (mi & 1)), b0, b1, b2, b3);
                mma_bf16_16816(sc[0], qf[kk], b0, b1);
                mma_bf16_16816(sc[1], qf[kk], b2, b3);
            }
        }
        // scale, mask keys past the split end or with a rejected slot, row max
        float mx0 = -INFINITY, mx1 = -INFINITY;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
                const int pos = kbase + nt * 8 + (lane & 3) * 2 + c;
                const bool ok = pos < n && idx[pos] >= 0;
                const float s0 = ok ? sc[nt][c] * p.scale_log2 : -INFINITY;
                const float s1 = ok ? sc[nt][c + 2] * p.scale_log2 : -INFINITY;
                sc[nt][c] = s0;
                sc[nt][c + 2] = s1;
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
        const float corr0 = fast_exp2(m0 - mu0), corr1 = fast_exp2(m1 - mu1);
        m0 = mn0;
        m1 = mn1;
        float ps0 = 0.f, ps1 = 0.f;
#pragma unroll
        for (int nt = 0; nt < 2; ++nt) {
            sc[nt][0] = fast_exp2(sc[nt][0] - mu0);
            sc[nt][1] = fast_exp2(sc[nt][1] - mu0);
            sc[nt][2] = fast_exp2(sc[nt][2] - mu1);
            sc[nt][3] = fast_exp2(sc[nt][3] - mu1);
            ps0 += sc[nt][0] + sc[nt][1];
            ps1 += sc[nt][2] + sc[nt][3];
        }
        l0 = l0 * corr0 + ps0;
        l1 = l1 * corr1 + ps1;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
            o[j][0] *= corr0;
            o[j][1] *= corr0;
            o[j][2] *= corr1;
            o[j][3] *= corr1;
        }
        uint32_t pa[4];
        pa[0] = pack_bf16x2(sc[0][0], sc[0][1]);
        pa[1] = pack_bf16x2(sc[0][2], sc[0][3]);
        pa[2] = pack_bf16x2(sc[1][0], sc[1][1]);
        pa[3] = pack_bf16x2(sc[1][2], sc[1][3]);
        // O += P V  (V^T fragments through ldmatrix.trans)
        {
            const int mi = lane >> 3;
            const int key = warp * 16 + (mi & 1) * 8 + (lane & 7);
#pragma unroll
            for (int dp = 0; dp < 8; ++dp) {
                uint32_t b0, b1, b2, b3;
                ldmatrix_x4_trans(vt + swz(key, 2 * dp + (mi >> 1)), b0, b1, b2, b3);
                mma_bf16_16816(o[2 * dp], pa, b0, b1);
                mma_bf16_16816(o[2 * dp + 1], pa, b2, b3);
            }
        }
    }

    // ---- merge the 4 warps' partial states
    l0 += __shfl_xor_sync(0xffffffffu, l0, 1);
    l0 += __shfl_xor_sync(0xffffffffu, l0, 2);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 1);
    l1 += __shfl_xor_sync(0xffffffffu, l1, 2);
    cp_async_wait<0>();
    __syncthreads();  // ring is idle: reuse it as merge scratch
    const int ra = lane >> 2, rb = ra + 8;
    if ((lane & 3) == 0) {
        red_m[warp][ra] = m0;
        red_m[warp][rb] = m1;
        red_l[warp][ra] = l0;
        red_l[warp][rb] = l1;
    }
    __syncthreads();
    float Ma = -INFINITY, Mb = -INFINITY;
#pragma unroll
    for (int w = 0; w < kWarps; ++w) {
        Ma = fmaxf(Ma, red_m[w][ra]);
        Mb = fmaxf(Mb, red_m[w][rb]);
    }
    const float fa = m0 == -INFINITY ? 0.f : fast_exp2(m0 - Ma);
    const float fb = m1 == -INFINITY ? 0.f : fast_exp2(m1 - Mb);
    float *obuf = reinterpret_cast<float *>(smem);  // [warps][16 rows][128]
    const int g = p.group;
#pragma unroll
    for (int j = 0; j < 16; ++j) {
        const int d = j * 8 + (lane & 3) * 2;
        if (ra < g)
            *reinterpret_cast<float2 *>(obuf + (warp * kRows + ra) * kHeadDim + d) =
                make_float2(o[j][0] * fa, o[j][1] * fa);
        if (rb < g)
            *reinterpret_cast<float2 *>(obuf + (warp * kRows + rb) * kHeadDim + d) =
                make_float2(o[j][2] * fb, o[j][3] * fb);
    }
    __syncthreads();
    const int h0 = kvh * g;
    for (int e = tid; e < g * kHeadDim; e += kThreads) {
        const int rr = e / kHeadDim, d = e % kHeadDim;
        float M = -INFINITY;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) M = fmaxf(M, red_m[w][rr]);
        float Lsum = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kWarps; ++w) {
            const float mw = red_m[w][rr];
            if (mw != -INFINITY) Lsum += red_l[w][rr] * fast_exp2(mw - M);
            acc += obuf[(w * kRows + rr) * kHeadDim + d];
        }
        const float val = Lsum > 0.f ? acc / Lsum : 0.f;
        const int64_t oh = (int64_t)r * p.num_q_heads + h0 + rr;
        if (nsplit_r == 1) {
            p.out[oh * kHeadDim + d] = __float2bfloat16_rn(val);
        } else {
            p.part_o[(oh * p.num_splits + split) * kHeadDim + d] = val;
            if (d == 0) p.part_lse[oh * p.num_splits + split] = Lsum > 0.f ? M + __log2f(Lsum) : -INFINITY;
        }
    }
}

// One warp per (request, q head): combine the splits' partials.
__global__ void __launch_bounds__(128) decode_merge_kernel(const Params p) {
    const int wg = blockIdx.x * 4 + (threadIdx.x >> 5);
    const int lane = threadIdx.x & 31;
    if (wg >= p.batch * p.num_q_heads) return;
    const int r = wg / p.num_q_heads;
    int row;
    const int L = checked_length(p, r, row);
    if (L <= 0) return;  // flagged by the split kernel
    const int ns = (L + p.chunk - 1) / p.chunk;
    if (ns <= 1) return;  // written directly by the split kernel
    const int64_t oh = wg;  // == r * Hq + h
    const float *lse = p.part_lse + oh * p.num_splits;
    float mx = -INFINITY;
    for (int s = lane; s < ns; s += 32) mx = fmaxf(mx, lse[s]);
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
    float wsum = 0.f;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    const float4 *po = reinterpret_cast<const float4 *>(p.part_o + oh * p.num_splits * kHeadDim) + lane;
    for (int s = 0; s < ns; ++s) {
        const float ls = lse[s];
        const float w = ls == -INFINITY ? 0.f : fast_exp2(ls - mx);
        const float4 v = po[s * (kHeadDim / 4)];
        wsum += w;
        acc.x += w * v.x;
        acc.y += w * v.y;
        acc.z += w * v.z;
        acc.w += w * v.w;
    }
    const float inv = wsum > 0.f ? 1.f / wsum : 0.f;
    uint2 packed;
    packed.x = pack_bf16x2(acc.x * inv, acc.y * inv);
    packed.y = pack_bf16x2(acc.z * inv, acc.w * inv);
    *reinterpret_cast<uint2 *>(p.out + oh * kHeadDim + lane * 4) = packed;
}

}  // namespace decode
}  // namespace mg
