// store_kv.cuh -- the KV write: scatter the new tokens' K/V rows into pool
// slots at out_loc ("手写 mini-sglang 阶段一 · Engine 与采样器", §手工驱动引擎:
// out_loc = page_table[table_idx, cached_len:device_len]; Mini-SGLang tag page,
// Engine post §一: the KV-cache write precedes attention in every layer).
//
// One thread moves one 16-byte vector of K and the matching vector of V.  A
// token's row (num_kv_heads * head_dim bf16) is contiguous both in k/v and in
// the pool, so consecutive threads read and write consecutive 16-byte pieces:
// loads and stores are fully coalesced within each token.  The kernel is
// HBM/launch bound; there is nothing to compute.
#pragma once

#include "common.cuh"

namespace mg {

struct StoreParams {
    const uint4 *k;
    const uint4 *v;
    const int32_t *out_loc;
    uint4 *k_cache;
    uint4 *v_cache;
    int64_t num_slots;
    int64_t total_vecs;   // num_tokens * vecs_per_token
    int32_t vecs_per_token;
};

__global__ void __launch_bounds__(256) store_kv_kernel(const StoreParams p) {
    griddep_launch_dependents();  // attention may launch and wait on the store
    griddep_wait();               // k / v / out_loc written by the previous kernel
    const int64_t stride = (int64_t)gridDim.x * blockDim.x;
    for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < p.total_vecs; i += stride) {
        const int64_t t = i / p.vecs_per_token;
        const int64_t c = i - t * p.vecs_per_token;
        const int32_t slot = __ldg(p.out_loc + t);
        if (slot < 0 || (int64_t)slot >= p.num_slots) {
            atomicOr(&g_mg_device_error, MG_DEVERR_SLOT_RANGE);
            continue;
        }
        const uint4 kv = __ldcs(p.k + i);
        const uint4 vv = __ldcs(p.v + i);
        const int64_t dst = (int64_t)slot * p.vecs_per_token + c;
        p.k_cache[dst] = kv;
        p.v_cache[dst] = vv;
    }
}

}  // namespace mg
