// mg.cu -- the C ABI of libmg (declared in include/mg.h): argument checks,
// the decode split plan, and kernel launches on the caller's stream.
//
// Everything is one translation unit so the kernels share the device error
// word without relocatable device code.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <mutex>

#include "common.cuh"
#include "decode.cuh"
#include "extend.cuh"
#include "store_kv.cuh"

namespace mg {
namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxDecodeWorkers = 1 << 22;

// Per-device caches, filled on first use.  They are read without the lock,
// so they are atomics: a thread that sees a value also sees what was done
// before it was stored (the attributes set, the count read).  What belongs to
// a CUDA context (kernel attributes, a module global's address) is keyed on
// the context's unique id, so a context created after cudaDeviceReset is set
// up again instead of inheriting the old context's state.
std::atomic<int> g_sm_count[kMaxDevices];
std::atomic<unsigned long long> g_attr_ctx[kMaxDevices];  // context whose kernel attributes are set
std::mutex g_attr_mutex;

// mg_set_extend_wait_limit: process-wide, read at each extend launch.
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;
std::atomic<uint64_t> g_extend_wait_limit_ns{kDefaultWaitLimitNs};
std::atomic<int32_t> g_extend_inject_stall{0};

// mg_mixed_attn with a split: the extend half runs on a library stream of the
// device (non-blocking, created once per context), forked from and joined back
// to the caller's stream by events.
struct SideStream {
    unsigned long long ctx;
    cudaStream_t stream;
};
SideStream g_side[kMaxDevices];
std::mutex g_side_mutex;

using CtxGetCurrentFn = CUresult (*)(CUcontext *);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long *);

// Unique id of the calling thread's current CUDA context (0: none current, or
// the driver cannot tell).  Ids are never reused within a process.
unsigned long long current_context_id() {
    static const CtxGetCurrentFn get_current = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<CtxGetCurrentFn>(ptr);
        return static_cast<CtxGetCurrentFn>(nullptr);
    }();
    static const CtxGetIdFn get_id = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuCtxGetId", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<CtxGetIdFn>(ptr);
        return static_cast<CtxGetIdFn>(nullptr);
    }();
    CUcontext ctx = nullptr;
    unsigned long long id = 0;
    if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
    if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
    return id;
}

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

mg_status current_device(int &dev) {
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kMaxDevices) return MG_ERR_CUDA;
    return MG_OK;
}

mg_status sm_count(int &sms) {
    int dev;
    if (current_device(dev) != MG_OK) return MG_ERR_CUDA;
    int v = g_sm_count[dev].load(std::memory_order_acquire);
    if (v == 0) {
        if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
            return MG_ERR_CUDA;
        g_sm_count[dev].store(v, std::memory_order_release);
    }
    sms = v;
    return MG_OK;
}

mg_status side_stream(cudaStream_t &out) {
    int dev;
    if (current_device(dev) != MG_OK) return MG_ERR_CUDA;
    const unsigned long long ctx = current_context_id();
    std::lock_guard<std::mutex> lock(g_side_mutex);
    if (g_side[dev].stream == nullptr || g_side[dev].ctx != ctx) {
        cudaStream_t st = nullptr;
        if (cudaStreamCreateWithFlags(&st, cudaStreamNonBlocking) != cudaSuccess) return MG_ERR_CUDA;
        g_side[dev].stream = st;
        g_side[dev].ctx = ctx;
    }
    out = g_side[dev].stream;
    return MG_OK;
}

// Opt the kernels with large dynamic shared memory in, once per device.
mg_status ensure_kernel_attributes() {
    int dev;
    if (current_device(dev) != MG_OK) return MG_ERR_CUDA;
    const unsigned long long ctx = current_context_id();
    if (ctx != 0 && g_attr_ctx[dev].load(std::memory_order_acquire) == ctx) return MG_OK;
    std::lock_guard<std::mutex> lock(g_attr_mutex);
    if (ctx != 0 && g_attr_ctx[dev].load(std::memory_order_relaxed) == ctx) return MG_OK;
    if (cudaFuncSetAttribute(decode::decode_kernel<1, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(decode::decode_kernel<2, false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(decode::decode_kernel<1, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(decode::decode_kernel<2, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(decode::decode_kernel<2, false, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess ||
        cudaFuncSetAttribute(decode::decode_kernel<2, true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             decode::kSmemBytes) != cudaSuccess)
        return MG_ERR_CUDA;
    if (extend::set_attributes() != cudaSuccess) return MG_ERR_CUDA;
    // the calls above made the device's primary context current if none was
    const unsigned long long now = current_context_id();
    if (now != 0) g_attr_ctx[dev].store(now, std::memory_order_release);
    return MG_OK;
}

// Decode plan: the number of workers (warps) that share the work equally.
// Automatic: one per warp slot the device keeps resident (SMs x resident CTAs
// x warps per CTA), i.e. a single persistent wave.  Forced: num_partitions workers.
mg_status decode_plan(int batch, int hkv, int max_seq_len, int num_partitions, int &workers) {
    if (batch <= 0 || hkv <= 0 || max_seq_len <= 0 || num_partitions < 0) return MG_ERR_INVALID_ARGUMENT;
    if (batch > decode::kMaxBatch) return MG_ERR_UNSUPPORTED_SHAPE;
    if (num_partitions > 0) {
        if (num_partitions > kMaxDecodeWorkers) return MG_ERR_INVALID_ARGUMENT;
        workers = num_partitions;
    } else {
        int sms;
        if (sm_count(sms) != MG_OK) return MG_ERR_CUDA;
        workers = sms * MG_DECODE_MIN_BLOCKS * decode::kWarps;
    }
    return MG_OK;
}

size_t align256(size_t x) { return (x + 255) / 256 * 256; }

// Workspace: per-(virtual) request unit prefix (int64), then per-slot
// log-sum-exp and partial outputs (fp32) of `rows` q rows each; slots = pairs
// + workers.  Plain decode: one virtual request per request, rows = group.
// Shared-prefix decode: num_groups more virtual requests, rows = 16.
struct DecodeWorkspace {
    size_t prefix, lse, o, total;
};
DecodeWorkspace decode_ws_layout(int batch, int hq, int hkv, int workers, int num_groups = 0) {
    const size_t vreqs = (size_t)batch + (size_t)num_groups;
    const size_t slots = vreqs * hkv + (size_t)workers;
    const size_t rows = num_groups > 0 ? (size_t)decode::kRows : (size_t)(hq / hkv);
    DecodeWorkspace w;
    w.prefix = 0;
    w.lse = align256((vreqs + 1) * sizeof(int64_t));
    w.o = w.lse + align256(slots * rows * sizeof(float));
    w.total = w.o + slots * rows * kHeadDim * sizeof(float);
    return w;
}

mg_status check_attention_shape(int hq, int hkv, int head_dim) {
    if (hq <= 0 || hkv <= 0 || head_dim <= 0) return MG_ERR_INVALID_ARGUMENT;
    if (head_dim != kHeadDim || hq % hkv != 0 || hq / hkv > decode::kRows) return MG_ERR_UNSUPPORTED_SHAPE;
    return MG_OK;
}

// A softmax scale is finite and positive; the kernels take row maxima of the
// unscaled scores and scale them afterwards, which needs scale > 0.
bool valid_scale(float scale) { return scale > 0.f && scale <= 3.0e38f; }

}  // namespace
}  // namespace mg

namespace mg {
namespace {
// Decode attention; with k_new != nullptr the KV store of the step's new
// tokens (one per request) is fused into the same launch.
// With group_first != nullptr the shared-prefix (cascade) mode runs.
mg_status decode_impl(const void *q, const void *k_new, const void *v_new, const int32_t *out_loc,
                      const void *k_cache, const void *v_cache, int64_t num_slots, const int32_t *page_table,
                      int32_t page_table_rows, int32_t page_table_stride, const int32_t *table_idx,
                      const int32_t *seq_len, int32_t batch, int32_t max_seq_len, int32_t num_q_heads,
                      int32_t num_kv_heads, int32_t head_dim, float scale, int32_t num_partitions, void *out,
                      void *workspace, size_t workspace_bytes, void *stream, const int32_t *group_first = nullptr,
                      const int32_t *prefix_len = nullptr, int32_t num_groups = 0, const int32_t *row_map = nullptr,
                      int32_t total_rows = 0, bool check_only = false) {
    const bool fused = k_new != nullptr;
    const bool cascade = group_first != nullptr;
    if (cascade && (!prefix_len || num_groups <= 0)) return MG_ERR_INVALID_ARGUMENT;
    if (cascade && (int64_t)batch + num_groups > decode::kMaxBatch) return MG_ERR_UNSUPPORTED_SHAPE;
    mg_status st = check_attention_shape(num_q_heads, num_kv_heads, head_dim);
    if (st != MG_OK) return st;
    if (!valid_scale(scale)) return MG_ERR_INVALID_ARGUMENT;
    if (batch <= 0 || num_slots <= 0 || page_table_rows <= 0 || page_table_stride <= 0 ||
        max_seq_len <= 0 || max_seq_len > page_table_stride)
        return MG_ERR_INVALID_ARGUMENT;
    if (!q || !k_cache || !v_cache || !page_table || !table_idx || !seq_len || !out)
        return MG_ERR_INVALID_ARGUMENT;
    if (fused && (!v_new || !out_loc)) return MG_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return MG_ERR_MISALIGNED;
    if (fused && (!aligned16(k_new) || !aligned16(v_new))) return MG_ERR_MISALIGNED;
    int workers;
    st = decode_plan(batch, num_kv_heads, max_seq_len, num_partitions, workers);
    if (st != MG_OK) return st;
    // units <= batch * Hkv * ceil(max_seq_len / 16); the partition math multiplies by workers
    const double max_units = (double)batch * num_kv_heads * ((max_seq_len + 15) / 16);
    if (max_units * (double)(workers + 1) >= 4.0e18) return MG_ERR_UNSUPPORTED_SHAPE;
    const DecodeWorkspace ws = decode_ws_layout(batch, num_q_heads, num_kv_heads, workers, cascade ? num_groups : 0);
    if (!workspace || workspace_bytes < ws.total) return MG_ERR_WORKSPACE_TOO_SMALL;
    if (!aligned16(workspace)) return MG_ERR_MISALIGNED;
    if (check_only) return MG_OK;  // the host checks alone (a caller about to launch other work first)
    if (ensure_kernel_attributes() != MG_OK) return MG_ERR_CUDA;

    decode::Params p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
    p.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
    p.page_table = page_table;
    p.table_idx = table_idx;
    p.seq_len = seq_len;
    p.out = static_cast<__nv_bfloat16 *>(out);
    uint8_t *wsb = static_cast<uint8_t *>(workspace);
    p.prefix = reinterpret_cast<int64_t *>(wsb + ws.prefix);
    p.part_lse = reinterpret_cast<float *>(wsb + ws.lse);
    p.part_o = reinterpret_cast<float *>(wsb + ws.o);
    p.k_new = static_cast<const __nv_bfloat16 *>(k_new);
    p.v_new = static_cast<const __nv_bfloat16 *>(v_new);
    p.out_loc = out_loc;
    p.k_store = const_cast<__nv_bfloat16 *>(p.k_cache);
    p.v_store = const_cast<__nv_bfloat16 *>(p.v_cache);
    p.num_slots = num_slots;
    p.pt_rows = page_table_rows;
    p.pt_stride = page_table_stride;
    p.batch = batch;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_q_heads / num_kv_heads;
    p.num_workers = workers;
    p.max_seq_len = max_seq_len;
    p.scale_log2 = scale * kLog2e;
    p.group_first = group_first;
    p.prefix_len = prefix_len;
    p.num_groups = cascade ? num_groups : 0;
    p.max_members = decode::kRows / p.group;
    p.rows_per_slot = cascade ? decode::kRows : p.group;
    p.num_vreqs = batch + p.num_groups;
    p.row_map = row_map;
    p.total_rows = total_rows;

    cudaStream_t s = static_cast<cudaStream_t>(stream);
    const int ctas = (workers + decode::kWarps - 1) / decode::kWarps;
    const dim3 grid(ctas), block(decode::kThreads);
    const size_t smem = decode::kSmemBytes;
    if (cascade)
        st = fused ? launch_pdl(decode::decode_kernel<2, true, true>, grid, block, smem, s, p)
                   : launch_pdl(decode::decode_kernel<2, false, true>, grid, block, smem, s, p);
    else if (p.group <= 8)
        st = fused ? launch_pdl(decode::decode_kernel<1, true>, grid, block, smem, s, p)
                   : launch_pdl(decode::decode_kernel<1, false>, grid, block, smem, s, p);
    else
        st = fused ? launch_pdl(decode::decode_kernel<2, true>, grid, block, smem, s, p)
                   : launch_pdl(decode::decode_kernel<2, false>, grid, block, smem, s, p);
    if (st != MG_OK) return st;
    const int warps = batch * num_q_heads;
    return launch_pdl(decode::decode_merge_kernel, dim3((warps + 3) / 4), dim3(128), 0, s, p);
}
}  // namespace
}  // namespace mg

namespace mg {
namespace {
// Extend attention; with skip_single the requests with exactly one new token
// are left to the decode kernel (mixed batches).
mg_status extend_impl(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                      const int32_t *page_table, int32_t page_table_rows, int32_t page_table_stride,
                      const int32_t *table_idx, const int32_t *cached_len, const int32_t *seq_len,
                      const int32_t *q_offset, int32_t batch, int32_t total_q, int32_t max_q_len,
                      int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                      void *out, void *stream, bool skip_single, int max_ctas = 0) {
    mg_status st = check_attention_shape(num_q_heads, num_kv_heads, head_dim);
    if (st != MG_OK) return st;
    if (!valid_scale(scale)) return MG_ERR_INVALID_ARGUMENT;
    if (batch <= 0 || total_q < 0 || max_q_len < 0 || num_slots <= 0 || page_table_rows <= 0 ||
        page_table_stride <= 0 || max_seq_len <= 0 || max_seq_len > page_table_stride)
        return MG_ERR_INVALID_ARGUMENT;
    if (total_q == 0 || max_q_len == 0) return MG_OK;
    if (!q || !k_cache || !v_cache || !page_table || !table_idx || !cached_len || !seq_len ||
        !q_offset || !out)
        return MG_ERR_INVALID_ARGUMENT;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out))
        return MG_ERR_MISALIGNED;
    if (ensure_kernel_attributes() != MG_OK) return MG_ERR_CUDA;
    extend::Params p;
    p.q = static_cast<const __nv_bfloat16 *>(q);
    p.k_cache = static_cast<const __nv_bfloat16 *>(k_cache);
    p.v_cache = static_cast<const __nv_bfloat16 *>(v_cache);
    p.page_table = page_table;
    p.table_idx = table_idx;
    p.cached_len = cached_len;
    p.seq_len = seq_len;
    p.q_offset = q_offset;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.num_slots = num_slots;
    p.pt_rows = page_table_rows;
    p.pt_stride = page_table_stride;
    p.batch = batch;
    p.total_q = total_q;
    p.max_q_len = max_q_len;
    p.max_seq_len = max_seq_len;
    p.num_q_heads = num_q_heads;
    p.num_kv_heads = num_kv_heads;
    p.group = num_q_heads / num_kv_heads;
    p.scale_log2 = scale * kLog2e;
    p.wait_limit_ns = g_extend_wait_limit_ns.load(std::memory_order_relaxed);
    p.inject_stall = g_extend_inject_stall.load(std::memory_order_relaxed);
    p.skip_single = skip_single ? 1 : 0;
    int sms;
    if (sm_count(sms) != MG_OK) return MG_ERR_CUDA;
    return extend::launch(p, max_ctas > 0 && max_ctas < sms ? max_ctas : sms, static_cast<cudaStream_t>(stream));
}
}  // namespace
}  // namespace mg

using namespace mg;

extern "C" {

const char *mg_status_string(mg_status s) {
    switch (s) {
        case MG_OK: return "MG_OK";
        case MG_ERR_INVALID_ARGUMENT: return "MG_ERR_INVALID_ARGUMENT";
        case MG_ERR_UNSUPPORTED_SHAPE: return "MG_ERR_UNSUPPORTED_SHAPE";
        case MG_ERR_MISALIGNED: return "MG_ERR_MISALIGNED";
        case MG_ERR_WORKSPACE_TOO_SMALL: return "MG_ERR_WORKSPACE_TOO_SMALL";
        case MG_ERR_CUDA: return "MG_ERR_CUDA";
        case MG_ERR_DEVICE_CHECK: return "MG_ERR_DEVICE_CHECK";
        case MG_ERR_DEVICE_TIMEOUT: return "MG_ERR_DEVICE_TIMEOUT";
    }
    return "MG_ERR_UNKNOWN";
}

int32_t mg_abi_version(void) { return 2; }

mg_status mg_store_kv(const void *k, const void *v, const int32_t *out_loc, int32_t num_tokens,
                      void *k_cache, void *v_cache, int64_t num_slots, int32_t num_kv_heads,
                      int32_t head_dim, void *stream) {
    if (num_tokens < 0 || num_slots <= 0 || num_kv_heads <= 0 || head_dim <= 0)
        return MG_ERR_INVALID_ARGUMENT;
    if (num_tokens == 0) return MG_OK;
    if (!k || !v || !out_loc || !k_cache || !v_cache) return MG_ERR_INVALID_ARGUMENT;
    const int64_t row_bytes = (int64_t)num_kv_heads * head_dim * 2;
    if (row_bytes % 16 != 0) return MG_ERR_UNSUPPORTED_SHAPE;
    if (!aligned16(k) || !aligned16(v) || !aligned16(k_cache) || !aligned16(v_cache))
        return MG_ERR_MISALIGNED;
    int sms;
    if (sm_count(sms) != MG_OK) return MG_ERR_CUDA;
    StoreParams p;
    p.k = static_cast<const uint4 *>(k);
    p.v = static_cast<const uint4 *>(v);
    p.out_loc = out_loc;
    p.k_cache = static_cast<uint4 *>(k_cache);
    p.v_cache = static_cast<uint4 *>(v_cache);
    p.num_slots = num_slots;
    p.vecs_per_token = (int32_t)(row_bytes / 16);
    p.total_vecs = (int64_t)num_tokens * p.vecs_per_token;
    const int threads = 256;
    long long blocks = (p.total_vecs + threads - 1) / threads;
    const long long cap = (long long)sms * 8;
    if (blocks > cap) blocks = cap;
    return launch_pdl(store_kv_kernel, dim3((unsigned)blocks), dim3(threads), 0, static_cast<cudaStream_t>(stream), p);
}

mg_status mg_decode_plan(int32_t batch, int32_t num_kv_heads, int32_t max_seq_len,
                         int32_t num_partitions, int32_t *workers_out, int64_t *slots_out) {
    int workers;
    mg_status st = decode_plan(batch, num_kv_heads, max_seq_len, num_partitions, workers);
    if (st != MG_OK) return st;
    if (workers_out) *workers_out = workers;
    if (slots_out) *slots_out = (int64_t)batch * num_kv_heads + workers;
    return MG_OK;
}

size_t mg_decode_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads,
                                 int32_t head_dim, int32_t max_seq_len, int32_t num_partitions) {
    int workers;
    if (check_attention_shape(num_q_heads, num_kv_heads, head_dim) != MG_OK) return 0;
    if (decode_plan(batch, num_kv_heads, max_seq_len, num_partitions, workers) != MG_OK) return 0;
    return decode_ws_layout(batch, num_q_heads, num_kv_heads, workers).total;
}

mg_status mg_decode_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                         const int32_t *page_table, int32_t page_table_rows,
                         int32_t page_table_stride, const int32_t *table_idx,
                         const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                         int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                         int32_t num_partitions, void *out, void *workspace, size_t workspace_bytes,
                         void *stream) {
    return decode_impl(q, nullptr, nullptr, nullptr, k_cache, v_cache, num_slots, page_table, page_table_rows,
                       page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                       head_dim, scale, num_partitions, out, workspace, workspace_bytes, stream);
}

mg_status mg_store_decode_attn(const void *q, const void *k_new, const void *v_new, const int32_t *out_loc,
                               void *k_cache, void *v_cache, int64_t num_slots, const int32_t *page_table,
                               int32_t page_table_rows, int32_t page_table_stride, const int32_t *table_idx,
                               const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                               int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim, float scale,
                               int32_t num_partitions, void *out, void *workspace, size_t workspace_bytes,
                               void *stream) {
    if (!k_new) return MG_ERR_INVALID_ARGUMENT;
    return decode_impl(q, k_new, v_new, out_loc, k_cache, v_cache, num_slots, page_table, page_table_rows,
                       page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                       head_dim, scale, num_partitions, out, workspace, workspace_bytes, stream);
}

size_t mg_decode_shared_prefix_workspace_bytes(int32_t batch, int32_t num_groups, int32_t num_q_heads,
                                               int32_t num_kv_heads, int32_t head_dim, int32_t max_seq_len,
                                               int32_t num_partitions) {
    int workers;
    if (num_groups <= 0 || (int64_t)batch + num_groups > decode::kMaxBatch) return 0;
    if (check_attention_shape(num_q_heads, num_kv_heads, head_dim) != MG_OK) return 0;
    if (decode_plan(batch, num_kv_heads, max_seq_len, num_partitions, workers) != MG_OK) return 0;
    return decode_ws_layout(batch, num_q_heads, num_kv_heads, workers, num_groups).total;
}

mg_status mg_decode_attn_shared_prefix(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                                       const int32_t *page_table, int32_t page_table_rows,
                                       int32_t page_table_stride, const int32_t *table_idx,
                                       const int32_t *seq_len, int32_t batch, int32_t max_seq_len,
                                       const int32_t *group_first, const int32_t *prefix_len,
                                       int32_t num_groups, int32_t num_q_heads, int32_t num_kv_heads,
                                       int32_t head_dim, float scale, int32_t num_partitions, void *out,
                                       void *workspace, size_t workspace_bytes, void *stream) {
    if (!group_first || !prefix_len || num_groups <= 0) return MG_ERR_INVALID_ARGUMENT;
    return decode_impl(q, nullptr, nullptr, nullptr, k_cache, v_cache, num_slots, page_table, page_table_rows,
                       page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                       head_dim, scale, num_partitions, out, workspace, workspace_bytes, stream, group_first,
                       prefix_len, num_groups);
}

mg_status mg_store_decode_attn_shared_prefix(const void *q, const void *k_new, const void *v_new,
                                             const int32_t *out_loc, void *k_cache, void *v_cache,
                                             int64_t num_slots, const int32_t *page_table,
                                             int32_t page_table_rows, int32_t page_table_stride,
                                             const int32_t *table_idx, const int32_t *seq_len, int32_t batch,
                                             int32_t max_seq_len, const int32_t *group_first,
                                             const int32_t *prefix_len, int32_t num_groups,
                                             int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                             float scale, int32_t num_partitions, void *out, void *workspace,
                                             size_t workspace_bytes, void *stream) {
    if (!k_new || !group_first || !prefix_len || num_groups <= 0) return MG_ERR_INVALID_ARGUMENT;
    return decode_impl(q, k_new, v_new, out_loc, k_cache, v_cache, num_slots, page_table, page_table_rows,
                       page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                       head_dim, scale, num_partitions, out, workspace, workspace_bytes, stream, group_first,
                       prefix_len, num_groups);
}

mg_status mg_extend_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                         const int32_t *page_table, int32_t page_table_rows,
                         int32_t page_table_stride, const int32_t *table_idx,
                         const int32_t *cached_len, const int32_t *seq_len,
                         const int32_t *q_offset, int32_t batch, int32_t total_q,
                         int32_t max_q_len, int32_t max_seq_len, int32_t num_q_heads,
                         int32_t num_kv_heads, int32_t head_dim, float scale, void *out,
                         void *stream) {
    return extend_impl(q, k_cache, v_cache, num_slots, page_table, page_table_rows, page_table_stride, table_idx,
                       cached_len, seq_len, q_offset, batch, total_q, max_q_len, max_seq_len, num_q_heads,
                       num_kv_heads, head_dim, scale, out, stream, false);
}

size_t mg_mixed_workspace_bytes(int32_t batch, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                                int32_t max_seq_len, int32_t num_partitions) {
    return mg_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len, num_partitions);
}

mg_status mg_mixed_attn(const void *q, const void *k_cache, const void *v_cache, int64_t num_slots,
                        const int32_t *page_table, int32_t page_table_rows, int32_t page_table_stride,
                        const int32_t *table_idx, const int32_t *cached_len, const int32_t *seq_len,
                        const int32_t *q_offset, int32_t batch, int32_t total_q, int32_t max_q_len,
                        int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
                        float scale, int32_t num_partitions, int32_t extend_ctas, void *out, void *workspace,
                        size_t workspace_bytes, void *stream) {
    // the same checks as mg_extend_attn, before anything is launched
    mg_status st = check_attention_shape(num_q_heads, num_kv_heads, head_dim);
    if (st != MG_OK) return st;
    if (!valid_scale(scale)) return MG_ERR_INVALID_ARGUMENT;
    if (batch <= 0 || total_q < 0 || max_q_len < 0 || num_slots <= 0 || page_table_rows <= 0 ||
        page_table_stride <= 0 || max_seq_len <= 0 || max_seq_len > page_table_stride || extend_ctas < 0)
        return MG_ERR_INVALID_ARGUMENT;
    if (total_q == 0 || max_q_len == 0) return MG_OK;
    if (!q_offset) return MG_ERR_INVALID_ARGUMENT;
    int sms = 1;  // the device is asked only when a split is requested
    if (extend_ctas > 0 && max_q_len > 1 && sm_count(sms) != MG_OK) return MG_ERR_CUDA;
    if (extend_ctas > 0 && max_q_len > 1 && sms > 1) {
        // The split: the extend kernel on extend_ctas SMs, on a side stream,
        // while the decode kernel's workers fill the other SMs (the decode
        // kernel is bound by HBM, the extend kernel by its softmax and tensor
        // cores, so the two overlap instead of following each other).
        const int e = extend_ctas < sms ? extend_ctas : sms - 1;
        int32_t workers = MG_DECODE_MIN_BLOCKS * decode::kWarps * (sms - e);
        if (num_partitions > 0 && num_partitions < workers) workers = num_partitions;
        // every host check of both halves before anything is enqueued
        if (!cached_len) return MG_ERR_INVALID_ARGUMENT;
        st = decode_impl(q, nullptr, nullptr, nullptr, k_cache, v_cache, num_slots, page_table, page_table_rows,
                         page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                         head_dim, scale, workers, out, workspace, workspace_bytes, stream, nullptr, nullptr, 0,
                         q_offset, total_q, true);
        if (st != MG_OK) return st;
        cudaStream_t side, s = static_cast<cudaStream_t>(stream);
        if (side_stream(side) != MG_OK) return MG_ERR_CUDA;
        cudaEvent_t fork = nullptr, join = nullptr;
        if (cudaEventCreateWithFlags(&fork, cudaEventDisableTiming) != cudaSuccess) return MG_ERR_CUDA;
        if (cudaEventCreateWithFlags(&join, cudaEventDisableTiming) != cudaSuccess) {
            cudaEventDestroy(fork);
            return MG_ERR_CUDA;
        }
        st = MG_OK;
        if (cudaEventRecord(fork, s) != cudaSuccess || cudaStreamWaitEvent(side, fork, 0) != cudaSuccess)
            st = MG_ERR_CUDA;
        if (st == MG_OK)
            st = extend_impl(q, k_cache, v_cache, num_slots, page_table, page_table_rows, page_table_stride,
                             table_idx, cached_len, seq_len, q_offset, batch, total_q, max_q_len, max_seq_len,
                             num_q_heads, num_kv_heads, head_dim, scale, out, side, true, e);
        if (st == MG_OK)
            st = decode_impl(q, nullptr, nullptr, nullptr, k_cache, v_cache, num_slots, page_table, page_table_rows,
                             page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads,
                             head_dim, scale, workers, out, workspace, workspace_bytes, stream, nullptr, nullptr, 0,
                             q_offset, total_q);
        // the join is recorded whatever happened above, so the caller's stream
        // never runs ahead of work already enqueued on the side stream
        const bool joined = cudaEventRecord(join, side) == cudaSuccess && cudaStreamWaitEvent(s, join, 0) == cudaSuccess;
        cudaEventDestroy(fork);
        cudaEventDestroy(join);
        if (st == MG_OK && !joined) st = MG_ERR_CUDA;
        return st;
    }
    // one-token requests: the split-KV decode kernel and its merge, rows by q_offset
    st = decode_impl(q, nullptr, nullptr, nullptr, k_cache, v_cache, num_slots, page_table, page_table_rows,
                     page_table_stride, table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim,
                     scale, num_partitions, out, workspace, workspace_bytes, stream, nullptr, nullptr, 0, q_offset,
                     total_q);
    if (st != MG_OK || max_q_len <= 1) return st;
    // every other request: the extend kernel, which leaves the one-token ones alone
    return extend_impl(q, k_cache, v_cache, num_slots, page_table, page_table_rows, page_table_stride, table_idx,
                       cached_len, seq_len, q_offset, batch, total_q, max_q_len, max_seq_len, num_q_heads,
                       num_kv_heads, head_dim, scale, out, stream, true);
}

mg_status mg_set_extend_wait_limit(uint64_t limit_ns, int32_t inject_stall) {
    g_extend_wait_limit_ns.store(limit_ns ? limit_ns : kDefaultWaitLimitNs, std::memory_order_relaxed);
    g_extend_inject_stall.store(inject_stall ? 1 : 0, std::memory_order_relaxed);
    return MG_OK;
}

mg_status mg_read_device_error(void *stream, uint32_t *bits_out) {
    if (cudaStreamSynchronize(static_cast<cudaStream_t>(stream)) != cudaSuccess) return MG_ERR_CUDA;
    unsigned int bits = 0, zero = 0;
    if (cudaMemcpyFromSymbol(&bits, g_mg_device_error, sizeof bits) != cudaSuccess) return MG_ERR_CUDA;
    if (bits && cudaMemcpyToSymbol(g_mg_device_error, &zero, sizeof zero) != cudaSuccess)
        return MG_ERR_CUDA;
    if (bits_out) *bits_out = bits;
    if (bits & MG_DEVERR_WAIT_TIMEOUT) return MG_ERR_DEVICE_TIMEOUT;
    return bits ? MG_ERR_DEVICE_CHECK : MG_OK;
}

}  // extern "C"

// ---------------------------------------------------------------- decode without a caller workspace
//
// Some callers cannot hand the library device scratch memory: code whose
// device memory is entirely owned by another allocator (a serving engine's
// pre-sized pool, a framework's caching allocator) where an extra cudaMalloc
// would fail or fragment it, plug-ins that receive only their inputs and
// outputs, and step loops that must not pay an allocation (which can
// synchronise the device) in the middle of a step.  For them decode can use a
// workspace that lives in this library: a fixed-size array in device global
// memory that every device which loads the library holds until the process
// exits.
namespace mg {
namespace {

constexpr size_t kStaticDecodeWorkspaceBytes = MG_DECODE_STATIC_WORKSPACE_BYTES;
static __device__ __align__(256) unsigned char g_decode_static_workspace[kStaticDecodeWorkspaceBytes];

// The array's device address, per device, with the context it belongs to.
struct StaticWorkspaceAddress {
    unsigned long long ctx = 0;
    void *ptr = nullptr;
};
StaticWorkspaceAddress g_static_ws[kMaxDevices];  // guarded by g_static_ws_mutex
std::mutex g_static_ws_mutex;

// The array's device address on the current device.  In host code the
// array's name is only a host-side stand-in, so the address is looked up with
// the device current, once per device and context, and cached.  A module
// global lives in a context: after cudaDeviceReset the next context holds it
// at another address, so the cache is keyed on the context's unique id.
mg_status static_workspace(void *&ptr) {
    int dev;
    if (current_device(dev) != MG_OK) return MG_ERR_CUDA;
    std::lock_guard<std::mutex> lock(g_static_ws_mutex);
    StaticWorkspaceAddress &c = g_static_ws[dev];
    unsigned long long ctx = current_context_id();
    if (ctx == 0 || ctx != c.ctx) {
        void *p = nullptr;
        if (cudaGetSymbolAddress(&p, g_decode_static_workspace) != cudaSuccess || p == nullptr)
            return MG_ERR_CUDA;
        ctx = current_context_id();  // the lookup makes the primary context current if none was
        if (ctx == 0) return MG_ERR_CUDA;
        c.ctx = ctx;
        c.ptr = p;
    }
    ptr = c.ptr;
    return MG_OK;
}

}  // namespace
}  // namespace mg

extern "C" mg_status mg_decode_attn_static_workspace(
    const void *q, const void *k_cache, const void *v_cache, int64_t num_slots, const int32_t *page_table,
    int32_t page_table_rows, int32_t page_table_stride, const int32_t *table_idx, const int32_t *seq_len,
    int32_t batch, int32_t max_seq_len, int32_t num_q_heads, int32_t num_kv_heads, int32_t head_dim,
    float scale, int32_t num_partitions, void *out, void *stream) {
    // the plan's workspace must fit the fixed array: refuse larger batches up front
    const size_t need = mg_decode_workspace_bytes(batch, num_q_heads, num_kv_heads, head_dim, max_seq_len,
                                                  num_partitions);
    if (need > kStaticDecodeWorkspaceBytes) return MG_ERR_WORKSPACE_TOO_SMALL;
    void *ws = nullptr;
    const mg_status st = static_workspace(ws);
    if (st != MG_OK) return st;
    return mg_decode_attn(q, k_cache, v_cache, num_slots, page_table, page_table_rows, page_table_stride,
                          table_idx, seq_len, batch, max_seq_len, num_q_heads, num_kv_heads, head_dim, scale,
                          num_partitions, out, ws, kStaticDecodeWorkspaceBytes, stream);
}
