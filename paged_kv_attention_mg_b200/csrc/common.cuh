// common.cuh -- definitions shared by the kernels of libmg (one translation unit).
#pragma once

#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include "mg.h"
#include "ptx.cuh"

namespace mg {

// Device error word: kernels OR MG_DEVERR_* bits into it instead of reading or
// writing out of bounds; mg_read_device_error() reads and clears it.
__device__ unsigned int g_mg_device_error;

constexpr int kHeadDim = 128;
constexpr float kLog2e = 1.4426950408889634f;

// ---------------------------------------------------------------- host: launches

// Launch with programmatic stream serialization: the kernel may start while
// the previous kernel in the stream finishes; it calls griddepcontrol.wait
// before touching anything that kernel wrote.
template <typename... KArgs, typename... Args>
inline mg_status launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t stream,
                            Args &&...args) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...) == cudaSuccess ? MG_OK : MG_ERR_CUDA;
}

// ---------------------------------------------------------------- host: TMA tensor maps

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda link).
inline EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    if (!fn) {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(ptr);
    }
    return fn;
}

// A pool [num_slots, num_kv_heads, 128] bf16 seen as 2-D rows (slot * Hkv + head)
// x 128 columns, box 64 columns x 1 row, 128-byte swizzle: the map tile::gather4
// reads four (slot, head) rows through.  Rows past the end read as zeros.
inline bool make_pool_tmap(CUtensorMap *map, const void *pool, int64_t num_slots, int num_kv_heads) {
    EncodeTiledFn enc = encode_fn();
    const cuuint64_t rows = (cuuint64_t)num_slots * (cuuint64_t)num_kv_heads;
    if (!enc || rows >= (1ull << 31)) return false;  // gather4 row coordinates are int32
    cuuint64_t dims[2] = {(cuuint64_t)kHeadDim, rows};
    cuuint64_t strides[1] = {(cuuint64_t)kHeadDim * 2};
    cuuint32_t box[2] = {64, 1};
    cuuint32_t es[2] = {1, 1};
    return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void *>(pool), dims, strides, box, es,
               CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
               CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace mg
