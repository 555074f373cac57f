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

// ---------------------------------------------------------------- host: TMA tensor maps (extend's Q tiles)

using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *, const cuuint64_t *,
                                   const cuuint64_t *, const cuuint32_t *, const cuuint32_t *,
                                   CUtensorMapInterleave, CUtensorMapSwizzle, CUtensorMapL2promotion,
                                   CUtensorMapFloatOOBfill);

// cuTensorMapEncodeTiled through the runtime's driver entry point (no libcuda
// link), looked up once; the function-local static makes the lookup thread-safe.
inline EncodeTiledFn encode_fn() {
    static const EncodeTiledFn fn = [] {
        void *ptr = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            return reinterpret_cast<EncodeTiledFn>(ptr);
        return static_cast<EncodeTiledFn>(nullptr);
    }();
    return fn;
}

}  // namespace mg
