// common.cuh -- definitions shared by the kernels of libmg (one translation unit).
#pragma once

#include <cstdint>
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

}  // namespace mg
