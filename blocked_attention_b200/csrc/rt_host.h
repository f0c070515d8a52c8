// rt_host.h -- host-side helpers shared by librtlayer's translation units
// (defined in rt_api.cu). Internal: not part of the C ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace rt {

// eps inside the square root of every RMSNorm, r(v) = sqrt(mean v^2 + eps)
constexpr float kEps = 1e-6f;

// Records `e` as the calling thread's last CUDA error (rt_last_cuda_error
// reads it) and returns RT_ERR_CUDA. Every RT_ERR_CUDA status of the library
// is returned through this function.
int cuda_failure(cudaError_t e);

// Loads cuTensorMapEncodeTiled once per process; false if the driver lacks it.
bool load_tensor_map_encoder();

// 2-D bf16 tensor map over a row-major [rows][inner] matrix; box 64 x
// box_rows, 128-byte swizzle (the K-major UMMA operand layout). Out-of-range
// rows read 0. False if the base is not 16-byte aligned or encoding fails.
// load_tensor_map_encoder() must have succeeded.
bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows);

// Output-tile width of the batched projection GEMM: the widest tile
// (256, 128, 64, else 32) that still gives >= 120 output tiles.
int choose_bn(int M, int N);

}  // namespace rt
