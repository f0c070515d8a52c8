// rt_rownorm.cuh -- per-row RMS statistics (sm_100a).
//
// RMSNorm of the "Recurrent Transformer" paper page (paper §2, notation),
// read as rms(v) = v / sqrt(mean(v^2) + eps) with unit gain. The library
// never materialises rms(x): it computes the per-row factor 1/r(x) here and
// the GEMM epilogues apply it, since rms(x) W^T = (x W^T) / r(x).
#pragma once

#include "rt_common.cuh"

namespace rt {

// inv[r] = 1 / sqrt(mean(x_r^2) + eps), one warp per row of width d
template <class T>
__global__ void __launch_bounds__(256) k_row_inv_rms(const T* __restrict__ x, float* __restrict__ inv,
                                                     size_t rows, int d, float eps) {
  pdl_launch_dependents();
  pdl_wait();
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const T* xr = x + r * d;
  float s = 0.f;
  for (int e = lane; e < d; e += 32) {
    const float v = to_f(xr[e]);
    s += v * v;
  }
  s = warp_sum(s);
  if (lane == 0) inv[r] = rsqrtf(s / (float)d + eps);
}

}  // namespace rt
