// rt_simt.cuh -- fp32 SIMT GEMM of the fp32 storage mode (true fp32 FMA, no
// TF32), with the layer's epilogues. C[M][N] = A[M][K] * W[N][K]^T.
// The fp32 mode materialises each RMSNorm (k_rmsnorm_f32) instead of folding
// it into the epilogue; it exists for the 1e-4 parity bar, not for speed.
#pragma once

#include "rt_common.cuh"

namespace rt {

struct SimtEpi {
  int B, Nseq, d, d_ff, j;
  float* c32;            // PLAIN
  float* qkv;            // PROJ  [N][B][3d]
  const float* x;        // WO    [B][N][d]
  float* u;              // WO out / W2 in [B][d]
  float* h;              // W1 out [B][d_ff]
  float* zout;           // W2 out [B][N][d]
  float* zs;             // W2 out [B][d]
  float* Kout;           // WKV out [N][B][d]
  float* Vout;
};

template <int EPI>
__device__ __forceinline__ void simt_epilogue(const SimtEpi& p, int r, int c, int N, float v) {
  if constexpr (EPI == 0) {          // PLAIN
    p.c32[(size_t)r * N + c] = v;
  } else if constexpr (EPI == 1) {   // PROJ: row r = b*Nseq + n
    const int b = r / p.Nseq, n = r - b * p.Nseq;
    p.qkv[((size_t)n * p.B + b) * (size_t)(3 * p.d) + c] = v;
  } else if constexpr (EPI == 2) {   // WO
    p.u[(size_t)r * p.d + c] = p.x[((size_t)r * p.Nseq + p.j) * p.d + c] + v;
  } else if constexpr (EPI == 3) {   // W1
    p.h[(size_t)r * p.d_ff + c] = gelu_erf(v);
  } else if constexpr (EPI == 4) {   // W2
    const float z = p.u[(size_t)r * p.d + c] + v;
    p.zout[((size_t)r * p.Nseq + p.j) * p.d + c] = z;
    p.zs[(size_t)r * p.d + c] = z;
  } else if constexpr (EPI == 5) {   // WKV
    const size_t base = ((size_t)p.j * p.B + r) * p.d;
    if (c < p.d) p.Kout[base + c] = v;
    else p.Vout[base + c - p.d] = v;
  }
}

// 64 x 64 tile per CTA of 256 threads, 4 x 4 outputs per thread.
template <int EPI>
__global__ void __launch_bounds__(256) k_gemm_simt(const float* __restrict__ A, const float* __restrict__ W,
                                                   int M, int N, int K, SimtEpi p) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int row0 = blockIdx.y * 64, col0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      const int r = i >> 4, kk = i & 15;
      const int gr = row0 + r, gc = col0 + r, gk = k0 + kk;
      As[kk][r] = (gr < M && gk < K) ? A[(size_t)gr * K + gk] : 0.f;
      Ws[kk][r] = (gc < N && gk < K) ? W[(size_t)gc * K + gk] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < 16; ++kk) {
      float a[4], w[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { a[i] = As[kk][ty * 4 + i]; w[i] = Ws[kk][tx * 4 + i]; }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) acc[i][jj] = fmaf(a[i], w[jj], acc[i][jj]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int jj = 0; jj < 4; ++jj) {
      const int r = row0 + ty * 4 + i, c = col0 + tx * 4 + jj;
      if (r < M && c < N) simt_epilogue<EPI>(p, r, c, N, acc[i][jj]);
    }
}

}  // namespace rt
