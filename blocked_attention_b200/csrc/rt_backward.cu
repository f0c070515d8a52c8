// rt_backward.cu -- backward pass of the Recurrent Transformer layer: fp32
// arithmetic (SIMT), fp32 storage (the 1e-4 parity mode) or bf16 storage
// (inputs widened to fp32 working copies, gradients rounded to bf16 at the
// end).
//
// Source: "Recurrent Transformer" paper page (www.lshu.cn/news/403416):
//   paper §2.2 : the layer (queries and temporary pairs from x_t, persistent
//                pairs from z_t);
//   paper §6.1 : activation checkpointing -- with the layer's inputs x and
//                outputs z (and the persistent pairs K, V) stored, every
//                intermediate of the forward is rebuilt in parallel;
//   notes §5.3 : the backward's weight gradients batched outside the
//                per-position loop;
//   paper §6.4 : the backward pass itself (its body is missing from the
//                extracted text; the steps below are the exact derivatives of
//                the forward definition).
//
// Gradients of the scalar sum(z * dz) + sum(K * dK) + sum(V * dV):
//  1. Rebuild (all B*N positions at once): r = rms(x), q / k~ / v~, the
//     attention output a_t and its log-sum-exp per head (over the stored
//     persistent pairs of positions < t plus the temporary pair), u, rms(u),
//     the MLP pre-activation, rms(z).
//  2. Reverse loop over positions t = N..1, M = B rows per step:
//       dk_t, dv_t are complete (every later query has contributed);
//       d rms(z_t) = dk_t W_k + dv_t W_v;  dz_t += rms'(z_t) ...
//       MLP backward -> du_t;  da_t = du_t W_o;
//       attention backward: query t's temporary pair, then the forward's
//       block whose earliest query is t (its keys' dk, dv and its queries'
//       dq, added in place) -- the exact blocked schedule in reverse.
//  3. Batched over all positions: dx = du + rms'(x)(dq W_q + dk~ W_k +
//     dv~ W_v), and every weight gradient as one [out][B*N] x [B*N][in]
//     product.
// Per-position buffers are position-major (row t*B + b), like K and V.
#include <algorithm>
#include <cmath>
#include <cstring>

#include "../../include/rtlayer.h"
#include "rt_common.cuh"
#include "rt_host.h"

namespace rt {
namespace bwd {

// C[m][n] (+)= sum_k A(m, k) * W(n, k), fp32, 64 x 64 tile per CTA of 256
// threads; A(m, k) = ta ? A[k * lda + m] : A[m * lda + k], likewise W.
__global__ void __launch_bounds__(256) k_gemm(const float* __restrict__ A, int lda, int ta,
                                              const float* __restrict__ W, int ldw, int tw, float* __restrict__ C,
                                              int ldc, int M, int N, int K, int accumulate) {
  __shared__ float As[16][64 + 4];
  __shared__ float Ws[16][64 + 4];
  const int row0 = blockIdx.y * 64, col0 = blockIdx.x * 64;
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  float acc[4][4] = {};
  for (int k0 = 0; k0 < K; k0 += 16) {
    for (int i = threadIdx.x; i < 1024; i += 256) {
      // ta / tw: consecutive threads walk the non-K index (coalesced for the
      // transposed operand), else the K index
      int r, kk;
      if (ta) { kk = i >> 6; r = i & 63; } else { r = i >> 4; kk = i & 15; }
      const int gr = row0 + r, gk = k0 + kk;
      As[kk][r] = (gr < M && gk < K) ? (ta ? A[(size_t)gk * lda + gr] : A[(size_t)gr * lda + gk]) : 0.f;
      int c, kw;
      if (tw) { kw = i >> 6; c = i & 63; } else { c = i >> 4; kw = i & 15; }
      const int gc = col0 + c, gkw = k0 + kw;
      Ws[kw][c] = (gc < N && gkw < K) ? (tw ? W[(size_t)gkw * ldw + gc] : W[(size_t)gc * ldw + gkw]) : 0.f;
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
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], w[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int r = row0 + ty * 4 + i, c = col0 + tx * 4 + j;
      if (r < M && c < N) {
        float* dst = C + (size_t)r * ldc + c;
        *dst = accumulate ? *dst + acc[i][j] : acc[i][j];
      }
    }
}

// dst[i] = float(src[i]) (bf16 storage -> the fp32 working copies) and back
__global__ void k_bf16_to_f32(const __nv_bfloat16* __restrict__ src, float* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __bfloat162float(src[i]);
}
__global__ void k_f32_to_bf16(const float* __restrict__ src, __nv_bfloat16* __restrict__ dst, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    dst[i] = __float2bfloat16_rn(src[i]);
}

// dst[n][b][:] = src[b][n][:] (to = 1), or the inverse (to = 0)
__global__ void k_permute(const float* __restrict__ src, float* __restrict__ dst, int B, int N, int d, int to) {
  const size_t total = (size_t)B * N * d;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int e = (int)(i % d);
    const size_t r = i / d;
    if (to) {   // i indexes src [B][N][d]
      const int n = (int)(r % N), b = (int)(r / N);
      dst[((size_t)n * B + b) * d + e] = src[i];
    } else {    // i indexes src [N][B][d]
      const int b = (int)(r % B), n = (int)(r / B);
      dst[((size_t)b * N + n) * d + e] = src[i];
    }
  }
}

// out[r] = in[r] * c_r, c_r = 1 / sqrt(mean(in[r]^2) + eps); one warp per row
__global__ void __launch_bounds__(256) k_rms_rows(const float* __restrict__ in, float* __restrict__ out,
                                                  float* __restrict__ cinv, size_t rows, int d, float eps) {
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* v = in + r * d;
  float s = 0.f;
  for (int e = lane; e < d; e += 32) s += v[e] * v[e];
  s = warp_sum(s);
  const float c = rsqrtf(s / (float)d + eps);
  for (int e = lane; e < d; e += 32) out[r * d + e] = v[e] * c;
  if (lane == 0) cinv[r] = c;
}

// Backward of y = v * c(v), c = (mean(v^2) + eps)^(-1/2), for upstream g:
//   dv = c g - c^3 (v . g) / d * v;   out[r] = add[r] + dv  (add may be null)
__global__ void __launch_bounds__(256) k_rms_bwd(const float* __restrict__ v, const float* __restrict__ g,
                                                 const float* __restrict__ cinv, const float* __restrict__ add,
                                                 float* __restrict__ out, size_t rows, int d) {
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* vr = v + r * d;
  const float* gr = g + r * d;
  float s = 0.f;
  for (int e = lane; e < d; e += 32) s += vr[e] * gr[e];
  s = warp_sum(s);
  const float c = cinv[r];
  const float k = c * c * c * s / (float)d;
  for (int e = lane; e < d; e += 32) {
    const float dv = c * gr[e] - k * vr[e];
    out[r * d + e] = (add ? add[r * d + e] : 0.f) + dv;
  }
}

// y = GELU(h) (exact erf form) and its derivative dGELU/dh = Phi(h) + h phi(h)
__global__ void k_gelu(const float* __restrict__ h, float* __restrict__ y, size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x)
    y[i] = gelu_erf(h[i]);
}
__global__ void k_gelu_bwd(const float* __restrict__ dy, const float* __restrict__ h, float* __restrict__ dh,
                           size_t n) {
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    const float x = h[i];
    const float Phi = 0.5f * (1.f + erff(x * 0.70710678118654752f));
    const float phi = 0.39894228040143268f * expf(-0.5f * x * x);
    dh[i] = dy[i] * (Phi + x * phi);
  }
}

// Attention of every position at once over the stored persistent pairs
// (rows 0..t-1 of K, V) plus its temporary pair, natural-log units:
//   a_t = sum_i softmax(s)_i v_i,  lse_t = log sum_i exp(s_i),  s_i = <q, k_i> * scale.
// One warp per (t, b, h); lane i owns keys i, i + 32, ... (key t is the
// temporary pair) with whole-row dot products, its own online-softmax state
// and DH-wide numerator; the lanes are merged at the end.
template <int DH>
__global__ void __launch_bounds__(128) k_attn_lse(const float* __restrict__ qkv, const float* __restrict__ K,
                                                  const float* __restrict__ V, float* __restrict__ a,
                                                  float* __restrict__ lse, int B, int N, int H, float scale) {
  const long w = (long)blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= (long)N * B * H) return;
  const int h = (int)(w % H);
  const long rb = w / H;                       // position-major row t * B + b
  const int b = (int)(rb % B), t = (int)(rb / B);
  const int d = H * DH;
  const float* q = qkv + (size_t)rb * 3 * d + h * DH;
  float qr[DH], acc[DH];
#pragma unroll
  for (int e = 0; e < DH; ++e) { qr[e] = q[e]; acc[e] = 0.f; }
  float m = -INFINITY, l = 0.f;
  for (int i = lane; i <= t; i += 32) {
    const float* k = i < t ? K + ((size_t)i * B + b) * d + h * DH : q + d;
    const float* v = i < t ? V + ((size_t)i * B + b) * d + h * DH : q + 2 * d;
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) s += qr[e] * k[e];
    s *= scale;
    const float mn = fmaxf(m, s);
    const float al = m == -INFINITY ? 0.f : expf(m - mn), p = expf(s - mn);
    l = l * al + p;
#pragma unroll
    for (int e = 0; e < DH; ++e) acc[e] = acc[e] * al + p * v[e];
    m = mn;
  }
  // merge the lanes' states
  const float M = warp_max(m);
  const float f = m == -INFINITY ? 0.f : expf(m - M);
  const float L = warp_sum(l * f);
#pragma unroll
  for (int e = 0; e < DH; ++e) {
    const float v = warp_sum(acc[e] * f);
    if (lane == (e & 31)) a[(size_t)rb * d + h * DH + e] = v / L;
  }
  if (lane == 0) lse[(size_t)rb * H + h] = M + logf(L);
}

// Attention backward, exact blocked schedule (the forward's dyadic blocks in
// reverse). With p_ji = exp(s_ji - lse_j), s_ji = <q_j, k_i> * scale,
// dp_ji = <da_j, v_i>, delta_j = <da_j, a_j>, ds_ji = p_ji (dp_ji - delta_j):
//   dk_i += scale sum_j ds_ji q_j,  dv_i += sum_j p_ji da_j,  dq_j += scale sum_i ds_ji k_i.
// The pairs (key i < query j) are the forward's blocks: the block the forward
// folds at step t (keys (t - lb, t], queries (t, t + lb]) is back-propagated
// in the reverse loop right after query t + 1's gradient da is known (every
// other query of the block is later, so already done) and before key t's
// gradient is needed; each pair once, Theta(N log N) traffic like the forward.
//
// The temporary pair of query t: dk~ = scale ds~ q, dv~ = p~ da, and dq_t is
// initialised with its term (the blocks add the rest later); delta_t stored.
// One warp per (b, h); lanes over dims.
template <int DH>
__global__ void __launch_bounds__(128) k_attn_bwd_temp(const float* __restrict__ qkv, const float* __restrict__ a,
                                                       const float* __restrict__ lse, const float* __restrict__ da,
                                                       float* __restrict__ delta, float* __restrict__ dqkv, int B,
                                                       int H, int t, float scale) {
  const int w = blockIdx.x * 4 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (w >= B * H) return;
  const int b = w / H, h = w - b * H;
  const int d = H * DH;
  const size_t r = (size_t)t * B + b;
  const float* q = qkv + r * 3 * d + h * DH;
  const float* dav = da + r * d + h * DH;
  const float* av = a + r * d + h * DH;
  float s = 0.f, dp = 0.f, dl = 0.f;
  for (int e = lane; e < DH; e += 32) {
    s += q[e] * q[d + e];
    dp += dav[e] * q[2 * d + e];
    dl += dav[e] * av[e];
  }
  s = warp_sum(s);
  dp = warp_sum(dp);
  dl = warp_sum(dl);
  const float p = expf(s * scale - lse[r * H + h]);
  const float ds = p * (dp - dl);
  float* dq = dqkv + r * 3 * d + h * DH;
  for (int e = lane; e < DH; e += 32) {
    dq[e] = scale * ds * q[d + e];
    dq[d + e] = scale * ds * q[e];
    dq[2 * d + e] = p * dav[e];
  }
  if (lane == 0) delta[r * H + h] = dl;
}

// One block, key side: thread = key row i of keys [k0, k0 + nk), all of one
// (b, h) per blockIdx.x; loops over the block's queries.
template <int DH>
__global__ void __launch_bounds__(128) k_attn_bwd_block_kv(const float* __restrict__ qkv, const float* __restrict__ K,
                                                           const float* __restrict__ V,
                                                           const float* __restrict__ lse,
                                                           const float* __restrict__ delta,
                                                           const float* __restrict__ da, float* __restrict__ dK,
                                                           float* __restrict__ dV, int B, int H, int q0, int nq,
                                                           int k0, int nk, float scale) {
  const int b = blockIdx.x / H, h = blockIdx.x - b * H;
  const int i = k0 + blockIdx.y * 128 + threadIdx.x;
  if (i >= k0 + nk) return;
  const int d = H * DH;
  const size_t ri = (size_t)i * B + b;
  float k[DH], v[DH], gk[DH], gv[DH];
#pragma unroll
  for (int e = 0; e < DH; ++e) { k[e] = K[ri * d + h * DH + e]; v[e] = V[ri * d + h * DH + e]; gk[e] = gv[e] = 0.f; }
  for (int j = q0; j < q0 + nq; ++j) {
    const size_t rj = (size_t)j * B + b;
    const float* q = qkv + rj * 3 * d + h * DH;
    const float* dav = da + rj * d + h * DH;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) { s += q[e] * k[e]; dp += dav[e] * v[e]; }
    const float p = expf(s * scale - lse[rj * H + h]);
    const float ds = p * (dp - delta[rj * H + h]);
#pragma unroll
    for (int e = 0; e < DH; ++e) { gk[e] += scale * ds * q[e]; gv[e] += p * dav[e]; }
  }
#pragma unroll
  for (int e = 0; e < DH; ++e) { dK[ri * d + h * DH + e] += gk[e]; dV[ri * d + h * DH + e] += gv[e]; }
}

// One block, query side: thread = query row j of queries [q0, q0 + nq);
// adds its block term to dq_j.
template <int DH>
__global__ void __launch_bounds__(128) k_attn_bwd_block_q(const float* __restrict__ qkv, const float* __restrict__ K,
                                                          const float* __restrict__ V,
                                                          const float* __restrict__ lse,
                                                          const float* __restrict__ delta,
                                                          const float* __restrict__ da, float* __restrict__ dqkv,
                                                          int B, int H, int q0, int nq, int k0, int nk,
                                                          float scale) {
  const int b = blockIdx.x / H, h = blockIdx.x - b * H;
  const int j = q0 + blockIdx.y * 128 + threadIdx.x;
  if (j >= q0 + nq) return;
  const int d = H * DH;
  const size_t rj = (size_t)j * B + b;
  float q[DH], dav[DH], gq[DH];
#pragma unroll
  for (int e = 0; e < DH; ++e) { q[e] = qkv[rj * 3 * d + h * DH + e]; dav[e] = da[rj * d + h * DH + e]; gq[e] = 0.f; }
  const float L = lse[rj * H + h], dl = delta[rj * H + h];
  for (int i = k0; i < k0 + nk; ++i) {
    const size_t ri = (size_t)i * B + b;
    const float* k = K + ri * d + h * DH;
    const float* v = V + ri * d + h * DH;
    float s = 0.f, dp = 0.f;
#pragma unroll
    for (int e = 0; e < DH; ++e) { s += q[e] * k[e]; dp += dav[e] * v[e]; }
    const float ds = expf(s * scale - L) * (dp - dl);
#pragma unroll
    for (int e = 0; e < DH; ++e) gq[e] += scale * ds * k[e];
  }
#pragma unroll
  for (int e = 0; e < DH; ++e) dqkv[rj * 3 * d + h * DH + e] += gq[e];
}

// ---------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------
struct BwdPlan {
  size_t off_in, off_out;   // bf16 storage: fp32 copies of the 13 inputs / the 7 outputs
  size_t off_err, off_xp, off_xr, off_cx, off_qkv, off_a, off_lse, off_delta, off_u, off_ur, off_cu, off_hp, off_g, off_zp,
      off_zr, off_cz, off_dzu, off_dKa, off_dVa, off_dZ, off_dH, off_dU, off_dA, off_dqkv, off_dzr, off_dg,
      off_dur, off_dxr, off_dxp, total;
};

static size_t al(size_t x) { return (x + 255) / 256 * 256; }

// element counts of the backward's inputs (x, W_q, W_k, W_v, W_o, W_1, W_2,
// z, K, V, dz, dK, dV) and outputs (dx, dW_q, dW_k, dW_v, dW_o, dW_1, dW_2)
static void bwd_counts(int B, int N, int d, int d_ff, size_t (&in)[13], size_t (&out)[7]) {
  const size_t act = (size_t)B * N * d, dd = (size_t)d * d, df = (size_t)d * d_ff;
  const size_t i_[13] = {act, dd, dd, dd, dd, df, df, act, act, act, act, act, act};
  const size_t o_[7] = {act, dd, dd, dd, dd, df, df};
  for (int i = 0; i < 13; ++i) in[i] = i_[i];
  for (int i = 0; i < 7; ++i) out[i] = o_[i];
}

static BwdPlan bwd_plan(int B, int N, int d, int H, int d_ff, int dtype) {
  BwdPlan P;
  std::memset(&P, 0, sizeof(P));
  const size_t R = (size_t)B * N, f = 4;
  size_t off = 0;
  auto take = [&](size_t bytes) { const size_t o = off; off += al(bytes); return o; };
  if (dtype == RT_BF16) {
    size_t in[13], out[7], ni = 0, no = 0;
    bwd_counts(B, N, d, d_ff, in, out);
    for (size_t c : in) ni += al(c * f);
    for (size_t c : out) no += al(c * f);
    P.off_in = take(ni);
    P.off_out = take(no);
  }
  P.off_err = take(256);
  P.off_xp = take(R * d * f);
  P.off_xr = take(R * d * f);
  P.off_cx = take(R * f);
  P.off_qkv = take(R * 3 * d * f);
  P.off_a = take(R * d * f);
  P.off_lse = take(R * H * f);
  P.off_delta = take(R * H * f);
  P.off_u = take(R * d * f);
  P.off_ur = take(R * d * f);
  P.off_cu = take(R * f);
  P.off_hp = take(R * d_ff * f);
  P.off_g = take(R * d_ff * f);
  P.off_zp = take(R * d * f);
  P.off_zr = take(R * d * f);
  P.off_cz = take(R * f);
  P.off_dzu = take(R * d * f);
  P.off_dKa = take(R * d * f);
  P.off_dVa = take(R * d * f);
  P.off_dZ = take(R * d * f);
  P.off_dH = take(R * d_ff * f);
  P.off_dU = take(R * d * f);
  P.off_dA = take(R * d * f);
  P.off_dqkv = take(R * 3 * d * f);
  P.off_dzr = take((size_t)B * d * f);
  P.off_dg = take((size_t)B * d_ff * f);
  P.off_dur = take((size_t)B * d * f);
  P.off_dxr = take(R * d * f);
  P.off_dxp = take(R * d * f);
  P.total = off;
  return P;
}

static int bwd_validate(int B, int N, int d, int H, int d_ff, int dtype) {
  if (B <= 0 || N <= 0 || d <= 0 || H <= 0 || d_ff <= 0 || d % H != 0) return RT_ERR_INVALID_ARG;
  if (dtype != RT_F32 && dtype != RT_BF16) return RT_ERR_INVALID_ARG;
  const int dh = d / H;
  if ((dh != 32 && dh != 64 && dh != 128) || (long)B * N > (1l << 24)) return RT_ERR_UNSUPPORTED;
  return RT_OK;
}

static cudaError_t gemm(const float* A, int lda, int ta, const float* W, int ldw, int tw, float* C, int ldc, int M,
                        int N, int K, int acc, cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  k_gemm<<<grid, 256, 0, st>>>(A, lda, ta, W, ldw, tw, C, ldc, M, N, K, acc);
  return cudaGetLastError();
}

static unsigned grid_for(size_t n) { return (unsigned)std::min<size_t>((n + 255) / 256, 65535); }

// Attention backward of reverse step t (0-based position row t): the
// temporary pair of query t, then the forward's block of step t (1-based:
// keys rows [t - lb, t), queries rows [t, t + lb) clipped at N), whose
// earliest query is row t.
template <int DH>
static cudaError_t attn_bwd_dh(const float* qkv, const float* K, const float* V, const float* a, const float* lse,
                               const float* da, float* delta, float* dK, float* dV, float* dqkv, int B, int N, int H,
                               int t, float scale, cudaStream_t st) {
  k_attn_bwd_temp<DH><<<(unsigned)((B * H + 3) / 4), 128, 0, st>>>(qkv, a, lse, da, delta, dqkv, B, H, t, scale);
  if (t >= 1) {
    const int lb = lowbit(t), nq = std::min(lb, N - t), k0 = t - lb;
    k_attn_bwd_block_kv<DH><<<dim3((unsigned)(B * H), (unsigned)((lb + 127) / 128)), 128, 0, st>>>(
        qkv, K, V, lse, delta, da, dK, dV, B, H, t, nq, k0, lb, scale);
    k_attn_bwd_block_q<DH><<<dim3((unsigned)(B * H), (unsigned)((nq + 127) / 128)), 128, 0, st>>>(
        qkv, K, V, lse, delta, da, dqkv, B, H, t, nq, k0, lb, scale);
  }
  return cudaGetLastError();
}
static cudaError_t attn_bwd(int dh, const float* qkv, const float* K, const float* V, const float* a,
                            const float* lse, const float* da, float* delta, float* dK, float* dV, float* dqkv, int B,
                            int N, int H, int t, float scale, cudaStream_t st) {
  if (dh == 32) return attn_bwd_dh<32>(qkv, K, V, a, lse, da, delta, dK, dV, dqkv, B, N, H, t, scale, st);
  if (dh == 64) return attn_bwd_dh<64>(qkv, K, V, a, lse, da, delta, dK, dV, dqkv, B, N, H, t, scale, st);
  return attn_bwd_dh<128>(qkv, K, V, a, lse, da, delta, dK, dV, dqkv, B, N, H, t, scale, st);
}

}  // namespace bwd
}  // namespace rt

using namespace rt;
using namespace rt::bwd;

extern "C" size_t rt_layer_backward_workspace_bytes(int B, int N, int d, int H, int d_ff, int dtype) {
  if (bwd_validate(B, N, d, H, d_ff, dtype) != RT_OK) return 0;
  return bwd_plan(B, N, d, H, d_ff, dtype).total;
}

#define RT_BCK(call)                                    \
  do {                                                  \
    cudaError_t e_ = (call);                            \
    if (e_ != cudaSuccess) return rt::cuda_failure(e_); \
  } while (0)

extern "C" int rt_layer_backward(const void* x_, const void* Wq_, const void* Wk_, const void* Wv_, const void* Wo_,
                                 const void* W1_, const void* W2_, const void* z_, const void* K_, const void* V_,
                                 const void* dz_, const void* dK_, const void* dV_, int B, int N, int d, int H,
                                 int d_ff, int dtype, void* dx_, void* dWq_, void* dWk_, void* dWv_, void* dWo_,
                                 void* dW1_, void* dW2_, void* workspace, size_t workspace_bytes, void* stream) {
  int rc = bwd_validate(B, N, d, H, d_ff, dtype);
  if (rc != RT_OK) return rc;
  const void* in[13] = {x_, Wq_, Wk_, Wv_, Wo_, W1_, W2_, z_, K_, V_, dz_, dK_, dV_};
  void* out[7] = {dx_, dWq_, dWk_, dWv_, dWo_, dW1_, dW2_};
  for (const void* p : in)
    if (!p) return RT_ERR_INVALID_ARG;
  for (void* p : out)
    if (!p) return RT_ERR_INVALID_ARG;
  const BwdPlan P = bwd_plan(B, N, d, H, d_ff, dtype);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  int dev = 0, major = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) !=
                                                cudaSuccess || major != 10)
    return RT_ERR_DEVICE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  // bf16 storage: widen the inputs into fp32 working copies, run the fp32
  // backward on them, round the results to bf16 at the end
  void* out_dst[7] = {dx_, dWq_, dWk_, dWv_, dWo_, dW1_, dW2_};
  size_t in_n[13], out_n[7];
  bwd_counts(B, N, d, d_ff, in_n, out_n);
  if (dtype == RT_BF16) {
    size_t o = P.off_in;
    for (int i = 0; i < 13; ++i) {
      float* dst = reinterpret_cast<float*>(ws + o);
      k_bf16_to_f32<<<grid_for(in_n[i]), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(in[i]), dst, in_n[i]);
      in[i] = dst;
      o += al(in_n[i] * 4);
    }
    o = P.off_out;
    for (int i = 0; i < 7; ++i) {
      out[i] = ws + o;
      o += al(out_n[i] * 4);
    }
    RT_BCK(cudaGetLastError());
    x_ = in[0]; Wq_ = in[1]; Wk_ = in[2]; Wv_ = in[3]; Wo_ = in[4]; W1_ = in[5]; W2_ = in[6];
    z_ = in[7]; K_ = in[8]; V_ = in[9]; dz_ = in[10]; dK_ = in[11]; dV_ = in[12];
    dx_ = out[0]; dWq_ = out[1]; dWk_ = out[2]; dWv_ = out[3]; dWo_ = out[4]; dW1_ = out[5]; dW2_ = out[6];
  }
  auto F = [&](size_t off) { return reinterpret_cast<float*>(ws + off); };
  const float *x = static_cast<const float*>(x_), *z = static_cast<const float*>(z_);
  const float *Wq = static_cast<const float*>(Wq_), *Wk = static_cast<const float*>(Wk_),
              *Wv = static_cast<const float*>(Wv_), *Wo = static_cast<const float*>(Wo_),
              *W1 = static_cast<const float*>(W1_), *W2 = static_cast<const float*>(W2_);
  const float *K = static_cast<const float*>(K_), *V = static_cast<const float*>(V_);
  const float *dz = static_cast<const float*>(dz_), *dK = static_cast<const float*>(dK_),
              *dV = static_cast<const float*>(dV_);
  float *dx = static_cast<float*>(dx_), *dWq = static_cast<float*>(dWq_), *dWk = static_cast<float*>(dWk_),
        *dWv = static_cast<float*>(dWv_), *dWo = static_cast<float*>(dWo_), *dW1 = static_cast<float*>(dW1_),
        *dW2 = static_cast<float*>(dW2_);
  float *xp = F(P.off_xp), *xr = F(P.off_xr), *cx = F(P.off_cx), *qkv = F(P.off_qkv), *a = F(P.off_a),
        *lse = F(P.off_lse), *delta = F(P.off_delta), *u = F(P.off_u), *ur = F(P.off_ur), *cu = F(P.off_cu), *hp = F(P.off_hp),
        *g = F(P.off_g), *zp = F(P.off_zp), *zr = F(P.off_zr), *cz = F(P.off_cz), *dzu = F(P.off_dzu),
        *dKa = F(P.off_dKa), *dVa = F(P.off_dVa), *dZ = F(P.off_dZ), *dH = F(P.off_dH), *dU = F(P.off_dU),
        *dA = F(P.off_dA), *dqkv = F(P.off_dqkv), *dzr = F(P.off_dzr), *dg = F(P.off_dg), *dur = F(P.off_dur),
        *dxr = F(P.off_dxr), *dxp = F(P.off_dxp);
  const size_t R = (size_t)B * N;
  const int dh = d / H;
  const float scale = 1.f / std::sqrt((float)dh);
  const unsigned rows_grid = (unsigned)((R + 7) / 8);

  // 1. rebuild the forward's intermediates, all positions at once
  k_permute<<<grid_for(R * d), 256, 0, st>>>(x, xp, B, N, d, 1);
  k_permute<<<grid_for(R * d), 256, 0, st>>>(z, zp, B, N, d, 1);
  k_permute<<<grid_for(R * d), 256, 0, st>>>(dz, dzu, B, N, d, 1);
  RT_BCK(cudaGetLastError());
  k_rms_rows<<<rows_grid, 256, 0, st>>>(xp, xr, cx, R, d, kEps);
  k_rms_rows<<<rows_grid, 256, 0, st>>>(zp, zr, cz, R, d, kEps);
  RT_BCK(cudaGetLastError());
  RT_BCK(gemm(xr, d, 0, Wq, d, 0, qkv, 3 * d, (int)R, d, d, 0, st));
  RT_BCK(gemm(xr, d, 0, Wk, d, 0, qkv + d, 3 * d, (int)R, d, d, 0, st));
  RT_BCK(gemm(xr, d, 0, Wv, d, 0, qkv + 2 * d, 3 * d, (int)R, d, d, 0, st));
  {
    const unsigned g = (unsigned)((R * H + 3) / 4);
    if (dh == 32) k_attn_lse<32><<<g, 128, 0, st>>>(qkv, K, V, a, lse, B, N, H, scale);
    else if (dh == 64) k_attn_lse<64><<<g, 128, 0, st>>>(qkv, K, V, a, lse, B, N, H, scale);
    else k_attn_lse<128><<<g, 128, 0, st>>>(qkv, K, V, a, lse, B, N, H, scale);
  }
  RT_BCK(cudaGetLastError());
  RT_BCK(cudaMemcpyAsync(u, xp, R * d * 4, cudaMemcpyDeviceToDevice, st));
  RT_BCK(gemm(a, d, 0, Wo, d, 0, u, d, (int)R, d, d, 1, st));
  k_rms_rows<<<rows_grid, 256, 0, st>>>(u, ur, cu, R, d, kEps);
  RT_BCK(cudaGetLastError());
  RT_BCK(gemm(ur, d, 0, W1, d, 0, hp, d_ff, (int)R, d_ff, d, 0, st));
  k_gelu<<<grid_for(R * d_ff), 256, 0, st>>>(hp, g, R * d_ff);
  RT_BCK(cudaGetLastError());

  // 2. reverse loop over positions
  RT_BCK(cudaMemcpyAsync(dKa, dK, R * d * 4, cudaMemcpyDeviceToDevice, st));
  RT_BCK(cudaMemcpyAsync(dVa, dV, R * d * 4, cudaMemcpyDeviceToDevice, st));
  const unsigned brows = (unsigned)((B + 7) / 8);
  for (int t = N - 1; t >= 0; --t) {
    const size_t r0 = (size_t)t * B;
    // d rms(z_t) = dk_t W_k + dv_t W_v; dz_t = dz(upstream) + rms'(z_t)
    RT_BCK(gemm(dKa + r0 * d, d, 0, Wk, d, 1, dzr, d, B, d, d, 0, st));
    RT_BCK(gemm(dVa + r0 * d, d, 0, Wv, d, 1, dzr, d, B, d, d, 1, st));
    k_rms_bwd<<<brows, 256, 0, st>>>(zp + r0 * d, dzr, cz + r0, dzu + r0 * d, dZ + r0 * d, B, d);
    RT_BCK(cudaGetLastError());
    // MLP: dh = dz W_2 ; dpre = dh * GELU'(pre) ; d rms(u) = dpre W_1 ; du = dz + rms'(u)
    RT_BCK(gemm(dZ + r0 * d, d, 0, W2, d_ff, 1, dg, d_ff, B, d_ff, d, 0, st));
    k_gelu_bwd<<<grid_for((size_t)B * d_ff), 256, 0, st>>>(dg, hp + r0 * d_ff, dH + r0 * d_ff, (size_t)B * d_ff);
    RT_BCK(cudaGetLastError());
    RT_BCK(gemm(dH + r0 * d_ff, d_ff, 0, W1, d, 1, dur, d, B, d, d_ff, 0, st));
    k_rms_bwd<<<brows, 256, 0, st>>>(u + r0 * d, dur, cu + r0, dZ + r0 * d, dU + r0 * d, B, d);
    RT_BCK(cudaGetLastError());
    // da = du W_o, then the attention backward of query t
    RT_BCK(gemm(dU + r0 * d, d, 0, Wo, d, 1, dA + r0 * d, d, B, d, d, 0, st));
    RT_BCK(attn_bwd(dh, qkv, K, V, a, lse, dA, delta, dKa, dVa, dqkv, B, N, H, t, scale, st));
    RT_BCK(cudaGetLastError());
  }

  // 3. batched: dx and the weight gradients
  RT_BCK(gemm(dqkv, 3 * d, 0, Wq, d, 1, dxr, d, (int)R, d, d, 0, st));
  RT_BCK(gemm(dqkv + d, 3 * d, 0, Wk, d, 1, dxr, d, (int)R, d, d, 1, st));
  RT_BCK(gemm(dqkv + 2 * d, 3 * d, 0, Wv, d, 1, dxr, d, (int)R, d, d, 1, st));
  k_rms_bwd<<<rows_grid, 256, 0, st>>>(xp, dxr, cx, dU, dxp, R, d);
  RT_BCK(cudaGetLastError());
  k_permute<<<grid_for(R * d), 256, 0, st>>>(dxp, dx, B, N, d, 0);
  RT_BCK(cudaGetLastError());
  const int Ri = (int)R;
  RT_BCK(gemm(dqkv, 3 * d, 1, xr, d, 1, dWq, d, d, d, Ri, 0, st));
  RT_BCK(gemm(dqkv + d, 3 * d, 1, xr, d, 1, dWk, d, d, d, Ri, 0, st));
  RT_BCK(gemm(dKa, d, 1, zr, d, 1, dWk, d, d, d, Ri, 1, st));
  RT_BCK(gemm(dqkv + 2 * d, 3 * d, 1, xr, d, 1, dWv, d, d, d, Ri, 0, st));
  RT_BCK(gemm(dVa, d, 1, zr, d, 1, dWv, d, d, d, Ri, 1, st));
  RT_BCK(gemm(dU, d, 1, a, d, 1, dWo, d, d, d, Ri, 0, st));
  RT_BCK(gemm(dH, d_ff, 1, ur, d, 1, dW1, d, d_ff, d, Ri, 0, st));
  RT_BCK(gemm(dZ, d, 1, g, d_ff, 1, dW2, d_ff, d, d_ff, Ri, 0, st));
  if (dtype == RT_BF16) {
    for (int i = 0; i < 7; ++i)
      k_f32_to_bf16<<<grid_for(out_n[i]), 256, 0, st>>>(static_cast<const float*>(out[i]),
                                                       static_cast<__nv_bfloat16*>(out_dst[i]), out_n[i]);
    RT_BCK(cudaGetLastError());
  }
  return RT_OK;
}
