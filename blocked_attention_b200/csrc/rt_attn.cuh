// rt_attn.cuh -- attention side of the Recurrent Transformer layer.
//
// Source: "Recurrent Transformer" paper page (www.lshu.cn/news/403416):
//   notes §2.2 / paper §2.2 : the temporary pair (from x_t) is used only by
//                             position t's own attention;
//   notes §4.2 / paper §5   : exact blocked schedule with online-softmax
//                             statistics (running max m, normaliser l,
//                             numerator o);
//   notes §4.1              : the naive schedule (query t reads all revealed
//                             pairs at step t), kept as the ablation;
//   paper §6.3              : position-major KV cache.
//
// Storage (position-major; row (j, b) = position j of sequence b):
//   QKV [N][B][3d]  : q | k~ | v~ of every position (from the projection)
//   K, V [N][B][d]  : persistent pairs
//   m, l [N][B][H]  : fp32 statistics; m is kept in log2 units of the scaled
//                     score, s2 = <q, k> * log2(e) / sqrt(d_h)
//   o [N][B][d]     : fp32 numerators
// Head h occupies columns h*d_h .. h*d_h + d_h - 1 of every row.
#pragma once

#include "rt_common.cuh"
#include "rt_rownorm.cuh"

namespace rt {

template <class T, int DPL>
__device__ __forceinline__ void load_lane(const T* src, float (&v)[DPL]) {
#pragma unroll
  for (int i = 0; i < DPL; ++i) v[i] = to_f(src[i]);
}

// ---------------------------------------------------------------------------
// finalise position j: merge the temporary pair into the accumulator of
// query j, then a_j = o / l per head. One warp per (b, h).
// has_acc = false: the accumulator of j was never folded into (position 1).
// ---------------------------------------------------------------------------
template <class T, int DPL>
__global__ void __launch_bounds__(128)
    k_finalize(const T* __restrict__ qkv, const float* __restrict__ m, const float* __restrict__ l,
               const float* __restrict__ o, T* __restrict__ a_out, int B, int H, int j, float sc2,
               int has_acc) {
  constexpr int DH = DPL * 32;
  pdl_launch_dependents();
  pdl_wait();
  const int pair = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pair >= B * H) return;
  const int b = pair / H, h = pair - b * H;
  const int d = H * DH;
  const size_t row = (size_t)j * B + b;
  const T* qp = qkv + row * (size_t)(3 * d) + h * DH + lane * DPL;
  float q[DPL], kt[DPL], vt[DPL];
  load_lane<T, DPL>(qp, q);
  load_lane<T, DPL>(qp + d, kt);
  load_lane<T, DPL>(qp + 2 * d, vt);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) dot += q[i] * kt[i];
  const float s = warp_sum(dot) * sc2;
  float mo = -INFINITY, lo = 0.f, oo[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) oo[i] = 0.f;
  if (has_acc) {
    mo = m[row * H + h];
    lo = l[row * H + h];
    const float* op = o + row * (size_t)d + h * DH + lane * DPL;
#pragma unroll
    for (int i = 0; i < DPL; ++i) oo[i] = op[i];
  }
  const float mn = fmaxf(mo, s);
  const float al = rescale(mo, mn), pt = exp2f(s - mn);
  const float ln = lo * al + pt;
  const float inv = 1.f / ln;
  T* ap = a_out + (size_t)b * d + h * DH + lane * DPL;
#pragma unroll
  for (int i = 0; i < DPL; ++i) ap[i] = from_f<T>((oo[i] * al + pt * vt[i]) * inv);
}

// ---------------------------------------------------------------------------
// naive schedule (ablation; also the decode step's attention): a_j from all
// persistent pairs i < j plus the temporary pair of the query at row qpos of
// qkv. One CTA of 8 warps per (b, h): warp w scores keys
// w*32 + lane, w*32 + 256 + lane, ... (one key per lane, 16-byte loads), keeps
// its own online-softmax state, and the 8 partial states are merged in shared
// memory at the end.
// ---------------------------------------------------------------------------
template <class T, int DPL>
__global__ void __launch_bounds__(256)
    k_naive_attn(const T* __restrict__ qkv, const T* __restrict__ K, const T* __restrict__ V,
                 T* __restrict__ a_out, int B, int H, int j, int qpos, float sc2) {
  constexpr int DH = DPL * 32, NW = 8;
  __shared__ float sq[DH];
  __shared__ float sm[NW], sl[NW], so[NW][DH];
  pdl_launch_dependents();
  pdl_wait();
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int b = pair / H, h = pair - b * H;
  const int d = H * DH;
  const size_t row = (size_t)qpos * B + b;   // the query's row of qkv (the layer: qpos = j)
  const T* qp = qkv + row * (size_t)(3 * d) + h * DH;
  if (threadIdx.x < DH) sq[threadIdx.x] = to_f(qp[threadIdx.x]);
  __syncthreads();
  float mo = -INFINITY, lo = 0.f, oo[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) oo[i] = 0.f;
  for (int c0 = w * 32; c0 < j; c0 += NW * 32) {
    const int n = min(32, j - c0);
    float s = -INFINITY;
    if (lane < n) {
      const T* kp = K + ((size_t)(c0 + lane) * B + b) * d + h * DH;
      float acc = 0.f;
      if constexpr (sizeof(T) == 2 && DH % 8 == 0) {
#pragma unroll
        for (int e0 = 0; e0 < DH; e0 += 8) {
          const uint4 wv = *reinterpret_cast<const uint4*>(kp + e0);
          const __nv_bfloat162* p2 = reinterpret_cast<const __nv_bfloat162*>(&wv);
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const float2 f = __bfloat1622float2(p2[k]);
            acc += sq[e0 + 2 * k] * f.x + sq[e0 + 2 * k + 1] * f.y;
          }
        }
      } else {
#pragma unroll 8
        for (int e = 0; e < DH; ++e) acc += sq[e] * to_f(kp[e]);
      }
      s = acc * sc2;
    }
    const float mn = fmaxf(mo, warp_max(s));
    const float al = rescale(mo, mn);
    const float pl = (lane < n) ? exp2f(s - mn) : 0.f;
    lo = lo * al + warp_sum(pl);
#pragma unroll
    for (int i = 0; i < DPL; ++i) oo[i] *= al;
#pragma unroll 8
    for (int i = 0; i < n; ++i) {
      const float pi = __shfl_sync(0xffffffffu, pl, i);
      const T* vp = V + ((size_t)(c0 + i) * B + b) * d + h * DH + lane * DPL;
#pragma unroll
      for (int e = 0; e < DPL; ++e) oo[e] += pi * to_f(vp[e]);
    }
    mo = mn;
  }
  if (lane == 0) { sm[w] = mo; sl[w] = lo; }
#pragma unroll
  for (int i = 0; i < DPL; ++i) so[w][lane * DPL + i] = oo[i];
  __syncthreads();
  if (w != 0) return;
  // merge the warps' partial states, then the temporary pair
  float mt = -INFINITY;
  for (int k = 0; k < NW; ++k) mt = fmaxf(mt, sm[k]);
  float lt = 0.f, ot[DPL];
#pragma unroll
  for (int i = 0; i < DPL; ++i) ot[i] = 0.f;
  for (int k = 0; k < NW; ++k) {
    const float f = rescale(sm[k], mt);
    lt += sl[k] * f;
#pragma unroll
    for (int i = 0; i < DPL; ++i) ot[i] += so[k][lane * DPL + i] * f;
  }
  float kt[DPL], vt[DPL];
  load_lane<T, DPL>(qp + d + lane * DPL, kt);
  load_lane<T, DPL>(qp + 2 * d + lane * DPL, vt);
  float dot = 0.f;
#pragma unroll
  for (int i = 0; i < DPL; ++i) dot += sq[lane * DPL + i] * kt[i];
  const float s = warp_sum(dot) * sc2;
  const float mn = fmaxf(mt, s);
  const float al = rescale(mt, mn), pt = exp2f(s - mn);
  const float inv = 1.f / (lt * al + pt);
  T* ap = a_out + (size_t)b * d + h * DH + lane * DPL;
#pragma unroll
  for (int i = 0; i < DPL; ++i) ap[i] = from_f<T>((ot[i] * al + pt * vt[i]) * inv);
}

// ---------------------------------------------------------------------------
// block fold, warp kernel: one warp per (b, h) folds keys [k0, k0+nk) into
// queries [q0, q0+nq). Used for every block in fp32 and, through
// rt_block_fold, for bf16 blocks whose key count none of the other kernels
// takes (neither <= 8 nor a multiple of 16). init = 1: the queries'
// accumulators are empty (first fold into them), so they are written without
// being read.
// ---------------------------------------------------------------------------
template <class T, int DPL>
__global__ void __launch_bounds__(128)
    k_fold_warp(const T* __restrict__ Q, int q_stride, const T* __restrict__ K,
                const T* __restrict__ V, int kv_stride, float* __restrict__ m,
                float* __restrict__ l, float* __restrict__ o, int B, int H, int q0, int nq,
                int k0, int nk, float sc2, int init) {
  constexpr int DH = DPL * 32, KC = 8;
  pdl_launch_dependents();
  pdl_wait();
  const int pair = blockIdx.x * 4 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (pair >= B * H) return;
  const int b = pair / H, h = pair - b * H;
  const int d = H * DH;
  for (int jq = q0; jq < q0 + nq; ++jq) {
    const size_t row = (size_t)jq * B + b;
    float q[DPL];
    load_lane<T, DPL>(Q + row * (size_t)q_stride + h * DH + lane * DPL, q);
    float mo = -INFINITY, lo = 0.f, oo[DPL];
    float* op = o + row * (size_t)d + h * DH + lane * DPL;
    if (init) {
#pragma unroll
      for (int i = 0; i < DPL; ++i) oo[i] = 0.f;
    } else {
      mo = m[row * H + h];
      lo = l[row * H + h];
#pragma unroll
      for (int i = 0; i < DPL; ++i) oo[i] = op[i];
    }
    for (int c0 = 0; c0 < nk; c0 += KC) {
      const int n = min(KC, nk - c0);
      float s[KC];
      float cm = -INFINITY;
#pragma unroll
      for (int i = 0; i < KC; ++i) {
        s[i] = -INFINITY;
        if (i < n) {
          float kk[DPL];
          load_lane<T, DPL>(K + ((size_t)(k0 + c0 + i) * B + b) * kv_stride + h * DH + lane * DPL, kk);
          float dot = 0.f;
#pragma unroll
          for (int e = 0; e < DPL; ++e) dot += q[e] * kk[e];
          s[i] = warp_sum(dot) * sc2;
          cm = fmaxf(cm, s[i]);
        }
      }
      const float mn = fmaxf(mo, cm);
      const float al = rescale(mo, mn);
      lo *= al;
#pragma unroll
      for (int e = 0; e < DPL; ++e) oo[e] *= al;
#pragma unroll
      for (int i = 0; i < KC; ++i) {
        if (i < n) {
          const float p = exp2f(s[i] - mn);
          float vv[DPL];
          load_lane<T, DPL>(V + ((size_t)(k0 + c0 + i) * B + b) * kv_stride + h * DH + lane * DPL, vv);
          lo += p;
#pragma unroll
          for (int e = 0; e < DPL; ++e) oo[e] += p * vv[e];
        }
      }
      mo = mn;
    }
    if (lane == 0) {
      m[row * H + h] = mo;
      l[row * H + h] = lo;
    }
#pragma unroll
    for (int i = 0; i < DPL; ++i) op[i] = oo[i];
  }
}

// ---------------------------------------------------------------------------
// block fold for small blocks (at most 8 keys), bf16, d_h = 64: eight lanes
// per (b, h, query), eight dims (16 bytes of q/k/v, 32 bytes of o) per lane.
// fin = 1: the first query of the block (q0) receives no later fold, so it
// is finalised here -- its temporary pair is merged and a_{q0} = o / l is
// written to a_out [B][d]; its (m, l, o) are not stored.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void load_bf16x8(const __nv_bfloat16* src, float (&v)[8]) {
  const uint4 w = *reinterpret_cast<const uint4*>(src);
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(p[k]);
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}


// Work split: a CTA of 128 threads holds 16 octets. With S = min(16, the
// power of two >= max(nq, nk)) query slots per (b, h) pair, a CTA serves
// 16 / S pairs (S < 16) or 16 queries of one pair (nq > 16: the pair's
// queries cut into ceil(nq / 16) CTAs). For nk >= 2 the CTA's keys -- at
// most 16 (pair, key) rows of k and of v -- are staged once in shared memory
// by cp.async, so every query of a pair reads them from there; a single key
// (nk = 1, half of all steps) has no reuse and is loaded by each octet
// directly. All index arithmetic precedes the wait for the predecessor
// kernel, and every global load of a thread is issued before the first use
// (one round of memory latency). NK > 0 fixes nk = NK and S = NK at compile
// time (the layer's blocks, nq <= nk); NK = 0 takes them at run time.
__host__ __device__ __forceinline__ int fold_small_slots(int nq, int nk) {
  int s = 1;
  while (s < nq || s < nk) s <<= 1;
  return s < 16 ? s : 16;
}

template <int NK>
__global__ void __launch_bounds__(128)
    k_fold_small(const __nv_bfloat16* __restrict__ qkv, int q_stride, const __nv_bfloat16* __restrict__ K,
                 const __nv_bfloat16* __restrict__ V, int kv_stride, float* __restrict__ m, float* __restrict__ l,
                 float* __restrict__ o, __nv_bfloat16* __restrict__ a_out, int B, int H, int q0, int nq,
                 int k0, int nk_rt, float sc2, int init, int fin) {
  constexpr int DH = 64, KMAX = 8;
  constexpr bool STAGED = NK != 1;
  __shared__ __align__(16) uint4 skv[STAGED ? 2 : 1][STAGED ? 16 * 8 : 1];   // [k | v][(pair_local * n + key) * 8 + part]
  const int n = NK > 0 ? NK : min(nk_rt, KMAX);      // callers use this kernel for nk <= 8
  const int pairs = B * H;
  const int S = NK > 0 ? NK : fold_small_slots(nq, n);
  const int chunks = NK > 0 ? 1 : (nq + S - 1) / S;  // > 1 only when S = 16
  const int P = 16 / S;                              // pairs per CTA (1 when chunks > 1)
  const int pair0 = (chunks == 1 ? (int)blockIdx.x : (int)blockIdx.x / chunks) * P;
  const int qbase = chunks == 1 ? 0 : ((int)blockIdx.x % chunks) * S;
  const int d = H * DH;
  // ---- this octet's query ----
  const int oct = threadIdx.x >> 3, sl = threadIdx.x & 7;
  const unsigned omask = 0xFFu << ((threadIdx.x & 31) & 24);
  const int pl = oct / S, qi = qbase + (oct - pl * S);
  const int pair = pair0 + pl;
  const bool active = pair < pairs && qi < nq;
  const int b = active ? pair / H : 0, h = active ? pair - b * H : 0;
  const size_t row = (size_t)(q0 + (active ? qi : 0)) * B + b;
  const __nv_bfloat16* qp = qkv + row * (size_t)q_stride + h * DH + sl * 8;
  const bool finrow = active && fin && qi == 0;
  float* op = o + row * (size_t)d + h * DH + sl * 8;
  const size_t kv0 = ((size_t)k0 * B + b) * kv_stride + h * DH + sl * 8;   // key k0 of this pair (nk = 1 path)

  pdl_launch_dependents();
  pdl_wait();

  if (STAGED) {
    // ---- stage the keys of the CTA's pairs ----
    const int E = P * n;                             // (pair, key) rows, <= 16
    for (int u = threadIdx.x; u < 2 * E * 8; u += blockDim.x) {
      const int kv = u >= E * 8 ? 1 : 0, r = u - kv * (E * 8);
      const int e = r >> 3, part = r & 7;
      const int pe = e / n, i = e - pe * n;
      const int pr = pair0 + pe;
      if (pr < pairs) {
        const int bb = pr / H, hh = pr - bb * H;
        const __nv_bfloat16* src = (kv ? V : K) + ((size_t)(k0 + i) * B + bb) * kv_stride + hh * DH + part * 8;
        asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(&skv[kv][e * 8 + part])), "l"(src)
                     : "memory");
      }
    }
    asm volatile("cp.async.commit_group;" ::: "memory");
  }
  uint4 qw = make_uint4(0, 0, 0, 0), ktw = qw, vtw = qw, k1w = qw, v1w = qw;
  float mo = -INFINITY, lo = 0.f;
  float4 o0 = make_float4(0.f, 0.f, 0.f, 0.f), o1 = o0;
  if (active) {
    qw = *reinterpret_cast<const uint4*>(qp);
    if (!STAGED) {
      k1w = *reinterpret_cast<const uint4*>(K + kv0);
      v1w = *reinterpret_cast<const uint4*>(V + kv0);
    }
    if (finrow) {
      ktw = *reinterpret_cast<const uint4*>(qp + d);
      vtw = *reinterpret_cast<const uint4*>(qp + 2 * d);
    }
    if (!init) {
      mo = m[row * H + h];
      lo = l[row * H + h];
      o0 = reinterpret_cast<const float4*>(op)[0];
      o1 = reinterpret_cast<const float4*>(op)[1];
    }
  }
  if (STAGED) {
    asm volatile("cp.async.wait_all;" ::: "memory");
    __syncthreads();
  }
  if (!active) return;   // whole octets leave together; no barrier follows

  float oo[8] = {o0.x, o0.y, o0.z, o0.w, o1.x, o1.y, o1.z, o1.w};
  float q[8];
  unpack_bf16x8(qw, q);
  const uint4* sk = &skv[0][STAGED ? (pl * n) * 8 + sl : 0];
  const uint4* sv = &skv[STAGED ? 1 : 0][STAGED ? (pl * n) * 8 + sl : 0];
  // ---- scores ----
  float s[KMAX];
  float mx = -INFINITY;
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    s[i] = -INFINITY;
    if (i < n) {
      float kk[8];
      unpack_bf16x8(STAGED ? sk[i * 8] : k1w, kk);
      float dot = 0.f;
#pragma unroll
      for (int e = 0; e < 8; ++e) dot += q[e] * kk[e];
      dot += __shfl_xor_sync(omask, dot, 1);
      dot += __shfl_xor_sync(omask, dot, 2);
      dot += __shfl_xor_sync(omask, dot, 4);
      s[i] = dot * sc2;
      mx = fmaxf(mx, s[i]);
    }
  }
  float st = -INFINITY;
  if (finrow) {
    float kt[8];
    unpack_bf16x8(ktw, kt);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dot += q[e] * kt[e];
    dot += __shfl_xor_sync(omask, dot, 1);
    dot += __shfl_xor_sync(omask, dot, 2);
    dot += __shfl_xor_sync(omask, dot, 4);
    st = dot * sc2;
  }
  // ---- online-softmax merge (block keys, then the temporary pair if finalising) ----
  const float mn = fmaxf(mo, mx);
  const float al = rescale(mo, mn);
  lo *= al;
#pragma unroll
  for (int e = 0; e < 8; ++e) oo[e] *= al;
#pragma unroll
  for (int i = 0; i < KMAX; ++i) {
    if (i < n) {
      const float p = ex2_ftz(s[i] - mn);
      float vv[8];
      unpack_bf16x8(STAGED ? sv[i * 8] : v1w, vv);
      lo += p;
#pragma unroll
      for (int e = 0; e < 8; ++e) oo[e] += p * vv[e];
    }
  }
  if (finrow) {
    const float m2 = fmaxf(mn, st);
    const float a2 = rescale(mn, m2), pt = exp2f(st - m2);
    const float inv = 1.f / (lo * a2 + pt);
    float vt[8];
    unpack_bf16x8(vtw, vt);
    uint4 w;
    uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      __nv_bfloat162 v2 = __floats2bfloat162_rn((oo[2 * k] * a2 + pt * vt[2 * k]) * inv,
                                                (oo[2 * k + 1] * a2 + pt * vt[2 * k + 1]) * inv);
      wp[k] = *reinterpret_cast<uint32_t*>(&v2);
    }
    *reinterpret_cast<uint4*>(a_out + (size_t)b * d + h * DH + sl * 8) = w;
  } else {
    if (sl == 0) {
      m[row * H + h] = mn;
      l[row * H + h] = lo;
    }
    reinterpret_cast<float4*>(op)[0] = make_float4(oo[0], oo[1], oo[2], oo[3]);
    reinterpret_cast<float4*>(op)[1] = make_float4(oo[4], oo[5], oo[6], oo[7]);
  }
}

// ---------------------------------------------------------------------------
// block-wise (chunked) recurrence, bf16, d_h = 64: the attention of the nc
// positions p0 .. p0 + nc - 1 of one chunk. Query t of sequence b, head h
// has folded into its (m, l, o) every persistent pair of the earlier chunks
// (has_acc = 0 for the first chunk: none); it now attends causally to the
// temporary pairs of the chunk's positions p0 .. t, merged one by one into
// the same online-softmax statistics, and writes a_t = o / l to row
// (t - p0) * B + b of a_out [nc * B][d]. An octet of lanes (8 dims each) per
// (position, sequence, head); 16 octets per CTA.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    k_chunk_attend(const __nv_bfloat16* __restrict__ qkv, const float* __restrict__ m,
                   const float* __restrict__ l, const float* __restrict__ o, __nv_bfloat16* __restrict__ a_out,
                   int B, int H, int p0, int nc, float sc2, int has_acc, unsigned* err) {
  pdl_launch_dependents();
  pdl_wait();
  const int oct = threadIdx.x >> 3, sl = threadIdx.x & 7;
  const unsigned omask = 0xFFu << ((threadIdx.x & 31) & 24);
  const long unit = (long)blockIdx.x * 16 + oct;           // ((t - p0) * B + b) * H + h
  if (unit >= (long)nc * B * H) return;                     // whole octets together
  const int h = (int)(unit % H);
  const long rb = unit / H;                                 // chunk row (t - p0) * B + b
  const int b = (int)(rb % B), i = (int)(rb / B);
  const int d = H * 64;
  const int t = p0 + i;
  if (!idx_ok(i < nc && b < B, err)) return;
  const size_t row = (size_t)t * B + b;
  float q[8];
  load_bf16x8(qkv + row * (size_t)(3 * d) + h * 64 + sl * 8, q);
  float mo = -INFINITY, lo = 0.f, oo[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
  if (has_acc) {
    mo = m[row * H + h];
    lo = l[row * H + h];
    const float4* op = reinterpret_cast<const float4*>(o + row * (size_t)d + h * 64 + sl * 8);
    const float4 a0 = op[0], a1 = op[1];
    oo[0] = a0.x; oo[1] = a0.y; oo[2] = a0.z; oo[3] = a0.w; oo[4] = a1.x; oo[5] = a1.y; oo[6] = a1.z; oo[7] = a1.w;
  }
  for (int s = p0; s <= t; ++s) {
    const __nv_bfloat16* tp = qkv + ((size_t)s * B + b) * (size_t)(3 * d) + h * 64 + sl * 8;
    float kt[8], vt[8];
    load_bf16x8(tp + d, kt);
    load_bf16x8(tp + 2 * d, vt);
    float dot = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) dot += q[e] * kt[e];
    dot += __shfl_xor_sync(omask, dot, 1);
    dot += __shfl_xor_sync(omask, dot, 2);
    dot += __shfl_xor_sync(omask, dot, 4);
    const float sc = dot * sc2;
    const float mn = fmaxf(mo, sc);
    const float al = rescale(mo, mn), p = exp2f(sc - mn);
    lo = lo * al + p;
#pragma unroll
    for (int e = 0; e < 8; ++e) oo[e] = oo[e] * al + p * vt[e];
    mo = mn;
  }
  const float inv = 1.f / lo;
  uint4 w;
  uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    __nv_bfloat162 v2 = __floats2bfloat162_rn(oo[2 * k] * inv, oo[2 * k + 1] * inv);
    wp[k] = *reinterpret_cast<uint32_t*>(&v2);
  }
  *reinterpret_cast<uint4*>(a_out + (size_t)rb * d + h * 64 + sl * 8) = w;
}

// ---------------------------------------------------------------------------
// decode-step attention (bf16, d_h = 64): the query at row 0 of a
// one-position qkv [B][3d] against cached keys 0..j-1 (position-major K, V
// [.][B][d]) plus its temporary pair. One CTA of 4 warps per (b, h); each
// lane owns whole keys (c = thread, thread + 128, ...): it loads the key's k
// and v rows (2 x 128 bytes, sixteen 16-byte loads in flight), and keeps its
// own online-softmax state (m, l) and 64-wide numerator. Lanes, then warps,
// are merged at the end; warp 0 adds the temporary pair and writes a [B][d].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(128)
    k_decode_attn(const __nv_bfloat16* __restrict__ qkv, const __nv_bfloat16* __restrict__ K,
                  const __nv_bfloat16* __restrict__ V, __nv_bfloat16* __restrict__ a_out, int B, int H, int j,
                  float sc2) {
  constexpr int DH = 64, NW = 4;
  __shared__ __align__(16) float sq[DH];
  __shared__ float sm[NW], sl[NW];
  __shared__ __align__(16) float so[NW][DH];
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int pair = blockIdx.x;
  const int b = pair / H, h = pair - b * H;
  const int d = H * DH;
  const __nv_bfloat16* qp = qkv + (size_t)b * (3 * d) + h * DH;
  pdl_launch_dependents();
  pdl_wait();
  if (threadIdx.x < DH) sq[threadIdx.x] = __bfloat162float(qp[threadIdx.x]);
  __syncthreads();
  float m = -INFINITY, l = 0.f, oacc[DH];
#pragma unroll
  for (int i = 0; i < DH; ++i) oacc[i] = 0.f;
  const float4* sq4 = reinterpret_cast<const float4*>(sq);
  for (int c = threadIdx.x; c < j; c += blockDim.x) {
    const size_t off = ((size_t)c * B + b) * d + h * DH;
    const uint4* kp = reinterpret_cast<const uint4*>(K + off);
    const uint4* vp = reinterpret_cast<const uint4*>(V + off);
    uint4 kw[8], vw[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) kw[e] = kp[e];
#pragma unroll
    for (int e = 0; e < 8; ++e) vw[e] = vp[e];
    float s = 0.f;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float kk[8];
      unpack_bf16x8(kw[e], kk);
      const float4 q0 = sq4[2 * e], q1 = sq4[2 * e + 1];
      s += q0.x * kk[0] + q0.y * kk[1] + q0.z * kk[2] + q0.w * kk[3] + q1.x * kk[4] + q1.y * kk[5] +
           q1.z * kk[6] + q1.w * kk[7];
    }
    s *= sc2;
    if (s > m) {   // new running maximum of this lane: rescale its state
      const float al = rescale(m, s);
      l *= al;
#pragma unroll
      for (int i = 0; i < DH; ++i) oacc[i] *= al;
      m = s;
    }
    const float p = exp2f(s - m);
    l += p;
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      float vv[8];
      unpack_bf16x8(vw[e], vv);
#pragma unroll
      for (int i = 0; i < 8; ++i) oacc[e * 8 + i] += p * vv[i];
    }
  }
  // merge the warp's lanes (a lane without keys has m = -inf and weight 0)
  const float mw = warp_max(m);
  const float f = rescale(m, mw);
  l = warp_sum(l * f);
#pragma unroll
  for (int i = 0; i < DH; ++i) oacc[i] = warp_sum(oacc[i] * f);
  if (lane == 0) {
    sm[w] = mw;
    sl[w] = l;
#pragma unroll
    for (int i = 0; i < DH; ++i) so[w][i] = oacc[i];
  }
  __syncthreads();
  if (w != 0) return;
  // warp 0: merge the warps' states, then the temporary pair; lane owns dims 2*lane, 2*lane + 1
  float mt = -INFINITY;
#pragma unroll
  for (int k = 0; k < NW; ++k) mt = fmaxf(mt, sm[k]);
  float lt = 0.f, ot0 = 0.f, ot1 = 0.f;
#pragma unroll
  for (int k = 0; k < NW; ++k) {
    const float fk = rescale(sm[k], mt);
    lt += sl[k] * fk;
    ot0 += so[k][2 * lane] * fk;
    ot1 += so[k][2 * lane + 1] * fk;
  }
  const float2 kt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qp + d + 2 * lane));
  const float2 vt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(qp + 2 * d + 2 * lane));
  const float st = warp_sum(sq[2 * lane] * kt.x + sq[2 * lane + 1] * kt.y) * sc2;
  const float mn = fmaxf(mt, st);
  const float al = rescale(mt, mn), pt = exp2f(st - mn);
  const float inv = 1.f / (lt * al + pt);
  *reinterpret_cast<__nv_bfloat162*>(a_out + (size_t)b * d + h * DH + 2 * lane) =
      __floats2bfloat162_rn((ot0 * al + pt * vt.x) * inv, (ot1 * al + pt * vt.y) * inv);
}

// ---------------------------------------------------------------------------
// block fold, tensor-core kernel (bf16, d_h = 64, nk a multiple of 16):
// S = Q K^T and O += P V with mma.sync m16n8k16 (fp32 accumulate), online
// softmax over key chunks of 64, then one merge into the fp32 (m, l, o) of
// each query. CTA = 4 warps = 64 queries of one (b, h); K/V chunks are
// double-buffered in shared memory by cp.async.
// ---------------------------------------------------------------------------
namespace mma_detail {
constexpr int LDS = 72;  // padded smem row (bf16): 144 bytes, conflict-free ldmatrix

__device__ __forceinline__ void cp_async16(void* dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(dst)), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ void ldsm_x4(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t (&r)[4], const void* p) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(smem_u32(p)));
}
__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}
__device__ __forceinline__ uint32_t pack2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}
}  // namespace mma_detail

// P (b, h) pairs per CTA: P = 1 for blocks >= 64 keys (64 queries of one pair,
// keys in 64-key chunks); P = 2 / 4 for 32- / 16-key blocks (64/P queries and
// the 64/P keys of each pair share one 64-row tile), so no warp idles.
// NB = K/V chunk buffers: 2 (double-buffered chunks) for blocks of more than
// one chunk, 1 for blocks of one chunk (16 keys at P = 4, 32 at P = 2), whose
// smaller footprint (and register bound) lets 5 CTAs share an SM instead of 4.
template <int P, int NB = 2>
__global__ void __launch_bounds__(128, NB == 1 ? 5 : 4)
    k_fold_mma(const __nv_bfloat16* __restrict__ Q, int q_stride, const __nv_bfloat16* __restrict__ K,
               const __nv_bfloat16* __restrict__ V, int kv_stride, float* __restrict__ m,
               float* __restrict__ l, float* __restrict__ o, __nv_bfloat16* __restrict__ a_out, int B, int H,
               int q0, int nq, int k0, int nk, float sc2, int init, int fin, unsigned* err) {
  using namespace mma_detail;
  constexpr int DH = 64, QT = 64, KC = 64, QTP = QT / P, KCP = KC / P;
  __shared__ __align__(128) __nv_bfloat16 sQ[QT * LDS];
  __shared__ __align__(128) __nv_bfloat16 sK[NB][KC * LDS];
  __shared__ __align__(128) __nv_bfloat16 sV[NB][KC * LDS];
  pdl_launch_dependents();
  pdl_wait();
  if (NB == 1 && nk > KCP) {             // one buffer holds one chunk only
    if (threadIdx.x == 0) set_error(err, RT_DEVERR_INDEX);
    return;
  }

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int npairs = B * H;
  const int d = H * DH;
  const int qt0 = q0 + blockIdx.x * QTP;                 // first query of every pair in this CTA
  const int nrows = min(QTP, q0 + nq - qt0);             // valid query rows per pair
  // pair of tile row r (query rows and key rows alike)
  auto pair_of = [&](int r) { return (int)blockIdx.y * P + r / QTP; };

  // Q tile (rows beyond nrows, or of a missing pair, are zero)
  for (int c = tid; c < QT * 8; c += 128) {
    const int r = c >> 3, cc = c & 7;
    const int pr = pair_of(r), qr = r % QTP;
    __nv_bfloat16* dst = &sQ[r * LDS + cc * 8];
    if (qr < nrows && pr < npairs) {
      const int b = pr / H, h = pr - b * H;
      cp_async16(dst, Q + ((size_t)(qt0 + qr) * B + b) * q_stride + h * DH + cc * 8);
    } else {
      *reinterpret_cast<uint4*>(dst) = make_uint4(0, 0, 0, 0);
    }
  }
  // keys [kc0, kc0 + kcn) of every pair; pair p occupies rows p*KCP .. p*KCP + KCP - 1
  auto load_kv = [&](int buf, int kc0, int kcn) {
    for (int c = tid; c < KC * 8; c += 128) {
      const int r = c >> 3, cc = c & 7;
      const int pr = (int)blockIdx.y * P + r / KCP, kr = r % KCP;
      if (kr < kcn && pr < npairs) {
        const int b = pr / H, h = pr - b * H;
        const size_t src = ((size_t)(k0 + kc0 + kr) * B + b) * kv_stride + h * DH + cc * 8;
        cp_async16(&sK[buf][r * LDS + cc * 8], K + src);
        cp_async16(&sV[buf][r * LDS + cc * 8], V + src);
      }
    }
  };
  load_kv(0, 0, min(KCP, nk));
  cp_async_commit();

  const int wpair = pair_of(warp * 16);                  // this warp's pair
  const int wq0 = (warp * 16) % QTP;                     // its first query row within the pair
  const int kbase = (warp * 16 / QTP) * KCP;             // its pair's first key row in sK / sV
  const int b = wpair / H, h = wpair - (wpair / H) * H;
  const int nchunks = (nk + KCP - 1) / KCP;
  const bool warp_active = wq0 < nrows && wpair < npairs;
  float mrow[2] = {-INFINITY, -INFINITY}, lrow[2] = {0.f, 0.f};
  float oacc[8][4];
#pragma unroll
  for (int i = 0; i < 8; ++i) oacc[i][0] = oacc[i][1] = oacc[i][2] = oacc[i][3] = 0.f;
  uint32_t qf[4][4];

  for (int ci = 0; ci < nchunks; ++ci) {
    const int buf = NB == 2 ? (ci & 1) : 0;
    if (ci + 1 < nchunks) {
      load_kv(NB == 2 ? buf ^ 1 : 0, (ci + 1) * KCP, min(KCP, nk - (ci + 1) * KCP));
      cp_async_commit();
      cp_async_wait<1>();
    } else {
      cp_async_wait<0>();
    }
    __syncthreads();
    if (warp_active) {
      if (ci == 0) {
#pragma unroll
        for (int ks = 0; ks < 4; ++ks)
          ldsm_x4(qf[ks], &sQ[(warp * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + ks * 16 + (lane >> 4) * 8]);
      }
      const int kcn = min(KCP, nk - ci * KCP);
      const int ntiles = kcn >> 3;  // even: kcn is a multiple of 16
      float sacc[8][4];
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        sacc[nt][0] = sacc[nt][1] = sacc[nt][2] = sacc[nt][3] = 0.f;
        if (nt < ntiles) {
#pragma unroll
          for (int kk = 0; kk < 2; ++kk) {
            uint32_t r[4];
            ldsm_x4(r, &sK[buf][(kbase + nt * 8 + (lane & 7)) * LDS + kk * 32 + (lane >> 3) * 8]);
            mma16816(sacc[nt], qf[2 * kk], r[0], r[1]);
            mma16816(sacc[nt], qf[2 * kk + 1], r[2], r[3]);
          }
        }
      }
      // online softmax: rows g = lane/4 (regs 0,1) and g+8 (regs 2,3)
      float cmax[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int nt = 0; nt < 8; ++nt) {
        if (nt < ntiles) {
#pragma unroll
          for (int e = 0; e < 4; ++e) sacc[nt][e] *= sc2;
          cmax[0] = fmaxf(cmax[0], fmaxf(sacc[nt][0], sacc[nt][1]));
          cmax[1] = fmaxf(cmax[1], fmaxf(sacc[nt][2], sacc[nt][3]));
        }
      }
      float al[2];
#pragma unroll
      for (int rr = 0; rr < 2; ++rr) {
        cmax[rr] = fmaxf(cmax[rr], __shfl_xor_sync(0xffffffffu, cmax[rr], 1));
        cmax[rr] = fmaxf(cmax[rr], __shfl_xor_sync(0xffffffffu, cmax[rr], 2));
        const float mn = fmaxf(mrow[rr], cmax[rr]);
        al[rr] = rescale(mrow[rr], mn);
        mrow[rr] = mn;
        lrow[rr] *= al[rr];
      }
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) {
        oacc[nd][0] *= al[0]; oacc[nd][1] *= al[0];
        oacc[nd][2] *= al[1]; oacc[nd][3] *= al[1];
      }
#pragma unroll
      for (int kj = 0; kj < 4; ++kj) {
        if (2 * kj < ntiles) {
          float p[2][4];
#pragma unroll
          for (int u = 0; u < 2; ++u) {
            p[u][0] = ex2_ftz(sacc[2 * kj + u][0] - mrow[0]);
            p[u][1] = ex2_ftz(sacc[2 * kj + u][1] - mrow[0]);
            p[u][2] = ex2_ftz(sacc[2 * kj + u][2] - mrow[1]);
            p[u][3] = ex2_ftz(sacc[2 * kj + u][3] - mrow[1]);
            lrow[0] += p[u][0] + p[u][1];
            lrow[1] += p[u][2] + p[u][3];
          }
          uint32_t pa[4];
          pa[0] = pack2(p[0][0], p[0][1]);
          pa[1] = pack2(p[0][2], p[0][3]);
          pa[2] = pack2(p[1][0], p[1][1]);
          pa[3] = pack2(p[1][2], p[1][3]);
#pragma unroll
          for (int nd = 0; nd < 8; nd += 2) {
            uint32_t r[4];
            ldsm_x4_t(r, &sV[buf][(kbase + kj * 16 + (lane & 7) + ((lane >> 3) & 1) * 8) * LDS + nd * 8 + (lane >> 4) * 8]);
            mma16816(oacc[nd], pa, r[0], r[1]);
            mma16816(oacc[nd + 1], pa, r[2], r[3]);
          }
        }
      }
    }
    __syncthreads();
  }

  if (!warp_active) return;
  // merge the block result into the global statistics of each query row
#pragma unroll
  for (int rr = 0; rr < 2; ++rr) {
    float lsum = lrow[rr];
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 1);
    lsum += __shfl_xor_sync(0xffffffffu, lsum, 2);
    const int r = wq0 + (lane >> 2) + rr * 8;             // query row within the pair
    if (r >= nrows) continue;
    // (uniform across the four lanes of a row, like the test above)
    if (!idx_ok(qt0 + r >= q0 && qt0 + r < q0 + nq && b < B && h < H, err)) continue;
    const size_t row = (size_t)(qt0 + r) * B + b;
    float mg = -INFINITY, lg = 0.f;
    if (!init) { mg = m[row * H + h]; lg = l[row * H + h]; }
    const float mn = fmaxf(mg, mrow[rr]);
    const float ag = rescale(mg, mn), ab = rescale(mrow[rr], mn);
    const float ln = lg * ag + lsum * ab;
    float* op = o + row * (size_t)d + h * DH + (lane & 3) * 2;
    float on[16];
#pragma unroll
    for (int nd = 0; nd < 8; ++nd) {
      float2 og = make_float2(0.f, 0.f);
      if (!init) og = *reinterpret_cast<const float2*>(op + nd * 8);
      on[2 * nd] = og.x * ag + oacc[nd][rr * 2 + 0] * ab;
      on[2 * nd + 1] = og.y * ag + oacc[nd][rr * 2 + 1] * ab;
    }
    if (fin && blockIdx.x == 0 && r == 0) {
      // query q0 receives no later fold: merge its temporary pair, write a_{q0}
      const __nv_bfloat16* tp = Q + row * (size_t)q_stride + h * DH + (lane & 3) * 2;
      const __nv_bfloat16* qrow = &sQ[(warp * 16) * LDS];   // tile row of this pair's query q0
      float dot = 0.f;
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) {
        const float2 kt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tp + d + nd * 8));
        const float2 qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(&qrow[nd * 8 + (lane & 3) * 2]));
        dot += qv.x * kt.x + qv.y * kt.y;
      }
      dot += __shfl_xor_sync(0xFu, dot, 1);
      dot += __shfl_xor_sync(0xFu, dot, 2);
      const float st = dot * sc2;
      const float m2 = fmaxf(mn, st);
      const float a2 = rescale(mn, m2), pt = exp2f(st - m2);
      const float inv = 1.f / (ln * a2 + pt);
      __nv_bfloat16* ap = a_out + (size_t)b * d + h * DH + (lane & 3) * 2;
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) {
        const float2 vt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tp + 2 * d + nd * 8));
        *reinterpret_cast<__nv_bfloat162*>(ap + nd * 8) =
            __floats2bfloat162_rn((on[2 * nd] * a2 + pt * vt.x) * inv, (on[2 * nd + 1] * a2 + pt * vt.y) * inv);
      }
    } else {
      if ((lane & 3) == 0) {
        m[row * H + h] = mn;
        l[row * H + h] = ln;
      }
#pragma unroll
      for (int nd = 0; nd < 8; ++nd) *reinterpret_cast<float2*>(op + nd * 8) = make_float2(on[2 * nd], on[2 * nd + 1]);
    }
  }
}

// ---------------------------------------------------------------------------
// small helpers
// ---------------------------------------------------------------------------
// out[r] = in[r] / rms(in[r]) (fp32 path)
__global__ void __launch_bounds__(256) k_rmsnorm_f32(const float* __restrict__ in, float* __restrict__ out,
                                                     size_t rows, int d, float eps) {
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  const float* xr = in + r * d;
  float s = 0.f;
  for (int e = lane; e < d; e += 32) s += xr[e] * xr[e];
  s = warp_sum(s);
  const float inv = rsqrtf(s / (float)d + eps);
  for (int e = lane; e < d; e += 32) out[r * d + e] = xr[e] * inv;
}

// x[r][:] = E[ids[r]][:]
template <class T>
__global__ void k_embed(const int32_t* __restrict__ ids, const T* __restrict__ E, T* __restrict__ x,
                        size_t rows, int vocab, int d, unsigned* err) {
  const size_t r = blockIdx.x;
  if (r >= rows) return;
  const int id = ids[r];
  const bool ok = id >= 0 && id < vocab;
  if (!ok && threadIdx.x == 0) set_error(err, RT_DEVERR_INDEX);
  for (int e = threadIdx.x; e < d; e += blockDim.x)
    x[r * d + e] = ok ? E[(size_t)id * d + e] : from_f<T>(0.f);
}

}  // namespace rt
