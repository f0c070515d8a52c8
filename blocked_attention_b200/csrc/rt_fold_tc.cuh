// rt_fold_tc.cuh -- block fold on the sm_100a tensor cores for large blocks.
//
// Folds keys [k0, k0 + nk) into the online-softmax statistics (m, l, o) of
// queries [q0, q0 + nq) ("Recurrent Transformer" paper page, notes §4.2 /
// paper §5: when (k_t, v_t) is revealed, keys (t - lowbit(t), t] are folded
// into queries (t, t + lowbit(t)]). bf16 q/k/v, d_h = 64, nk a multiple of 128.
//
// Persistent CTAs (one per SM) loop over work items = one (sequence b, head h)
// and 128 queries each; 192 threads:
//   warp 0     : TMA producer (3-D boxes over the position-major cache:
//                128 positions x 64 dims of one (b, h))
//   warp 1     : TMEM allocator + MMA issuer
//   warps 2..5 : softmax / accumulate / merge; thread = one query row
// For each 128-key chunk c (double-buffered everywhere):
//   S_c = Q K_c^T         tcgen05.mma, M=128 N=128 K=64, fp32 in TMEM
//   P_c = exp2(S_c*sc2 - m_c) in bf16, written by the softmax warps to shared
//         memory in the 128-byte-swizzled K-major operand layout
//   O_c = P_c V_c         tcgen05.mma, M=128 N=64 K=128, V as MN-major operand
//   o  <- o * exp2(m_{c-1} - m_c) + O_c   (registers; one chunk behind, so the
//         PV product of chunk c overlaps the softmax of chunk c+1)
// Finally each row merges (m, l, o) into its global statistics, or, when
// fin = 1 and the row is query q0, merges the temporary pair and writes a_{q0}.
#pragma once

#include "rt_common.cuh"
#include "rt_gemm_tc.cuh"

namespace rt {

struct FoldTcCfg {
  static constexpr int QT = 128, KC = 128, DH = 64, KVS = 3;
  static constexpr uint32_t Q_BYTES = QT * DH * 2;    // 16 KB
  static constexpr uint32_t KV_BYTES = KC * DH * 2;   // 16 KB (K or V chunk)
  static constexpr uint32_t P_BYTES = QT * KC * 2;    // 32 KB (two 64-key swizzle atoms)
  static constexpr uint32_t OFF_Q = 0;                             // [2]
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;           // [KVS]
  static constexpr uint32_t OFF_V = OFF_K + KVS * KV_BYTES;        // [KVS]
  static constexpr uint32_t OFF_P = OFF_V + KVS * KV_BYTES;        // [2]
  static constexpr uint32_t OFF_BAR = OFF_P + 2 * P_BYTES;
  static constexpr size_t SMEM_BYTES = 1024 + OFF_BAR + 256;
  static constexpr uint32_t TMEM_COLS = 512;          // S[2] at 0/128, O[2] at 256/320
};

__device__ __forceinline__ void tma_load_3d(const CUtensorMap* m, uint64_t* bar, void* dst, int c0, int c1,
                                            int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// MN-major operand with 128-byte swizzle, one 64-element swizzle row along MN:
// K rows of 128 bytes, 8-row groups 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128_mn(const void* p) {
  const uint32_t a = smem_u32(p);
  uint64_t d = 0;
  d |= (uint64_t)((a >> 4) & 0x3FFFu);   // start address
  d |= (uint64_t)(8192u >> 4) << 16;     // leading byte offset (next 64-element MN group; unused for N = 64)
  d |= (uint64_t)(1024u >> 4) << 32;     // stride byte offset: 8 K rows x 128 B
  d |= (uint64_t)1u << 46;               // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;               // layout: 128-byte swizzle
  return d;
}

__device__ __forceinline__ void fence_async_shared() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// Persistent: CTA i takes work items i, i + gridDim.x, ... where an item is one
// (b, h) pair and one tile of 128 queries (query tile fastest). All its chunks
// form one global sequence g = 0, 1, ... (chunk c = g % nch of local item
// g / nch), so the K/V ring, S/P/O buffers and their barrier phases run on
// across items and the next item's Q and K/V load while the current finishes.
__global__ void __launch_bounds__(192, 1)
    k_fold_tc(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
              const __grid_constant__ CUtensorMap tmV, const __nv_bfloat16* __restrict__ Q, int q_stride,
              float* __restrict__ m, float* __restrict__ l, float* __restrict__ o,
              __nv_bfloat16* __restrict__ a_out, int B, int H, int q0, int nq, int k0, int nk, float sc2,
              int init, int fin, unsigned* err) {
  using C = FoldTcCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;     // [2]
  uint64_t* q_empty = bars + 2;    // [2]
  uint64_t* kv_full = bars + 4;    // [KVS]
  uint64_t* kv_empty = bars + 7;   // [KVS]
  uint64_t* s_full = bars + 10;    // [2]
  uint64_t* s_free = bars + 12;    // [2]
  uint64_t* p_full = bars + 14;    // [2]
  uint64_t* o_full = bars + 16;    // [2]
  uint64_t* o_free = bars + 18;    // [2]
  uint64_t* mma_done = bars + 20;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 21);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = H * C::DH;
  const int ntq = (nq + C::QT - 1) / C::QT;
  const int nitems = B * H * ntq;
  const int nch = nk / C::KC;
  // items of this CTA and its total chunk count
  const int my_items = blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = my_items * nch;
  auto item_of = [&](int li, int& b, int& h, int& qt0) {
    const int it = (int)blockIdx.x + li * (int)gridDim.x;
    const int pair = it / ntq, qt = it - pair * ntq;
    b = pair / H;
    h = pair - b * H;
    qt0 = q0 + qt * C::QT;
  };

  if (threadIdx.x == 0) {
    for (int i = 0; i < 2; ++i) {
      mbar_init(&q_full[i], 1);
      mbar_init(&q_empty[i], 5);   // the MMA thread's commit + the four softmax warps
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
      mbar_init(&p_full[i], 4);
      mbar_init(&o_full[i], 1);
      mbar_init(&o_free[i], 4);
    }
    for (int i = 0; i < C::KVS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int g = 0;
      bool ok = true;
      int issued_q = 0;
      for (int li = 0; li < my_items && ok; ++li) {
        int b, h, qt0;
        item_of(li, b, h, qt0);
        const int qb = li & 1;
        if (!mbar_wait(&q_empty[qb], ((li >> 1) & 1u) ^ 1u, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[qb], C::Q_BYTES);
        tma_load_3d(&tmQ, &q_full[qb], smem + C::OFF_Q + qb * C::Q_BYTES, h * C::DH, b, qt0);
        ++issued_q;
        for (int c = 0; c < nch; ++c, ++g) {
          const int st = g % C::KVS;
          const uint32_t ph = (g / C::KVS) & 1u;
          if (!mbar_wait(&kv_empty[st], ph ^ 1u, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], 2 * C::KV_BYTES);
          tma_load_3d(&tmK, &kv_full[st], smem + C::OFF_K + st * C::KV_BYTES, h * C::DH, b, k0 + c * C::KC);
          tma_load_3d(&tmV, &kv_full[st], smem + C::OFF_V + st * C::KV_BYTES, h * C::DH, b, k0 + c * C::KC);
        }
      }
      if (!ok) {
        // aborted: wait (bounded) for the copies this thread issued
        if (issued_q > 0) mbar_wait(&q_full[0], (issued_q - 1) & 1u, err);
        for (int i = (g >= C::KVS ? g - C::KVS : 0); i < g; ++i) mbar_wait(&kv_full[i % C::KVS], (i / C::KVS) & 1u, err);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64) | (1u << 16);   // B (= V) MN-major
      bool ok = true;
      auto issue_s = [&](int g) -> bool {
        const int li = g / nch, c = g - li * nch;
        const int qb = li & 1, st = g % C::KVS, bb = g & 1;
        if (c == 0 && !mbar_wait(&q_full[qb], (li >> 1) & 1u, err)) return false;
        if (!mbar_wait(&kv_full[st], (g / C::KVS) & 1u, err) || !mbar_wait(&s_free[bb], ((g >> 1) & 1u) ^ 1u, err))
          return false;
        tc_fence_after();
        const uint8_t* qt = smem + C::OFF_Q + qb * C::Q_BYTES;
        const uint8_t* kt = smem + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
        for (int k = 0; k < C::DH / 16; ++k)
          tc_mma_f16(tmem_base + bb * 128, smem_desc_sw128(qt + k * 32), smem_desc_sw128(kt + k * 32), idesc_s,
                     k != 0 ? 1u : 0u);
        tc_commit(&s_full[bb]);
        return true;
      };
      auto issue_pv = [&](int g) -> bool {
        const int li = g / nch, c = g - li * nch;
        const int st = g % C::KVS, bb = g & 1;
        const uint32_t ph = (g >> 1) & 1u;
        if (!mbar_wait(&p_full[bb], ph, err) || !mbar_wait(&o_free[bb], ph ^ 1u, err)) return false;
        tc_fence_after();
        const uint8_t* pt = smem + C::OFF_P + bb * C::P_BYTES;
        const uint8_t* vt = smem + C::OFF_V + st * C::KV_BYTES;
#pragma unroll
        for (int ks = 0; ks < C::KC / 16; ++ks) {
          // A = P: K-major, 64-key atoms 16 KB apart, 32 bytes per 16 keys inside an atom
          // B = V: MN-major, 16 keys = 16 rows of 128 bytes
          tc_mma_f16(tmem_base + 256 + bb * 64, smem_desc_sw128(pt + (ks >> 2) * 16384 + (ks & 3) * 32),
                     smem_desc_sw128_mn(vt + ks * 16 * 128), idesc_o, ks != 0 ? 1u : 0u);
        }
        tc_commit(&o_full[bb]);
        tc_commit(&kv_empty[st]);
        if (c == nch - 1) tc_commit(&q_empty[li & 1]);   // the item's S products are all done
        return true;
      };
      if (total > 0) ok = issue_s(0);
      for (int g = 0; g < total && ok; ++g) {
        if (g + 1 < total) ok = issue_s(g + 1);
        if (ok) ok = issue_pv(g);
      }
      // every MMA this thread issued has finished before the CTA can free TMEM
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, err);
    }
  } else {
    // ---------------- softmax / accumulate / merge ----------------
    const int qq = warp & 3;
    const int r = qq * 32 + lane;
    const uint32_t lane_base = (uint32_t)(qq * 32) << 16;
    uint8_t* sP = smem + C::OFF_P;
    float m_run = -INFINITY, l_run = 0.f, alpha_prev = 0.f;
    float oacc[64];
    bool ok = true;

    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
      int v = 1;
      if (lane == 0) v = mbar_wait(bar, parity, err) ? 1 : 0;
      return __shfl_sync(0xffffffffu, v, 0) != 0;
    };
    auto accumulate = [&](int g, float alpha) -> bool {
      const int bb = g & 1;
      if (!wait_warp(&o_full[bb], (g >> 1) & 1u)) return false;
      tc_fence_after();
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t rv[32];
        tmem_ld_32x32b_x32(tmem_base + lane_base + 256 + bb * 64 + half * 32, rv);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) oacc[half * 32 + i] = oacc[half * 32 + i] * alpha + __uint_as_float(rv[i]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[bb]);
      return true;
    };
    // merge the finished item li into the global statistics (or finalise q0)
    auto merge = [&](int li) {
      int b, h, qt0;
      item_of(li, b, h, qt0);
      const int nrows = min(C::QT, q0 + nq - qt0);
      if (r < nrows && idx_ok(qt0 + r >= q0 && qt0 + r < q0 + nq && b < B && h < H, err)) {
        const size_t row = (size_t)(qt0 + r) * B + b;
        float mg = -INFINITY, lg = 0.f;
        float* op = o + row * (size_t)d + h * C::DH;
        if (!init) { mg = m[row * H + h]; lg = l[row * H + h]; }
        const float mn = fmaxf(mg, m_run);
        const float ag = rescale(mg, mn), ab = rescale(m_run, mn);
        const float ln = lg * ag + l_run * ab;
        if (fin && qt0 == q0 && r == 0) {
          // query q0 receives no later fold: merge its temporary pair, write a_{q0}
          const __nv_bfloat16* tp = Q + row * (size_t)q_stride + h * C::DH;
          const __nv_bfloat16* qrow = reinterpret_cast<const __nv_bfloat16*>(smem + C::OFF_Q + (li & 1) * C::Q_BYTES);
          float dot = 0.f;
#pragma unroll 8
          for (int e = 0; e < C::DH; ++e) dot += __bfloat162float(qrow[e]) * __bfloat162float(tp[d + e]);
          const float s2 = dot * sc2;
          const float m2 = fmaxf(mn, s2);
          const float a2 = rescale(mn, m2), pt = exp2f(s2 - m2);
          const float inv = 1.f / (ln * a2 + pt);
          __nv_bfloat16* ap = a_out + (size_t)b * d + h * C::DH;
#pragma unroll
          for (int e = 0; e < C::DH; e += 2) {
            float og0 = 0.f, og1 = 0.f;
            if (!init) { og0 = op[e]; og1 = op[e + 1]; }
            const float o0 = og0 * ag + oacc[e] * ab, o1 = og1 * ag + oacc[e + 1] * ab;
            const float2 vt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(tp + 2 * d + e));
            *reinterpret_cast<__nv_bfloat162*>(ap + e) =
                __floats2bfloat162_rn((o0 * a2 + pt * vt.x) * inv, (o1 * a2 + pt * vt.y) * inv);
          }
        } else {
          m[row * H + h] = mn;
          l[row * H + h] = ln;
#pragma unroll
          for (int e = 0; e < C::DH; e += 4) {
            float4 og = make_float4(0.f, 0.f, 0.f, 0.f);
            if (!init) og = *reinterpret_cast<const float4*>(op + e);
            og.x = og.x * ag + oacc[e] * ab;
            og.y = og.y * ag + oacc[e + 1] * ab;
            og.z = og.z * ag + oacc[e + 2] * ab;
            og.w = og.w * ag + oacc[e + 3] * ab;
            *reinterpret_cast<float4*>(op + e) = og;
          }
        }
      }
      // this item's Q buffer may be refilled (the MMA thread also arrives)
      __syncwarp();
      if (lane == 0) mbar_arrive(&q_empty[li & 1]);
    };

    for (int g = 0; g < total && ok; ++g) {
      const int li = g / nch, c = g - li * nch;
      const int bb = g & 1;
      if (c == 0) {
        if (g > 0) {
          // finish the previous item before its running state is reset
          if (!accumulate(g - 1, alpha_prev)) { ok = false; break; }
          merge(li - 1);
        }
        m_run = -INFINITY;
        l_run = 0.f;
#pragma unroll
        for (int i = 0; i < 64; ++i) oacc[i] = 0.f;
      }
      if (!wait_warp(&s_full[bb], (g >> 1) & 1u)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sbase = tmem_base + lane_base + bb * 128;
      float mx = -INFINITY;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t rv[32];
        tmem_ld_32x32b_x32(sbase + cc * 32, rv);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 32; ++i) mx = fmaxf(mx, __uint_as_float(rv[i]));
      }
      const float m_new = fmaxf(m_run, mx * sc2);
      const float alpha = rescale(m_run, m_new);
      float lsum = 0.f;
      uint8_t* prow = sP + bb * C::P_BYTES + r * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t rv[32];
        tmem_ld_32x32b_x32(sbase + cc * 32, rv);
        tmem_ld_wait();
        uint8_t* atom = prow + (cc >> 1) * 16384;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2_ftz(__uint_as_float(rv[gq * 8 + e]) * sc2 - m_new);
            lsum += p[e];
          }
          uint4 w;
          w.x = pack_bf16x2(p[0], p[1]);
          w.y = pack_bf16x2(p[2], p[3]);
          w.z = pack_bf16x2(p[4], p[5]);
          w.w = pack_bf16x2(p[6], p[7]);
          const int chunk = (cc & 1) * 4 + gq;
          *reinterpret_cast<uint4*>(atom + ((chunk ^ (r & 7)) << 4)) = w;
        }
      }
      l_run = l_run * alpha + lsum;
      m_run = m_new;
      tc_fence_before();
      fence_async_shared();   // P stores -> visible to the tensor core
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&s_free[bb]);
        mbar_arrive(&p_full[bb]);
      }
      if (c > 0 && !accumulate(g - 1, alpha_prev)) { ok = false; break; }
      alpha_prev = alpha;
    }
    if (ok && total > 0 && accumulate(total - 1, alpha_prev)) merge(my_items - 1);
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------
// k_fold_tc2: two softmax warpgroups. Work item = one (b, h) pair and a super
// tile of 256 queries (tile A = queries 0..127, tile B = 128..255 of it), so
// every K/V chunk feeds two 128-query tiles. 320 threads:
//   warp 0 : TMA producer (Q of both tiles per item; K/V ring)
//   warp 1 : MMA issuer, order S_A(0) S_B(0) | S_A(g+1) PV_A(g) S_B(g+1)
//            PV_B(g) | ...: the next chunk's scores go ahead of this chunk's
//            PV product, since the softmax frees S as soon as it has read it
//   warps 2..5 (tile A), 6..9 (tile B): softmax and merge
// Per chunk a softmax thread (one query row) reads its 128 scores from tensor
// memory once and releases S; exponentials are taken against a reference
// maximum that moves only when a chunk's maximum exceeds it by more than 8
// (in log2 units; p <= 2^8 is exact enough in bf16), and only then are O and
// l rescaled (O read, scaled and written back in tensor memory once the
// previous PV product has completed). O accumulates over an item's chunks in
// tensor memory (the first chunk's PV overwrites it) and is read once, at the
// item's end, for the merge. P is double-buffered per tile in shared memory.
// Q is single-buffered: the producer reloads it once the item's last S
// products have completed.
// TMEM: S_A 0..127, S_B 128..255, O_A 256..319, O_B 320..383.
// ---------------------------------------------------------------------------
// q . k over d_h = 64 bf16 elements (one thread; kept out of line so that the
// finalising row's dot product adds no registers to the softmax loop)
__device__ __noinline__ float dot64_bf16(const __nv_bfloat16* q, const __nv_bfloat16* k) {
  float dot = 0.f;
  for (int e = 0; e < 64; e += 2) {
    const float2 qv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(q + e));
    const float2 kv = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(k + e));
    dot += qv.x * kv.x + qv.y * kv.y;
  }
  return dot;
}

struct FoldTc2Cfg {
  static constexpr int QT = 128, KC = 128, DH = 64, KVS = 2;
  static constexpr uint32_t Q_BYTES = QT * DH * 2;    // 16 KB per tile
  static constexpr uint32_t KV_BYTES = KC * DH * 2;   // 16 KB
  static constexpr uint32_t P_BYTES = QT * KC * 2;    // 32 KB per tile and buffer
  static constexpr uint32_t OFF_Q = 0;                           // [2 tiles]
  static constexpr uint32_t OFF_K = OFF_Q + 2 * Q_BYTES;         // [KVS]
  static constexpr uint32_t OFF_V = OFF_K + KVS * KV_BYTES;      // [KVS]
  static constexpr uint32_t OFF_P = OFF_V + KVS * KV_BYTES;      // [2 tiles][2 buffers]
  static constexpr uint32_t OFF_BAR = OFF_P + 4 * P_BYTES;
  static constexpr size_t SMEM_BYTES = 1024 + OFF_BAR + 512;
  static constexpr uint32_t TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory per block");
};

__global__ void __launch_bounds__(320, 1)
    k_fold_tc2(const __grid_constant__ CUtensorMap tmQ, const __grid_constant__ CUtensorMap tmK,
               const __grid_constant__ CUtensorMap tmV, const __nv_bfloat16* __restrict__ Q, int q_stride,
               float* __restrict__ m, float* __restrict__ l, float* __restrict__ o,
               __nv_bfloat16* __restrict__ a_out, int B, int H, int q0, int nq, int k0, int nk, float sc2,
               int init, int fin, unsigned* err) {
  using C = FoldTc2Cfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + C::OFF_BAR);
  uint64_t* q_full = bars + 0;      // [1]
  uint64_t* q_empty = bars + 2;     // [1]
  uint64_t* kv_full = bars + 4;     // [KVS]
  uint64_t* kv_empty = bars + 6;    // [KVS]
  uint64_t* s_full = bars + 8;      // [tile]
  uint64_t* s_free = bars + 10;     // [tile]
  uint64_t* p_full = bars + 12;     // [tile][2]
  uint64_t* p_free = bars + 16;     // [tile][2]
  uint64_t* o_done = bars + 20;     // [tile]: a PV product has completed (one phase per chunk)
  uint64_t* mma_done = bars + 28;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(bars + 29);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int d = H * C::DH;
  const int nts = (nq + 2 * C::QT - 1) / (2 * C::QT);   // super tiles per pair
  const int nitems = B * H * nts;
  const int nch = nk / C::KC;
  const int my_items = blockIdx.x < nitems ? (nitems - 1 - (int)blockIdx.x) / (int)gridDim.x + 1 : 0;
  const int total = my_items * nch;
  auto item_of = [&](int li, int& b, int& h, int& st0) {
    const int it = (int)blockIdx.x + li * (int)gridDim.x;
    const int pair = it / nts, stt = it - pair * nts;
    b = pair / H;
    h = pair - b * H;
    st0 = q0 + stt * 2 * C::QT;
  };

  if (threadIdx.x == 0) {
    mbar_init(&q_full[0], 1);
    mbar_init(&q_empty[0], 1);   // MMA commit after the item's last S products
    for (int i = 0; i < 2; ++i) {
      mbar_init(&s_full[i], 1);
      mbar_init(&s_free[i], 4);
    }
    for (int i = 0; i < 4; ++i) {
      mbar_init(&p_full[i], 4);
      mbar_init(&p_free[i], 1);
    }
    mbar_init(&o_done[0], 1);
    mbar_init(&o_done[1], 1);
    for (int i = 0; i < C::KVS; ++i) {
      mbar_init(&kv_full[i], 1);
      mbar_init(&kv_empty[i], 1);
    }
    mbar_init(mma_done, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    fence_async_shared();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmQ);
    tma_prefetch_desc(&tmK);
    tma_prefetch_desc(&tmV);
  }
  if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  pdl_launch_dependents();
  pdl_wait();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      int g = 0, issued_q = 0;
      bool ok = true;
      for (int li = 0; li < my_items && ok; ++li) {
        int b, h, st0;
        item_of(li, b, h, st0);
        if (!mbar_wait(&q_empty[0], (li & 1u) ^ 1u, err)) { ok = false; break; }
        mbar_arrive_expect_tx(&q_full[0], 2 * C::Q_BYTES);
        tma_load_3d(&tmQ, &q_full[0], smem + C::OFF_Q, h * C::DH, b, st0);
        tma_load_3d(&tmQ, &q_full[0], smem + C::OFF_Q + C::Q_BYTES, h * C::DH, b, st0 + C::QT);
        ++issued_q;
        for (int c = 0; c < nch; ++c, ++g) {
          const int st = g % C::KVS;
          const uint32_t ph = (g / C::KVS) & 1u;
          if (!mbar_wait(&kv_empty[st], ph ^ 1u, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&kv_full[st], 2 * C::KV_BYTES);
          tma_load_3d(&tmK, &kv_full[st], smem + C::OFF_K + st * C::KV_BYTES, h * C::DH, b, k0 + c * C::KC);
          tma_load_3d(&tmV, &kv_full[st], smem + C::OFF_V + st * C::KV_BYTES, h * C::DH, b, k0 + c * C::KC);
        }
      }
      if (!ok) {
        if (issued_q > 0) mbar_wait(&q_full[0], (issued_q - 1) & 1u, err);
        for (int i = (g >= C::KVS ? g - C::KVS : 0); i < g; ++i) mbar_wait(&kv_full[i % C::KVS], (i / C::KVS) & 1u, err);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    if (lane == 0) {
      const uint32_t idesc_s = idesc_bf16_f32(128, 128);
      const uint32_t idesc_o = idesc_bf16_f32(128, 64) | (1u << 16);   // B (= V) MN-major
      auto issue_s = [&](int g, int t) -> bool {
        const int li = g / nch, c = g - li * nch;
        const int st = g % C::KVS;
        if (t == 0 && c == 0 && !mbar_wait(&q_full[0], li & 1u, err)) return false;
        if (t == 0 && !mbar_wait(&kv_full[st], (g / C::KVS) & 1u, err)) return false;
        if (!mbar_wait(&s_free[t], (g & 1u) ^ 1u, err)) return false;
        tc_fence_after();
        const uint8_t* qt = smem + C::OFF_Q + t * C::Q_BYTES;
        const uint8_t* kt = smem + C::OFF_K + st * C::KV_BYTES;
#pragma unroll
        for (int k = 0; k < C::DH / 16; ++k)
          tc_mma_f16(tmem_base + t * 128, smem_desc_sw128(qt + k * 32), smem_desc_sw128(kt + k * 32), idesc_s,
                     k != 0 ? 1u : 0u);
        tc_commit(&s_full[t]);
        // the item's last S products release Q to the producer
        if (t == 1 && c == nch - 1) tc_commit(&q_empty[0]);
        return true;
      };
      auto issue_pv = [&](int g, int t) -> bool {
        const int li = g / nch, c = g - li * nch;
        const int st = g % C::KVS, pb = g & 1;
        if (!mbar_wait(&p_full[t * 2 + pb], (g >> 1) & 1u, err)) return false;
        tc_fence_after();
        const uint8_t* pt = smem + C::OFF_P + (t * 2 + pb) * C::P_BYTES;
        const uint8_t* vt = smem + C::OFF_V + st * C::KV_BYTES;
        // O accumulates over the item's chunks; its first chunk overwrites it
#pragma unroll
        for (int ks = 0; ks < C::KC / 16; ++ks)
          tc_mma_f16(tmem_base + 256 + t * 64, smem_desc_sw128(pt + (ks >> 2) * 16384 + (ks & 3) * 32),
                     smem_desc_sw128_mn(vt + ks * 16 * 128), idesc_o, (ks != 0 || c != 0) ? 1u : 0u);
        tc_commit(&o_done[t]);
        tc_commit(&p_free[t * 2 + pb]);
        if (t == 1) tc_commit(&kv_empty[st]);
        (void)li;
        return true;
      };
      bool ok = true;
      if (total > 0) ok = issue_s(0, 0) && issue_s(0, 1);
      // Within an item the next chunk's S products go ahead of this chunk's
      // PV products. At an item's last chunk the PV products go first: the
      // next item's S products wait for its Q tiles, and the merge must not.
      for (int g = 0; g < total && ok; ++g) {
        if ((g + 1) % nch == 0) {
          ok = issue_pv(g, 0) && issue_pv(g, 1);
          if (ok && g + 1 < total) ok = issue_s(g + 1, 0) && issue_s(g + 1, 1);
          continue;
        }
        if (g + 1 < total) ok = issue_s(g + 1, 0);
        if (ok) ok = issue_pv(g, 0);
        if (ok && g + 1 < total) ok = issue_s(g + 1, 1);
        if (ok) ok = issue_pv(g, 1);
      }
      tc_commit(mma_done);
      mbar_wait(mma_done, 0, err);
    }
  } else {
    // ---------------- softmax warpgroups ----------------
    const int t = (warp - 2) >> 2;          // tile of this warpgroup
    const int qq = warp & 3;                // TMEM lane quarter of this warp
    const int r = qq * 32 + lane;           // query row within the tile
    const uint32_t lane_base = (uint32_t)(qq * 32) << 16;
    uint8_t* const sP = smem + C::OFF_P + t * 2 * C::P_BYTES + r * 128;   // this row in P buffer 0
    uint64_t* const pfull = p_full + t * 2;
    uint64_t* const pfree = p_free + t * 2;
    float m_ref = -INFINITY, m_true = -INFINITY, l_run = 0.f;   // reference and true row maximum
    bool ok = true;
    const uint32_t obase = tmem_base + lane_base + 256 + t * 64;   // this row's O

    auto wait_warp = [&](uint64_t* bar, uint32_t parity) -> bool {
      int v = 1;
      if (lane == 0) v = mbar_wait(bar, parity, err) ? 1 : 0;
      return __shfl_sync(0xffffffffu, v, 0) != 0;
    };
    // The merge runs warp-wide on coalesced rows: lane i owns columns 2i, 2i+1
    // of each of the warp's 32 rows, so a row's 256 bytes of o move in one
    // access. The running o of item li is loaded that way before the item's
    // last PV product completes (its latency overlaps it); the block's
    // result leaves tensor memory one row per thread and is transposed
    // through this warp's own 4 KB slices of the tile's P buffer 0 (rows
    // 32qq..32qq+31 of both key halves: columns 0-31 and 32-63, 128 bytes a
    // row, 16-byte chunks XOR-swizzled by row). Both P buffers are idle from
    // the item's last PV product until this warp writes its next P rows.
    uint8_t* const stg = smem + C::OFF_P + t * 2 * C::P_BYTES + qq * 4096;
    constexpr int NPRE = 14;   // rows of the running o loaded ahead (registers allow no more)
    struct RowPos { int b, h, qt0, nrows; };
    auto pos_of = [&](int li) {
      RowPos p;
      int st0;
      item_of(li, p.b, p.h, st0);
      p.qt0 = st0 + t * C::QT;
      p.nrows = min(C::QT, q0 + nq - p.qt0);   // may be <= 0 for an empty tile B
      return p;
    };
    auto load_prev = [&](const RowPos& p, float2 (&prev)[NPRE], float& mg, float& lg) {
      mg = -INFINITY;
      lg = 0.f;
      if (!init && r < p.nrows) {   // this thread's row: its running maximum and sum
        const size_t row = (size_t)(p.qt0 + r) * B + p.b;
        mg = m[row * H + p.h];
        lg = l[row * H + p.h];
      }
      const float* const o_w = o + ((size_t)(p.qt0 + qq * 32) * B + p.b) * d + p.h * C::DH + 2 * lane;
#pragma unroll
      for (int k = 0; k < NPRE; ++k) {
        prev[k] = make_float2(0.f, 0.f);
        if (!init && qq * 32 + k < p.nrows) prev[k] = *reinterpret_cast<const float2*>(o_w + k * (size_t)B * d);
      }
    };
    // af: the factor that takes O from the lazy reference to the true maximum
    auto merge = [&](const RowPos& p, float af, const float2 (&prev)[NPRE], float mg, float lg) {
      const bool valid =
          r < p.nrows && idx_ok(p.qt0 + r >= q0 && p.qt0 + r < q0 + nq && p.b < B && p.h < H, err);
      const size_t row = (size_t)(p.qt0 + r) * B + p.b;
      const float mn = fmaxf(mg, m_ref);
      const float ag = rescale(mg, mn), ab = rescale(m_ref, mn);
      const float abo = ab * af;   // on O, still relative to the lazy reference
      const float ln = lg * ag + l_run * ab;
      const bool fin_row = fin && p.qt0 == q0 && r == 0;   // lane 0 of warp 0 of the first tile
      // finalisation of query q0 with its own temporary pair (q . k_tmp)
      float a2 = 0.f, pt = 0.f, inv = 0.f;
      if (fin_row && valid) {
        const __nv_bfloat16* tp = Q + row * (size_t)q_stride + p.h * C::DH;   // q, k_tmp at +d
        const float s2 = dot64_bf16(tp, tp + d) * sc2;
        const float m2 = fmaxf(mn, s2);
        a2 = rescale(mn, m2);
        pt = exp2f(s2 - m2);
        inv = 1.f / (ln * a2 + pt);
      } else if (valid) {
        m[row * H + p.h] = mn;
        l[row * H + p.h] = ln;
      }
      // this row's new-block part, abo * O, from tensor memory into the staging slices
#pragma unroll
      for (int half = 0; half < 2; ++half) {
        uint32_t ov[32];
        tmem_ld_32x32b_x32(obase + half * 32, ov);
        tmem_ld_wait();
#pragma unroll
        for (int jj = 0; jj < 8; ++jj) {
          const int j = half * 8 + jj;
          const float4 v = make_float4(__uint_as_float(ov[4 * jj]) * abo, __uint_as_float(ov[4 * jj + 1]) * abo,
                                       __uint_as_float(ov[4 * jj + 2]) * abo, __uint_as_float(ov[4 * jj + 3]) * abo);
          *reinterpret_cast<float4*>(stg + half * 16384 + lane * 128 + (((j & 7) ^ (lane & 7)) << 4)) = v;
        }
      }
      tc_fence_before();
      __syncwarp();
      const bool fin_warp = fin && p.qt0 == q0 && qq == 0;
      a2 = __shfl_sync(0xffffffffu, a2, 0);
      pt = __shfl_sync(0xffffffffu, pt, 0);
      inv = __shfl_sync(0xffffffffu, inv, 0);
      const uint32_t rd = (uint32_t)(lane >> 4) * 16384u + (uint32_t)(lane & 1) * 8u;
      const size_t ostep = (size_t)B * d;   // floats from one query row of o to the next
      float* const o_w = o + ((size_t)(p.qt0 + qq * 32) * B + p.b) * d + p.h * C::DH + 2 * lane;
      const int nk_rows = min(32, p.nrows - qq * 32);   // rows of this warp in the block (warp-uniform)
      auto put_row = [&](int k, float2 pk) {
        const float agk = __shfl_sync(0xffffffffu, ag, k);
        const float2 nb = *reinterpret_cast<const float2*>(stg + rd + k * 128 + ((((lane & 15) >> 1) ^ (k & 7)) << 4));
        const float o0 = pk.x * agk + nb.x, o1 = pk.y * agk + nb.y;
        if (fin_warp && k == 0) {
          const __nv_bfloat16* vt_p = Q + ((size_t)p.qt0 * B + p.b) * q_stride + 2 * d + p.h * C::DH + 2 * lane;
          const float2 vt = __bfloat1622float2(*reinterpret_cast<const __nv_bfloat162*>(vt_p));
          *reinterpret_cast<__nv_bfloat162*>(a_out + (size_t)p.b * d + p.h * C::DH + 2 * lane) =
              __floats2bfloat162_rn((o0 * a2 + pt * vt.x) * inv, (o1 * a2 + pt * vt.y) * inv);
        } else {
          *reinterpret_cast<float2*>(o_w + k * ostep) = make_float2(o0, o1);
        }
      };
      // the other rows' running o, all in flight together
      float2 rest[32 - NPRE];
#pragma unroll
      for (int k = NPRE; k < 32; ++k) {
        rest[k - NPRE] = make_float2(0.f, 0.f);
        if (!init && k < nk_rows) rest[k - NPRE] = *reinterpret_cast<const float2*>(o_w + k * ostep);
      }
#pragma unroll
      for (int k = 0; k < NPRE; ++k)
        if (k < nk_rows) put_row(k, prev[k]);
#pragma unroll
      for (int k = NPRE; k < 32; ++k)
        if (k < nk_rows) put_row(k, rest[k - NPRE]);
      __syncwarp();   // the staging slices are rewritten by this warp's next P rows
    };

    for (int g = 0; g < total && ok; ++g) {
      const int li = g / nch, c = g - li * nch;
      if (!wait_warp(&s_full[t], g & 1u)) { ok = false; break; }
      tc_fence_after();
      // the row's 128 scores, read once; S is then free for the next chunk
      uint32_t sv[4][32];
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) tmem_ld_32x32b_x32(tmem_base + lane_base + t * 128 + cc * 32, sv[cc]);
      tmem_ld_wait();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[t]);
      // row maximum and, below, row sum in 8 independent partials (a single
      // running value would chain 128 dependent operations per chunk)
      float mxp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) mxp[e] = -INFINITY;
#pragma unroll
      for (int cc = 0; cc < 4; ++cc)
#pragma unroll
        for (int i = 0; i < 32; ++i) mxp[i & 7] = fmaxf(mxp[i & 7], __uint_as_float(sv[cc][i]));
      float mx = fmaxf(fmaxf(fmaxf(mxp[0], mxp[1]), fmaxf(mxp[2], mxp[3])),
                       fmaxf(fmaxf(mxp[4], mxp[5]), fmaxf(mxp[6], mxp[7])));
      mx *= sc2;
      // The reference moves only when a row's chunk maximum passes it by
      // more than 8; then O and l are rescaled, warp-wide (the warp's rows
      // share the tensor-memory access) and after this chunk's exponentials,
      // before its PV product may start.
      float alpha = 1.f;
      bool rescale_o = false;
      if (c == 0) {
        m_ref = mx;   // a new item: O is overwritten by this chunk's PV product
        m_true = mx;
        l_run = 0.f;
      } else if (__any_sync(0xffffffffu, mx > m_ref + 8.f)) {
        const float m_new = fmaxf(m_ref, mx);
        alpha = rescale(m_ref, m_new);
        m_ref = m_new;
        rescale_o = true;
      }
      // P buffer g % 2 must have been consumed by the PV product of chunk g - 2
      const int pb = g & 1;
      if (!wait_warp(pfree + pb, ((g >> 1) & 1u) ^ 1u)) { ok = false; break; }
      float lsp[8];
#pragma unroll
      for (int e = 0; e < 8; ++e) lsp[e] = 0.f;
      uint8_t* prow = sP + (pb ? C::P_BYTES : 0u);
#pragma unroll
      for (int cc = 0; cc < 4; ++cc) {
        uint8_t* atom = prow + (cc >> 1) * 16384;
#pragma unroll
        for (int gq = 0; gq < 4; ++gq) {
          float p[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            p[e] = ex2_ftz(__uint_as_float(sv[cc][gq * 8 + e]) * sc2 - m_ref);
            lsp[e] += p[e];
          }
          uint4 w;
          w.x = pack_bf16x2(p[0], p[1]);
          w.y = pack_bf16x2(p[2], p[3]);
          w.z = pack_bf16x2(p[4], p[5]);
          w.w = pack_bf16x2(p[6], p[7]);
          const int chunk = (cc & 1) * 4 + gq;
          *reinterpret_cast<uint4*>(atom + ((chunk ^ (r & 7)) << 4)) = w;
        }
      }
      const float lsum = ((lsp[0] + lsp[1]) + (lsp[2] + lsp[3])) + ((lsp[4] + lsp[5]) + (lsp[6] + lsp[7]));
      // o_done completes one phase per PV product, and a parity wait only
      // tells the phase it waits for from the one before it. Chunk g - 1's
      // product has had no wait of its own (the next chunk's S products are
      // issued ahead of it), so it is waited for here -- before this chunk's
      // P is released, while chunk g's product cannot have started -- when O
      // is rescaled and at an item's last chunk, whose merge then waits for
      // phase g alone.
      if ((rescale_o || c == nch - 1) && g > 0 && !wait_warp(&o_done[t], (uint32_t)(g - 1) & 1u)) {
        ok = false;
        break;
      }
      if (rescale_o) {
        // O of chunks up to g - 1 is final: rescale it
        tc_fence_after();
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          uint32_t ov[32];
          tmem_ld_32x32b_x32(obase + half * 32, ov);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 32; ++i) ov[i] = __float_as_uint(__uint_as_float(ov[i]) * alpha);
          tmem_st_32x32b_x32(obase + half * 32, ov);
        }
        tmem_st_wait();
      }
      l_run = l_run * alpha + lsum;
      m_true = fmaxf(m_true, mx);
      tc_fence_before();
      fence_async_shared();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull + pb);
      if (c == nch - 1) {
        // the item's last chunk: O is final once its PV product completes
        const RowPos pos = pos_of(li);
        float2 prev[NPRE];   // the warp's first NPRE rows; the others load in the merge
        float mg, lg;
        load_prev(pos, prev, mg, lg);
        if (!wait_warp(&o_done[t], (uint32_t)g & 1u)) { ok = false; break; }
        tc_fence_after();
        // the statistics in canonical form: relative to the true maximum
        float af = 1.f;
        if (m_true > m_ref) {
          af = rescale(m_ref, m_true);
          l_run *= af;
          m_ref = m_true;
        }
        merge(pos, af, prev, mg, lg);
      }
    }
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace rt
