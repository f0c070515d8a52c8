// rt_foldunits.cuh -- the small block fold (at most 8 keys) as a device
// routine over (sequence, query) units of one head, shared by the persistent
// step kernel's fold tasks and the W_kv GEMM's fused fold.
//
// "Recurrent Transformer" paper page, notes §4.2: when (k_t, v_t) is
// revealed, keys (t - lowbit(t), t] are folded into the online-softmax
// statistics (m, l, o) of queries (t, t + lowbit(t)]; the first query of the
// block is finalised with its temporary pair (paper §2.2).
#pragma once

#include "rt_common.cuh"

namespace rt {

// Operands of the fold (device pointers; position-major [N][B][...] rows)
struct FoldUnitArgs {
  int B, H, d, Nseq;
  const __nv_bfloat16* K;     // [N][B][d] persistent keys
  const __nv_bfloat16* V;
  const __nv_bfloat16* qkv;   // [N][B][3d]: q, k~, v~
  float* m;                   // [N][B][H]
  float* l;
  float* o;                   // [N][B][d]
  __nv_bfloat16* a16;         // [B][d]: a of the finalised query
  float sc2;                  // log2(e) x the softmax scale
  unsigned* err;
};

// One call folds the block's NK keys, starting at key k0, for one head h and
// sequences [s0, s0 + ns) into queries [q0, q0 + nq): every (sequence, query) unit is served by an octet of lanes
// holding 8 of the head's 64 dims; each thread takes R units at a time and
// issues all their loads before any use. With fin, the first query q0 is
// finalised (temporary pair merged, a = o / l written, statistics not
// stored); the other queries' (m, l, o) are updated in place, or written when
// the fold is the first into them (init).
// ---------------------------------------------------------------------------
template <int NK, int R>
__device__ __forceinline__ void fold_units(const FoldUnitArgs& P, int q0, int nq, int k0, int init, int h, int s0,
                                           int ns, int tid, int fin) {
  const int B = P.B, H = P.H, d = P.d;
  const int oct = tid >> 3, sl = tid & 7;
  const unsigned omask = 0xFFu << ((tid & 31) & 24);
  const int U = ns * nq;
  const __nv_bfloat16* K = P.K;
  const __nv_bfloat16* V = P.V;
  for (int u0 = 0; u0 < U; u0 += 16 * R) {
    uint4 qw[R], kw[R][NK], vw[R][NK], ktw[R], vtw[R];
    float4 oa[R], ob[R];
    float mo[R], lo[R];
    bool live[R];
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int u = u0 + r * 16 + oct;
      bool act = u < U;
      const int s = act ? u / nq : 0, qi = act ? u - s * nq : 0;
      const int b = s0 + s;
      const size_t row = (size_t)(q0 + qi) * B + b;
      const __nv_bfloat16* qp = P.qkv + row * (size_t)(3 * d) + h * 64 + sl * 8;
      qw[r] = ktw[r] = vtw[r] = make_uint4(0, 0, 0, 0);
      act = act && idx_ok(b < B && q0 + qi < P.Nseq && k0 >= 0 && k0 + NK <= q0 && h < H, P.err);
      oa[r] = ob[r] = make_float4(0.f, 0.f, 0.f, 0.f);
      mo[r] = -INFINITY;
      lo[r] = 0.f;
#pragma unroll
      for (int i = 0; i < NK; ++i) kw[r][i] = vw[r][i] = make_uint4(0, 0, 0, 0);
      live[r] = act;
      if (act) {
        // k, v, m, l and o were written by other CTAs of this kernel: loads
        // through L2 only (no stale L1 lines); q and the temporary pair come
        // from the projection kernel
        qw[r] = *reinterpret_cast<const uint4*>(qp);
#pragma unroll
        for (int i = 0; i < NK; ++i) {
          const size_t kv = ((size_t)(k0 + i) * B + b) * d + h * 64 + sl * 8;
          kw[r][i] = __ldcg(reinterpret_cast<const uint4*>(K + kv));
          vw[r][i] = __ldcg(reinterpret_cast<const uint4*>(V + kv));
        }
        if (fin && qi == 0) {   // the finalised query's temporary pair
          ktw[r] = *reinterpret_cast<const uint4*>(qp + d);
          vtw[r] = *reinterpret_cast<const uint4*>(qp + 2 * d);
        }
        if (!init) {
          const float* op = P.o + row * (size_t)d + h * 64 + sl * 8;
          mo[r] = __ldcg(P.m + row * H + h);
          lo[r] = __ldcg(P.l + row * H + h);
          oa[r] = __ldcg(reinterpret_cast<const float4*>(op));
          ob[r] = __ldcg(reinterpret_cast<const float4*>(op) + 1);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < R; ++r) {
      const int u = u0 + r * 16 + oct;
      if (!live[r]) continue;   // whole octets together; shuffles stay inside the octet
      const int s = u / nq, qi = u - s * nq;
      const int b = s0 + s;
      const size_t row = (size_t)(q0 + qi) * B + b;
      float q[8];
      unpack_bf16x8(qw[r], q);
      float sc[NK];
      float mx = -INFINITY;
#pragma unroll
      for (int i = 0; i < NK; ++i) {
        float kk[8];
        unpack_bf16x8(kw[r][i], kk);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) dot += q[e] * kk[e];
        dot += __shfl_xor_sync(omask, dot, 1);
        dot += __shfl_xor_sync(omask, dot, 2);
        dot += __shfl_xor_sync(omask, dot, 4);
        sc[i] = dot * P.sc2;
        mx = fmaxf(mx, sc[i]);
      }
      float oo[8] = {oa[r].x, oa[r].y, oa[r].z, oa[r].w, ob[r].x, ob[r].y, ob[r].z, ob[r].w};
      const float mn = fmaxf(mo[r], mx);
      const float al = rescale(mo[r], mn);
      float ln = lo[r] * al;
#pragma unroll
      for (int e = 0; e < 8; ++e) oo[e] *= al;
#pragma unroll
      for (int i = 0; i < NK; ++i) {
        const float p = ex2_ftz(sc[i] - mn);
        float vv[8];
        unpack_bf16x8(vw[r][i], vv);
        ln += p;
#pragma unroll
        for (int e = 0; e < 8; ++e) oo[e] += p * vv[e];
      }
      if (fin && qi == 0) {
        float kt[8];
        unpack_bf16x8(ktw[r], kt);
        float dot = 0.f;
#pragma unroll
        for (int e = 0; e < 8; ++e) dot += q[e] * kt[e];
        dot += __shfl_xor_sync(omask, dot, 1);
        dot += __shfl_xor_sync(omask, dot, 2);
        dot += __shfl_xor_sync(omask, dot, 4);
        const float st = dot * P.sc2;
        const float m2 = fmaxf(mn, st);
        const float a2 = rescale(mn, m2), pt = exp2f(st - m2);
        const float inv = 1.f / (ln * a2 + pt);
        float vt[8];
        unpack_bf16x8(vtw[r], vt);
        uint4 w;
        uint32_t* wp = reinterpret_cast<uint32_t*>(&w);
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          __nv_bfloat162 v2 = __floats2bfloat162_rn((oo[2 * k] * a2 + pt * vt[2 * k]) * inv,
                                                    (oo[2 * k + 1] * a2 + pt * vt[2 * k + 1]) * inv);
          wp[k] = *reinterpret_cast<uint32_t*>(&v2);
        }
        if (idx_ok(b < B && h < H, P.err, 16, b, h))
          *reinterpret_cast<uint4*>(P.a16 + (size_t)b * d + h * 64 + sl * 8) = w;
      } else {
        float* op = P.o + row * (size_t)d + h * 64 + sl * 8;
        if (sl == 0) {
          P.m[row * H + h] = mn;
          P.l[row * H + h] = ln;
        }
        reinterpret_cast<float4*>(op)[0] = make_float4(oo[0], oo[1], oo[2], oo[3]);
        reinterpret_cast<float4*>(op)[1] = make_float4(oo[4], oo[5], oo[6], oo[7]);
      }
    }
  }
}

}  // namespace rt
