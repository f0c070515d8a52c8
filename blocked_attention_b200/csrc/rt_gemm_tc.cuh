// rt_gemm_tc.cuh -- bf16 x bf16 -> fp32 GEMM on the sm_100a tensor cores
// (tcgen05.mma, accumulators in tensor memory, operands staged by TMA), with
// the fused epilogues of the Recurrent Transformer layer.
//
//   C[M][N] = A[M][K] * W[N][K]^T      (A, W row-major = K-major operands)
//
// Kernel shape: persistent CTAs of 224 threads (one output tile per CTA of a
// thread-block cluster under split-K).
//   warp 0      : TMA producer (one elected lane), STAGES-deep smem ring of
//                 KSUB 64-wide K slices per stage
//   warps 1, 2  : MMA issuers (one lane each; warp 1 also allocates TMEM),
//                 taking alternate stages into their own accumulators
//   warps 3..6  : epilogue; warp w reads TMEM lanes 32*(w%4) .. +31 and sums
//                 the issuers' accumulators
// Tile 128 x BN; two tiles' accumulators in TMEM so that the epilogue of tile
// i overlaps the MMAs of tile i+1.
//
// Epilogues (one thread owns one output row, 32 columns at a time):
//   PLAIN : C fp32
//   PROJ  : batched projection of all positions, scaled by 1/rms(x) of the
//           row, written position-major [N][B][3d] (queries and temporary
//           pairs, "Recurrent Transformer" paper page, notes §4.2: queries
//           depend only on the layer input and are computed up front)
//   WO    : u = x_t + a W_o^T (fp32 and bf16 copies) + per-tile sum of u^2
//   W1    : h = GELU((u W_1^T) / rms(u))            (rms from the WO partials)
//   W2    : z_t = u + h W_2^T -> output z, bf16 copy, per-tile sum of z^2
//   WKV   : [k_t | v_t] = (z_t [W_k; W_v]^T) / rms(z_t) -> position-major K, V
//   RKV   : the same for all B*N rows of a stored output z [B][N][d] at once
//           (activation-checkpoint recompute of the persistent pairs, paper
//           §6.1), scaled by 1/rms(z) of the row -> position-major K, V
// The identity rms(v) W^T = (v W^T) / r(v), r(v) = sqrt(mean v^2 + eps), moves
// each RMSNorm into the next GEMM's epilogue; it changes only rounding.
#pragma once

#include "rt_common.cuh"

namespace rt {

enum EpiKind { EPI_PLAIN = 0, EPI_PROJ = 1, EPI_WO = 2, EPI_W1 = 3, EPI_W2 = 4, EPI_WKV = 5, EPI_RKV = 6 };

struct EpiParams {
  int B, Nseq, d, d_ff, j;   // batch, sequence length, width, MLP width, position (0-based)
  // x is stored as [ceil(Nseq / xc)][B][xc][d]: chunks of xc positions, each
  // chunk sequence-major (xc = Nseq is the plain [B][Nseq][d] layout)
  int xc;
  int n0;                    // PROJ: the launch's rows are one chunk, [B][xc], from position n0
  float eps;
  float* c32;                // PLAIN out [M][N]
  const float* inv_rms;      // PROJ: 1/rms per input row [B*N]
  __nv_bfloat16* qkv;        // PROJ out [N][B][3d]
  const __nv_bfloat16* x;    // WO: layer input [B][N][d]
  float* u32;                // WO out / W2 in: [B][d]
  __nv_bfloat16* u16;        // WO out: [B][d]
  float* ssq_out;            // WO / W2 out: [n_tiles][B]
  const float* ssq_in;       // W1 / WKV in: [ssq_tiles][B]
  int ssq_tiles;
  __nv_bfloat16* h16;        // W1 out: [B][d_ff]
  __nv_bfloat16* zout;       // W2 out: [B][N][d]
  __nv_bfloat16* z16;        // W2 out: [B][d]
  __nv_bfloat16* Kout;       // WKV out: [N][B][d]
  __nv_bfloat16* Vout;
  // split-K: `splits` CTAs (one thread-block cluster, launched with cluster
  // dimension `splits`) share one output tile, each over K/splits; each
  // stages its fp32 partial tile in its own shared memory, and after a
  // cluster barrier CTA rank r sums rows [r*128/splits, (r+1)*128/splits) of
  // all ranks' partials over distributed shared memory, in rank order, and
  // runs the epilogue for them. BN/splits must be a multiple of 32.
  int splits;
  // the paper's own parameterisation ("Recurrent Transformer" paper page,
  // paper §2 notation and §2.1): pages = 1 normalises every head of q, k~
  // (PROJ) and k (WKV, RKV) to unit RMS, and scales the W_o and W_2 branches
  // by inv_sqrt_L = 1/sqrt(L) (the caller also sets eps = 0 and drops the
  // softmax scale). pages = 0: the single-layer configuration.
  int pages;
  float inv_sqrt_L;
  // Rows of the per-position GEMMs (WO, W1, W2, WKV) are position-major:
  // row r is sequence r % B at position j + r / B (one position per launch:
  // row = sequence; a chunk of positions: B rows per position). ssq_rows is
  // the row count of the launch, the stride of the sum-of-squares partials
  // (0 = B).
  int ssq_rows;
};

__device__ __forceinline__ int ssq_stride(const EpiParams& p) { return p.ssq_rows ? p.ssq_rows : p.B; }

__device__ __forceinline__ uint32_t dsmem_map(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
// bulk copy of `bytes` (multiple of 16, 16-byte aligned) from this CTA's shared
// memory into the shared memory of a CTA of the cluster, completing on that
// CTA's mbarrier (both addresses already mapped with mapa)
__device__ __forceinline__ void bulk_copy_to_cluster(uint32_t dst, uint32_t src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.shared::cta.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "r"(src), "r"(bytes), "r"(bar)
               : "memory");
}
__device__ __forceinline__ void bulk_commit_group() { asm volatile("cp.async.bulk.commit_group;" ::: "memory"); }
__device__ __forceinline__ void bulk_wait_read_all() {
  asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");
}
__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 v = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&v);
}

// store 32 floats as 32 bf16 (64 contiguous bytes, 16-byte aligned)
__device__ __forceinline__ void store_bf16x32(__nv_bfloat16* dst, const float (&v)[32]) {
  uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w;
    w.x = pack_bf16x2(v[8 * i + 0], v[8 * i + 1]);
    w.y = pack_bf16x2(v[8 * i + 2], v[8 * i + 3]);
    w.z = pack_bf16x2(v[8 * i + 4], v[8 * i + 5]);
    w.w = pack_bf16x2(v[8 * i + 6], v[8 * i + 7]);
    d4[i] = w;
  }
}

__device__ __forceinline__ void load_bf16x32(const __nv_bfloat16* src, float (&v)[32]) {
  const uint4* s4 = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w = s4[i];
    const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float2 f = __bfloat1622float2(p[k]);
      v[8 * i + 2 * k] = f.x;
      v[8 * i + 2 * k + 1] = f.y;
    }
  }
}

// Tile configuration. A pipeline stage holds KSUB 64-wide K slices of the A
// tile (128 rows) and of the B tile (BN rows), each slice one 128-byte-swizzle
// TMA box, so one mbarrier wait gates 4 * KSUB MMAs. For BN <= 128 two
// MMA-issuing warps take alternate stages into their own TMEM accumulators
// (summed in the epilogue): an mbarrier wait of the issuing thread costs
// about as long as four 128 x BN x 16 MMAs at BN <= 128, so with one issuer
// the tensor pipe drains at every wait; the second issuer's MMAs fill it.
// BN = 256 MMAs outlast the wait: one issuer, one slice per stage.
template <int BN>
struct GemmCfg {
  static constexpr int BM = 128, BK = 64, KSUB = BN == 256 ? 1 : 2;
  static constexpr int KB = BK * KSUB;                       // K per stage
  static constexpr uint32_t A_SUB = BM * BK * 2, B_SUB = BN * BK * 2;
  static constexpr uint32_t A_BYTES = A_SUB * KSUB, B_BYTES = B_SUB * KSUB;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = (200 * 1024) / STAGE_BYTES;  // 5 / 4 / 3 / 4 for BN 32 / 64 / 128 / 256
  static constexpr int NACC = BN == 256 ? 1 : 2;             // accumulators (issuing warps) per tile
  static constexpr uint32_t TMEM_COLS = 2 * NACC * BN;       // two tiles in flight
  static constexpr int THREADS = 224;                        // producer, 2 issuers, 4 epilogue warps
  // split-K staging in the ring: the CTA's partial tile plus splits - 1
  // receive slots of one row block each (fp32 rows padded to BN + 4)
  static constexpr bool split_fits(int splits) {
    return splits >= 1 && (BN / splits) % 32 == 0 &&
           (size_t)(BM + (splits - 1) * (BM / splits)) * (BN + 4) * 4 <= (size_t)STAGES * STAGE_BYTES;
  }
  static constexpr size_t SMEM_BYTES = 1024 /*align slack*/ + STAGES * STAGE_BYTES + 256;
  static_assert(BN == 32 || BN == 64 || BN == 128 || BN == 256, "BN");
  static_assert(STAGES >= 2, "stages");
};

// Pulls into L1 the residual operand the epilogue will read for `ncols`
// columns of a row from col0 on (WO: the layer input x, bf16).
template <int EPI>
__device__ __forceinline__ void epilogue_prefetch(const EpiParams& p, int row, int col0, int N, int ncols) {
  for (int c = 0; c < ncols; c += 32) {
    if (col0 + c >= N) break;
    const void* ptr = nullptr;
    if constexpr (EPI == EPI_WO) {
      const int b = row % p.B, jj = p.j + row / p.B;
      const int ch = jj / p.xc;
      ptr = p.x + (((size_t)ch * p.B + b) * p.xc + (jj - ch * p.xc)) * p.d + col0 + c;
    }
    if (ptr) asm volatile("prefetch.global.L1 [%0];" ::"l"(ptr));   // one 128-byte line per chunk
  }
}

// Row-wise epilogue for one 32-column chunk; returns the chunk's sum of squares
// of the value that feeds the next RMSNorm (WO: u, W2: z), else 0.
template <int EPI>
__device__ __forceinline__ float epilogue_chunk(const EpiParams& p, int row, int col0, int N,
                                                float (&v)[32], float row_scale, unsigned* dbg_err = nullptr) {
  float ssq = 0.f;
  if constexpr (EPI == EPI_WO || EPI == EPI_W2 || EPI == EPI_WKV) {
    // (debug build) the step rows and the output columns
    if (!idx_ok(p.j + row / p.B < p.Nseq && col0 + 32 <= (EPI == EPI_WKV ? 2 * p.d : p.d) && (col0 & 31) == 0,
                dbg_err, 20 + EPI, row, col0))
      return 0.f;
  } else if constexpr (EPI == EPI_W1) {
    if (!idx_ok(col0 + 32 <= p.d_ff && (col0 & 31) == 0, dbg_err, 20 + EPI, row, col0)) return 0.f;
  }
  if constexpr (EPI == EPI_PLAIN) {
    float* dst = p.c32 + (size_t)row * N + col0;
    if (col0 + 32 <= N && (N % 4) == 0) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(dst)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    } else {
      for (int i = 0; i < 32; ++i)
        if (col0 + i < N) dst[i] = v[i];
    }
  } else if constexpr (EPI == EPI_PROJ) {
    const int b = row / p.xc, n = p.n0 + (row - b * p.xc);
    if (n >= p.Nseq) return 0.f;   // padding rows of a last, shorter chunk
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= row_scale;
    store_bf16x32(p.qkv + ((size_t)n * p.B + b) * (size_t)(3 * p.d) + col0, v);
  } else if constexpr (EPI == EPI_WO) {
    const int b = row % p.B, jj = p.j + row / p.B;
    float xv[32];
    const int c = jj / p.xc;
    load_bf16x32(p.x + (((size_t)c * p.B + b) * p.xc + (jj - c * p.xc)) * p.d + col0, xv);
    if (p.pages) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= p.inv_sqrt_L;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      v[i] += xv[i];
      ssq += v[i] * v[i];
    }
    float4* u4 = reinterpret_cast<float4*>(p.u32 + (size_t)row * p.d + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) u4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    store_bf16x32(p.u16 + (size_t)row * p.d + col0, v);
  } else if constexpr (EPI == EPI_W1) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = gelu_as7126(v[i] * row_scale);
    store_bf16x32(p.h16 + (size_t)row * p.d_ff + col0, v);
  } else if constexpr (EPI == EPI_W2) {
    const int b = row % p.B, jj = p.j + row / p.B;
    // u was written by other CTAs (L2-coherent loads: no stale L1 lines)
    const float4* u4 = reinterpret_cast<const float4*>(p.u32 + (size_t)row * p.d + col0);
    if (p.pages) {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] *= p.inv_sqrt_L;
    }
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float4 w = __ldcg(u4 + i);
      v[4 * i] += w.x; v[4 * i + 1] += w.y; v[4 * i + 2] += w.z; v[4 * i + 3] += w.w;
    }
#pragma unroll
    for (int i = 0; i < 32; ++i) ssq += v[i] * v[i];
    store_bf16x32(p.zout + ((size_t)b * p.Nseq + jj) * p.d + col0, v);
    store_bf16x32(p.z16 + (size_t)row * p.d + col0, v);
  } else if constexpr (EPI == EPI_WKV) {
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= row_scale;
    const size_t base = ((size_t)p.j * p.B + row) * p.d;   // position j + row / B, sequence row % B
    if (col0 < p.d) store_bf16x32(p.Kout + base + col0, v);
    else store_bf16x32(p.Vout + base + (col0 - p.d), v);
  } else if constexpr (EPI == EPI_RKV) {
    // row = b * Nseq + n of z [B][N][d]; outputs position-major [N][B][d]
    const int b = row / p.Nseq, n = row - b * p.Nseq;
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] *= row_scale;
    const size_t base = ((size_t)n * p.B + b) * p.d;
    if (col0 < p.d) store_bf16x32(p.Kout + base + col0, v);
    else store_bf16x32(p.Vout + base + (col0 - p.d), v);
  }
  return ssq;
}

// The paper's per-head query/key normalisation (paper §2.1, RMS applied to
// each head's d_h = 64 entries): 64 columns = one head of one row, scaled by
// the row factor, then, for the q / k~ columns of PROJ ([0, 2d)) and the k
// columns of WKV and RKV ([0, d)), normalised to unit RMS; then stored by the
// 32-column epilogue with a row factor of 1.
template <int EPI>
__device__ __forceinline__ void epilogue_head64(const EpiParams& p, int row, int col0, int N, float (&va)[32],
                                                float (&vb)[32], float row_scale) {
  static_assert(EPI == EPI_PROJ || EPI == EPI_WKV || EPI == EPI_RKV, "head normalisation epilogues");
#pragma unroll
  for (int i = 0; i < 32; ++i) { va[i] *= row_scale; vb[i] *= row_scale; }
  const bool normed = EPI == EPI_PROJ ? col0 < 2 * p.d : col0 < p.d;
  if (normed) {
    float ss = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) ss += va[i] * va[i] + vb[i] * vb[i];
    const float sc = rsqrtf(ss * (1.f / 64.f));
#pragma unroll
    for (int i = 0; i < 32; ++i) { va[i] *= sc; vb[i] *= sc; }
  }
  epilogue_chunk<EPI>(p, row, col0, N, va, 1.f);
  epilogue_chunk<EPI>(p, row, col0 + 32, N, vb, 1.f);
}

// 32 columns of a tile's accumulator for this thread's row: the sum of the
// two issuers' partial accumulators (BN columns apart) when both wrote one.
template <int NACC, int BN>
__device__ __forceinline__ void tmem_ld_acc(uint32_t taddr, bool two, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  if (NACC == 2 && two) {
    uint32_t r2[32];
    tmem_ld_32x32b_x32(taddr + BN, r2);
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]) + __uint_as_float(r2[i]);
  } else {
    tmem_ld_wait();
#pragma unroll
    for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
  }
}

template <int EPI>
__device__ __forceinline__ float row_scale_for(const EpiParams& p, int row) {
  if constexpr (EPI == EPI_PROJ || EPI == EPI_RKV) {
    return p.inv_rms[row];
  } else if constexpr (EPI == EPI_W1 || EPI == EPI_WKV) {
    float s = 0.f;
    for (int t = 0; t < p.ssq_tiles; ++t) s += __ldcg(p.ssq_in + (size_t)t * ssq_stride(p) + row);
    return rsqrtf(s / (float)p.d + p.eps);
  } else {
    return 1.f;
  }
}

template <int BN, int EPI>
__global__ void __launch_bounds__(224, 1)
    k_gemm_tc(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
              int M, int N, int K, EpiParams p, unsigned* err) {
  using C = GemmCfg<BN>;
  constexpr int STAGES = C::STAGES, NACC = C::NACC, KSUB = C::KSUB;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2]
  uint64_t* tempty = tfull + 2;       // [2]
  uint64_t* rbar = tempty + 2;        // split-K: the other ranks' row blocks have landed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(rbar + 1);
  volatile uint32_t* seen = tmem_holder + 1;   // [STAGES]: see ring_round_wait

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ntn = (N + BN - 1) / BN, ntm = (M + C::BM - 1) / C::BM;
  const int nmn = ntn * ntm;
  const int splits = p.splits > 1 ? p.splits : 1;
  // splits == 1: persistent loop over output tiles; splits > 1: one tile per
  // CTA, tile = mn * splits + ks, so a cluster of `splits` CTAs holds one mn.
  const int num_tiles = nmn * splits;
  // stages per tile (per split). K is a multiple of 64; a last stage with
  // fewer than KSUB slices loads and multiplies only those. With splits > 1
  // the host keeps K / splits a multiple of the stage depth.
  const int nk = splits > 1 ? K / C::KB / splits : (K + C::KB - 1) / C::KB;
  const int ksl = K / C::BK;   // 64-wide K slices in all
  auto slices = [&](int kblock) { const int r = ksl - kblock * KSUB; return r < KSUB ? r : KSUB; };
  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); seen[s] = 0; }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], NACC); mbar_init(&tempty[a], 4); }
    mbar_init(rbar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0) { tma_prefetch_desc(&tmA); tma_prefetch_desc(&tmB); }
  if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;
  // everything above overlaps the predecessor kernel. The producer also loads
  // the weight (B) tiles of its first pipeline stages before waiting: weights
  // are never written by a predecessor. Every thread waits before touching
  // anything a predecessor writes.
  pdl_launch_dependents();

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t it = 0;
      bool ok = true;
      // weight tiles of the first tile's first stages (all stages start empty)
      int pre = 0;
      if ((int)blockIdx.x < num_tiles) {
        const int mn = (int)blockIdx.x / splits, ks = (int)blockIdx.x - mn * splits;
        const int mt = mn / ntn, nt = mn - mt * ntn;
        pre = nk < STAGES ? nk : STAGES;
        for (int kb = 0; kb < pre; ++kb) {
          const int kk = (ks * nk + kb) * KSUB, ns = slices(ks * nk + kb);
          mbar_arrive_expect_tx(&full[kb], ns * (C::A_SUB + C::B_SUB));
          for (int j = 0; j < ns; ++j)
            tma_load_2d(&tmB, &full[kb], sB + kb * C::B_BYTES + j * C::B_SUB, (kk + j) * C::BK, nt * BN);
        }
      }
      pdl_wait();
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        const int mn = tile / splits, ks = tile - mn * splits;
        const int mt = mn / ntn, nt = mn - mt * ntn;
        const int kb0 = ks * nk;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
          const int kk = (kb0 + kb) * KSUB, ns = slices(kb0 + kb);
          uint8_t* a_st = sA + s * C::A_BYTES;
          if ((int)it < pre) {   // B already in flight; add A
            for (int j = 0; j < ns; ++j)
              tma_load_2d(&tmA, &full[s], a_st + j * C::A_SUB, (kk + j) * C::BK, mt * C::BM);
            continue;
          }
          if (!mbar_wait(&empty[s], ph ^ 1u, err)) { ok = false; break; }
          mbar_arrive_expect_tx(&full[s], ns * (C::A_SUB + C::B_SUB));
          for (int j = 0; j < ns; ++j) {
            tma_load_2d(&tmA, &full[s], a_st + j * C::A_SUB, (kk + j) * C::BK, mt * C::BM);
            tma_load_2d(&tmB, &full[s], sB + s * C::B_BYTES + j * C::B_SUB, (kk + j) * C::BK, nt * BN);
          }
        }
      }
      if (!ok) {
        // wait (bounded) for copies still in flight before the CTA can exit
        const uint32_t first = it > (uint32_t)STAGES ? it - STAGES : 0u;
        for (uint32_t i = first; i < it; ++i) mbar_wait(&full[i % STAGES], (i / STAGES) & 1u, err);
      }
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: stage kb of a tile goes to issuer kb % NACC ----------------
    pdl_wait();
    const int par = warp - 1;
    if (lane == 0 && par < NACC) {
      const uint32_t idesc = idesc_bf16_f32(C::BM, BN);
      uint32_t it = 0, local = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++local) {
        const uint32_t acc = local & 1u, aph = (local >> 1) & 1u;
        if (!mbar_wait(&tempty[acc], aph ^ 1u, err)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (acc * NACC + par) * BN;
        uint32_t accumulate = 0;
        const int kb0 = (tile - (tile / splits) * splits) * nk;
        for (int kb = 0; kb < nk; ++kb, ++it) {
          if ((kb % NACC) != par) continue;
          const uint32_t s = it % STAGES, ph = (it / STAGES) & 1u;
          if (NACC > 1 && !ring_round_wait(&seen[s], it / STAGES, err)) { ok = false; break; }
          if (!mbar_wait(&full[s], ph, err)) { ok = false; break; }
          if (NACC > 1) seen[s] = it / STAGES + 1;
          tc_fence_after();
          const uint8_t* a_st = sA + s * C::A_BYTES;
          const uint8_t* b_st = sB + s * C::B_BYTES;
          const int nmma = slices(kb0 + kb) * (C::BK / 16);
#pragma unroll
          for (int k = 0; k < KSUB * (C::BK / 16); ++k) {
            if (k >= nmma) break;
            // slice k / 4; inside it advance 16 bf16 (32 bytes) along K in the 128-byte swizzle atom
            const int j = k / (C::BK / 16), kk = k % (C::BK / 16);
            tc_mma_f16(d_tmem, smem_desc_sw128(a_st + j * C::A_SUB + kk * 32),
                       smem_desc_sw128(b_st + j * C::B_SUB + kk * 32), idesc, accumulate);
            accumulate = 1u;
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&tfull[acc]);   // with no stage of its own in this tile it arrives at once
      }
    }
  } else {
    // ---------------- epilogue warps ----------------
    pdl_wait();
    const int q = warp & 3;
    uint32_t local = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++local) {
      const int mn = tile / splits;
      const int mt = mn / ntn, nt = mn - mt * ntn;
      const uint32_t acc = local & 1u, aph = (local >> 1) & 1u;
      const int lrow = q * 32 + lane;
      const int row = mt * C::BM + lrow;
      const bool row_ok = row < M;
      // while the tile's MMAs run: the row's RMS scale (reads the previous
      // kernel's partial sums) and the epilogue's residual operand into L1
      const float rs = (splits == 1 && row_ok) ? row_scale_for<EPI>(p, row) : 0.f;
      if (splits == 1 && row_ok) epilogue_prefetch<EPI>(p, row, nt * BN, N, BN);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(&tfull[acc], aph, err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      if (!ok) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * NACC * BN;
      const bool two = NACC == 2 && nk >= 2;   // issuer 1 wrote its accumulator in this tile
      if (splits == 1) {
        float ssq = 0.f;
        bool head_norm = false;
        if constexpr ((EPI == EPI_PROJ || EPI == EPI_WKV || EPI == EPI_RKV) && BN >= 64) head_norm = p.pages != 0;
        if (head_norm) {
#pragma unroll 1
          for (int c = 0; c < BN; c += 64) {
            float va[32], vb[32];
            tmem_ld_acc<NACC, BN>(taddr + c, two, va);
            tmem_ld_acc<NACC, BN>(taddr + c + 32, two, vb);
            const int col0 = nt * BN + c;
            if constexpr ((EPI == EPI_PROJ || EPI == EPI_WKV || EPI == EPI_RKV) && BN >= 64)
              if (row_ok && col0 < N) epilogue_head64<EPI>(p, row, col0, N, va, vb, rs);
          }
        }
#pragma unroll 1
        for (int c = 0; c < BN && !head_norm; c += 32) {
          float v[32];
          tmem_ld_acc<NACC, BN>(taddr + c, two, v);
          const int col0 = nt * BN + c;
          if (row_ok && col0 < N) ssq += epilogue_chunk<EPI>(p, row, col0, N, v, rs);
        }
        if constexpr (EPI == EPI_WO || EPI == EPI_W2) {
          if (row_ok) p.ssq_out[(size_t)nt * ssq_stride(p) + row] = ssq;
        }
      } else {
        // stage this CTA's partial tile (fp32, rows padded to BN + 4 floats) in the
        // shared memory of the operand ring: every TMA load and MMA has completed
        fence_proxy_async_smem();
        float* stage = reinterpret_cast<float*>(smem) + (size_t)lrow * (BN + 4);
#pragma unroll 1
        for (int c = 0; c < BN; c += 32) {
          float v[32];
          tmem_ld_acc<NACC, BN>(taddr + c, two, v);
#pragma unroll
          for (int i = 0; i < 8; ++i)
            reinterpret_cast<float4*>(stage + c)[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[acc]);
    }
  }
  if (splits > 1) {
    // One output tile per cluster, reduce-scattered over distributed shared
    // memory: rank r owns rows [r * rows_per, (r + 1) * rows_per) of the tile.
    // Every rank bulk-copies each row block it does not own from its staged
    // partial into that owner's receive slot (slot = sender's rank among the
    // others); each owner sums its block over the ranks in rank order and runs
    // the epilogue on it.
    const int rank = blockIdx.x % splits;            // == %cluster_ctarank for a 1-D cluster of `splits`
    const int rows_per = C::BM / splits, cpt = BN / splits;
    const uint32_t rb_floats = (uint32_t)rows_per * (BN + 4), rb_bytes = rb_floats * 4u;
    float* stage = reinterpret_cast<float*>(smem);
    float* recv = stage + (size_t)C::BM * (BN + 4);
    if (threadIdx.x == 96) mbar_arrive_expect_tx(rbar, (uint32_t)(splits - 1) * rb_bytes);
    fence_proxy_async_smem();   // this thread's staging writes -> the bulk copies' reads
    cluster_sync();             // every rank's partial is staged and its receive barrier armed
    if (threadIdx.x == 96) {
      for (int rr = 0; rr < splits; ++rr) {
        if (rr == rank) continue;
        const int slot = rank < rr ? rank : rank - 1;
        bulk_copy_to_cluster(dsmem_map(smem_u32(recv + (size_t)slot * rb_floats), (uint32_t)rr),
                             smem_u32(stage + (size_t)rr * rb_floats), rb_bytes,
                             dsmem_map(smem_u32(rbar), (uint32_t)rr));
      }
      bulk_commit_group();
    }
    if (warp >= 3) {
      const int t = threadIdx.x - 96;                  // 0..127
      const int mn = blockIdx.x / splits;
      const int mt = mn / ntn, nt = mn - mt * ntn;
      const int brow = t / splits, cbase = (t % splits) * cpt;
      const int lrow = rank * rows_per + brow;
      const int row = mt * C::BM + lrow;
      const bool in_range = row < M && blockIdx.x < num_tiles;
      // while the other ranks' blocks are in flight
      const float rs = in_range ? row_scale_for<EPI>(p, row) : 0.f;
      if (in_range) epilogue_prefetch<EPI>(p, row, nt * BN + cbase, N, cpt);
      int ok = 1;
      if (lane == 0) ok = mbar_wait(rbar, 0u, err) ? 1 : 0;
      ok = __shfl_sync(0xffffffffu, ok, 0);
      const bool row_ok = ok && in_range;
      float ssq = 0.f;
#pragma unroll 1
      for (int c = 0; c < cpt; c += 32) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = 0.f;
        for (int rr = 0; rr < splits; ++rr) {
          const float* src = rr == rank ? stage + (size_t)lrow * (BN + 4)
                                        : recv + (size_t)(rr < rank ? rr : rr - 1) * rb_floats +
                                              (size_t)brow * (BN + 4);
          const float4* s4 = reinterpret_cast<const float4*>(src + cbase + c);
#pragma unroll
          for (int i = 0; i < 8; ++i) {
            const float4 w = s4[i];
            v[4 * i] += w.x; v[4 * i + 1] += w.y; v[4 * i + 2] += w.z; v[4 * i + 3] += w.w;
          }
        }
        const int col0 = nt * BN + cbase + c;
        if (row_ok && col0 < N) ssq += epilogue_chunk<EPI>(p, row, col0, N, v, rs);
      }
      if constexpr (EPI == EPI_WO || EPI == EPI_W2) {
        // the `splits` consecutive lanes sharing a row add their column sums
        for (int o = 1; o < splits; o <<= 1) ssq += __shfl_xor_sync(0xffffffffu, ssq, o);
        if (row_ok && (t % splits) == 0) p.ssq_out[(size_t)nt * ssq_stride(p) + row] = ssq;
      }
    }
    // this CTA's outgoing copies have read its staging before it can exit;
    // incoming ones completed before the owner's barrier wait returned
    if (threadIdx.x == 96) bulk_wait_read_all();
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace rt
