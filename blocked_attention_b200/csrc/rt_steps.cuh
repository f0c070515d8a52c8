// rt_steps.cuh -- the layer's N-step loop as one persistent kernel per segment
// of steps (sm_100a: tcgen05 tensor cores, TMEM accumulators, TMA operands).
//
// Source: "Recurrent Transformer" paper page (www.lshu.cn/news/403416):
//   paper §2.2  : the per-position chain u = x_t + W_o a_t ->
//                 z_t = u + W_2 GELU(W_1 rms(u)) -> (k_t, v_t) = [W_k; W_v] rms(z_t);
//   notes §4.2  : when (k_t, v_t) is revealed, keys (t - lowbit(t), t] are
//                 folded into the online-softmax statistics of queries
//                 (t, t + lowbit(t)];
//   paper §6.2  : O(N) medium-sized launches dominate a per-step loop.
//
// A segment is a run of steps j0 .. j1-1 (0-based positions; step j reveals
// the pair of position t = j + 1) whose folds all have at most 8 keys, except
// the fold of its last step, which has >= 16 keys (run afterwards by the block
// fold kernels) or does not exist (t = N). Sequences never interact, so the
// batch is cut into row blocks of 128 sequences (the GEMM tile height) and
// every dependency below stays inside one row block: the row blocks run as
// independent chains that overlap on the machine.
//
// Work of one step, per row block rb ("tasks"):
//   WO   : u = x_j + a W_o^T (+ per-tile sums of u^2)        tiles of BN_o columns
//   W1   : h = GELU((u W_1^T) / r(u))                         tiles of BN_1
//   W2   : z_j = u + h W_2^T (+ sums of z^2)                  tiles of BN_2, K split S ways
//   WKV  : [k_j | v_j] = (z_j [W_k; W_v]^T) / r(z_j)          tiles of BN_kv
//   FOLD : keys (t - lb, t] into queries (t, t + lb] for one head and 32
//          sequences; the first query (t + 1) is finalised: its temporary pair
//          is merged and a_{t+1} = o / l is written (the A operand of the next
//          step's WO).                                        lb <= 8, not on the segment's last step
// Tasks are numbered in the order (step, phase, row block, tile, split) and
// dealt round-robin to the grid's CTAs (one per SM, co-resident: cooperative
// launch); each CTA processes its tasks in that order. Every task waits only
// for tasks earlier in the order, except that the S splits of a W_2 tile wait
// for one another's partial tiles; those are S consecutive tasks of one phase
// on S different CTAs, each reached after earlier tasks only, so the earliest
// unfinished task can always run: no deadlock.
//
// Dependencies are flags in global memory holding "last step done + 1"
// (monotonic within a forward; cleared before it), one per output tile, or per
// 1 / S of a W_2 tile. A task's TMA producer loads the weight operand of its
// first pipeline stages, then polls every flag its A operand depends on (the
// warp's lanes in parallel) and streams A. Every thread that reads data another CTA
// wrote first observes (acquire) the flag that covers it, then fences, and
// reads that data through L2 (ld.global.cg or TMA), never from a possibly
// stale L1 line; every writer fences its stores (also to the async proxy,
// since the next phase reads them with TMA) before it releases its flag. The
// W_2 split-K partial tiles go to global slots; once all S have arrived, every
// split sums its 1 / S of the columns over the S slots in split order
// (deterministic) and runs the epilogue on them.
//
// Every poll and every mbarrier wait is bounded by %globaltimer. A poll that
// runs out records RT_DEVERR_TIMEOUT and returns; once the error word is set,
// every later poll returns at once and the tasks run on with whatever data is
// there, so the kernel always ends. An mbarrier wait that runs out (or sees
// the error word set) stops its warp's task loop; before the CTA frees its
// tensor memory, the MMA warps wait (bounded) for their issued MMAs and the
// producer for its copies in flight.
#pragma once

#include "rt_common.cuh"
#include "rt_foldunits.cuh"
#include "rt_gemm_tc.cuh"

namespace rt {

enum StepPhase { PH_WO = 0, PH_W1 = 1, PH_W2 = 2, PH_WKV = 3, PH_FOLD = 4, PH_DEFER = 5, PH_COUNT = 6 };
// the order of the phases inside a step
__device__ __forceinline__ int phase_at(int i) {
  switch (i) {
    case 0: return PH_WO;
    case 1: return PH_W1;
    case 2: return PH_DEFER;
    case 3: return PH_W2;
    case 4: return PH_WKV;
    default: return PH_FOLD;
  }
}

constexpr int kFlagStride = 256;   // flags per (phase, row block): tiles, or heads x fold groups
constexpr int kFoldSeqs = 32;      // sequences per fold task
constexpr int kSmallFoldMax = 8;   // largest block folded inside the step kernel

struct StepsCfg {
  static constexpr int BM = 128, BK = 64, KSUB = 2, BN_MAX = 128;
  static constexpr uint32_t A_SUB = BM * BK * 2;            // one 64-wide K slice of A (16 KB)
  static constexpr uint32_t B_SUB = BN_MAX * BK * 2;        // slot for one K slice of B (16 KB)
  static constexpr uint32_t A_BYTES = A_SUB * KSUB, B_BYTES = B_SUB * KSUB;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = 3;
  static constexpr uint32_t TMEM_COLS = 512;                // 2 tiles in flight x 2 issuers x 128
  static constexpr int THREADS = 352;                       // producer, 2 MMA issuers, 4 epilogue, 4 fold warps
  static constexpr size_t SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
};

// One GEMM phase: C[B][N] = A[B][K] W[N][K]^T, output tiles of 128 x BN, the
// reduction split S ways (S > 1 only for W2).
struct GemmPhase {
  int N, K, BN, S, tiles;
};

struct StepsParams {
  CUtensorMap tA[4], tB[4];    // per GEMM phase: A (activations, box 64 x 128) and W (box 64 x BN)
  GemmPhase g[4];
  EpiParams ep;                // shapes, x, u32, u16, h16, zout, z16, Kout, Vout, xc, eps
  float* ssq_u;                // [d / BN_o][B]
  float* ssq_z;                // [d / BN_2][B]
  const __nv_bfloat16* qkv;    // [N][B][3d]
  float* m;                    // [N][B][H]
  float* l;
  float* o;                    // [N][B][d]
  __nv_bfloat16* a16;          // [B][d]
  unsigned* flags;             // [PH_COUNT][nrb][kFlagStride]
  unsigned* w2cnt;             // [nrb][tiles of W2]: split arrivals, cumulative over the forward
  float* w2part;               // [nrb][tiles][S][BN_2][128] fp32 partial tiles
  unsigned* err;
  unsigned* progress;          // (debug build) [gridDim][10]: the task and the wait each role of each CTA is at
  unsigned long long* trace;   // (trace build) [tasks of the segment][16] event times, or null
  float sc2;                   // log2(e) / sqrt(d_h)
  int H, nrb, G;               // heads, row blocks, fold groups of 32 sequences per row block
  int j0, j1;                  // the segment's steps
};

// ---------------------------------------------------------------------------
// synchronisation helpers
// ---------------------------------------------------------------------------
// generic-proxy global stores <-> async-proxy (TMA) global accesses
__device__ __forceinline__ void fence_proxy_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
// barrier of the four epilogue warps (named barrier 1, 128 threads)
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
// barrier of the four fold warps (named barrier 2, 128 threads)
__device__ __forceinline__ void fold_bar() { asm volatile("bar.sync 2, 128;" ::: "memory"); }

// mbarrier wait bounded by time and abandoned once the error word is set.
__device__ __forceinline__ bool mbar_wait_g(uint64_t* bar, unsigned parity, unsigned* err, unsigned id = 0,
                                            long long where = 0) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0) {
      if (ld_volatile_u32(err) != 0) return false;
      if (globaltimer() - t0 > kWaitLimitNs) {
        set_error(err, RT_DEVERR_TIMEOUT);
        timeout_record(err, id, where, parity);
        return false;
      }
    }
  }
}

// where a wait is: CTA, step, phase and the task's index in its phase
__device__ __forceinline__ long long wait_site(int ph, int j, int loc) {
  return ((long long)blockIdx.x << 24) | ((long long)(j & 0xfff) << 12) | ((ph & 7) << 9) | (loc & 0x1ff);
}

// (debug build) after an error the flags stay as they were, so that the
// record shows the dependency state at the first failure
__device__ __forceinline__ bool release_allowed(const StepsParams& P) {
#ifdef RT_BOUNDS_CHECK
  return ld_volatile_u32(P.err) == 0;
#else
  return true;
#endif
}

// (debug build) role r of this CTA is at task (ph, j, loc): producer 0, MMA
// issuers 1 and 2, epilogue 3, folds 4 (word 2r), and in which wait (word 2r + 1:
// kind in bits 28..30 -- 1 ring slot free, 2 dependency flag, 3 accumulator
// free, 4 stage loaded, 5 accumulator full, 6 slot's previous round seen --
// then the ring stage counter or task counter in bits 0..27)
__device__ __forceinline__ void note_progress(const StepsParams& P, int role, int ph, int j, int loc) {
#ifdef RT_BOUNDS_CHECK
  // frozen once the error word is set: the record shows where each role was
  if (P.progress && ld_volatile_u32(P.err) == 0)
    *reinterpret_cast<volatile unsigned*>(P.progress + blockIdx.x * 10 + 2 * role) =
        ((unsigned)(j & 0xfff) << 12) | ((ph & 7) << 9) | (loc & 0x1ff) | 0x80000000u;
#endif
}
__device__ __forceinline__ void note_wait(const StepsParams& P, int role, unsigned kind, unsigned counter) {
#ifdef RT_BOUNDS_CHECK
  if (P.progress && ld_volatile_u32(P.err) == 0)
    *reinterpret_cast<volatile unsigned*>(P.progress + blockIdx.x * 10 + 2 * role + 1) =
        (kind << 28) | (counter & 0x0fffffffu) | 0x80000000u;
#endif
}

// (trace build) event ev of the segment's task gi happened now (%globaltimer
// ns): 0 producer starts the task, 1 producer issued its last A load (every
// dependency seen), 2 / 3 issuer 0 / 1 has its accumulator, 4 / 5 issuer 0 /
// 1 issued its last MMA, 6 epilogue starts, 7 epilogue dependencies seen, 8
// accumulator full, 9 flag released (a fold: 6, 7 and 9); per pipeline stage
// k < 16: 16 + k producer has the slot, 48 + k an issuer saw the stage
// loaded; 32 producer saw every dependency; epilogue sub-steps: 10 outputs
// stored, 11 fences done, 40 + 2c / 41 + 2c chunk c (< 4) read from tensor
// memory / written; a W2 split: 12 partial written, 13 every split arrived,
// 14 its columns summed
constexpr int kTraceSlots = 64;
__device__ __forceinline__ void trace_ev(const StepsParams& P, int gi, int ev) {
#ifdef RT_TRACE
  if (P.trace && ev < kTraceSlots) P.trace[(size_t)gi * kTraceSlots + ev] = globaltimer();
#endif
}

// ---------------------------------------------------------------------------
// task enumeration (identical in every warp role of a CTA)
// ---------------------------------------------------------------------------
// Queries of the block folded at step j - 1 (t = j) after its first one: the
// deferred part of that fold, run at step j (0 when the block has one query).
__device__ __forceinline__ int deferred_queries(const StepsParams& P, int j) {
  return min(lowbit(j), P.ep.Nseq - j) - 1;
}
__device__ __forceinline__ int phase_tasks(const StepsParams& P, int ph, int j) {
  if (ph < 4) return P.nrb * P.g[ph].tiles * P.g[ph].S;
  if (ph == PH_FOLD) return (j + 1 < P.j1) ? P.nrb * P.H * P.G : 0;   // the segment's last fold runs elsewhere
  return (j > P.j0 && deferred_queries(P, j) > 0) ? P.nrb * P.H * P.G : 0;
}

// Calls f(phase, step, local index, index in the segment) for this CTA's
// tasks in order; stops when f returns false.
template <class F>
__device__ __forceinline__ void for_my_tasks(const StepsParams& P, F&& f) {
  const long G = gridDim.x, bid = blockIdx.x;
  long base = 0;
  for (int j = P.j0; j < P.j1; ++j) {
    for (int oi = 0; oi < PH_COUNT; ++oi) {
      const int ph = phase_at(oi);
      const int n = phase_tasks(P, ph, j);
      long first = (bid - base) % G;
      if (first < 0) first += G;
      for (long loc = first; loc < n; loc += G)
        if (!f(ph, j, (int)loc, (int)(base + loc))) return;
      base += n;
    }
  }
}

struct GemmTask {
  int rb, tile, split, sl0, sl1;   // row block, output tile, K split, 64-wide K slices [sl0, sl1)
};
__device__ __forceinline__ GemmTask decode_gemm(const GemmPhase& g, int loc) {
  GemmTask t;
  const int per_rb = g.tiles * g.S;
  t.rb = loc / per_rb;
  const int r = loc - t.rb * per_rb;
  t.tile = r / g.S;
  t.split = r - t.tile * g.S;
  const int ksl = g.K / 64;
  t.sl0 = t.split * ksl / g.S;
  t.sl1 = (t.split + 1) * ksl / g.S;
  return t;
}

__device__ __forceinline__ unsigned* flag_ptr(const StepsParams& P, int ph, int rb, int i) {
  if (!idx_ok(ph >= 0 && ph < PH_COUNT && rb >= 0 && rb < P.nrb && i >= 0 && i < kFlagStride, P.err))
    i = 0, rb = 0, ph = 0;   // (debug build) a bad flag index reads flag 0 instead
  return P.flags + ((size_t)(ph * P.nrb + rb) * kFlagStride + i);
}

// The flags the A operand of a GEMM task depends on: K slice kk of phase ph
// is made by flags [lo(kk), hi(kk)) of phase dep_phase(ph), complete once
// they reach dep_target.
__device__ __forceinline__ int dep_phase(int ph) { return ph == PH_WO ? PH_FOLD : ph - 1; }
// Columns one flag of a GEMM phase covers: a tile, or with a split
// reduction one tile / S (every split finishes that share of its tile).
__device__ __forceinline__ int flag_cols(const GemmPhase& g) { return g.BN / g.S; }
__device__ __forceinline__ int phase_flags(const GemmPhase& g) { return g.tiles * g.S; }
__device__ __forceinline__ void slice_flags(const StepsParams& P, int ph, int kk, int& lo, int& hi) {
  if (ph == PH_WO) {   // a of head kk (d_h = 64): the fold groups of head kk
    lo = kk * P.G;
    hi = lo + P.G;
  } else {             // columns [64 kk, 64 kk + 64) of the previous phase's output
    const int fc = flag_cols(P.g[ph - 1]);
    lo = (64 * kk) / fc;
    hi = (64 * kk + 63) / fc + 1;
  }
}


// ---------------------------------------------------------------------------
// epilogue of one GEMM tile (split == whole K): 32 columns at a time, the sum
// of the two issuers' accumulators
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_ld_pair(uint32_t taddr, bool two, float (&v)[32]) {
  uint32_t r[32];
  tmem_ld_32x32b_x32(taddr, r);
  if (two) {
    uint32_t r2[32];
    tmem_ld_32x32b_x32(taddr + StepsCfg::BN_MAX, r2);
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
__device__ __forceinline__ float epi_tile_tmem(const EpiParams& e, int row, bool row_ok, int col_base, int BN,
                                               uint32_t taddr, bool two, float rs, unsigned* dbg_err,
                                               const StepsParams& P, int gi) {
  float ssq = 0.f;
  if constexpr (EPI == EPI_WKV) {
    if (e.pages) {   // per-head unit RMS of k (the paper's parameterisation)
#pragma unroll 1
      for (int c = 0; c < BN; c += 64) {
        float va[32], vb[32];
        tmem_ld_pair(taddr + c, two, va);
        tmem_ld_pair(taddr + c + 32, two, vb);
        if (row_ok) epilogue_head64<EPI_WKV>(e, row, col_base + c, e.d * 2, va, vb, rs);
      }
      return 0.f;
    }
  }
#pragma unroll 1
  for (int c = 0; c < BN; c += 32) {
    float v[32];
    tmem_ld_pair(taddr + c, two, v);
    if (threadIdx.x == 96 && c < 128) trace_ev(P, gi, 40 + (c >> 4));
    if (row_ok) ssq += epilogue_chunk<EPI>(e, row, col_base + c, EPI == EPI_W1 ? e.d_ff : (EPI == EPI_WKV ? 2 * e.d : e.d), v, rs, dbg_err);
    if (threadIdx.x == 96 && c < 128) trace_ev(P, gi, 41 + (c >> 4));
  }
  return ssq;
}

// W_o tile epilogue (BN = 64) with the residual x already in registers (the
// epilogue loads it before it waits for the accumulator): u = x + a W_o^T,
// written fp32 and bf16; returns the row's sum of squares over the tile.
__device__ __forceinline__ float epi_wo_tile64(const EpiParams& e, int row, bool row_ok, int col_base,
                                               uint32_t taddr, bool two, const uint4 (&xw)[8], unsigned* dbg_err) {
  float ssq = 0.f;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    float v[32];
    tmem_ld_pair(taddr + 32 * h, two, v);
    const int col0 = col_base + 32 * h;
    if (!row_ok || !idx_ok(e.j + row / e.B < e.Nseq && col0 + 32 <= e.d, dbg_err, 20 + EPI_WO, row, col0)) continue;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float xf[8];
      unpack_bf16x8(xw[4 * h + k], xf);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float w = v[8 * k + i];
        if (e.pages) w *= e.inv_sqrt_L;
        w += xf[i];
        v[8 * k + i] = w;
        ssq += w * w;
      }
    }
    float4* u4 = reinterpret_cast<float4*>(e.u32 + (size_t)row * e.d + col0);
#pragma unroll
    for (int i = 0; i < 8; ++i) u4[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
    store_bf16x32(e.u16 + (size_t)row * e.d + col0, v);
  }
  return ssq;
}

// W_2 epilogue of one 32-column chunk with the residual u already in
// registers: z = u + h W_2^T, written to the layer output and the bf16
// operand of W_kv; returns the chunk's sum of squares.
__device__ __forceinline__ float epi_w2_chunk_pre(const EpiParams& e, int row, bool row_ok, int col0,
                                                  float (&v)[32], const uint4 (&uw)[8], unsigned* dbg_err) {
  if (!row_ok || !idx_ok(e.j + row / e.B < e.Nseq && col0 + 32 <= e.d, dbg_err, 20 + EPI_W2, row, col0)) return 0.f;
  const int b = row % e.B, jj = e.j + row / e.B;
  float ssq = 0.f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const float u[4] = {__uint_as_float(uw[i].x), __uint_as_float(uw[i].y), __uint_as_float(uw[i].z),
                        __uint_as_float(uw[i].w)};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      float w = v[4 * i + k];
      if (e.pages) w *= e.inv_sqrt_L;
      w += u[k];
      v[4 * i + k] = w;
      ssq += w * w;
    }
  }
  store_bf16x32(e.zout + ((size_t)b * e.Nseq + jj) * e.d + col0, v);
  store_bf16x32(e.z16 + (size_t)row * e.d + col0, v);
  return ssq;
}

// The epilogue-side dependencies of a task, polled in parallel by the 128
// epilogue threads (thread i polls flag i of a contiguous range; the polls
// are acquire loads), then the epilogue barrier, which orders every epilogue
// thread's later loads after those acquires.
__device__ __forceinline__ void epi_poll_range(const StepsParams& P, int ph, int rb, int lo, int hi, unsigned target,
                                               int tid, int task_ph = 7, int task_loc = 0) {
  for (int i = lo + tid; i < hi; i += 128)
    poll_ge(flag_ptr(P, ph, rb, i), target, P.err, 46, wait_site(task_ph, (int)target, (ph << 6) | (i & 63)));
}

// ---------------------------------------------------------------------------
// the kernel
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(StepsCfg::THREADS, 1) k_steps(const __grid_constant__ StepsParams P) {
  using C = StepsCfg;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = smem + C::STAGES * C::A_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + C::STAGES * C::STAGE_BYTES);
  uint64_t* empty = full + C::STAGES;
  uint64_t* tfull = empty + C::STAGES;   // [2]
  uint64_t* tempty = tfull + 2;          // [2]
  uint64_t* drain = tempty + 2;          // [2]: an issuer's MMAs have all completed
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(drain + 2);
  volatile uint32_t* seen = tmem_holder + 2;   // [STAGES]: see ring_round_wait

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < C::STAGES; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); seen[s] = 0; }
    for (int a = 0; a < 2; ++a) { mbar_init(&tfull[a], 2); mbar_init(&tempty[a], 4); mbar_init(&drain[a], 1); }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 0 && lane == 0)
    for (int i = 0; i < 4; ++i) { tma_prefetch_desc(&P.tA[i]); tma_prefetch_desc(&P.tB[i]); }
  if (warp == 1) tmem_alloc(tmem_holder, C::TMEM_COLS);
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  if (warp == 0) {
    // ---------------- TMA producer (lane 0 issues; the warp polls flags) ----------------
    uint32_t it = 0;
    bool ok = true;
    for_my_tasks(P, [&](int ph, int j, int loc, int gi) -> bool {
      if (ph >= PH_FOLD) return true;
      if (lane == 0) note_progress(P, 0, ph, j, loc);
      if (lane == 0) trace_ev(P, gi, 0);
      const GemmPhase& g = P.g[ph];
      const GemmTask T = decode_gemm(g, loc);
      const bool deps = !(ph == PH_WO && j == P.j0);   // a of the first step comes from an earlier kernel
      const int dph = dep_phase(ph);
      const unsigned target = ph == PH_WO ? (unsigned)j : (unsigned)(j + 1);
      int flo = 0, fhi = 0, tmp;
      if (deps) {
        slice_flags(P, ph, T.sl0, flo, tmp);
        slice_flags(P, ph, T.sl1 - 1, tmp, fhi);
      }
      // The weight (B) halves of the first ring stages are loaded before the
      // dependencies are seen (weights are never written here); then the
      // lanes poll every flag the task's A operand depends on at once, one
      // fence orders those writes before the async-proxy loads, and the A
      // halves follow.
      const uint32_t bn_bytes = (uint32_t)g.BN * C::BK * 2;
      const int nst = (T.sl1 - T.sl0 + C::KSUB - 1) / C::KSUB;
      const int pre = deps ? min(nst, C::STAGES) : 0;
      auto take_slot = [&](int k) -> bool {   // wait for stage k's slot, then arm it and load its B half
        const uint32_t ik = it + k, s = ik % C::STAGES, par = (ik / C::STAGES) & 1u;
        const int kb = T.sl0 + k * C::KSUB, ns = min(C::KSUB, T.sl1 - kb);
        int w = 1;
        if (lane == 0) note_wait(P, 0, 1, ik);
        if (lane == 0) w = mbar_wait_g(&empty[s], par ^ 1u, P.err, 41, wait_site(ph, j, loc)) ? 1 : 0;
        w = __shfl_sync(0xffffffffu, w, 0);
        if (!w) return false;
        if (lane == 0) {
          trace_ev(P, gi, 16 + min(k, 15));
          mbar_arrive_expect_tx(&full[s], ns * (C::A_SUB + bn_bytes));
          for (int q = 0; q < ns; ++q)
            if (idx_ok((kb + q + 1) * C::BK <= g.K && (T.tile + 1) * g.BN <= g.N && s < (uint32_t)C::STAGES &&
                           g.BN <= C::BN_MAX, P.err, 11, kb + q, T.tile))
              tma_load_2d(&P.tB[ph], &full[s], sB + s * C::B_BYTES + q * C::B_SUB, (kb + q) * C::BK, T.tile * g.BN);
        }
        return true;
      };
      auto load_a = [&](int k) {
        const uint32_t ik = it + k, s = ik % C::STAGES;
        const int kb = T.sl0 + k * C::KSUB, ns = min(C::KSUB, T.sl1 - kb);
        if (lane == 0)
          for (int q = 0; q < ns; ++q)
            if (idx_ok((kb + q + 1) * C::BK <= g.K && T.rb * C::BM < P.ep.B, P.err, 12, kb + q, T.rb))
              tma_load_2d(&P.tA[ph], &full[s], sA + s * C::A_BYTES + q * C::A_SUB, (kb + q) * C::BK, T.rb * C::BM);
      };
      // (an abort leaves no armed stage without its A half, so that every
      // copy in flight completes its barrier before the CTA exits)
      for (int k = 0; k < pre; ++k)
        if (!take_slot(k)) {
          for (int q = 0; q < k; ++q) load_a(q);
          it += k;
          ok = false;
          return false;
        }
      if (deps) {
        if (lane == 0) note_wait(P, 0, 2, it);
        for (int f = flo + lane; f < fhi; f += 32)
          poll_ge(flag_ptr(P, dph, T.rb, f), target, P.err, 42, wait_site(ph, j, f));
        __syncwarp();
        if (lane == 0) fence_proxy_async_global();
        if (lane == 0) trace_ev(P, gi, 32);
      }
      for (int k = 0; k < pre; ++k) load_a(k);
      for (int k = pre; k < nst; ++k) {
        if (!take_slot(k)) {
          it += k;
          ok = false;
          return false;
        }
        load_a(k);
      }
      it += nst;
      if (lane == 0) trace_ev(P, gi, 1);
      return true;
    });
    if (!ok && lane == 0) {
      // wait (bounded) for copies still in flight before the CTA can exit
      const uint32_t first = it > (uint32_t)C::STAGES ? it - C::STAGES : 0u;
      for (uint32_t i = first; i < it; ++i) mbar_wait(&full[i % C::STAGES], (i / C::STAGES) & 1u, P.err);
    }
  } else if (warp == 1 || warp == 2) {
    // ---------------- MMA issuers: stage kb of a task goes to issuer kb % 2 ----------------
    const int par = warp - 1;
    if (lane == 0) {
      uint32_t it = 0, local = 0;
      for_my_tasks(P, [&](int ph, int j, int loc, int gi) -> bool {
        if (ph >= PH_FOLD) return true;
        note_progress(P, 1 + par, ph, j, loc);
        const GemmPhase& g = P.g[ph];
        const GemmTask T = decode_gemm(g, loc);
        const int nst = (T.sl1 - T.sl0 + C::KSUB - 1) / C::KSUB;
        const uint32_t acc = local & 1u, aph = (local >> 1) & 1u;
        ++local;
        note_wait(P, 1 + par, 3, local - 1);
        if (!mbar_wait_g(&tempty[acc], aph ^ 1u, P.err, 43, wait_site(ph, j, loc))) return false;
        trace_ev(P, gi, 2 + par);
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + (acc * 2 + par) * C::BN_MAX;
        idx_ok((acc * 2 + par) * C::BN_MAX + g.BN <= C::TMEM_COLS && nst >= 1, P.err, 13, acc, nst);
        const uint32_t idesc = idesc_bf16_f32(C::BM, g.BN);
        uint32_t accumulate = 0;
        for (int kb = 0; kb < nst; ++kb, ++it) {
          if ((kb & 1) != par) continue;
          const uint32_t s = it % C::STAGES, sp = (it / C::STAGES) & 1u;
          note_wait(P, 1 + par, 6, it);
          if (!ring_round_wait(&seen[s], it / C::STAGES, P.err, 48, wait_site(ph, j, loc))) return false;
          note_wait(P, 1 + par, 4, it);
          if (!mbar_wait_g(&full[s], sp, P.err, 44, wait_site(ph, j, loc))) return false;
          seen[s] = it / C::STAGES + 1;
          trace_ev(P, gi, 48 + min(kb, 15));
          tc_fence_after();
          const uint8_t* a_st = sA + s * C::A_BYTES;
          const uint8_t* b_st = sB + s * C::B_BYTES;
          const int nmma = min(C::KSUB, T.sl1 - T.sl0 - kb * C::KSUB) * (C::BK / 16);
#pragma unroll
          for (int k = 0; k < C::KSUB * (C::BK / 16); ++k) {
            if (k >= nmma) break;
            const int q = k / (C::BK / 16), kk = k % (C::BK / 16);
            tc_mma_f16(d_tmem, smem_desc_sw128(a_st + q * C::A_SUB + kk * 32),
                       smem_desc_sw128(b_st + q * C::B_SUB + kk * 32), idesc, accumulate);
            accumulate = 1u;
          }
          tc_commit(&empty[s]);
        }
        tc_commit(&tfull[acc]);   // with no stage of its own in this task it arrives at once
        trace_ev(P, gi, 4 + par);
        return true;
      });
      // every MMA this thread issued has completed before the CTA frees TMEM
      tc_commit(&drain[par]);
      mbar_wait(&drain[par], 0u, P.err);
    }
  } else if (warp < 7) {
    // ---------------- epilogue warps: the GEMM epilogues ----------------
    const int tid = threadIdx.x - 96;   // 0..127
    const int q = warp & 3;             // TMEM lanes 32q .. 32q + 31
    const int lrow = q * 32 + lane;
    uint32_t local = 0;
    for_my_tasks(P, [&](int ph, int j, int loc, int gi) -> bool {
      if (ph >= PH_FOLD) return true;   // the fold warps' tasks
      if (tid == 0) note_progress(P, 3, ph, j, loc);
      if (tid == 0) trace_ev(P, gi, 6);
      const GemmPhase& g = P.g[ph];
      const GemmTask T = decode_gemm(g, loc);
      const int nst = (T.sl1 - T.sl0 + C::KSUB - 1) / C::KSUB;
      const uint32_t acc = local & 1u, aph = (local >> 1) & 1u;
      ++local;
      const int row = T.rb * C::BM + lrow;
      const int col_base = T.tile * g.BN;
      const bool row_ok = row < P.ep.B &&
                          idx_ok(T.rb < P.nrb && col_base + g.BN <= g.N && T.sl1 <= g.K / 64 && j < P.ep.Nseq, P.err);
      // dependencies of what this epilogue reads or overwrites (see the file comment)
      if (ph == PH_WO) {
        if (j > P.j0) epi_poll_range(P, PH_FOLD, T.rb, 0, P.H * P.G, (unsigned)j, tid);
      } else if (ph == PH_W1) {
        epi_poll_range(P, PH_WO, T.rb, 0, P.g[PH_WO].tiles, (unsigned)(j + 1), tid);
      } else if (ph == PH_W2) {
        epi_poll_range(P, PH_WO, T.rb, 0, P.g[PH_WO].tiles, (unsigned)(j + 1), tid);   // the residual u
      } else {
        epi_poll_range(P, PH_W2, T.rb, 0, phase_flags(P.g[PH_W2]), (unsigned)(j + 1), tid);
      }
      epi_bar();
      if (tid == 0) trace_ev(P, gi, 7);
      EpiParams e = P.ep;
      e.j = j;
      float rs = 1.f;
      if (ph == PH_W1) {
        e.ssq_in = P.ssq_u; e.ssq_tiles = P.g[PH_WO].tiles;
        if (row_ok) rs = row_scale_for<EPI_W1>(e, row);
      } else if (ph == PH_WKV) {
        e.ssq_in = P.ssq_z; e.ssq_tiles = phase_flags(P.g[PH_W2]);
        if (row_ok) rs = row_scale_for<EPI_WKV>(e, row);
      }
      // W_o: the residual x (an input of the layer, never written here) is
      // loaded now, while the tile's MMAs run
      const bool wo64 = ph == PH_WO && g.BN == 64;
      // a W_2 split finishes 32 columns: their residual u, loaded now as well
      const bool w2pre = ph == PH_W2 && g.S > 1 && flag_cols(g) == 32;
      uint4 xw[8];   // W_o: 64 bf16 of x; a W_2 split: 32 fp32 of u (their bits)
#pragma unroll
      for (int i = 0; i < 8; ++i) xw[i] = make_uint4(0, 0, 0, 0);
      if (w2pre && row_ok) {
        const uint4* up = reinterpret_cast<const uint4*>(P.ep.u32 + (size_t)row * P.ep.d + col_base + T.split * 32);
#pragma unroll
        for (int i = 0; i < 8; ++i) xw[i] = __ldcg(up + i);
      } else if (wo64 && row_ok) {
        const int b = row % P.ep.B, jj = j + row / P.ep.B, ch = jj / P.ep.xc;
        const uint4* xp = reinterpret_cast<const uint4*>(
            P.ep.x + (((size_t)ch * P.ep.B + b) * P.ep.xc + (jj - ch * P.ep.xc)) * P.ep.d + col_base);
#pragma unroll
        for (int i = 0; i < 8; ++i) xw[i] = __ldg(xp + i);
      } else if (row_ok && ph == PH_WO) {
        epilogue_prefetch<EPI_WO>(e, row, col_base, g.N, g.BN);
      }
      // A wait that gives up (error word set) does not end the task: the four
      // epilogue warps must reach every named barrier together, so they run
      // on with whatever tensor memory holds.
      if (tid == 0) note_wait(P, 3, 5, local - 1);
      if (lane == 0) mbar_wait_g(&tfull[acc], aph, P.err, 45, wait_site(ph, j, loc));
      if (tid == 0) trace_ev(P, gi, 8);
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + acc * 2 * C::BN_MAX;
      const bool two = nst >= 2;
      const int fu = T.tile * g.S + T.split;   // the flag (and Σ² unit) this task finishes
      if (g.S == 1) {
        float ssq = 0.f;
        switch (ph) {
          case PH_WO:
            ssq = wo64 ? epi_wo_tile64(e, row, row_ok, col_base, taddr, two, xw, P.err)
                       : epi_tile_tmem<EPI_WO>(e, row, row_ok, col_base, g.BN, taddr, two, rs, P.err, P, gi);
            break;
          case PH_W1: epi_tile_tmem<EPI_W1>(e, row, row_ok, col_base, g.BN, taddr, two, rs, P.err, P, gi); break;
          case PH_W2: ssq = epi_tile_tmem<EPI_W2>(e, row, row_ok, col_base, g.BN, taddr, two, rs, P.err, P, gi); break;
          default: epi_tile_tmem<EPI_WKV>(e, row, row_ok, col_base, g.BN, taddr, two, rs, P.err, P, gi); break;
        }
        if (row_ok && ph == PH_WO && idx_ok(T.tile <= P.ep.d / 32, P.err, 15, T.tile, 0))
          P.ssq_u[(size_t)T.tile * P.ep.B + row] = ssq;
        if (row_ok && ph == PH_W2 && idx_ok(fu <= P.ep.d / 32, P.err, 15, fu, 1))
          P.ssq_z[(size_t)fu * P.ep.B + row] = ssq;
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
      } else {
        // split of W2: this split's partial tile to its slot ([col][row], so
        // that a warp's stores and loads are 128-byte lines)
        const size_t tile_i = (size_t)T.rb * g.tiles + T.tile;
        const size_t slot_i = tile_i * g.S + T.split;
        idx_ok(slot_i < (size_t)P.nrb * g.tiles * g.S && T.split < g.S, P.err, 14, (long long)slot_i, T.split);
        float* slot = P.w2part + slot_i * (size_t)g.BN * C::BM;
#pragma unroll 1
        for (int c = 0; c < g.BN; c += 32) {
          float v[32];
          tmem_ld_pair(taddr + c, two, v);
#pragma unroll
          for (int i = 0; i < 32; ++i) slot[(size_t)(c + i) * C::BM + lrow] = v[i];
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&tempty[acc]);
        if (tid == 0) trace_ev(P, gi, 12);
        epi_bar();
        // Every split of the tile has written its slot once the tile's
        // arrival count reaches S (j + 1). The S splits run on S different
        // CTAs at about the same time, and each then sums its 1 / S of the
        // tile's columns over the S slots (in split order: deterministic)
        // and runs the W2 epilogue on them. (The wait ends: a split's
        // arrival needs only its own MMAs and earlier tasks of its CTA, and
        // those never wait on this phase of this step.)
        if (tid == 0) {
          unsigned* cnt = P.w2cnt + tile_i;
          __threadfence();   // the CTA's slot stores (ordered before by the barrier)
          atom_add_acq_rel(cnt, 1u);
          poll_ge(cnt, (unsigned)(g.S * (j + 1)), P.err, 49, wait_site(ph, j, loc));
        }
        epi_bar();
        if (tid == 0) trace_ev(P, gi, 13);
        const int fc = flag_cols(g), c0 = T.split * fc;
        const float* slots = P.w2part + tile_i * g.S * (size_t)g.BN * C::BM;
        float ssq = 0.f;
#pragma unroll 1
        for (int c = c0; c < c0 + fc; c += 32) {
          float v[32];
#pragma unroll
          for (int i = 0; i < 32; ++i) v[i] = 0.f;
          for (int sp = 0; sp < g.S; ++sp) {
            const float* src = slots + (size_t)sp * g.BN * C::BM + (size_t)c * C::BM + lrow;
#pragma unroll
            for (int i = 0; i < 32; ++i) v[i] += __ldcg(src + (size_t)i * C::BM);
          }
          if (tid == 0 && c == c0) trace_ev(P, gi, 14);
          if (w2pre) ssq += epi_w2_chunk_pre(e, row, row_ok, col_base + c, v, xw, P.err);
          else if (row_ok) ssq += epilogue_chunk<EPI_W2>(e, row, col_base + c, g.N, v, 1.f, P.err);
        }
        if (row_ok && idx_ok(fu <= P.ep.d / 32, P.err, 15, fu, 2)) P.ssq_z[(size_t)fu * P.ep.B + row] = ssq;
      }
      // every thread's stores are issued; after the epilogue barrier one
      // thread fences (also toward the async proxy: the next phase reads
      // these outputs with TMA) and releases the flag
      if (tid == 0) trace_ev(P, gi, 10);
      epi_bar();
      if (tid == 0) {
        fence_proxy_async_global();
        __threadfence();
        trace_ev(P, gi, 11);
        if (release_allowed(P)) st_release_u32(flag_ptr(P, ph, T.rb, fu), (unsigned)(j + 1));
      }
      if (tid == 0) trace_ev(P, gi, 9);
      return true;
    });
  } else {
    // ---------------- fold warps: the small folds (FOLD and DEFER tasks) ----------------
    const int ftid = threadIdx.x - 224;   // 0..127
    FoldUnitArgs fa;
    fa.B = P.ep.B; fa.H = P.H; fa.d = P.ep.d; fa.Nseq = P.ep.Nseq;
    fa.K = P.ep.Kout; fa.V = P.ep.Vout; fa.qkv = P.qkv;
    fa.m = P.m; fa.l = P.l; fa.o = P.o; fa.a16 = P.a16; fa.sc2 = P.sc2; fa.err = P.err;
    for_my_tasks(P, [&](int ph, int j, int loc, int gi) -> bool {
      if (ph < PH_FOLD) return true;
      if (ftid == 0) note_progress(P, 4, ph, j, loc);
      if (ftid == 0) trace_ev(P, gi, 6);
      // FOLD (step j, t = j + 1): the block's keys into its first query t,
      // which is finalised (a_t, read by the next step's W_o). DEFER (step
      // j, t = j): the same block of the previous step into its other
      // queries t + 1 .. t + nq - 1, off the critical path; the fold of
      // step j (query t + 1 = j + 1) waits for it.
      const bool urgent = ph == PH_FOLD;
      const int per_rb = P.H * P.G;
      const int rb = loc / per_rb, r = loc - rb * per_rb;
      const int h = r / P.G, gq = r - h * P.G;
      const int t = urgent ? j + 1 : j, lb = lowbit(t), nq = min(lb, P.ep.Nseq - t);
      const unsigned kv_ready = urgent ? (unsigned)(j + 1) : (unsigned)j;   // k, v of position t - 1
      // this head's k and v of step t - 1 (and, through them, everything before)
      const int kt = (64 * h) / P.g[PH_WKV].BN, vt = (P.ep.d + 64 * h) / P.g[PH_WKV].BN;
      if (ftid == 0) poll_ge(flag_ptr(P, PH_WKV, rb, kt), kv_ready, P.err, 47, wait_site(ph, j, kt));
      if (ftid == 32) poll_ge(flag_ptr(P, PH_WKV, rb, vt), kv_ready, P.err, 47, wait_site(ph, j, vt));
      if (urgent && ftid == 64 && phase_tasks(P, PH_DEFER, j) > 0)
        poll_ge(flag_ptr(P, PH_DEFER, rb, r), (unsigned)(j + 1), P.err, 50, wait_site(ph, j, r));
      fold_bar();
      if (ftid == 0) trace_ev(P, gi, 7);
      const int s0 = rb * 128 + gq * kFoldSeqs;
      const int ns = min(kFoldSeqs, min(P.ep.B - s0, (rb + 1) * 128 - s0));
      const int init = t == lb ? 1 : 0;
      if (ns > 0 && urgent && nq > 0) {
        switch (lb) {
          case 1: fold_units<1, 2>(fa, t, 1, t - 1, init, h, s0, ns, ftid, 1); break;
          case 2: fold_units<2, 2>(fa, t, 1, t - 2, init, h, s0, ns, ftid, 1); break;
          case 4: fold_units<4, 2>(fa, t, 1, t - 4, init, h, s0, ns, ftid, 1); break;
          default: fold_units<8, 1>(fa, t, 1, t - 8, init, h, s0, ns, ftid, 1); break;
        }
      } else if (ns > 0 && !urgent && nq > 1) {
        switch (lb) {
          case 2: fold_units<2, 2>(fa, t + 1, nq - 1, t - 2, init, h, s0, ns, ftid, 0); break;
          case 4: fold_units<4, 2>(fa, t + 1, nq - 1, t - 4, init, h, s0, ns, ftid, 0); break;
          default: fold_units<8, 1>(fa, t + 1, nq - 1, t - 8, init, h, s0, ns, ftid, 0); break;
        }
      }
      if (ftid == 0) trace_ev(P, gi, 10);
      fold_bar();
      if (ftid == 0) {
        fence_proxy_async_global();   // a is read by the next step's TMA loads
        __threadfence();
        trace_ev(P, gi, 11);
        if (release_allowed(P)) st_release_u32(flag_ptr(P, ph, rb, r), (unsigned)(j + 1));
      }
      if (ftid == 0) trace_ev(P, gi, 9);
      return true;
    });
  }
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace rt
