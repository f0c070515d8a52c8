// rt_common.cuh -- shared device helpers of librtlayer (sm_100a only).
//
// Every spin-wait in this library is bounded by a wall-clock limit read from
// %globaltimer. A wait that runs out records RT_DEVERR_TIMEOUT in the
// caller's error word and returns false; the kernel then unwinds without
// issuing further work.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#if defined(__CUDA_ARCH__) && (__CUDA_ARCH__ < 1000)
#error "librtlayer is written for sm_100a (B200) only"
#endif

namespace rt {

// device error word bits
enum : unsigned { RT_DEVERR_TIMEOUT = 1u, RT_DEVERR_INDEX = 2u };

// 2 s per wait: far above any legitimate wait in these kernels.
constexpr unsigned long long kWaitLimitNs = 2000000000ull;

constexpr float kLog2e = 1.4426950408889634f;

__host__ __device__ inline int lowbit(int t) { return t & (-t); }

__device__ __forceinline__ unsigned long long globaltimer() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ void set_error(unsigned* err, unsigned bits) {
  if (err) atomicOr(err, bits);
}

// Debug build (compiled with -DRT_BOUNDS_CHECK, library librtlayer_check.so):
// the global indexes the layer's kernels compute are checked against the
// ranges their arguments declare; a failed check records RT_DEVERR_INDEX in
// the error word (rt_layer_sync_status then returns RT_ERR_INVALID_ARG) and
// the access is skipped. Nothing traps. In the normal build the check is the
// constant true and compiles away.
// The first failed check also leaves a record after the error word: word 1 =
// the check's id (1-based), words 2 and 3 = two of its values (the caller's
// error word must have room for four words; the layer's workspace reserves
// 256 bytes).
#ifdef RT_BOUNDS_CHECK
__device__ __forceinline__ bool idx_ok(bool ok, unsigned* err, unsigned id = 0, long long a = 0,
                                       long long b = 0) {
  if (!ok) {
    set_error(err, RT_DEVERR_INDEX);
    if (err && id && atomicCAS(err + 1, 0u, id) == 0u) {
      err[2] = (unsigned)a;
      err[3] = (unsigned)b;
    }
  }
  return ok;
}
// (debug build) the first bounded wait that ran out leaves the same kind of
// record: id, then two values describing the wait
__device__ __forceinline__ void timeout_record(unsigned* err, unsigned id, long long a, long long b) {
  if (err && atomicCAS(err + 1, 0u, id) == 0u) {
    err[2] = (unsigned)a;
    err[3] = (unsigned)b;
  }
}
#else
__device__ __forceinline__ constexpr bool idx_ok(bool, unsigned*, unsigned = 0, long long = 0, long long = 0) {
  return true;
}
__device__ __forceinline__ void timeout_record(unsigned*, unsigned, long long, long long) {}
#endif

// ---------------------------------------------------------------------------
// programmatic dependent launch: a kernel launched with programmatic stream
// serialisation may start while its predecessor runs; it must call
// pdl_wait() before touching anything the predecessor writes, and every
// kernel calls it before it can finish so that completion stays transitive.
// Both are no-ops for a normal launch.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------------------
// small numeric helpers
// ---------------------------------------------------------------------------
__device__ __forceinline__ float to_f(float v) { return v; }
__device__ __forceinline__ float to_f(__nv_bfloat16 v) { return __bfloat162float(v); }
template <class T> __device__ __forceinline__ T from_f(float v);
template <> __device__ __forceinline__ float from_f<float>(float v) { return v; }
template <> __device__ __forceinline__ __nv_bfloat16 from_f<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

// exact GELU, y * Phi(y)
__device__ __forceinline__ float gelu_erf(float y) {
  return 0.5f * y * (1.0f + erff(y * 0.70710678118654752f));
}

// erf by the rational approximation of Abramowitz & Stegun, Handbook of
// Mathematical Functions, formula 7.1.26 (|error| <= 1.5e-7 for x >= 0; erf
// is odd): erf(x) = 1 - t (a1 + t (a2 + t (a3 + t (a4 + t a5)))) exp(-x^2),
// t = 1 / (1 + p x). One reciprocal and one base-2 exponential (the PTX
// approximate instructions) and six FMAs.
__device__ __forceinline__ float erf_as7126(float x) {
  const float ax = fabsf(x);
  float t;
  asm("rcp.approx.ftz.f32 %0, %1;" : "=f"(t) : "f"(fmaf(0.3275911f, ax, 1.f)));
  float poly = fmaf(t, 1.061405429f, -1.453152027f);
  poly = fmaf(t, poly, 1.421413741f);
  poly = fmaf(t, poly, -0.284496736f);
  poly = fmaf(t, poly, 0.254829592f);
  poly *= t;
  float e;   // exp(-x^2) = 2^(-x^2 log2 e)
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(e) : "f"(-ax * ax * 1.44269504088896341f));
  return copysignf(fmaf(-poly, e, 1.f), x);
}
// GELU with that erf: the layer's bf16 path (its outputs are bf16-rounded,
// 2^-9 relative, far above the approximation's error)
__device__ __forceinline__ float gelu_as7126(float y) {
  return 0.5f * y * (1.0f + erf_as7126(y * 0.70710678118654752f));
}

// eight bf16 (one 16-byte word) to float
__device__ __forceinline__ void unpack_bf16x8(const uint4& w, float (&v)[8]) {
  const __nv_bfloat162* p = reinterpret_cast<const __nv_bfloat162*>(&w);
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const float2 f = __bfloat1622float2(p[k]);
    v[2 * k] = f.x;
    v[2 * k + 1] = f.y;
  }
}

// 2^x on the special-function unit, results below 2^-126 flushed to zero
// (ex2(-inf) = +0). For softmax weights of bf16 folds: a weight that small
// is negligible against the row's largest (>= 2^-8 of the reference).
__device__ __forceinline__ float ex2_ftz(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

// scale of an empty accumulator: exp2(m_old - m_new) with m_old = -inf -> 0
__device__ __forceinline__ float rescale(float m_old, float m_new) {
  return (m_old == -INFINITY) ? 0.f : exp2f(m_old - m_new);
}

// ---------------------------------------------------------------------------
// shared-memory mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, unsigned count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, unsigned bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, unsigned parity) {
  unsigned ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Bounded wait for the phase with the given parity to complete.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, unsigned parity, unsigned* err,
                                          unsigned long long limit_ns = kWaitLimitNs) {
  if (mbar_try_wait(bar, parity)) return true;
  const unsigned long long t0 = globaltimer();
  for (unsigned it = 0;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 255u && globaltimer() - t0 > limit_ns) {
      set_error(err, RT_DEVERR_TIMEOUT);
      return false;
    }
  }
}

// ---------------------------------------------------------------------------
// flags in global memory between CTAs of one kernel
// ---------------------------------------------------------------------------
__device__ __forceinline__ unsigned ld_acquire_u32(const unsigned* p) {
  unsigned v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}
__device__ __forceinline__ void st_release_u32(unsigned* p, unsigned v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(p), "r"(v) : "memory");
}
__device__ __forceinline__ unsigned atom_add_acq_rel(unsigned* p, unsigned v) {
  unsigned old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(p), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ unsigned ld_volatile_u32(const unsigned* p) {
  return *reinterpret_cast<const volatile unsigned*>(p);
}
// Bounded poll until *f >= target (acquire). Returns at once once the error
// word is set; a poll that runs out sets RT_DEVERR_TIMEOUT. Either way the
// caller proceeds.
// (debug build: a wait that runs out records `id` and `where`, and the value
// it saw, after the error word)
static __device__ __noinline__ void poll_ge(const unsigned* f, unsigned target, unsigned* err, unsigned id = 0,
                                     long long where = 0) {
  if (ld_acquire_u32(f) >= target) return;
  const unsigned long long t0 = globaltimer();
  for (unsigned it = 1;; ++it) {
    __nanosleep(64);
    const unsigned v = ld_acquire_u32(f);
    if (v >= target) return;
    if ((it & 15u) == 0) {
      if (err && ld_volatile_u32(err) != 0) return;
      if (globaltimer() - t0 > kWaitLimitNs) {
        set_error(err, RT_DEVERR_TIMEOUT);
        timeout_record(err, id, where, ((long long)v << 16) | (target & 0xffff));
        return;
      }
    }
  }
}

// Rings consumed by two issuers that take alternate stages: the previous
// round of a slot may belong to the other issuer, and if that round's copy
// has not landed yet when this issuer reaches the slot, a parity wait for
// the slot's next round reads the pending phase as "the one before" and
// passes with the wrong data. So each issuer records, per slot, the last
// round whose data it saw land (seen[s] = round + 1), and before waiting on a
// slot's barrier for round r an issuer waits (bounded) for seen[s] >= r. The
// barrier is then exactly one phase from round r, which the parity tells
// apart.
// (debug build: a wait that runs out records `id` and `where`)
__device__ __forceinline__ bool ring_round_wait(const volatile uint32_t* seen, uint32_t round, unsigned* err,
                                                unsigned id = 0, long long where = 0,
                                                unsigned long long limit_ns = kWaitLimitNs) {
  if (*seen >= round) return true;
  const unsigned long long t0 = globaltimer();
  for (unsigned it = 0;; ++it) {
    if (*seen >= round) return true;
    if ((it & 255u) == 255u) {
      if (*reinterpret_cast<volatile unsigned*>(err) != 0) return false;
      if (globaltimer() - t0 > limit_ns) {
        set_error(err, RT_DEVERR_TIMEOUT);
        if (id) timeout_record(err, id, where, round);
        return false;
      }
    }
  }
}

// ---------------------------------------------------------------------------
// TMA (tiled, no multicast)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* m) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(m)) : "memory");
}

// 2-D tile load; c0 = innermost (element) coordinate, c1 = row coordinate.
__device__ __forceinline__ void tma_load_2d(const CUtensorMap* m, uint64_t* bar, void* dst, int c0,
                                            int c1) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4}], [%2];" ::"r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(m)), "r"(smem_u32(bar)), "r"(c0), "r"(c1)
      : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05 (5th-generation tensor cores, accumulators in tensor memory)
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, unsigned ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, unsigned ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 inputs, fp32 accumulate)
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// mbarrier arrives once all previously issued tcgen05 ops of this thread complete
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// 32 lanes x 32 columns of 32-bit: thread i of the warp gets row (lane base + i),
// columns [col, col + 32).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// the inverse: thread i writes row (lane base + i), columns [col, col + 32)
__device__ __forceinline__ void tmem_st_32x32b_x32(uint32_t taddr, const uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16,"
      "%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"
      ::"r"(taddr), "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
        "r"(r[7]), "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15]), "r"(r[16]), "r"(r[17]), "r"(r[18]), "r"(r[19]), "r"(r[20]), "r"(r[21]), "r"(r[22]),
        "r"(r[23]), "r"(r[24]), "r"(r[25]), "r"(r[26]), "r"(r[27]), "r"(r[28]), "r"(r[29]), "r"(r[30]),
        "r"(r[31])
      : "memory");
}
__device__ __forceinline__ void tmem_st_wait() { asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory"); }

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// Shared-memory matrix descriptor, K-major operand with 128-byte swizzle:
// rows of 128 bytes (64 bf16), 8-row swizzle atoms 1024 bytes apart.
__device__ __forceinline__ uint64_t smem_desc_sw128(const void* p) {
  const uint32_t a = smem_u32(p);
  uint64_t d = 0;
  d |= (uint64_t)((a >> 4) & 0x3FFFu);         // start address
  d |= (uint64_t)1u << 16;                     // leading byte offset (unused for SW128 K-major)
  d |= (uint64_t)(1024u >> 4) << 32;           // stride byte offset: 8 rows x 128 B
  d |= (uint64_t)1u << 46;                     // descriptor version (sm_100)
  d |= (uint64_t)2u << 61;                     // layout: 128-byte swizzle
  return d;
}

// Instruction descriptor, kind::f16: bf16 A and B (both K-major), fp32 D.
__host__ __device__ constexpr uint32_t idesc_bf16_f32(int M, int N) {
  return (1u << 4)                       // D format F32
         | (1u << 7)                     // A format BF16
         | (1u << 10)                    // B format BF16
         | ((uint32_t)(N >> 3) << 17)    // N / 8
         | ((uint32_t)(M >> 4) << 24);   // M / 16
}

}  // namespace rt
