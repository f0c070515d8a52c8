// rt_api.cu -- host side of librtlayer: argument validation, workspace plan,
// TMA descriptors, the N-step driver (host loop or one CUDA-graph replay) and
// the extern "C" entry points declared in include/rtlayer.h.
//
// One forward of the Recurrent Transformer layer ("Recurrent Transformer"
// paper page, www.lshu.cn/news/403416, paper §2.2 and notes §4.2):
//   1. inv_rms(x) for all B*N rows; batched projection QKV = [W_q;W_k;W_v] rms(x)
//      (queries and temporary pairs of every position, position-major);
//   2. for t = 1..N (j = t-1):
//        finalise a_j (temporary-pair merge, a = o/l)      [naive: full attention]
//        u = x_j + a W_o^T ; h = GELU(rms(u) W_1^T) ; z_j = u + h W_2^T
//        (k_j, v_j) = rms(z_j) [W_k; W_v]^T  -> position-major K, V
//        fold keys (t - lb, t] into queries (t, t + lb], lb = lowbit(t)   [blocked only]
// No accumulator initialisation pass: at t = 2^k the block (0, t] x (t, 2t] is
// the first fold into each of its queries, so those folds write (m, l, o)
// without reading them, and position 1 is never folded into.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <map>
#include <mutex>
#include <vector>

#include "../../include/rtlayer.h"
#include "rt_attn.cuh"
#include "rt_common.cuh"
#include "rt_fold_tc.cuh"
#include "rt_gemm_tc.cuh"
#include "rt_host.h"
#include "rt_simt.cuh"
#include "rt_steps.cuh"

namespace rt {

typedef __nv_bfloat16 bf16;

// The CUDA error behind the calling thread's last RT_ERR_CUDA status
// (rt_last_cuda_error reads it).
static thread_local int g_last_cuda_error = 0;
int cuda_failure(cudaError_t e) {
  g_last_cuda_error = (int)e;
  return RT_ERR_CUDA;
}
#define RT_CK(call)                                  \
  do {                                               \
    cudaError_t e_ = (call);                         \
    if (e_ != cudaSuccess) return cuda_failure(e_);  \
  } while (0)

static inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// Launch with programmatic stream serialisation: the kernel may start while the
// previous kernel in the stream runs; every kernel calls pdl_wait() before it
// reads its predecessor's outputs.
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl_cluster(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                                      int cluster, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute at[2];
  at[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  at[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.numAttrs = 1;
  if (cluster > 1) {
    at[1].id = cudaLaunchAttributeClusterDimension;
    at[1].val.clusterDim.x = cluster;
    at[1].val.clusterDim.y = 1;
    at[1].val.clusterDim.z = 1;
    cfg.numAttrs = 2;
  }
  cfg.attrs = at;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}
template <typename... KArgs, typename... Args>
static cudaError_t launch_pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                              Args&&... args) {
  return launch_pdl_cluster(kern, grid, block, smem, st, 1, std::forward<Args>(args)...);
}

// The persistent step kernel: one CTA per SM, all co-resident, since its
// tasks wait on flags set by other CTAs. The launch is cooperative (the
// driver guarantees co-residency or refuses); `coop` = false launches the
// same grid plainly -- one CTA per SM fits (shared memory allows no second)
// and the previous kernel of the stream has finished, so the CTAs are
// resident together in practice, and every wait is bounded regardless.
#ifdef RT_TRACE
// (trace build) the segment starting at step g_trace_j0 records its task
// events into g_trace (kTraceSlots times per task), if it has room for them
static unsigned long long* g_trace = nullptr;
static size_t g_trace_bytes = 0;
static int g_trace_j0 = -1;
extern "C" void rt_debug_trace_segment(void* buf, size_t bytes, int j0) {
  g_trace = static_cast<unsigned long long*>(buf);
  g_trace_bytes = bytes;
  g_trace_j0 = j0;
}
#endif
static cudaError_t launch_steps(const StepsParams& sp_in, int sms, cudaStream_t st, bool coop) {
  StepsParams sp = sp_in;
#ifdef RT_TRACE
  if (g_trace && sp.j0 == g_trace_j0) {
    size_t tasks = 0;
    for (int j = sp.j0; j < sp.j1; ++j) {
      for (int ph = 0; ph < 4; ++ph) tasks += (size_t)sp.nrb * sp.g[ph].tiles * sp.g[ph].S;
      if (j + 1 < sp.j1) tasks += (size_t)sp.nrb * sp.H * sp.G;
    }
    if (tasks * kTraceSlots * 8 <= g_trace_bytes) sp.trace = g_trace;
  }
#endif
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3((unsigned)sms);
  cfg.blockDim = dim3(StepsCfg::THREADS);
  cfg.dynamicSmemBytes = StepsCfg::SMEM_BYTES;
  cfg.stream = st;
  cudaLaunchAttribute at[1];
  at[0].id = cudaLaunchAttributeCooperative;
  at[0].val.cooperative = 1;
  cfg.attrs = at;
  cfg.numAttrs = coop ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, k_steps, sp);
}

// ---------------------------------------------------------------------------
// device set-up
// ---------------------------------------------------------------------------
typedef CUresult (*PFN_encodeTiled_t)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                      const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                      const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                      CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DevState {
  bool ready = false;
  int sms = 0;
  // the step kernel's launches are cooperative unless this device's driver
  // refused a cooperative launch (then plain, see launch_steps)
  bool coop = true;
  cudaStream_t capture = nullptr;
  cudaStream_t h2d = nullptr, d2h = nullptr;   // transfer streams of the host-buffer entry point
  std::vector<cudaEvent_t> events;             // fork/join events of the host-buffer entry point
};
// Overlapped transfers of rt_layer_forward_host: x goes up in kIoXChunks
// chunks of sequences (each projected as soon as it lands) and z, K, V come
// down in kIoOutChunks ranges of positions as soon as the step loop has
// finished them.
static constexpr int kIoXChunks = 32, kIoOutChunks = 64, kIoEvents = 3 + kIoXChunks + kIoOutChunks;
static std::mutex g_io_mu;   // the transfer streams and events are per device
// positions per uploaded chunk of x
static int io_chunk_len(int N) { return (N + kIoXChunks - 1) / kIoXChunks; }
static std::mutex g_dev_mu;
static DevState g_dev[64];
static std::mutex g_encode_mu;
static PFN_encodeTiled_t g_encode = nullptr;

bool load_tensor_map_encoder() {
  std::lock_guard<std::mutex> lk(g_encode_mu);
  if (g_encode) return true;
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
          cudaSuccess ||
      q != cudaDriverEntryPointSuccess || !fn)
    return false;
  g_encode = reinterpret_cast<PFN_encodeTiled_t>(fn);
  return true;
}

template <int BN, int EPI>
static cudaError_t set_tc_attr() {
  return cudaFuncSetAttribute(k_gemm_tc<BN, EPI>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)GemmCfg<BN>::SMEM_BYTES);
}
template <int EPI>
static cudaError_t set_tc_attrs_epi() {
  cudaError_t e;
  if ((e = set_tc_attr<32, EPI>()) != cudaSuccess) return e;
  if ((e = set_tc_attr<64, EPI>()) != cudaSuccess) return e;
  if ((e = set_tc_attr<128, EPI>()) != cudaSuccess) return e;
  return set_tc_attr<256, EPI>();
}

// Checks the current device and performs one-time per-device set-up.
static int device_setup(DevState** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return RT_ERR_DEVICE;
  if (dev < 0 || dev >= 64) return RT_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_dev_mu);
  DevState& ds = g_dev[dev];
  if (!ds.ready) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess) return RT_ERR_DEVICE;
    if (major != 10) return RT_ERR_DEVICE;
    if (cudaDeviceGetAttribute(&ds.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RT_ERR_DEVICE;
    if (!load_tensor_map_encoder()) return RT_ERR_CUDA;
    RT_CK(set_tc_attrs_epi<EPI_PLAIN>());
    RT_CK(set_tc_attrs_epi<EPI_PROJ>());
    RT_CK(set_tc_attrs_epi<EPI_WO>());
    RT_CK(set_tc_attrs_epi<EPI_W1>());
    RT_CK(set_tc_attrs_epi<EPI_W2>());
    RT_CK(set_tc_attrs_epi<EPI_WKV>());
    RT_CK(set_tc_attrs_epi<EPI_RKV>());
    RT_CK(cudaFuncSetAttribute(k_fold_tc, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)FoldTcCfg::SMEM_BYTES));
    RT_CK(cudaFuncSetAttribute(k_fold_tc2, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               (int)FoldTc2Cfg::SMEM_BYTES));
    RT_CK(cudaFuncSetAttribute(k_steps, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)StepsCfg::SMEM_BYTES));
    RT_CK(cudaStreamCreateWithFlags(&ds.capture, cudaStreamNonBlocking));
    RT_CK(cudaStreamCreateWithFlags(&ds.h2d, cudaStreamNonBlocking));
    RT_CK(cudaStreamCreateWithFlags(&ds.d2h, cudaStreamNonBlocking));
    ds.events.resize(kIoEvents);
    for (auto& e : ds.events) RT_CK(cudaEventCreateWithFlags(&e, cudaEventDisableTiming));
    ds.ready = true;
  }
  *out = &ds;
  return RT_OK;
}

bool make_tmap(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 3-D bf16 tensor map over a position-major [npos][B][stride] buffer: box of
// 128 positions x one sequence x 64 elements (one head), 128-byte swizzle.
static bool make_tmap_pm(CUtensorMap* m, const void* base, uint64_t stride, uint64_t B, uint64_t npos) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0 || (stride * 2) % 16 != 0) return false;
  cuuint64_t dims[3] = {stride, B, npos};
  cuuint64_t strides[2] = {stride * 2, stride * 2 * B};
  cuuint32_t box[3] = {64, 1, 128};
  cuuint32_t es[3] = {1, 1, 1};
  return g_encode(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box, es,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

int choose_bn(int M, int N) {
  const long ntm = (M + 127) / 128;
  for (int bn : {256, 128, 64})
    if (ntm * ((N + bn - 1) / bn) >= 120) return bn;
  return 32;
}

// Per-step GEMMs (M = B rows): output tile width and split-K factor.
struct TileCfg {
  int bn, splits;
};
static TileCfg choose_tiles(int M, int N, int K, bool allow_split) {
  // Measured at M = 512 (per-step GEMM latency, graph of back-to-back
  // launches): for long K (W_2, K = 4096) 64-wide tiles with a 2-CTA cluster
  // split-K win (11.6 us vs 13.3 us unsplit); wider splits cost more in
  // staging than they save. For K = 1024: the widest tiles that still give
  // >= 120 CTAs (W_1: 128, 8.1 us vs 9.8 us at 64; W_kv: 64, 6.2 us vs 7.5
  // us at 128; W_o: 32 -- 64-wide tiles on 64 CTAs time alike in isolation
  // but 1.5 us slower inside the layer's step).
  const long ntm = (M + 127) / 128;
  if (allow_split && K / 64 >= 64 && K % (2 * GemmCfg<64>::KB) == 0 && N % 64 == 0) {
    const long mn = ntm * (N / 64);
    if (mn * 2 <= 160 && mn < 120) return {64, 2};
  }
  if (ntm * ((N + 127) / 128) >= 120) return {128, 1};
  if (ntm * ((N + 63) / 64) >= 120) return {64, 1};
  return {32, 1};
}
// Per-step GEMMs may use cluster split-K (see choose_tiles).
static constexpr bool kLayerSplitK = true;
// Smallest block size that uses the tcgen05 folds (smaller ones: mma.sync);
// measured at B = 512, d = 1024: mma.sync wins up to 128 keys, tcgen05 from 256.
static constexpr int kFoldTcMinBlock = 256;

template <int BN, int EPI>
static cudaError_t launch_tc_bn(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                                const EpiParams& p, unsigned* err, int sms, cudaStream_t st) {
  using C = GemmCfg<BN>;
  if (p.splits > 1) {
    if (!C::split_fits(p.splits) || p.splits > 8 || K % (C::KB * p.splits) != 0) return cudaErrorInvalidValue;
    // one output tile per cluster of `splits` CTAs, one tile per CTA
    const long tiles = (long)((M + 127) / 128) * ((N + BN - 1) / BN) * p.splits;
    return launch_pdl_cluster(k_gemm_tc<BN, EPI>, dim3((unsigned)tiles), dim3(C::THREADS), C::SMEM_BYTES, st,
                              p.splits, ta, tb, M, N, K, p, err);
  }
  const long tiles = (long)((M + 127) / 128) * ((N + BN - 1) / BN);
  const int grid = (int)std::min<long>(tiles, sms);
  return launch_pdl(k_gemm_tc<BN, EPI>, dim3(grid), dim3(C::THREADS), C::SMEM_BYTES, st, ta, tb, M, N, K, p, err);
}

template <int EPI>
static cudaError_t launch_tc(int bn, const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K,
                             const EpiParams& p, unsigned* err, int sms, cudaStream_t st) {
  switch (bn) {
    case 256: return launch_tc_bn<256, EPI>(ta, tb, M, N, K, p, err, sms, st);
    case 128: return launch_tc_bn<128, EPI>(ta, tb, M, N, K, p, err, sms, st);
    case 64: return launch_tc_bn<64, EPI>(ta, tb, M, N, K, p, err, sms, st);
    default: return launch_tc_bn<32, EPI>(ta, tb, M, N, K, p, err, sms, st);
  }
}

// ---------------------------------------------------------------------------
// shapes and workspace plan
// ---------------------------------------------------------------------------
struct Shape {
  int B, N, d, H, d_ff, dtype, schedule;
  // pages = 1: the paper's own parameterisation (per-head unit-RMS queries
  // and keys, no softmax scale, RMS without eps, branches scaled by
  // 1/sqrt(L)); 0: the single-layer configuration
  int pages = 0, L = 1;
  // chunk > 0: the block-wise recurrence with chunks of `chunk` positions
  // (a position's persistent pair is seen from the next chunk on; inside a
  // chunk, causal attention over the temporary pairs); 0: per position
  int chunk = 0;
  int dh() const { return d / H; }
  // rows of the per-step GEMMs: B sequences x positions per step
  int step_rows() const { return chunk > 0 ? B * std::min(chunk, N) : B; }
  float eps() const { return pages ? 0.f : kEps; }
  // softmax scale in log2 units: log2(e) / sqrt(d_h), or log2(e) unscaled
  float sc2() const { return pages ? kLog2e : kLog2e / std::sqrt((float)dh()); }
};

static int validate(const Shape& s) {
  if (s.B <= 0 || s.N <= 0 || s.d <= 0 || s.H <= 0 || s.d_ff <= 0) return RT_ERR_INVALID_ARG;
  if (s.d % s.H != 0) return RT_ERR_INVALID_ARG;
  if (s.dtype != RT_F32 && s.dtype != RT_BF16) return RT_ERR_INVALID_ARG;
  if (s.schedule != RT_SCHED_BLOCKED && s.schedule != RT_SCHED_NAIVE) return RT_ERR_INVALID_ARG;
  const long rows = (long)s.B * s.N;
  if (rows > (1l << 30) || (long)s.B * s.H > 65535) return RT_ERR_UNSUPPORTED;
  const int dh = s.dh();
  if (s.dtype == RT_F32) {
    if (dh != 32 && dh != 64 && dh != 128) return RT_ERR_UNSUPPORTED;
    if ((rows + 63) / 64 > 65535) return RT_ERR_UNSUPPORTED;
  } else {
    if (dh != 64 || s.d % 64 != 0 || s.d_ff % 64 != 0) return RT_ERR_UNSUPPORTED;
  }
  if (s.pages && (s.dtype != RT_BF16 || s.schedule != RT_SCHED_BLOCKED)) return RT_ERR_UNSUPPORTED;
  if (s.chunk < 0) return RT_ERR_INVALID_ARG;
  if (s.chunk > 0 && (s.dtype != RT_BF16 || s.schedule != RT_SCHED_BLOCKED || s.pages)) return RT_ERR_UNSUPPORTED;
  if ((long)s.step_rows() * s.d_ff > (1l << 31)) return RT_ERR_UNSUPPORTED;
  if (s.L < 1) return RT_ERR_INVALID_ARG;
  return RT_OK;
}

// Tile widths and splits of the persistent step kernel (bf16, blocked
// schedule). ok = false: a shape the step kernel does not take (flag ranges
// beyond its per-lane polling); the step loop then launches one GEMM kernel
// per phase and one fold per step.
struct StepsPlan {
  bool ok;
  GemmPhase g[4];
  int nrb, G;
};
static StepsPlan plan_steps(const Shape& s) {
  StepsPlan sp;
  std::memset(&sp, 0, sizeof(sp));
  if (s.dtype != RT_BF16 || s.schedule != RT_SCHED_BLOCKED || s.chunk > 0) return sp;
  const int d = s.d, dff = s.d_ff;
  auto phase = [](int N, int K, int BN, int S) { return GemmPhase{N, K, BN, S, N / BN}; };
  // W_o: 64-wide tiles (short tasks on the critical path); W_1, W_2, W_kv:
  // 128-wide where the width allows (fewer operand bytes per output); the
  // 4096-deep W_2 reduction split so that every task streams about 1024 of K.
  sp.g[PH_WO] = phase(d, d, 64, 1);
  sp.g[PH_W1] = phase(dff, d, dff % 128 == 0 ? 128 : 64, 1);
  const int bn2 = d % 128 == 0 ? 128 : 64;
  // every split finishes BN_2 / S >= 32 of its tile's columns
  const int s2 = std::max(1, std::min(std::min(4, bn2 / 32), (dff / 64) / 8));
  sp.g[PH_W2] = phase(d, dff, bn2, s2);
  sp.g[PH_WKV] = phase(2 * d, d, 128, 1);
  sp.nrb = (s.B + 127) / 128;
  sp.G = (std::min(s.B, 128) + kFoldSeqs - 1) / kFoldSeqs;
  // the flags of a phase fit its flag stride
  sp.ok = s.H * sp.G <= kFlagStride && sp.g[PH_WO].tiles <= kFlagStride && sp.g[PH_W1].tiles <= kFlagStride &&
          sp.g[PH_W2].tiles * s2 <= kFlagStride && sp.g[PH_WKV].tiles <= kFlagStride;
  return sp;
}

struct Plan {
  Shape s;
  size_t esz;
  size_t off_err, off_qkv, off_m, off_l, off_o, off_inv, off_xr, off_wqkv, off_a, off_u32, off_u16, off_ru,
      off_h, off_zs, off_rz, off_ssq_u, off_ssq_z, off_flags, off_w2cnt, off_w2part, off_progress, total;
  TileCfg t_wo, t_w1, t_w2, t_wkv;
  StepsPlan sp;
};

static Plan make_plan(const Shape& s) {
  Plan P;
  std::memset(&P, 0, sizeof(P));
  P.s = s;
  P.esz = s.dtype == RT_BF16 ? 2 : 4;
  const size_t rows = (size_t)s.B * s.N, d = s.d, B = (size_t)s.step_rows();   // B: rows per step
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off = align_up(off + bytes, 256);
    return o;
  };
  P.off_err = take(256);
  P.off_qkv = take(rows * 3 * d * P.esz);
  if (s.schedule == RT_SCHED_BLOCKED) {
    P.off_m = take(rows * s.H * 4);
    P.off_l = take(rows * s.H * 4);
    P.off_o = take(rows * d * 4);
  }
  if (s.dtype == RT_BF16) P.off_inv = take(rows * 4);
  else P.off_xr = take(rows * d * 4);
  P.off_wqkv = take(3 * d * d * P.esz);
  P.off_a = take(B * d * P.esz);
  P.off_u32 = take(B * d * 4);
  if (s.dtype == RT_BF16) P.off_u16 = take(B * d * 2);
  else P.off_ru = take(B * d * 4);
  P.off_h = take(B * (size_t)s.d_ff * P.esz);
  P.off_zs = take(B * d * P.esz);
  if (s.dtype == RT_F32) P.off_rz = take(B * d * 4);
  P.off_ssq_u = take((d / 32 + 1) * B * 4);
  P.off_ssq_z = take((d / 32 + 1) * B * 4);
  P.sp = plan_steps(s);
  if (P.sp.ok) {
    const GemmPhase& g2 = P.sp.g[PH_W2];
    P.off_flags = take((size_t)PH_COUNT * P.sp.nrb * kFlagStride * 4);
    P.off_w2cnt = take((size_t)P.sp.nrb * g2.tiles * 4);
    P.off_w2part = take((size_t)P.sp.nrb * g2.tiles * g2.S * g2.BN * StepsCfg::BM * 4);
    P.off_progress = take((size_t)1024 * 10 * 4);   // the debug build's per-CTA progress record
  }
  if (s.dtype == RT_BF16) {
    const int M = s.step_rows();
    P.t_wo = choose_tiles(M, s.d, s.d, kLayerSplitK);
    P.t_w1 = choose_tiles(M, s.d_ff, s.d, kLayerSplitK);
    P.t_w2 = choose_tiles(M, s.d, s.d_ff, kLayerSplitK);
    P.t_wkv = choose_tiles(M, 2 * s.d, s.d, kLayerSplitK);
    // the paper's parameterisation normalises every head of k inside the
    // W_kv epilogue, which needs a head's 64 columns in one tile
    if (s.pages && (P.t_wkv.bn < 64 || P.t_wkv.splits > 1)) P.t_wkv = TileCfg{64, 1};
  }
  P.total = off;
  return P;
}

struct Ptrs {
  const void *x, *Wq, *Wk, *Wv, *Wo, *W1, *W2;
  void *z, *K, *V, *ws;
};

// Host buffers of rt_layer_forward_host whose transfers the bf16 forward
// overlaps with its own work (x up in sequence chunks, outputs down in
// position ranges). Device-side copies are X.x / X.z / X.K / X.V.
struct HostIo {
  const void* x_host;
  void *z_host, *K_host, *V_host;
};

// ---------------------------------------------------------------------------
// per-kernel-class event timing (stream driver only)
// ---------------------------------------------------------------------------
enum KernelClass {
  KC_INV_RMS = 0, KC_PROJ, KC_ATTEND, KC_WO, KC_W1, KC_W2, KC_WKV, KC_FOLD_WARP, KC_FOLD_TENSOR, KC_STEPS,
  KC_FOLD_LEVEL0 = 16,   // + log2(block size): per-level fold timing
  KC_COUNT = 32
};

static int log2_int(int v) {
  int r = 0;
  while (v > 1) { v >>= 1; ++r; }
  return r;
}

struct Timer {
  std::vector<cudaEvent_t> pool;
  std::vector<int> cls;   // class of each recorded pair
  size_t used = 0;        // events used in the current forward
  cudaError_t err = cudaSuccess;
  cudaEvent_t next() {
    if (used == pool.size()) {
      cudaEvent_t e;
      cudaError_t c = cudaEventCreate(&e);
      if (c != cudaSuccess) { err = c; return nullptr; }
      pool.push_back(e);
    }
    return pool[used++];
  }
};

struct TimedScope {
  Timer* T;
  cudaStream_t st;
  TimedScope(Timer* t, int c, cudaStream_t s) : T(t), st(s) {
    if (T) {
      cudaEvent_t e = T->next();
      if (e) cudaEventRecord(e, st);
      T->cls.push_back(c);
    }
  }
  ~TimedScope() {
    if (T) {
      cudaEvent_t e = T->next();
      if (e) cudaEventRecord(e, st);
    }
  }
};

// ---------------------------------------------------------------------------
// fold launch (shared by the layer and rt_block_fold)
// ---------------------------------------------------------------------------
template <class T>
static cudaError_t launch_fold(const T* Q, int q_stride, const T* K, const T* V, int kv_stride, float* m,
                               float* l, float* o, T* a_out, int B, int H, int dh, int q0, int nq, int k0,
                               int nk, float sc2, int init, int fin, bool fast, cudaStream_t st,
                               unsigned* err = nullptr, int min_tc_block = 128, int sms = 148) {
  const int pairs = B * H;
  if constexpr (std::is_same<T, bf16>::value) {
    if (fast && dh == 64 && nk % 128 == 0 && nk >= min_tc_block && q_stride % 8 == 0 && kv_stride % 8 == 0) {
      CUtensorMap tq, tk, tv;
      if (!make_tmap_pm(&tq, Q, q_stride, B, q0 + nq) || !make_tmap_pm(&tk, K, kv_stride, B, k0 + nk) ||
          !make_tmap_pm(&tv, V, kv_stride, B, k0 + nk))
        return cudaErrorInvalidValue;
      if (nq > 128) {
        // two 128-query tiles per item share every K/V chunk
        const long items = (long)pairs * ((nq + 255) / 256);
        const dim3 grid((unsigned)std::min<long>(items, sms));
        return launch_pdl(k_fold_tc2, grid, dim3(320), FoldTc2Cfg::SMEM_BYTES, st, tq, tk, tv, Q, q_stride, m, l,
                          o, a_out, B, H, q0, nq, k0, nk, sc2, init, fin, err);
      }
      const long items = (long)pairs * ((nq + 127) / 128);
      const dim3 grid((unsigned)std::min<long>(items, sms));   // persistent over (pair, query tile) items
      return launch_pdl(k_fold_tc, grid, dim3(192), FoldTcCfg::SMEM_BYTES, st, tq, tk, tv, Q, q_stride, m, l, o,
                        a_out, B, H, q0, nq, k0, nk, sc2, init, fin, err);
    }
    if (fast && dh == 64 && nk >= 16 && nk % 16 == 0) {
      // pack 4 / 2 (b, h) pairs per CTA for 16- / 32-key blocks so that no warp idles
      // blocks of 16 or 32 keys are one chunk: the single-buffered variant (5 CTAs per SM)
      if (nk <= 16) {
        dim3 grid((nq + 15) / 16, (pairs + 3) / 4);
        return launch_pdl(k_fold_mma<4, 1>, grid, dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, a_out,
                          B, H, q0, nq, k0, nk, sc2, init, fin, err);
      }
      if (nk <= 32) {
        dim3 grid((nq + 31) / 32, (pairs + 1) / 2);
        return launch_pdl(k_fold_mma<2, 1>, grid, dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, a_out,
                          B, H, q0, nq, k0, nk, sc2, init, fin, err);
      }
      dim3 grid((nq + 63) / 64, pairs);
      return launch_pdl(k_fold_mma<1, 2>, grid, dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, a_out, B, H,
                        q0, nq, k0, nk, sc2, init, fin, err);
    }
    if (fast && dh == 64 && nk <= 8 && q_stride % 8 == 0 && kv_stride % 8 == 0) {
      // grid of k_fold_small: 16 / S pairs per CTA, or ceil(nq / 16) CTAs per pair
      const int S = fold_small_slots(nq, nk);
      const long ctas = (long)((pairs + 16 / S - 1) / (16 / S)) * ((nq + S - 1) / S);
      if (ctas > 0x7fffffffL) return cudaErrorInvalidValue;
      const dim3 grid((unsigned)ctas), block(128);
      if (nq <= nk && (nk == 1 || nk == 2 || nk == 4 || nk == 8)) {
        // the layer's blocks: compile-time key count (S == nk)
        auto kern = nk == 1 ? k_fold_small<1> : nk == 2 ? k_fold_small<2> : nk == 4 ? k_fold_small<4> : k_fold_small<8>;
        return launch_pdl(kern, grid, block, 0, st, Q, q_stride, K, V, kv_stride, m, l, o, a_out, B, H, q0, nq, k0,
                          nk, sc2, init, fin);
      }
      return launch_pdl(k_fold_small<0>, grid, block, 0, st, Q, q_stride, K, V, kv_stride, m, l, o,
                        a_out, B, H, q0, nq, k0, nk, sc2, init, fin);
    }
  }
  if (fin) return cudaErrorInvalidValue;   // only the bf16 kernels finalise
  const int blocks = (pairs + 3) / 4;
  switch (dh) {
    case 32: return launch_pdl(k_fold_warp<T, 1>, dim3(blocks), dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, B, H, q0, nq, k0, nk, sc2, init);
    case 64: return launch_pdl(k_fold_warp<T, 2>, dim3(blocks), dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, B, H, q0, nq, k0, nk, sc2, init);
    default: return launch_pdl(k_fold_warp<T, 4>, dim3(blocks), dim3(128), 0, st, Q, q_stride, K, V, kv_stride, m, l, o, B, H, q0, nq, k0, nk, sc2, init);
  }
}

template <class T, int DPL>
static cudaError_t launch_attend(const Plan& P, const T* qkv, const T* K, const T* V, const float* m,
                                 const float* l, const float* o, T* a, int j, float sc2, cudaStream_t st) {
  const Shape& s = P.s;
  const int blocks = (s.B * s.H + 3) / 4;
  if (s.schedule == RT_SCHED_BLOCKED)
    return launch_pdl(k_finalize<T, DPL>, dim3(blocks), dim3(128), 0, st, qkv, m, l, o, a, s.B, s.H, j, sc2,
                      j > 0 ? 1 : 0);
  // naive schedule: one CTA of 8 warps per (b, h), keys split across the warps
  return launch_pdl(k_naive_attn<T, DPL>, dim3(s.B * s.H), dim3(256), 0, st, qkv, K, V, a, s.B, s.H, j, j, sc2);
}

// ---------------------------------------------------------------------------
// bf16 forward
// ---------------------------------------------------------------------------
static int enqueue_bf16(const Plan& P, const Ptrs& X, const DevState& ds, cudaStream_t st, Timer* T,
                        const HostIo* io = nullptr, bool persistent = false) {
  const Shape& s = P.s;
  const bool steps = persistent && P.sp.ok;   // the persistent step kernel, else one kernel per phase
  char* ws = static_cast<char*>(X.ws);
  unsigned* err = reinterpret_cast<unsigned*>(ws + P.off_err);
  bf16* qkv = reinterpret_cast<bf16*>(ws + P.off_qkv);
  float* m = reinterpret_cast<float*>(ws + P.off_m);
  float* l = reinterpret_cast<float*>(ws + P.off_l);
  float* o = reinterpret_cast<float*>(ws + P.off_o);
  float* inv = reinterpret_cast<float*>(ws + P.off_inv);
  bf16* wqkv = reinterpret_cast<bf16*>(ws + P.off_wqkv);
  bf16* a16 = reinterpret_cast<bf16*>(ws + P.off_a);
  float* u32 = reinterpret_cast<float*>(ws + P.off_u32);
  bf16* u16 = reinterpret_cast<bf16*>(ws + P.off_u16);
  bf16* h16 = reinterpret_cast<bf16*>(ws + P.off_h);
  bf16* z16 = reinterpret_cast<bf16*>(ws + P.off_zs);
  float* ssq_u = reinterpret_cast<float*>(ws + P.off_ssq_u);
  float* ssq_z = reinterpret_cast<float*>(ws + P.off_ssq_z);
  const bf16* x = static_cast<const bf16*>(X.x);
  bf16* K = static_cast<bf16*>(X.K);
  bf16* V = static_cast<bf16*>(X.V);
  const int B = s.B, N = s.N, d = s.d, H = s.H, dff = s.d_ff;
  const size_t rows = (size_t)B * N;
  const size_t dd = (size_t)d * d * 2;

  RT_CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
  RT_CK(cudaMemcpyAsync(wqkv, X.Wq, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + dd, X.Wk, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + 2 * dd, X.Wv, dd, cudaMemcpyDeviceToDevice, st));

  // 1. queries and temporary pairs of all positions
  // (the paper's per-head normalisation needs whole 64-column heads per tile)
  const int bn_p = std::max(s.pages ? 64 : 32, choose_bn((int)rows, 3 * d));
  CUtensorMap tB_qkv;
  if (!make_tmap(&tB_qkv, wqkv, d, 3 * d, bn_p)) return RT_ERR_INVALID_ARG;
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = N; ep.d = d; ep.d_ff = dff; ep.eps = s.eps();
  ep.pages = s.pages; ep.inv_sqrt_L = 1.f / std::sqrt((float)s.L);
  ep.inv_rms = inv; ep.qkv = qkv; ep.x = x; ep.u32 = u32; ep.u16 = u16; ep.h16 = h16;
  ep.zout = static_cast<bf16*>(X.z); ep.z16 = z16; ep.Kout = K; ep.Vout = V;
  // x arrives in chunks of xc positions (the host-buffer path uploads chunk
  // c while earlier chunks are projected and the step loop runs); chunk c
  // is projected just before the first step that reads one of its
  // positions. Device layout of x: [n_chunks][B][xc][d].
  const int xc = io ? io_chunk_len(N) : N, n_chunks = (N + xc - 1) / xc;
  ep.xc = xc;
  int ev = 0;
  if (io) {   // fork the transfer streams off the main stream; queue every upload
    RT_CK(cudaEventRecord(ds.events[ev], st));
    RT_CK(cudaStreamWaitEvent(ds.h2d, ds.events[ev], 0));
    RT_CK(cudaStreamWaitEvent(ds.d2h, ds.events[ev], 0));
    ++ev;
    for (int c = 0; c < n_chunks; ++c) {
      const int len = std::min(xc, N - c * xc);
      RT_CK(cudaMemcpy2DAsync(const_cast<bf16*>(x) + (size_t)c * B * xc * d, (size_t)xc * d * 2,
                              static_cast<const bf16*>(io->x_host) + (size_t)c * xc * d, (size_t)N * d * 2,
                              (size_t)len * d * 2, B, cudaMemcpyHostToDevice, ds.h2d));
      RT_CK(cudaEventRecord(ds.events[ev + c], ds.h2d));
    }
  }
  const int ev_x = ev;
  if (io) ev += n_chunks;
  int projected = 0;   // chunks projected so far
  // project every chunk up to the one holding position `pos`
  auto project_through = [&](int pos) -> int {
    while (projected * xc <= pos) {
      const int c = projected++;
      const size_t nr = (size_t)B * xc;   // rows of the chunk, padding included
      const bf16* xs = x + (size_t)c * B * xc * d;
      if (io) RT_CK(cudaStreamWaitEvent(st, ds.events[ev_x + c], 0));
      {
        TimedScope ts(T, KC_INV_RMS, st);
        k_row_inv_rms<bf16><<<(unsigned)((nr + 7) / 8), 256, 0, st>>>(xs, inv, nr, d, s.eps());
      }
      RT_CK(cudaGetLastError());
      CUtensorMap tA_x;
      if (!make_tmap(&tA_x, xs, d, nr, 128)) return RT_ERR_INVALID_ARG;
      EpiParams epp = ep;
      epp.n0 = c * xc;
      TimedScope ts(T, KC_PROJ, st);
      RT_CK(launch_tc<EPI_PROJ>(bn_p, tA_x, tB_qkv, (int)nr, 3 * d, d, epp, err, ds.sms, st));
    }
    return RT_OK;
  };
  // outputs of positions [p0, p1) are final once step p1 - 1 has run
  int out_done = 0;
  auto ship_outputs = [&](int p1) -> int {
    const int p0 = out_done;
    if (!io || p1 <= p0) return RT_OK;
    RT_CK(cudaEventRecord(ds.events[ev], st));
    RT_CK(cudaStreamWaitEvent(ds.d2h, ds.events[ev], 0));
    ++ev;
    const size_t kv0 = (size_t)p0 * B * d, kvn = (size_t)(p1 - p0) * B * d;
    RT_CK(cudaMemcpyAsync(static_cast<bf16*>(io->K_host) + kv0, K + kv0, kvn * 2, cudaMemcpyDeviceToHost, ds.d2h));
    RT_CK(cudaMemcpyAsync(static_cast<bf16*>(io->V_host) + kv0, V + kv0, kvn * 2, cudaMemcpyDeviceToHost, ds.d2h));
    // z[b][p0:p1][:] for every b: B rows of (p1 - p0) * d elements, pitch N * d
    RT_CK(cudaMemcpy2DAsync(static_cast<bf16*>(io->z_host) + (size_t)p0 * d, (size_t)N * d * 2,
                            static_cast<const bf16*>(X.z) + (size_t)p0 * d, (size_t)N * d * 2,
                            (size_t)(p1 - p0) * d * 2, B, cudaMemcpyDeviceToHost, ds.d2h));
    out_done = p1;
    return RT_OK;
  };
  const int out_every = std::max(1, (N + kIoOutChunks - 1) / kIoOutChunks);

  // 2. the N-step loop
  const int bn_o = P.t_wo.bn, bn_1 = P.t_w1.bn, bn_2 = P.t_w2.bn, bn_kv = P.t_wkv.bn;
  CUtensorMap tA_a, tB_o, tA_u, tB_1, tA_h, tB_2, tA_z, tB_kv;
  if (!make_tmap(&tA_a, a16, d, B, 128) || !make_tmap(&tB_o, X.Wo, d, d, bn_o) ||
      !make_tmap(&tA_u, u16, d, B, 128) || !make_tmap(&tB_1, X.W1, d, dff, bn_1) ||
      !make_tmap(&tA_h, h16, dff, B, 128) || !make_tmap(&tB_2, X.W2, dff, d, bn_2) ||
      !make_tmap(&tA_z, z16, d, B, 128) || !make_tmap(&tB_kv, wqkv + (size_t)d * d, d, 2 * d, bn_kv))
    return RT_ERR_INVALID_ARG;
  const float sc2 = s.sc2();
  const bool blocked = s.schedule == RT_SCHED_BLOCKED;
  // step j reads queries and temporary pairs of positions up to 2j + 1
  // (the fold of step j covers queries j + 1 .. 2j + 1, 0-based) and x of j
  {
    const int rc = project_through(std::min(N - 1, 1));
    if (rc != RT_OK) return rc;
  }
  if (blocked) {
    // position 1: only its temporary pair; every later position is finalised
    // by the last fold into it (the fold of the previous step)
    TimedScope ts(T, KC_ATTEND, st);
    RT_CK((launch_attend<bf16, 2>(P, qkv, K, V, m, l, o, a16, 0, sc2, st)));
  }
  if (steps) {
    // persistent step kernel: one launch per segment of steps whose folds
    // have at most 8 keys; the segment's last fold (>= 16 keys) follows it
    StepsParams sp;
    std::memset(&sp, 0, sizeof(sp));
    const bf16* A_of[4] = {a16, u16, h16, z16};
    const void* W_of[4] = {X.Wo, X.W1, X.W2, wqkv + (size_t)d * d};
    for (int ph = 0; ph < 4; ++ph) {
      const GemmPhase& g = P.sp.g[ph];
      sp.g[ph] = g;
      if (!make_tmap(&sp.tA[ph], A_of[ph], g.K, B, 128) || !make_tmap(&sp.tB[ph], W_of[ph], g.K, g.N, g.BN))
        return RT_ERR_INVALID_ARG;
    }
    sp.ep = ep;
    sp.ssq_u = ssq_u;
    sp.ssq_z = ssq_z;
    sp.qkv = qkv;
    sp.m = m;
    sp.l = l;
    sp.o = o;
    sp.a16 = a16;
    sp.flags = reinterpret_cast<unsigned*>(ws + P.off_flags);
    sp.w2cnt = reinterpret_cast<unsigned*>(ws + P.off_w2cnt);
    sp.w2part = reinterpret_cast<float*>(ws + P.off_w2part);
    sp.err = err;
    sp.progress = reinterpret_cast<unsigned*>(ws + P.off_progress);
    sp.sc2 = sc2;
    sp.H = H;
    sp.nrb = P.sp.nrb;
    sp.G = P.sp.G;
    RT_CK(cudaMemsetAsync(sp.flags, 0, (size_t)PH_COUNT * P.sp.nrb * kFlagStride * 4, st));
    RT_CK(cudaMemsetAsync(sp.w2cnt, 0, (size_t)P.sp.nrb * P.sp.g[PH_W2].tiles * 4, st));
    for (int j = 0; j < N;) {
      // steps j .. j1-1; the last one reveals position t = j1, whose fold has
      // >= 16 keys (or which is the last position)
      int j1 = j + 1;
      while (j1 < N && lowbit(j1) < 16) ++j1;
      {
        const int rc = project_through(std::min(N - 1, 2 * (j1 - 1) + 1));
        if (rc != RT_OK) return rc;
      }
      sp.j0 = j;
      sp.j1 = j1;
      {
        TimedScope ts(T, KC_STEPS, st);
        cudaError_t e = launch_steps(sp, ds.sms, st, ds.coop);
        cudaStreamCaptureStatus cs = cudaStreamCaptureStatusNone;
        if (e != cudaSuccess && ds.coop && cudaStreamIsCapturing(st, &cs) == cudaSuccess &&
            cs == cudaStreamCaptureStatusNone) {
          cudaGetLastError();   // outside capture: the same grid, launched plainly
          e = launch_steps(sp, ds.sms, st, false);
        }
        RT_CK(e);
      }
      const int t = j1;
      if (t < N) {
        const int lb = lowbit(t), nq = std::min(lb, N - t);
        TimedScope ts(T, KC_FOLD_LEVEL0 + log2_int(lb), st);
        RT_CK(launch_fold<bf16>(qkv, 3 * d, K, V, d, m, l, o, a16, B, H, 64, t, nq, t - lb, lb, sc2,
                                t == lb ? 1 : 0, 1, true, st, err, kFoldTcMinBlock, ds.sms));
      }
      if (io && (j1 - out_done >= out_every || j1 == N)) {
        const int rc = ship_outputs(j1);
        if (rc != RT_OK) return rc;
      }
      j = j1;
    }
  }
  for (int j = 0; j < N && !steps; ++j) {
    ep.j = j;
    {
      const int rc = project_through(std::min(N - 1, 2 * j + 1));
      if (rc != RT_OK) return rc;
    }
    if (!blocked) {
      TimedScope ts(T, KC_ATTEND, st);
      RT_CK((launch_attend<bf16, 2>(P, qkv, K, V, m, l, o, a16, j, sc2, st)));
    }
    ep.ssq_out = ssq_u;
    ep.splits = P.t_wo.splits;
    {
      TimedScope ts(T, KC_WO, st);
      RT_CK(launch_tc<EPI_WO>(bn_o, tA_a, tB_o, B, d, d, ep, err, ds.sms, st));
    }
    ep.ssq_in = ssq_u; ep.ssq_tiles = (d + bn_o - 1) / bn_o;
    ep.splits = P.t_w1.splits;
    {
      TimedScope ts(T, KC_W1, st);
      RT_CK(launch_tc<EPI_W1>(bn_1, tA_u, tB_1, B, dff, d, ep, err, ds.sms, st));
    }
    ep.ssq_out = ssq_z;
    ep.splits = P.t_w2.splits;
    {
      TimedScope ts(T, KC_W2, st);
      RT_CK(launch_tc<EPI_W2>(bn_2, tA_h, tB_2, B, d, dff, ep, err, ds.sms, st));
    }
    ep.ssq_in = ssq_z; ep.ssq_tiles = (d + bn_2 - 1) / bn_2;
    ep.splits = P.t_wkv.splits;
    {
      TimedScope ts(T, KC_WKV, st);
      RT_CK(launch_tc<EPI_WKV>(bn_kv, tA_z, tB_kv, B, 2 * d, d, ep, err, ds.sms, st));
    }
    if (blocked) {
      // fold keys (t - lb, t] into queries (t, t + lb] and finalise query t + 1
      const int t = j + 1, lb = lowbit(t), nq = std::min(lb, N - t);
      if (nq > 0) {
        TimedScope ts(T, KC_FOLD_LEVEL0 + log2_int(lb), st);
        RT_CK(launch_fold<bf16>(qkv, 3 * d, K, V, d, m, l, o, a16, B, H, 64, t, nq, t - lb, lb, sc2,
                                t == lb ? 1 : 0, 1, true, st, err, kFoldTcMinBlock, ds.sms));
      }
    }
    if (io && ((j + 1) % out_every == 0 || j + 1 == N)) {
      const int rc = ship_outputs(j + 1);
      if (rc != RT_OK) return rc;
    }
  }
  if (io) {   // join the transfer streams back into the main stream
    RT_CK(cudaEventRecord(ds.events[ev], ds.h2d));
    RT_CK(cudaStreamWaitEvent(st, ds.events[ev], 0));
    ++ev;
    RT_CK(cudaEventRecord(ds.events[ev], ds.d2h));
    RT_CK(cudaStreamWaitEvent(st, ds.events[ev], 0));
    ++ev;
  }
  return RT_OK;
}

// ---------------------------------------------------------------------------
// fp32 forward (SIMT)
// ---------------------------------------------------------------------------
template <int EPI>
static cudaError_t launch_simt(const float* A, const float* W, int M, int N, int K, const SimtEpi& p,
                               cudaStream_t st) {
  dim3 grid((N + 63) / 64, (M + 63) / 64);
  k_gemm_simt<EPI><<<grid, 256, 0, st>>>(A, W, M, N, K, p);
  return cudaGetLastError();
}

static int enqueue_f32(const Plan& P, const Ptrs& X, cudaStream_t st, Timer* T) {
  const Shape& s = P.s;
  char* ws = static_cast<char*>(X.ws);
  unsigned* err = reinterpret_cast<unsigned*>(ws + P.off_err);
  float* qkv = reinterpret_cast<float*>(ws + P.off_qkv);
  float* m = reinterpret_cast<float*>(ws + P.off_m);
  float* l = reinterpret_cast<float*>(ws + P.off_l);
  float* o = reinterpret_cast<float*>(ws + P.off_o);
  float* xr = reinterpret_cast<float*>(ws + P.off_xr);
  float* wqkv = reinterpret_cast<float*>(ws + P.off_wqkv);
  float* a = reinterpret_cast<float*>(ws + P.off_a);
  float* u = reinterpret_cast<float*>(ws + P.off_u32);
  float* ru = reinterpret_cast<float*>(ws + P.off_ru);
  float* h = reinterpret_cast<float*>(ws + P.off_h);
  float* zs = reinterpret_cast<float*>(ws + P.off_zs);
  float* rz = reinterpret_cast<float*>(ws + P.off_rz);
  const float* x = static_cast<const float*>(X.x);
  float* K = static_cast<float*>(X.K);
  float* V = static_cast<float*>(X.V);
  const int B = s.B, N = s.N, d = s.d, H = s.H, dff = s.d_ff, dh = s.dh();
  const size_t rows = (size_t)B * N;
  const size_t dd = (size_t)d * d * 4;

  RT_CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
  RT_CK(cudaMemcpyAsync(wqkv, X.Wq, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + dd, X.Wk, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + 2 * dd, X.Wv, dd, cudaMemcpyDeviceToDevice, st));
  k_rmsnorm_f32<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(x, xr, rows, d, kEps);
  RT_CK(cudaGetLastError());
  SimtEpi p;
  std::memset(&p, 0, sizeof(p));
  p.B = B; p.Nseq = N; p.d = d; p.d_ff = dff;
  p.qkv = qkv; p.x = x; p.u = u; p.h = h; p.zout = static_cast<float*>(X.z); p.zs = zs; p.Kout = K; p.Vout = V;
  RT_CK(launch_simt<EPI_PROJ>(xr, wqkv, (int)rows, 3 * d, d, p, st));

  const float sc2 = kLog2e / std::sqrt((float)dh);
  const bool blocked = s.schedule == RT_SCHED_BLOCKED;
  for (int j = 0; j < N; ++j) {
    p.j = j;
    cudaError_t e;
    if (dh == 32) e = launch_attend<float, 1>(P, qkv, K, V, m, l, o, a, j, sc2, st);
    else if (dh == 64) e = launch_attend<float, 2>(P, qkv, K, V, m, l, o, a, j, sc2, st);
    else e = launch_attend<float, 4>(P, qkv, K, V, m, l, o, a, j, sc2, st);
    RT_CK(e);
    RT_CK(launch_simt<EPI_WO>(a, static_cast<const float*>(X.Wo), B, d, d, p, st));
    k_rmsnorm_f32<<<(B + 7) / 8, 256, 0, st>>>(u, ru, B, d, kEps);
    RT_CK(cudaGetLastError());
    RT_CK(launch_simt<EPI_W1>(ru, static_cast<const float*>(X.W1), B, dff, d, p, st));
    RT_CK(launch_simt<EPI_W2>(h, static_cast<const float*>(X.W2), B, d, dff, p, st));
    k_rmsnorm_f32<<<(B + 7) / 8, 256, 0, st>>>(zs, rz, B, d, kEps);
    RT_CK(cudaGetLastError());
    RT_CK(launch_simt<EPI_WKV>(rz, wqkv + (size_t)d * d, B, 2 * d, d, p, st));
    if (blocked) {
      const int t = j + 1, lb = lowbit(t), nq = std::min(lb, N - t);
      TimedScope ts(nq > 0 ? T : nullptr, KC_FOLD_LEVEL0 + log2_int(lb), st);
      if (nq > 0)
        RT_CK(launch_fold<float>(qkv, 3 * d, K, V, d, m, l, o, nullptr, B, H, dh, t, nq, t - lb, lb, sc2,
                                 t == lb ? 1 : 0, 0, false, st));
    }
  }
  return RT_OK;
}

// ---------------------------------------------------------------------------
// block-wise (chunked) recurrence, bf16: per chunk of C positions, the
// chunk's attention (fold state + causal temporary pairs), the four GEMMs at
// M = B * C rows (position-major), and the dyadic block fold at chunk
// granularity: when chunk cc (1-based) has revealed its persistent pairs,
// the pairs of chunks (cc - lb, cc] are folded into the queries of chunks
// (cc, cc + lb], lb = lowbit(cc).
// ---------------------------------------------------------------------------
static int enqueue_chunked(const Plan& P, const Ptrs& X, const DevState& ds, cudaStream_t st, Timer* T) {
  const Shape& s = P.s;
  char* ws = static_cast<char*>(X.ws);
  unsigned* err = reinterpret_cast<unsigned*>(ws + P.off_err);
  bf16* qkv = reinterpret_cast<bf16*>(ws + P.off_qkv);
  float* m = reinterpret_cast<float*>(ws + P.off_m);
  float* l = reinterpret_cast<float*>(ws + P.off_l);
  float* o = reinterpret_cast<float*>(ws + P.off_o);
  float* inv = reinterpret_cast<float*>(ws + P.off_inv);
  bf16* wqkv = reinterpret_cast<bf16*>(ws + P.off_wqkv);
  bf16* a16 = reinterpret_cast<bf16*>(ws + P.off_a);
  bf16* u16 = reinterpret_cast<bf16*>(ws + P.off_u16);
  bf16* h16 = reinterpret_cast<bf16*>(ws + P.off_h);
  bf16* z16 = reinterpret_cast<bf16*>(ws + P.off_zs);
  float* ssq_u = reinterpret_cast<float*>(ws + P.off_ssq_u);
  float* ssq_z = reinterpret_cast<float*>(ws + P.off_ssq_z);
  const bf16* x = static_cast<const bf16*>(X.x);
  bf16* K = static_cast<bf16*>(X.K);
  bf16* V = static_cast<bf16*>(X.V);
  const int B = s.B, N = s.N, d = s.d, H = s.H, dff = s.d_ff, C = std::min(s.chunk, s.N);
  const int Mmax = s.step_rows();
  const size_t rows = (size_t)B * N, dd = (size_t)d * d * 2;
  RT_CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
  RT_CK(cudaMemcpyAsync(wqkv, X.Wq, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + dd, X.Wk, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + 2 * dd, X.Wv, dd, cudaMemcpyDeviceToDevice, st));
  // queries and temporary pairs of every position
  {
    TimedScope ts(T, KC_INV_RMS, st);
    k_row_inv_rms<bf16><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(x, inv, rows, d, kEps);
  }
  RT_CK(cudaGetLastError());
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = N; ep.xc = N; ep.d = d; ep.d_ff = dff; ep.eps = kEps;
  ep.inv_rms = inv; ep.qkv = qkv; ep.x = x; ep.u32 = reinterpret_cast<float*>(ws + P.off_u32); ep.u16 = u16;
  ep.h16 = h16; ep.zout = static_cast<bf16*>(X.z); ep.z16 = z16; ep.Kout = K; ep.Vout = V;
  {
    const int bn_p = choose_bn((int)rows, 3 * d);
    CUtensorMap tA_x, tB_qkv;
    if (!make_tmap(&tA_x, x, d, rows, 128) || !make_tmap(&tB_qkv, wqkv, d, 3 * d, bn_p)) return RT_ERR_INVALID_ARG;
    TimedScope ts(T, KC_PROJ, st);
    RT_CK(launch_tc<EPI_PROJ>(bn_p, tA_x, tB_qkv, (int)rows, 3 * d, d, ep, err, ds.sms, st));
  }
  const int bn_o = P.t_wo.bn, bn_1 = P.t_w1.bn, bn_2 = P.t_w2.bn, bn_kv = P.t_wkv.bn;
  CUtensorMap tA_a, tB_o, tA_u, tB_1, tA_h, tB_2, tA_z, tB_kv;
  if (!make_tmap(&tA_a, a16, d, Mmax, 128) || !make_tmap(&tB_o, X.Wo, d, d, bn_o) ||
      !make_tmap(&tA_u, u16, d, Mmax, 128) || !make_tmap(&tB_1, X.W1, d, dff, bn_1) ||
      !make_tmap(&tA_h, h16, dff, Mmax, 128) || !make_tmap(&tB_2, X.W2, dff, d, bn_2) ||
      !make_tmap(&tA_z, z16, d, Mmax, 128) || !make_tmap(&tB_kv, wqkv + (size_t)d * d, d, 2 * d, bn_kv))
    return RT_ERR_INVALID_ARG;
  const float sc2 = s.sc2();
  const int nchunks = (N + C - 1) / C;
  for (int c = 0; c < nchunks; ++c) {
    const int p0 = c * C, nc = std::min(C, N - p0), M = B * nc;
    {
      TimedScope ts(T, KC_ATTEND, st);
      const long units = (long)M * H;
      RT_CK(launch_pdl(k_chunk_attend, dim3((unsigned)((units + 15) / 16)), dim3(128), 0, st,
                       static_cast<const bf16*>(qkv), static_cast<const float*>(m), static_cast<const float*>(l),
                       static_cast<const float*>(o), a16, B, H, p0, nc, sc2, c > 0 ? 1 : 0, err));
    }
    ep.j = p0;
    ep.ssq_rows = M;
    ep.ssq_out = ssq_u;
    ep.splits = P.t_wo.splits;
    {
      TimedScope ts(T, KC_WO, st);
      RT_CK(launch_tc<EPI_WO>(bn_o, tA_a, tB_o, M, d, d, ep, err, ds.sms, st));
    }
    ep.ssq_in = ssq_u; ep.ssq_tiles = (d + bn_o - 1) / bn_o;
    ep.splits = P.t_w1.splits;
    {
      TimedScope ts(T, KC_W1, st);
      RT_CK(launch_tc<EPI_W1>(bn_1, tA_u, tB_1, M, dff, d, ep, err, ds.sms, st));
    }
    ep.ssq_out = ssq_z;
    ep.splits = P.t_w2.splits;
    {
      TimedScope ts(T, KC_W2, st);
      RT_CK(launch_tc<EPI_W2>(bn_2, tA_h, tB_2, M, d, dff, ep, err, ds.sms, st));
    }
    ep.ssq_in = ssq_z; ep.ssq_tiles = (d + bn_2 - 1) / bn_2;
    ep.splits = P.t_wkv.splits;
    {
      TimedScope ts(T, KC_WKV, st);
      RT_CK(launch_tc<EPI_WKV>(bn_kv, tA_z, tB_kv, M, 2 * d, d, ep, err, ds.sms, st));
    }
    const int cc = c + 1;   // chunks revealed so far
    if (cc * C < N) {
      const int lb = lowbit(cc), q0 = cc * C, nq = std::min(lb * C, N - q0);
      TimedScope ts(T, KC_FOLD_LEVEL0 + log2_int(lb * C), st);
      RT_CK(launch_fold<bf16>(qkv, 3 * d, K, V, d, m, l, o, nullptr, B, H, 64, q0, nq, (cc - lb) * C, lb * C, sc2,
                              cc == lb ? 1 : 0, 0, true, st, err, kFoldTcMinBlock, ds.sms));
    }
  }
  return RT_OK;
}

static int enqueue_forward(const Plan& P, const Ptrs& X, const DevState& ds, cudaStream_t st,
                           Timer* T = nullptr, const HostIo* io = nullptr, bool persistent = false) {
  if (P.s.chunk > 0) {
    if (io) return RT_ERR_UNSUPPORTED;
    return enqueue_chunked(P, X, ds, st, T);
  }
  if (io) {
    if (P.s.dtype != RT_BF16) return RT_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_io_mu);
    return enqueue_bf16(P, X, ds, st, T, io, persistent);
  }
  return P.s.dtype == RT_BF16 ? enqueue_bf16(P, X, ds, st, T, nullptr, persistent) : enqueue_f32(P, X, st, T);
}

// Kernels one forward launches (must mirror enqueue_bf16 / enqueue_f32).
static long launch_count(const Shape& s, int driver) {
  long folds = 0;
  if (s.schedule == RT_SCHED_BLOCKED)
    for (int t = 1; t <= s.N; ++t) folds += (std::min(lowbit(t), s.N - t) > 0) ? 1 : 0;
  if (s.dtype == RT_BF16 && s.chunk > 0) {
    // inv_rms + projection; per chunk: attend + 4 GEMMs (+ a fold unless it is the last)
    const int C = std::min(s.chunk, s.N), nchunks = (s.N + C - 1) / C;
    return 2 + 5l * nchunks + (nchunks - 1);
  }
  if (s.dtype == RT_BF16) {
    if (driver == RT_DRIVER_PERSISTENT && plan_steps(s).ok) {
      // finalise(position 1) + one step kernel per segment + the folds of
      // >= 16 keys that end segments (each finalises the next position)
      long segments = 0, big = 0;
      for (int t = 1; t <= s.N; ++t) {
        if (t == s.N || lowbit(t) >= 16) ++segments;
        if (t < s.N && lowbit(t) >= 16) ++big;
      }
      return 2 + 1 + segments + big;
    }
    // blocked: finalise(position 1) + 4 GEMMs per step + folds (each finalises the next position)
    if (s.schedule == RT_SCHED_BLOCKED) return 2 + 1 + 4l * s.N + folds;
    return 2 + 5l * s.N;
  }
  return 2 + 8l * s.N + folds;
}

// ---------------------------------------------------------------------------
// CUDA-graph driver: the whole forward recorded once per argument set
// ---------------------------------------------------------------------------
struct GraphKey {
  uintptr_t p[15];
  int v[12];
  bool operator<(const GraphKey& o) const {
    int c = std::memcmp(p, o.p, sizeof(p));
    if (c) return c < 0;
    return std::memcmp(v, o.v, sizeof(v)) < 0;
  }
};
struct GraphEntry {
  cudaGraphExec_t exec;
  unsigned long long last_use;
};
static std::mutex g_graph_mu;
static std::map<GraphKey, GraphEntry> g_graphs;
static unsigned long long g_graph_clock = 0;
static constexpr size_t kMaxGraphs = 8;

// The persistent driver takes the bf16 blocked forward at shapes the step
// kernel's plan accepts.
static bool persistent_ok(const Plan& P) {
  return P.s.dtype == RT_BF16 && P.s.schedule == RT_SCHED_BLOCKED && P.s.chunk == 0 && P.sp.ok;
}

static int run_forward(const Plan& P, const Ptrs& X, int driver, cudaStream_t st, const HostIo* io = nullptr) {
  const bool persistent = driver == RT_DRIVER_PERSISTENT;
  if (persistent && !persistent_ok(P)) return RT_ERR_UNSUPPORTED;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  RT_CK(cudaStreamIsCapturing(st, &cap));
  if (driver == RT_DRIVER_STREAM || cap != cudaStreamCaptureStatusNone)
    return enqueue_forward(P, X, *ds, st, nullptr, io, persistent);

  int dev = 0;
  RT_CK(cudaGetDevice(&dev));
  GraphKey key;
  std::memset(&key, 0, sizeof(key));
  const void* ptrs[15] = {X.x, X.Wq, X.Wk, X.Wv, X.Wo, X.W1, X.W2, X.z, X.K, X.V, X.ws,
                          io ? io->x_host : nullptr, io ? io->z_host : nullptr,
                          io ? io->K_host : nullptr, io ? io->V_host : nullptr};
  for (int i = 0; i < 15; ++i) key.p[i] = reinterpret_cast<uintptr_t>(ptrs[i]);
  const int vals[12] = {P.s.B, P.s.N, P.s.d, P.s.H, P.s.d_ff, P.s.dtype, P.s.schedule, dev, P.s.pages, P.s.L,
                        P.s.chunk, driver};
  std::memcpy(key.v, vals, sizeof(vals));

  std::lock_guard<std::mutex> lk(g_graph_mu);
  auto it = g_graphs.find(key);
  if (it == g_graphs.end()) {
    cudaGraph_t graph = nullptr;
    cudaError_t ce = cudaSuccess;
    for (int attempt = 0; attempt < 2; ++attempt) {
      RT_CK(cudaStreamBeginCapture(ds->capture, cudaStreamCaptureModeThreadLocal));
      rc = enqueue_forward(P, X, *ds, ds->capture, nullptr, io, persistent);
      ce = cudaStreamEndCapture(ds->capture, &graph);
      // a capture that failed on the step kernel's cooperative launch is
      // recorded once more with plain launches
      if ((rc == RT_ERR_CUDA || ce != cudaSuccess) && persistent && ds->coop && attempt == 0) {
        if (graph) cudaGraphDestroy(graph);
        graph = nullptr;
        cudaGetLastError();
        ds->coop = false;
        continue;
      }
      break;
    }
    if (rc != RT_OK) {
      if (graph) cudaGraphDestroy(graph);
      return rc;
    }
    if (ce != cudaSuccess) return cuda_failure(ce);
    cudaGraphExec_t exec = nullptr;
    ce = cudaGraphInstantiate(&exec, graph, 0);
    cudaGraphDestroy(graph);
    if (ce != cudaSuccess) return cuda_failure(ce);
    if (g_graphs.size() >= kMaxGraphs) {
      auto victim = g_graphs.begin();
      for (auto i2 = g_graphs.begin(); i2 != g_graphs.end(); ++i2)
        if (i2->second.last_use < victim->second.last_use) victim = i2;
      cudaGraphExecDestroy(victim->second.exec);
      g_graphs.erase(victim);
    }
    it = g_graphs.emplace(key, GraphEntry{exec, 0}).first;
  }
  it->second.last_use = ++g_graph_clock;
  RT_CK(cudaGraphLaunch(it->second.exec, st));
  return RT_OK;
}

}  // namespace rt

// ===========================================================================
// extern "C" entry points
// ===========================================================================
using namespace rt;

extern "C" int rt_version(void) { return 100; }

extern "C" int rt_last_cuda_error(void) { return g_last_cuda_error; }

extern "C" const char* rt_cuda_error_string(int code) { return cudaGetErrorString((cudaError_t)code); }

extern "C" const char* rt_status_string(int status) {
  switch (status) {
    case RT_OK: return "ok";
    case RT_ERR_INVALID_ARG: return "invalid argument";
    case RT_ERR_UNSUPPORTED: return "unsupported shape or dtype";
    case RT_ERR_WORKSPACE: return "workspace missing, misaligned or too small";
    case RT_ERR_CUDA: return "CUDA runtime error";
    case RT_ERR_TIMEOUT: return "device-side wait timed out";
    case RT_ERR_DEVICE: return "no usable sm_100 device";
    default: return "unknown status";
  }
}

extern "C" size_t rt_layer_workspace_bytes(int B, int N, int d, int H, int d_ff, int dtype, int schedule) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  if (validate(s) != RT_OK) return 0;
  return make_plan(s).total;
}

extern "C" int rt_layer_forward(const void* x, const void* W_q, const void* W_k, const void* W_v,
                                const void* W_o, const void* W_1, const void* W_2, int B, int N, int d, int H,
                                int d_ff, int dtype, int schedule, int driver, void* z, void* K, void* V,
                                void* workspace, size_t workspace_bytes, void* stream) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (driver != RT_DRIVER_GRAPH && driver != RT_DRIVER_STREAM && driver != RT_DRIVER_PERSISTENT)
    return RT_ERR_INVALID_ARG;
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z || !K || !V) return RT_ERR_INVALID_ARG;
  const void* all[10] = {x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V};
  for (const void* p : all)
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  Ptrs X{x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V, workspace};
  return run_forward(P, X, driver, static_cast<cudaStream_t>(stream));
}

extern "C" int rt_layer_forward_pages(const void* x, const void* W_q, const void* W_k, const void* W_v,
                                      const void* W_o, const void* W_1, const void* W_2, int B, int N, int d, int H,
                                      int d_ff, int L, void* z, void* K, void* V, void* workspace,
                                      size_t workspace_bytes, void* stream, int driver) {
  Shape s{B, N, d, H, d_ff, RT_BF16, RT_SCHED_BLOCKED};
  s.pages = 1;
  s.L = L;
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (driver != RT_DRIVER_GRAPH && driver != RT_DRIVER_STREAM && driver != RT_DRIVER_PERSISTENT)
    return RT_ERR_INVALID_ARG;
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z || !K || !V) return RT_ERR_INVALID_ARG;
  const void* all[10] = {x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V};
  for (const void* p : all)
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  Ptrs X{x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V, workspace};
  return run_forward(P, X, driver, static_cast<cudaStream_t>(stream));
}

extern "C" size_t rt_layer_chunked_workspace_bytes(int B, int N, int d, int H, int d_ff, int C) {
  Shape s{B, N, d, H, d_ff, RT_BF16, RT_SCHED_BLOCKED};
  s.chunk = C;
  if (C < 1 || validate(s) != RT_OK) return 0;
  return make_plan(s).total;
}

extern "C" int rt_layer_forward_chunked(const void* x, const void* W_q, const void* W_k, const void* W_v,
                                        const void* W_o, const void* W_1, const void* W_2, int B, int N, int d,
                                        int H, int d_ff, int C, void* z, void* K, void* V, void* workspace,
                                        size_t workspace_bytes, void* stream) {
  Shape s{B, N, d, H, d_ff, RT_BF16, RT_SCHED_BLOCKED};
  s.chunk = C;
  if (C < 1) return RT_ERR_INVALID_ARG;
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z || !K || !V) return RT_ERR_INVALID_ARG;
  const void* all[10] = {x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V};
  for (const void* p : all)
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  Ptrs X{x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V, workspace};
  return run_forward(P, X, RT_DRIVER_GRAPH, static_cast<cudaStream_t>(stream));
}

extern "C" int rt_layer_sync_status(void* workspace, void* stream) {
  if (!workspace) return RT_ERR_INVALID_ARG;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  RT_CK(cudaStreamSynchronize(st));
  RT_CK(cudaMemcpyAsync(&h, workspace, sizeof(h), cudaMemcpyDeviceToHost, st));
  RT_CK(cudaMemsetAsync(workspace, 0, sizeof(h), st));
  RT_CK(cudaStreamSynchronize(st));
  if (h & RT_DEVERR_TIMEOUT) return RT_ERR_TIMEOUT;
  if (h & RT_DEVERR_INDEX) return RT_ERR_INVALID_ARG;
  return RT_OK;
}

static size_t host_io_bytes(const Shape& s, size_t esz) {
  const size_t rows = (size_t)s.B * s.N, d = s.d;
  size_t tot = 0;
  const size_t xc = (size_t)io_chunk_len(s.N), x_rows = (size_t)s.B * xc * ((s.N + xc - 1) / xc);
  tot += align_up(x_rows * d * esz, 256);                       // x, in chunks of positions
  tot += align_up(rows * d * esz, 256) * 3;                     // z, K, V
  tot += align_up(d * d * esz, 256) * 4;                        // W_q, W_k, W_v, W_o
  tot += align_up((size_t)s.d_ff * d * esz, 256) * 2;           // W_1, W_2
  return tot;
}

extern "C" size_t rt_layer_host_workspace_bytes(int B, int N, int d, int H, int d_ff, int dtype, int schedule) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  if (validate(s) != RT_OK) return 0;
  const Plan P = make_plan(s);
  return P.total + host_io_bytes(s, P.esz);
}

// True when `p` is page-locked host memory known to CUDA (cudaHostAlloc /
// cudaHostRegister); pageable memory cannot be copied asynchronously.
static bool is_pinned(const void* p) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    cudaGetLastError();
    return false;
  }
  return a.type == cudaMemoryTypeHost;
}

extern "C" int rt_layer_forward_host(const void* x, const void* W_q, const void* W_k, const void* W_v,
                                     const void* W_o, const void* W_1, const void* W_2, int B, int N, int d,
                                     int H, int d_ff, int dtype, int schedule, int driver, void* z, void* K,
                                     void* V, void* workspace, size_t workspace_bytes, void* stream) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z || !K || !V) return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total + host_io_bytes(s, P.esz) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const size_t rows = (size_t)B * N;
  const size_t act = rows * d * P.esz, wdd = (size_t)d * d * P.esz, wdf = (size_t)d_ff * d * P.esz;
  char* base = static_cast<char*>(workspace) + P.total;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    char* p = base + off;
    off += align_up(bytes, 256);
    return p;
  };
  const size_t xc = (size_t)io_chunk_len(N), x_act = (size_t)B * xc * ((N + xc - 1) / xc) * d * P.esz;
  char *xd = take(x_act), *zd = take(act), *Kd = take(act), *Vd = take(act);
  char *Wqd = take(wdd), *Wkd = take(wdd), *Wvd = take(wdd), *Wod = take(wdd), *W1d = take(wdf), *W2d = take(wdf);
  RT_CK(cudaMemcpyAsync(Wqd, W_q, wdd, cudaMemcpyHostToDevice, st));
  RT_CK(cudaMemcpyAsync(Wkd, W_k, wdd, cudaMemcpyHostToDevice, st));
  RT_CK(cudaMemcpyAsync(Wvd, W_v, wdd, cudaMemcpyHostToDevice, st));
  RT_CK(cudaMemcpyAsync(Wod, W_o, wdd, cudaMemcpyHostToDevice, st));
  RT_CK(cudaMemcpyAsync(W1d, W_1, wdf, cudaMemcpyHostToDevice, st));
  RT_CK(cudaMemcpyAsync(W2d, W_2, wdf, cudaMemcpyHostToDevice, st));
  Ptrs X{xd, Wqd, Wkd, Wvd, Wod, W1d, W2d, zd, Kd, Vd, workspace};
  // bf16 with page-locked x, z, K, V: the copies of x and of the outputs run
  // on transfer streams, overlapped with the projection and the step loop
  if (dtype == RT_BF16 && is_pinned(x) && is_pinned(z) && is_pinned(K) && is_pinned(V)) {
    HostIo io{x, z, K, V};
    return run_forward(P, X, driver, st, &io);
  }
  RT_CK(cudaMemcpyAsync(xd, x, act, cudaMemcpyHostToDevice, st));
  rc = run_forward(P, X, driver, st);
  if (rc != RT_OK) return rc;
  RT_CK(cudaMemcpyAsync(z, zd, act, cudaMemcpyDeviceToHost, st));
  RT_CK(cudaMemcpyAsync(K, Kd, act, cudaMemcpyDeviceToHost, st));
  RT_CK(cudaMemcpyAsync(V, Vd, act, cudaMemcpyDeviceToHost, st));
  return RT_OK;
}

extern "C" int rt_embed_forward(const int32_t* ids, const void* E, int B, int N, int vocab, int d, int dtype,
                                void* x, void* workspace, void* stream) {
  if (!ids || !E || !x || B <= 0 || N <= 0 || vocab <= 0 || d <= 0) return RT_ERR_INVALID_ARG;
  if (dtype != RT_F32 && dtype != RT_BF16) return RT_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned* err = static_cast<unsigned*>(workspace);
  const size_t rows = (size_t)B * N;
  if (rows > 0x7fffffffu) return RT_ERR_UNSUPPORTED;
  if (dtype == RT_BF16)
    k_embed<bf16><<<(unsigned)rows, 128, 0, st>>>(ids, static_cast<const bf16*>(E), static_cast<bf16*>(x), rows,
                                                  vocab, d, err);
  else
    k_embed<float><<<(unsigned)rows, 128, 0, st>>>(ids, static_cast<const float*>(E), static_cast<float*>(x),
                                                   rows, vocab, d, err);
  RT_CK(cudaGetLastError());
  return RT_OK;
}

extern "C" int rt_block_fold(const void* Q, int q_stride, const void* K, const void* V, int kv_stride, float* m,
                             float* l, float* o, int B, int H, int d_h, int q0, int nq, int k0, int nk, int dtype,
                             void* err_dev, void* stream) {
  if (!Q || !K || !V || !m || !l || !o || !err_dev) return RT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(err_dev) & 3u) != 0) return RT_ERR_INVALID_ARG;
  if (B <= 0 || H <= 0 || nq <= 0 || nk <= 0 || q0 < 0 || k0 < 0) return RT_ERR_INVALID_ARG;
  if (q_stride < H * d_h || kv_stride < H * d_h || (long)B * H > 65535) return RT_ERR_INVALID_ARG;
  if (dtype == RT_BF16 && d_h != 64) return RT_ERR_UNSUPPORTED;
  if (dtype == RT_F32 && d_h != 32 && d_h != 64 && d_h != 128) return RT_ERR_UNSUPPORTED;
  if (dtype == RT_BF16 && (q_stride % 8 != 0 || kv_stride % 8 != 0)) return RT_ERR_UNSUPPORTED;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  const float sc2 = kLog2e / std::sqrt((float)d_h);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaError_t e;
  if (dtype == RT_BF16)
    e = launch_fold<bf16>(static_cast<const bf16*>(Q), q_stride, static_cast<const bf16*>(K),
                          static_cast<const bf16*>(V), kv_stride, m, l, o, nullptr, B, H, d_h, q0, nq, k0, nk, sc2, 0,
                          0, true, st, static_cast<unsigned*>(err_dev), kFoldTcMinBlock, ds->sms);
  else if (dtype == RT_F32)
    e = launch_fold<float>(static_cast<const float*>(Q), q_stride, static_cast<const float*>(K),
                           static_cast<const float*>(V), kv_stride, m, l, o, nullptr, B, H, d_h, q0, nq, k0, nk, sc2, 0,
                           0, false, st);
  else
    return RT_ERR_INVALID_ARG;
  return e == cudaSuccess ? RT_OK : cuda_failure(e);
}

// ---------------------------------------------------------------------------
// autoregressive decode step (RT paper §7.3)
// ---------------------------------------------------------------------------
static Shape decode_shape(int B, int d, int H, int d_ff) { return Shape{B, 1, d, H, d_ff, RT_BF16, RT_SCHED_NAIVE}; }

extern "C" size_t rt_layer_decode_workspace_bytes(int B, int d, int H, int d_ff) {
  const Shape s = decode_shape(B, d, H, d_ff);
  if (validate(s) != RT_OK) return 0;
  return make_plan(s).total;
}

// Position t of B sequences: projection of x_t, attention of its query over
// the cached persistent pairs of positions 1..t-1 plus its temporary pair,
// W_o, MLP, and the new persistent pair written to row t-1 of the caches.
// The projection and GEMMs are the layer's own; the attention is a decode
// kernel (lanes own whole cached keys) with the query at row 0 of a
// one-position Q/K~/V~ buffer.
extern "C" int rt_layer_decode_step(const void* x_t, const void* W_q, const void* W_k, const void* W_v,
                                    const void* W_o, const void* W_1, const void* W_2, int B, int t, int capacity,
                                    int d, int H, int d_ff, void* z_t, void* K_cache, void* V_cache,
                                    void* workspace, size_t workspace_bytes, void* stream) {
  const Shape s = decode_shape(B, d, H, d_ff);
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (t < 1 || t > capacity || (long)capacity * B > (1l << 30)) return RT_ERR_INVALID_ARG;
  if (!x_t || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z_t || !K_cache || !V_cache) return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  DevState* ds = nullptr;
  rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  unsigned* err = reinterpret_cast<unsigned*>(ws + P.off_err);
  bf16* qkv = reinterpret_cast<bf16*>(ws + P.off_qkv);
  float* inv = reinterpret_cast<float*>(ws + P.off_inv);
  bf16* wqkv = reinterpret_cast<bf16*>(ws + P.off_wqkv);
  bf16* a16 = reinterpret_cast<bf16*>(ws + P.off_a);
  float* ssq_u = reinterpret_cast<float*>(ws + P.off_ssq_u);
  float* ssq_z = reinterpret_cast<float*>(ws + P.off_ssq_z);
  const bf16* x = static_cast<const bf16*>(x_t);
  const size_t dd = (size_t)d * d * 2;

  RT_CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
  RT_CK(cudaMemcpyAsync(wqkv, W_q, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + dd, W_k, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wqkv) + 2 * dd, W_v, dd, cudaMemcpyDeviceToDevice, st));
  k_row_inv_rms<bf16><<<(unsigned)((B + 7) / 8), 256, 0, st>>>(x, inv, (size_t)B, d, kEps);
  RT_CK(cudaGetLastError());

  // x_t, z_t are [B][d]: one position (Nseq = 1, position index 0) for the
  // projection, W_o and W_2 epilogues; K_cache / V_cache rows are positions
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = 1; ep.xc = 1; ep.d = d; ep.d_ff = d_ff; ep.eps = kEps;
  ep.inv_rms = inv; ep.qkv = qkv; ep.x = x;
  ep.u32 = reinterpret_cast<float*>(ws + P.off_u32); ep.u16 = reinterpret_cast<bf16*>(ws + P.off_u16);
  ep.h16 = reinterpret_cast<bf16*>(ws + P.off_h); ep.zout = static_cast<bf16*>(z_t);
  ep.z16 = reinterpret_cast<bf16*>(ws + P.off_zs);
  ep.Kout = static_cast<bf16*>(K_cache); ep.Vout = static_cast<bf16*>(V_cache);
  const int bn_p = choose_bn(B, 3 * d);
  CUtensorMap tA_x, tB_qkv;
  if (!make_tmap(&tA_x, x, d, B, 128) || !make_tmap(&tB_qkv, wqkv, d, 3 * d, bn_p)) return RT_ERR_INVALID_ARG;
  RT_CK(launch_tc<EPI_PROJ>(bn_p, tA_x, tB_qkv, B, 3 * d, d, ep, err, ds->sms, st));

  const float sc2 = kLog2e / std::sqrt((float)s.dh());
  RT_CK(launch_pdl(k_decode_attn, dim3(B * H), dim3(128), 0, st, static_cast<const bf16*>(qkv),
                   static_cast<const bf16*>(K_cache), static_cast<const bf16*>(V_cache), a16, B, H, t - 1, sc2));

  const int bn_o = P.t_wo.bn, bn_1 = P.t_w1.bn, bn_2 = P.t_w2.bn, bn_kv = P.t_wkv.bn;
  CUtensorMap tA_a, tB_o, tA_u, tB_1, tA_h, tB_2, tA_z, tB_kv;
  if (!make_tmap(&tA_a, a16, d, B, 128) || !make_tmap(&tB_o, W_o, d, d, bn_o) ||
      !make_tmap(&tA_u, ep.u16, d, B, 128) || !make_tmap(&tB_1, W_1, d, d_ff, bn_1) ||
      !make_tmap(&tA_h, ep.h16, d_ff, B, 128) || !make_tmap(&tB_2, W_2, d_ff, d, bn_2) ||
      !make_tmap(&tA_z, ep.z16, d, B, 128) || !make_tmap(&tB_kv, wqkv + (size_t)d * d, d, 2 * d, bn_kv))
    return RT_ERR_INVALID_ARG;
  ep.j = 0;
  ep.ssq_out = ssq_u;
  ep.splits = P.t_wo.splits;
  RT_CK(launch_tc<EPI_WO>(bn_o, tA_a, tB_o, B, d, d, ep, err, ds->sms, st));
  ep.ssq_in = ssq_u; ep.ssq_tiles = (d + bn_o - 1) / bn_o;
  ep.splits = P.t_w1.splits;
  RT_CK(launch_tc<EPI_W1>(bn_1, tA_u, tB_1, B, d_ff, d, ep, err, ds->sms, st));
  ep.ssq_out = ssq_z;
  ep.splits = P.t_w2.splits;
  RT_CK(launch_tc<EPI_W2>(bn_2, tA_h, tB_2, B, d, d_ff, ep, err, ds->sms, st));
  ep.ssq_in = ssq_z; ep.ssq_tiles = (d + bn_2 - 1) / bn_2;
  ep.splits = P.t_wkv.splits;
  ep.j = t - 1;   // the new persistent pair's row in the caches
  RT_CK(launch_tc<EPI_WKV>(bn_kv, tA_z, tB_kv, B, 2 * d, d, ep, err, ds->sms, st));
  return RT_OK;
}

extern "C" int rt_project_qkv(const void* x, const void* W_qkv, int B, int N, int d, int dtype, void* QKV,
                              void* scratch, void* err_dev, void* stream) {
  if (!x || !W_qkv || !QKV || !scratch || !err_dev || B <= 0 || N <= 0 || d <= 0) return RT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(err_dev) & 3u) != 0) return RT_ERR_INVALID_ARG;
  if (dtype == RT_BF16 && d % 64 != 0) return RT_ERR_UNSUPPORTED;
  const size_t rows = (size_t)B * N;
  if (rows > (1u << 30)) return RT_ERR_UNSUPPORTED;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  if (dtype == RT_BF16) {
    float* inv = static_cast<float*>(scratch);
    k_row_inv_rms<bf16><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(static_cast<const bf16*>(x), inv, rows, d, kEps);
    RT_CK(cudaGetLastError());
    const int bn = choose_bn((int)rows, 3 * d);
    CUtensorMap ta, tb;
    if (!make_tmap(&ta, x, d, rows, 128) || !make_tmap(&tb, W_qkv, d, 3 * d, bn)) return RT_ERR_INVALID_ARG;
    EpiParams ep;
    std::memset(&ep, 0, sizeof(ep));
    ep.B = B; ep.Nseq = N; ep.xc = N; ep.d = d; ep.inv_rms = inv; ep.qkv = static_cast<bf16*>(QKV);
    RT_CK(launch_tc<EPI_PROJ>(bn, ta, tb, (int)rows, 3 * d, d, ep, static_cast<unsigned*>(err_dev), ds->sms, st));
  } else if (dtype == RT_F32) {
    if ((rows + 63) / 64 > 65535) return RT_ERR_UNSUPPORTED;
    float* xr = static_cast<float*>(scratch);
    k_rmsnorm_f32<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(static_cast<const float*>(x), xr, rows, d, kEps);
    RT_CK(cudaGetLastError());
    SimtEpi p;
    std::memset(&p, 0, sizeof(p));
    p.B = B; p.Nseq = N; p.d = d; p.qkv = static_cast<float*>(QKV);
    RT_CK(launch_simt<EPI_PROJ>(xr, static_cast<const float*>(W_qkv), (int)rows, 3 * d, d, p, st));
  } else {
    return RT_ERR_INVALID_ARG;
  }
  return RT_OK;
}

// ---------------------------------------------------------------------------
// activation-checkpoint recompute of the persistent pairs (RT paper §6.1)
// ---------------------------------------------------------------------------
static size_t recompute_ws_bytes(int B, int N, int d) {
  return align_up(256, 256) + align_up((size_t)B * N * 4, 256) + align_up((size_t)2 * d * d * 2, 256);
}

extern "C" size_t rt_layer_recompute_workspace_bytes(int B, int N, int d) {
  if (B <= 0 || N <= 0 || d <= 0 || d % 64 != 0 || (long)B * N > (1l << 30)) return 0;
  return recompute_ws_bytes(B, N, d);
}

extern "C" int rt_layer_recompute_kv(const void* z, const void* W_k, const void* W_v, int B, int N, int d, void* K,
                                     void* V, void* workspace, size_t workspace_bytes, void* stream) {
  if (!z || !W_k || !W_v || !K || !V || B <= 0 || N <= 0 || d <= 0) return RT_ERR_INVALID_ARG;
  if (d % 64 != 0 || (long)B * N > (1l << 30)) return RT_ERR_UNSUPPORTED;
  const void* all[5] = {z, W_k, W_v, K, V};
  for (const void* p : all)
    if ((reinterpret_cast<uintptr_t>(p) & 15u) != 0) return RT_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < recompute_ws_bytes(B, N, d) ||
      (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  char* ws = static_cast<char*>(workspace);
  unsigned* err = reinterpret_cast<unsigned*>(ws);
  float* inv = reinterpret_cast<float*>(ws + 256);
  bf16* wkv = reinterpret_cast<bf16*>(ws + 256 + align_up((size_t)B * N * 4, 256));
  const size_t rows = (size_t)B * N, dd = (size_t)d * d * 2;
  RT_CK(cudaMemsetAsync(err, 0, sizeof(unsigned), st));
  RT_CK(cudaMemcpyAsync(wkv, W_k, dd, cudaMemcpyDeviceToDevice, st));
  RT_CK(cudaMemcpyAsync(reinterpret_cast<char*>(wkv) + dd, W_v, dd, cudaMemcpyDeviceToDevice, st));
  k_row_inv_rms<bf16><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(static_cast<const bf16*>(z), inv, rows, d, kEps);
  RT_CK(cudaGetLastError());
  const int bn = choose_bn((int)rows, 2 * d);
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, z, d, rows, 128) || !make_tmap(&tb, wkv, d, 2 * d, bn)) return RT_ERR_INVALID_ARG;
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = N; ep.xc = N; ep.d = d; ep.inv_rms = inv;
  ep.Kout = static_cast<bf16*>(K); ep.Vout = static_cast<bf16*>(V);
  RT_CK(launch_tc<EPI_RKV>(bn, ta, tb, (int)rows, 2 * d, d, ep, err, ds->sms, st));
  return RT_OK;
}

extern "C" int rt_gemm_bf16(const void* A, const void* W, float* C, int M, int Nout, int Kd, void* err_dev,
                            void* stream) {
  if (!A || !W || !C || !err_dev || M <= 0 || Nout <= 0 || Kd <= 0) return RT_ERR_INVALID_ARG;
  if ((reinterpret_cast<uintptr_t>(err_dev) & 3u) != 0) return RT_ERR_INVALID_ARG;
  if (Kd % 64 != 0) return RT_ERR_UNSUPPORTED;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  const int bn = choose_bn(M, Nout);
  CUtensorMap ta, tb;
  if (!make_tmap(&ta, A, Kd, M, 128) || !make_tmap(&tb, W, Kd, Nout, bn)) return RT_ERR_INVALID_ARG;
  EpiParams ep;
  std::memset(&ep, 0, sizeof(ep));
  ep.c32 = C;
  RT_CK(launch_tc<EPI_PLAIN>(bn, ta, tb, M, Nout, Kd, ep, static_cast<unsigned*>(err_dev), ds->sms,
                             static_cast<cudaStream_t>(stream)));
  return RT_OK;
}

extern "C" long rt_layer_launch_count(int B, int N, int d, int H, int d_ff, int dtype, int schedule, int driver) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  if (validate(s) != RT_OK) return -1;
  if (driver != RT_DRIVER_GRAPH && driver != RT_DRIVER_STREAM && driver != RT_DRIVER_PERSISTENT) return -1;
  if (driver == RT_DRIVER_PERSISTENT && !persistent_ok(make_plan(s))) return -1;
  return launch_count(s, driver);
}

extern "C" int rt_layer_forward_timed(const void* x, const void* W_q, const void* W_k, const void* W_v,
                                      const void* W_o, const void* W_1, const void* W_2, int B, int N, int d,
                                      int H, int d_ff, int dtype, int schedule, void* z, void* K, void* V,
                                      void* workspace, size_t workspace_bytes, void* stream, float* class_ms,
                                      int* class_launches, int n_classes) {
  Shape s{B, N, d, H, d_ff, dtype, schedule};
  int rc = validate(s);
  if (rc != RT_OK) return rc;
  if (!x || !W_q || !W_k || !W_v || !W_o || !W_1 || !W_2 || !z || !K || !V || !class_ms || !class_launches)
    return RT_ERR_INVALID_ARG;
  const Plan P = make_plan(s);
  if (!workspace || workspace_bytes < P.total || (reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return RT_ERR_WORKSPACE;
  DevState* ds = nullptr;
  rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  RT_CK(cudaStreamIsCapturing(st, &cap));
  if (cap != cudaStreamCaptureStatusNone) return RT_ERR_INVALID_ARG;
  static std::mutex mu;
  static Timer timer;
  std::lock_guard<std::mutex> lk(mu);
  timer.used = 0;
  timer.cls.clear();
  timer.err = cudaSuccess;
  Ptrs X{x, W_q, W_k, W_v, W_o, W_1, W_2, z, K, V, workspace};
  rc = enqueue_forward(P, X, *ds, st, &timer);
  if (rc != RT_OK) return rc;
  if (timer.err != cudaSuccess) return cuda_failure(timer.err);
  RT_CK(cudaStreamSynchronize(st));
  for (int c = 0; c < n_classes; ++c) { class_ms[c] = 0.f; class_launches[c] = 0; }
  for (size_t i = 0; i < timer.cls.size(); ++i) {
    float ms = 0.f;
    RT_CK(cudaEventElapsedTime(&ms, timer.pool[2 * i], timer.pool[2 * i + 1]));
    const int c = timer.cls[i];
    if (c < n_classes) { class_ms[c] += ms; class_launches[c] += 1; }
    if (c >= KC_FOLD_LEVEL0) {   // per-level folds also count towards the kernel that ran them
      const int kc = (s.dtype == RT_BF16 && c - KC_FOLD_LEVEL0 >= 4) ? KC_FOLD_TENSOR : KC_FOLD_WARP;
      if (kc < n_classes) { class_ms[kc] += ms; class_launches[kc] += 1; }
    }
  }
  return RT_OK;
}

// Self-test of the bounded wait: one thread waits on a barrier that nothing
// arrives on; the wait must give up after limit_ns and record the timeout.
namespace rt {
__global__ void k_selftest_wait(unsigned* err, unsigned long long limit_ns) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    mbar_wait(&bar, 0, err, limit_ns);   // phase 0 never completes
  }
}
}  // namespace rt

extern "C" int rt_selftest_wait_timeout(unsigned long long limit_ns, void* workspace, void* stream) {
  if (!workspace || limit_ns == 0 || limit_ns > 10000000000ull) return RT_ERR_INVALID_ARG;
  DevState* ds = nullptr;
  int rc = device_setup(&ds);
  if (rc != RT_OK) return rc;
  k_selftest_wait<<<1, 32, 0, static_cast<cudaStream_t>(stream)>>>(static_cast<unsigned*>(workspace), limit_ns);
  return cudaGetLastError() == cudaSuccess ? RT_OK : RT_ERR_CUDA;
}
