// rt_noalloc.cu -- rt_project_qkv_noalloc: the batched Q / temporary-pair
// projection of rt_project_qkv (bf16 storage) with its scratch -- one fp32
// 1/rms value per input row -- held in a fixed array inside this library
// instead of memory the caller allocates.
//
// Who needs it: callers that cannot allocate device memory at the point of the
// call -- runtimes that plan every device buffer at start-up and forbid later
// allocation, code running while another framework's caching allocator holds
// the free device memory, or latency-critical loops where an allocation's cost
// or possible failure is not acceptable. They still pass x, W_qkv and QKV.
//
// The array g_inv_rms_scratch below holds at most kMaxRows rows (4 MiB); every
// GPU that loads the library keeps it until the process exits. All calls share
// it: the kernels overwrite rows [0, B*N) on every call before reading them, so
// nothing has to start at zero, but calls that overlap on the GPU (different
// streams, or different host threads) race on it.
//
// Host code must not pass the symbol itself to a kernel: on the host it names
// a host-side stand-in, not device memory. The first call on each device (with
// that device current) looks up the device address with cudaGetSymbolAddress
// and caches it; make that first call before any stream capture.
#include <cstring>
#include <mutex>

#include "../../include/rtlayer.h"
#include "rt_common.cuh"
#include "rt_gemm_tc.cuh"

namespace {

constexpr size_t kMaxRows = size_t(1) << 20;   // B*N limit: 4 MiB of fp32
static __device__ __align__(256) float g_inv_rms_scratch[kMaxRows];

typedef CUresult (*EncodeFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                             const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                             CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

struct DeviceSlot {
  bool ready = false;
  int sms = 0;
  float* scratch = nullptr;   // device address of g_inv_rms_scratch on this device
};
std::mutex g_mu;
DeviceSlot g_slots[64];
EncodeFn g_encode_fn = nullptr;

template <int BN>
cudaError_t set_proj_attr() {
  return cudaFuncSetAttribute(rt::k_gemm_tc<BN, rt::EPI_PROJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)rt::GemmCfg<BN>::SMEM_BYTES);
}

// One-time set-up of the current device: sm_100 check, SM count, tensor-map
// encoder, kernel attributes and the device address of the scratch array.
int setup_current_device(DeviceSlot** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RT_ERR_DEVICE;
  std::lock_guard<std::mutex> lk(g_mu);
  DeviceSlot& s = g_slots[dev];
  if (!s.ready) {
    int major = 0;
    if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess || major != 10)
      return RT_ERR_DEVICE;
    if (cudaDeviceGetAttribute(&s.sms, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return RT_ERR_DEVICE;
    if (!g_encode_fn) {
      void* fn = nullptr;
      cudaDriverEntryPointQueryResult q;
      if (cudaGetDriverEntryPointByVersion("cuTensorMapEncodeTiled", &fn, 12000, cudaEnableDefault, &q) !=
              cudaSuccess ||
          q != cudaDriverEntryPointSuccess || !fn)
        return RT_ERR_CUDA;
      g_encode_fn = reinterpret_cast<EncodeFn>(fn);
    }
    if (set_proj_attr<32>() != cudaSuccess || set_proj_attr<64>() != cudaSuccess ||
        set_proj_attr<128>() != cudaSuccess || set_proj_attr<256>() != cudaSuccess)
      return RT_ERR_CUDA;
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_inv_rms_scratch) != cudaSuccess || !p) return RT_ERR_CUDA;
    s.scratch = static_cast<float*>(p);
    s.ready = true;
  }
  *out = &s;
  return RT_OK;
}

bool encode(CUtensorMap* m, const void* base, uint64_t inner, uint64_t rows, uint32_t box_rows) {
  if ((reinterpret_cast<uintptr_t>(base) & 15u) != 0) return false;
  cuuint64_t dims[2] = {inner, rows};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_rows};
  cuuint32_t es[2] = {1, 1};
  return g_encode_fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, es,
                     CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                     CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// inv[r] = 1 / sqrt(mean(x_r^2) + 1e-6), one warp per row
__global__ void __launch_bounds__(256) k_inv_rms_rows(const __nv_bfloat16* __restrict__ x, float* __restrict__ inv,
                                                      size_t rows, int d) {
  const size_t r = (size_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (r >= rows) return;
  float s = 0.f;
  for (int e = lane; e < d; e += 32) {
    const float v = __bfloat162float(x[r * d + e]);
    s += v * v;
  }
  s = rt::warp_sum(s);
  if (lane == 0) inv[r] = rsqrtf(s / (float)d + 1e-6f);
}

template <int BN>
cudaError_t launch_proj(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, const rt::EpiParams& p,
                        int sms, cudaStream_t st) {
  const long tiles = (long)((M + 127) / 128) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  rt::k_gemm_tc<BN, rt::EPI_PROJ>
      <<<grid, rt::GemmCfg<BN>::THREADS, rt::GemmCfg<BN>::SMEM_BYTES, st>>>(ta, tb, M, N, K, p, nullptr);
  return cudaGetLastError();
}

}  // namespace

extern "C" int rt_project_qkv_noalloc(const void* x, const void* W_qkv, int B, int N, int d, void* QKV,
                                      void* stream) {
  if (!x || !W_qkv || !QKV || B <= 0 || N <= 0 || d <= 0) return RT_ERR_INVALID_ARG;
  if (d % 64 != 0) return RT_ERR_UNSUPPORTED;
  const size_t rows = (size_t)B * N;
  if (rows > kMaxRows) return RT_ERR_WORKSPACE;   // beyond the fixed scratch array
  DeviceSlot* s = nullptr;
  int rc = setup_current_device(&s);
  if (rc != RT_OK) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  k_inv_rms_rows<<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(static_cast<const __nv_bfloat16*>(x), s->scratch,
                                                              rows, d);
  if (cudaGetLastError() != cudaSuccess) return RT_ERR_CUDA;
  // output-tile width: the widest with >= 120 tiles (as the allocating entry point)
  const long ntm = (long)((rows + 127) / 128);
  int bn = 32;
  for (int c : {256, 128, 64})
    if (ntm * ((3 * d + c - 1) / c) >= 120) { bn = c; break; }
  CUtensorMap ta, tb;
  if (!encode(&ta, x, d, rows, 128) || !encode(&tb, W_qkv, d, 3 * (uint64_t)d, bn)) return RT_ERR_INVALID_ARG;
  rt::EpiParams ep;
  memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = N; ep.xc = N; ep.d = d; ep.inv_rms = s->scratch; ep.qkv = static_cast<__nv_bfloat16*>(QKV);
  cudaError_t e;
  switch (bn) {
    case 256: e = launch_proj<256>(ta, tb, (int)rows, 3 * d, d, ep, s->sms, st); break;
    case 128: e = launch_proj<128>(ta, tb, (int)rows, 3 * d, d, ep, s->sms, st); break;
    case 64: e = launch_proj<64>(ta, tb, (int)rows, 3 * d, d, ep, s->sms, st); break;
    default: e = launch_proj<32>(ta, tb, (int)rows, 3 * d, d, ep, s->sms, st); break;
  }
  return e == cudaSuccess ? RT_OK : RT_ERR_CUDA;
}
