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
// streams, or different host threads) race on it. The error word
// g_noalloc_err, also file-scope, collects bounded-wait timeouts of every call
// on the device until rt_project_qkv_noalloc_status reads and clears it.
//
// Host code must not pass either symbol itself to a kernel: on the host it
// names a host-side stand-in, not device memory. The first call on each device
// (with that device current) looks up the device addresses with
// cudaGetSymbolAddress and caches them; make that first call before any stream
// capture.
#include <cstring>
#include <mutex>

#include "../../include/rtlayer.h"
#include "rt_common.cuh"
#include "rt_gemm_tc.cuh"
#include "rt_host.h"
#include "rt_rownorm.cuh"

namespace {

constexpr size_t kMaxRows = size_t(1) << 20;   // B*N limit: 4 MiB of fp32
static __device__ __align__(256) float g_inv_rms_scratch[kMaxRows];
static __device__ unsigned g_noalloc_err[4];   // error word (+ the debug build's failure record)

struct DeviceSlot {
  bool ready = false;
  int sms = 0;
  float* scratch = nullptr;   // device address of g_inv_rms_scratch on this device
  unsigned* err = nullptr;    // device address of g_noalloc_err on this device
};
std::mutex g_mu;
DeviceSlot g_slots[64];

template <int BN>
cudaError_t set_proj_attr() {
  return cudaFuncSetAttribute(rt::k_gemm_tc<BN, rt::EPI_PROJ>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              (int)rt::GemmCfg<BN>::SMEM_BYTES);
}

// One-time set-up of the current device: sm_100 check, SM count, tensor-map
// encoder, kernel attributes and the device addresses of the scratch array and
// the error word (the latter cleared once here).
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
    if (!rt::load_tensor_map_encoder()) return RT_ERR_CUDA;
    cudaError_t e;
    if ((e = set_proj_attr<32>()) != cudaSuccess || (e = set_proj_attr<64>()) != cudaSuccess ||
        (e = set_proj_attr<128>()) != cudaSuccess || (e = set_proj_attr<256>()) != cudaSuccess)
      return rt::cuda_failure(e);
    void* p = nullptr;
    if ((e = cudaGetSymbolAddress(&p, g_inv_rms_scratch)) != cudaSuccess) return rt::cuda_failure(e);
    if (!p) return RT_ERR_CUDA;
    void* q = nullptr;
    if ((e = cudaGetSymbolAddress(&q, g_noalloc_err)) != cudaSuccess) return rt::cuda_failure(e);
    if (!q) return RT_ERR_CUDA;
    if ((e = cudaMemset(q, 0, sizeof(g_noalloc_err))) != cudaSuccess) return rt::cuda_failure(e);
    s.scratch = static_cast<float*>(p);
    s.err = static_cast<unsigned*>(q);
    s.ready = true;
  }
  *out = &s;
  return RT_OK;
}

template <int BN>
cudaError_t launch_proj(const CUtensorMap& ta, const CUtensorMap& tb, int M, int N, int K, const rt::EpiParams& p,
                        unsigned* err, int sms, cudaStream_t st) {
  const long tiles = (long)((M + 127) / 128) * ((N + BN - 1) / BN);
  const int grid = (int)(tiles < sms ? tiles : sms);
  rt::k_gemm_tc<BN, rt::EPI_PROJ>
      <<<grid, rt::GemmCfg<BN>::THREADS, rt::GemmCfg<BN>::SMEM_BYTES, st>>>(ta, tb, M, N, K, p, err);
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
  // the same 1/rms kernel and tile choice as rt_project_qkv
  rt::k_row_inv_rms<__nv_bfloat16><<<(unsigned)((rows + 7) / 8), 256, 0, st>>>(
      static_cast<const __nv_bfloat16*>(x), s->scratch, rows, d, rt::kEps);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return rt::cuda_failure(e);
  const int bn = rt::choose_bn((int)rows, 3 * d);
  CUtensorMap ta, tb;
  if (!rt::make_tmap(&ta, x, d, rows, 128) || !rt::make_tmap(&tb, W_qkv, d, 3 * (uint64_t)d, bn))
    return RT_ERR_INVALID_ARG;
  rt::EpiParams ep;
  memset(&ep, 0, sizeof(ep));
  ep.B = B; ep.Nseq = N; ep.xc = N; ep.d = d; ep.inv_rms = s->scratch; ep.qkv = static_cast<__nv_bfloat16*>(QKV);
  switch (bn) {
    case 256: e = launch_proj<256>(ta, tb, (int)rows, 3 * d, d, ep, s->err, s->sms, st); break;
    case 128: e = launch_proj<128>(ta, tb, (int)rows, 3 * d, d, ep, s->err, s->sms, st); break;
    case 64: e = launch_proj<64>(ta, tb, (int)rows, 3 * d, d, ep, s->err, s->sms, st); break;
    default: e = launch_proj<32>(ta, tb, (int)rows, 3 * d, d, ep, s->err, s->sms, st); break;
  }
  return e == cudaSuccess ? RT_OK : rt::cuda_failure(e);
}

extern "C" int rt_project_qkv_noalloc_status(void* stream) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return RT_ERR_DEVICE;
  unsigned* err = nullptr;
  {
    std::lock_guard<std::mutex> lk(g_mu);
    if (!g_slots[dev].ready) return RT_ERR_DEVICE;
    err = g_slots[dev].err;
  }
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  unsigned h = 0;
  cudaError_t e;
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return rt::cuda_failure(e);
  if ((e = cudaMemcpyAsync(&h, err, sizeof(h), cudaMemcpyDeviceToHost, st)) != cudaSuccess) return rt::cuda_failure(e);
  if ((e = cudaMemsetAsync(err, 0, sizeof(h), st)) != cudaSuccess) return rt::cuda_failure(e);
  if ((e = cudaStreamSynchronize(st)) != cudaSuccess) return rt::cuda_failure(e);
  return (h & rt::RT_DEVERR_TIMEOUT) ? RT_ERR_TIMEOUT : RT_OK;
}
