// Allocation-free variant of the dynamic-scale NVFP4 entry point.
//
// kq_rht_quant_nvfp4 in dynamic mode needs a device workspace from the caller.
// Some callers cannot provide one: a plugin whose host framework owns all
// device memory and hands out no workspace, or a serving loop that reserves
// HBM up front and may not call cudaMalloc (which can also synchronize the
// device) on its hot path.  This entry point keeps that workspace in a
// fixed-size array in the library's own device memory instead.
//
// The array lives in every GPU that loads the library until the process exits.
// Host code only sees a host-side stand-in for it, so its device address is
// looked up with the device current and cached per device and context.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <mutex>

#include "kq.h"
#include "kq_internal.h"

namespace {

constexpr size_t kScratchBytes = KQ_NOALLOC_SCRATCH_BYTES;
static_assert(kScratchBytes % 256 == 0, "scratch size");

__device__ __align__(256) unsigned char g_nvfp4_scratch[kScratchBytes];

constexpr int kMaxDevices = 64;
std::mutex g_mu;
void* g_scratch_ptr[kMaxDevices] = {};
CUcontext g_scratch_ctx[kMaxDevices] = {};

// The driver's cuCtxGetCurrent, through the runtime (no link against libcuda).
PFN_cuCtxGetCurrent_v4000 get_ctx_fn() {
  static PFN_cuCtxGetCurrent_v4000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
  });
  return fn;
}

// Device address of g_nvfp4_scratch in the current context (nullptr on
// error).  The address is cached per device together with the context it was
// looked up in: after cudaDeviceReset, or with another context current, the
// module is loaded anew at another address and the lookup is repeated.
void* scratch_on_current_device(cudaError_t* err) {
  int dev = 0;
  *err = cudaGetDevice(&dev);
  if (*err != cudaSuccess) return nullptr;
  if (dev < 0 || dev >= kMaxDevices) {
    *err = cudaErrorInvalidDevice;
    return nullptr;
  }
  PFN_cuCtxGetCurrent_v4000 cur = get_ctx_fn();
  if (!cur) {
    *err = cudaErrorDeviceUninitialized;
    return nullptr;
  }
  CUcontext ctx = nullptr;
  if (cur(&ctx) != CUDA_SUCCESS) {
    *err = cudaErrorDeviceUninitialized;
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(g_mu);
  if (!ctx || !g_scratch_ptr[dev] || g_scratch_ctx[dev] != ctx) {
    // the lookup also creates the device's primary context if none is current
    void* p = nullptr;
    *err = cudaGetSymbolAddress(&p, g_nvfp4_scratch);
    if (*err != cudaSuccess) return nullptr;
    if (!ctx && (cur(&ctx) != CUDA_SUCCESS || !ctx)) {
      *err = cudaErrorDeviceUninitialized;
      return nullptr;
    }
    g_scratch_ptr[dev] = p;
    g_scratch_ctx[dev] = ctx;
  }
  return g_scratch_ptr[dev];
}

}  // namespace

extern "C" KQ_API kq_status kq_rht_quant_nvfp4_dynamic_noalloc(
    const void* x, int dtype, int64_t tokens, int dim, int block, const int8_t* signs,
    uint8_t* codes, uint8_t* block_scales, float* tensor_scale, kq_stream_t stream) {
  if (tokens < 0) return KQ_ERR_INVALID_ARG;
  if (tokens > (int64_t)KQ_NOALLOC_MAX_TOKENS) return KQ_ERR_UNSUPPORTED;
  const size_t need = kq_workspace_size(tokens, dim, block);
  if (need == 0) return KQ_ERR_UNSUPPORTED;   // bad dim/block
  if (need > kScratchBytes) return KQ_ERR_UNSUPPORTED;
  if (tokens == 0)
    return kq_rht_quant_nvfp4(x, dtype, 0, dim, block, signs, codes, block_scales,
                              tensor_scale, nullptr, need, KQ_SCALE_DYNAMIC, stream);
  cudaError_t err = cudaSuccess;
  void* ws = scratch_on_current_device(&err);
  if (!ws) {
    kq::set_last_cuda_error((int)err);
    return KQ_ERR_CUDA;
  }
  return kq_rht_quant_nvfp4(x, dtype, tokens, dim, block, signs, codes, block_scales,
                            tensor_scale, ws, kScratchBytes, KQ_SCALE_DYNAMIC, stream);
}
