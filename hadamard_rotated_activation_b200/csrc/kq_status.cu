// Device-side failure reports of the tensor-core kernels, and a diagnostic
// that exercises the reporting path.  Every wait of those kernels on an
// mbarrier is bounded; when one runs out the kernel records a bit in its
// family's error word and returns instead of hanging.  kq_device_errors reads
// and clears the words.  The diagnostic kernel waits on an mbarrier that
// nothing ever arrives at, with a short cycle limit, so its timeout (and only
// that) sets the diagnostic word.  The pages have no counterpart to either.
#include <cstdint>

#include "kq_internal.h"
#include "kq_sm100.cuh"

namespace kq {
namespace diag {

__device__ unsigned int g_diag_error = 0;

__global__ void k_diag_wait(long long limit_cycles) {
  __shared__ uint64_t bar;
  if (threadIdx.x == 0) {
    sm100::mbar_init(&bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    // phase 0 never completes: the single expected arrival never happens
    const uint32_t a = sm100::smem_u32(&bar);
    const long long start = clock64();
    for (;;) {
      uint32_t ok;
      asm volatile("{\n\t.reg .pred p;\n\t"
                   "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                   "selp.u32 %0, 1, 0, p;\n\t}"
                   : "=r"(ok) : "r"(a), "r"(0u), "r"(1000u) : "memory");
      if (ok) break;
      if (clock64() - start > limit_cycles) {
        atomicOr(&g_diag_error, 1u);
        break;
      }
    }
  }
}

}  // namespace diag

cudaError_t launch_diag_wait(long long limit_cycles, cudaStream_t s) {
  diag::k_diag_wait<<<1, 32, 0, s>>>(limit_cycles);
  return cudaGetLastError();
}

cudaError_t take_diag_errors(unsigned int* out) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, diag::g_diag_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(diag::g_diag_error, &zero, sizeof(unsigned int));
}

}  // namespace kq
