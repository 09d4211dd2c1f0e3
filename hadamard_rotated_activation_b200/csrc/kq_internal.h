// Internal interface between the C ABI (kq_api.cu) and the kernel files.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_runtime.h>

#include "kq_device.cuh"

namespace kq {

// Workspace of the dynamic NVFP4 tensor scale.
//   lower_bits: fp32 bits of a lower bound on max|S| over the tensor
//   gmax_bits:  fp64 bits of the exact max|S| (unnormalised)
//   rows[t]:    (computed row max |S_hat|, error bound) per row
struct NvWorkspace {
  unsigned int lower_bits;
  unsigned int pad_;
  unsigned long long gmax_bits;
  float2 rows[1];
};
constexpr size_t kNvWorkspaceHeader = 16;

// 2-D bf16 tensor map over a row-major [rows, cols] array (cols * 2 bytes a
// row, a multiple of 16), boxes of box_cols x box_rows.  False when the driver
// refuses it.
bool encode_tmap_bf16_2d(CUtensorMap* map, const void* base, uint64_t cols, uint64_t rows,
                         uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// General 2-D tensor map: `rows` rows of `row_bytes` bytes (a multiple of 16),
// `cols` elements of the given type a row, boxes of box_cols x box_rows.
bool encode_tmap_2d(CUtensorMap* map, const void* base, CUtensorMapDataType dtype,
                    uint32_t elem_bytes, uint64_t cols, uint64_t rows, uint64_t row_bytes,
                    uint32_t box_cols, uint32_t box_rows, CUtensorMapSwizzle swizzle);

// NVFP4 x NVFP4 GEMM on the block-scaled tensor cores (kq_gemm.cu):
// C[M, N] = t_a t_b sum_k A[m][k] B[n][k], codes K-major, block scales in the
// tensor-core layout (Geometry::sf_kc4), C fp32 or bf16 row-major.
cudaError_t launch_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                              const float* a_tscale, const uint8_t* b_codes,
                              const uint8_t* b_scales, const float* b_tscale, int64_t m,
                              int64_t n, int64_t k, void* c, int c_bf16, cudaStream_t s);
cudaError_t take_gemm_errors(unsigned int* out);

// Records a CUDA error for kq_last_cuda_error() on the calling thread.
void set_last_cuda_error(int err);

cudaError_t launch_rht(const void* x, int dtype, int64_t tokens, const Geometry& g,
                       const int8_t* signs, float* out, int inverse, cudaStream_t s);
cudaError_t launch_int4_sym(const void* x, int dtype, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, float* scales,
                            cudaStream_t s);
cudaError_t launch_int4_asym(const void* x, int dtype, int64_t tokens, const Geometry& g,
                             const int8_t* signs, int group, uint8_t* codes,
                             uint16_t* scales, uint16_t* zeros, cudaStream_t s);
cudaError_t launch_nvfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                         const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                         float* tensor_scale, NvWorkspace* ws, cudaStream_t s);
cudaError_t launch_nvfp4_global(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                const int8_t* signs, NvWorkspace* ws, cudaStream_t s);

// Fast kernels for 128-wide Hadamard blocks on bf16 rows (kq_block.cu).
bool blk128_supported(const Geometry& g, int dtype);
cudaError_t launch_blk128_nvfp4(const void* x, int64_t tokens, const Geometry& g,
                                const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                                float* tensor_scale, NvWorkspace* ws, cudaStream_t s);
cudaError_t launch_blk128_asym(const void* x, int64_t tokens, const Geometry& g,
                               const int8_t* signs, uint8_t* codes, uint16_t* scales,
                               uint16_t* zeros, const int64_t* slots, int64_t num_slots,
                            cudaStream_t s);

// Warp-per-row kernels for full-row transforms of 2048 or 4096 (kq_rowwarp.cu).
bool rowwarp_supported(const Geometry& g, int dtype);
cudaError_t launch_rowwarp_int4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                const int8_t* signs, uint8_t* codes, float* scales,
                                cudaStream_t s);
cudaError_t launch_rowwarp_nvfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                 const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                                 float* tensor_scale, NvWorkspace* ws, cudaStream_t s);

// Tensor-core kernels for full-row 4096 transforms of bf16 rows (kq_tc.cu).
bool tc_row_supported(const Geometry& g, int dtype, const void* x, int64_t tokens);
cudaError_t launch_tc_nvfp4(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                            float* tensor_scale, NvWorkspace* ws, cudaStream_t s);
cudaError_t launch_tc_rot(const void* x, int64_t tokens, const Geometry& g, const int8_t* signs,
                          float* out, cudaStream_t s);
int tc_error_flag();

// Tensor-core kernels for 12288-wide rows (H_12 kron H_1024) of bf16 input (kq_tcp.cu).
bool tcp_supported(const Geometry& g, int dtype, const void* x, int64_t tokens);
cudaError_t launch_tcp_int4(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, float* scales, cudaStream_t s);
cudaError_t launch_tcp_rot(const void* x, int64_t tokens, const Geometry& g,
                           const int8_t* signs, float* out, cudaStream_t s);
cudaError_t launch_diag_tc_steps(const uint16_t* a, const uint16_t* b, float* d1, float* d2,
                                 unsigned int* status, int fp16, cudaStream_t s);

cudaError_t launch_tc_mxfp4(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, uint8_t* scales,
                            cudaStream_t s);
cudaError_t launch_mxfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                         const int8_t* signs, uint8_t* codes, uint8_t* scales,
                         cudaStream_t s);
cudaError_t launch_dequant(int fmt, const uint8_t* codes, const void* scales,
                           const void* zeros, const float* tensor_scale, int64_t tokens,
                           int n, int group, float* out, cudaStream_t s);
cudaError_t launch_dequant_rht_inv(int fmt, const uint8_t* codes, const void* scales,
                                  const void* zeros, const float* tensor_scale,
                                  int64_t tokens, const Geometry& g, int group,
                                  const int8_t* signs, void* out, int out_bf16, cudaStream_t s);
// Block-128 rotation + asymmetric INT4 g128 on the tensor cores.
bool tcb_supported(const Geometry& g, int dtype, const void* x, int64_t tokens);
cudaError_t launch_tcb_asym(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, uint16_t* scales,
                            uint16_t* zeros, const int64_t* slots, int64_t num_slots,
                            cudaStream_t s);
// NVFP4 dequant + inverse rotation of 4096-wide rows on the tensor cores.
bool tci_supported(const Geometry& g, const uint8_t* codes, const uint8_t* scales,
                   const int8_t* signs, const void* out);
cudaError_t launch_tcinv_nvfp4(const uint8_t* codes, const uint8_t* scales,
                               const float* tensor_scale, int64_t tokens, const Geometry& g,
                               const int8_t* signs, void* out, int out_bf16, cudaStream_t s);

// Error words of the kernel families (read and cleared; device-synchronous).
cudaError_t take_tc_errors(unsigned int* out);
cudaError_t take_tcp_errors(unsigned int* out);
cudaError_t take_tcb_errors(unsigned int* out);
cudaError_t take_tci_errors(unsigned int* out);
cudaError_t take_diag_errors(unsigned int* out);
cudaError_t launch_diag_wait(long long limit_cycles, cudaStream_t s);

}  // namespace kq
