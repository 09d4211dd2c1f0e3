// C ABI of the kq library: host-side validation and dispatch (see include/kq.h).
//
// Every argument is checked here, before anything is enqueued; a rejected call
// leaves the stream untouched.  The library allocates nothing.
#include <cmath>
#include <cstdlib>
#include <cstdint>
#include <cstring>

#include "kq.h"
#include "kq_internal.h"

namespace {

thread_local int g_last_cuda_error = 0;

bool is_pow2(int64_t v) { return v > 0 && (v & (v - 1)) == 0; }

int ilog2(int64_t v) {
  int r = 0;
  while ((int64_t(1) << (r + 1)) <= v) ++r;
  return r;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

// Validates (dim, block) and fills the transform geometry.
kq_status make_geometry(int dim, int block, kq::Geometry* g) {
  const bool pow2 = is_pow2(dim) && dim >= 32 && dim <= 16384;
  const bool paley = (dim % 12 == 0) && is_pow2(dim / 12) && dim >= 384 && dim <= 12288;
  if (!pow2 && !paley) return KQ_ERR_UNSUPPORTED;
  int b = dim;
  if (block != 0) {
    if (block < 16 || !is_pow2(block) || block > dim || dim % block != 0)
      return KQ_ERR_UNSUPPORTED;
    b = block;
  }
  g->n = dim;
  g->b = b;
  g->paley = (b % 12 == 0 && !is_pow2(b)) ? 1 : 0;
  g->m = g->paley ? b / 12 : b;
  g->depth = ilog2(g->m) + (g->paley ? 11 : 0);
  g->sqrt_b = std::sqrt((double)b);
  g->inv_sqrt_b = (float)(1.0 / g->sqrt_b);
  g->sf_kc4 = 0;
  g->dyn = 0;
  return KQ_OK;
}

kq_status check_common(const void* x, int dtype, int64_t tokens, int dim, int block,
                       const int8_t* signs, kq::Geometry* g) {
  if (tokens < 0 || (tokens > 0 && !x)) return KQ_ERR_INVALID_ARG;
  if (dtype != KQ_F32 && dtype != KQ_BF16) return KQ_ERR_UNSUPPORTED;
  const kq_status st = make_geometry(dim, block, g);
  if (st != KQ_OK) return st;
  if (!aligned(x, 16)) return KQ_ERR_MISALIGNED;
  if (signs && !aligned(signs, 8)) return KQ_ERR_MISALIGNED;
  return KQ_OK;
}

kq_status finish(cudaError_t e) {
  if (e != cudaSuccess) {
    g_last_cuda_error = (int)e;
    return KQ_ERR_CUDA;
  }
  return KQ_OK;
}

// A simulated launch failure armed by kq_diag_fail_next_launch (this thread).
thread_local int g_fail_next_launch = 0;

// Runs a launcher (a validated call about to enqueue work) and turns its CUDA
// error into a status; an armed simulated failure is taken instead, and then
// nothing is enqueued.
template <class F>
kq_status dispatch(F&& launch) {
  if (g_fail_next_launch != 0) {
    const int e = g_fail_next_launch;
    g_fail_next_launch = 0;
    g_last_cuda_error = e;
    return KQ_ERR_CUDA;
  }
  return finish(launch());
}

// Format-specific argument checks shared by kq_dequant and
// kq_dequant_rht_inverse.
kq_status check_dequant(int fmt, const uint8_t* codes, const void* scales, const void* zeros,
                        const float* tensor_scale, int64_t tokens, int dim, int group,
                        const void* out) {
  if (!aligned(codes, 16) || !aligned(out, 16)) return KQ_ERR_MISALIGNED;
  switch (fmt) {
    case KQ_FMT_INT4_SYM:
      if (!aligned(scales, 4)) return KQ_ERR_MISALIGNED;
      break;
    case KQ_FMT_INT4_ASYM:
      if (group != 128 || dim % group != 0) return KQ_ERR_UNSUPPORTED;
      if (tokens > 0 && !zeros) return KQ_ERR_INVALID_ARG;
      if (!aligned(scales, 2) || !aligned(zeros, 2)) return KQ_ERR_MISALIGNED;
      break;
    case KQ_FMT_NVFP4:
      if (tokens > 0 && !tensor_scale) return KQ_ERR_INVALID_ARG;
      if (!aligned(tensor_scale, 4)) return KQ_ERR_MISALIGNED;
      break;
    case KQ_FMT_MXFP4:
      break;
    default:
      return KQ_ERR_INVALID_ARG;
  }
  return KQ_OK;
}

size_t nv_workspace_bytes(int64_t tokens) {
  return kq::kNvWorkspaceHeader + (size_t)tokens * sizeof(float2);
}

}  // namespace

namespace kq {
void set_last_cuda_error(int err) { g_last_cuda_error = err; }
}  // namespace kq

extern "C" {

KQ_API kq_status kq_rht(const void* x, int dtype, int64_t tokens, int dim, int block,
                        const int8_t* signs, float* out, int flags, kq_stream_t stream) {
  kq::Geometry g;
  kq_status st = check_common(x, dtype, tokens, dim, block, signs, &g);
  if (st != KQ_OK) return st;
  if (tokens > 0 && !out) return KQ_ERR_INVALID_ARG;
  if (flags & ~KQ_INVERSE) return KQ_ERR_INVALID_ARG;
  if (!aligned(out, 16)) return KQ_ERR_MISALIGNED;
  if (tokens == 0) return KQ_OK;
  if (!(flags & KQ_INVERSE) && kq::tc_row_supported(g, dtype, x, tokens))
    return dispatch([&] {
      return kq::launch_tc_rot(x, tokens, g, signs, out, reinterpret_cast<cudaStream_t>(stream));
    });
  if (!(flags & KQ_INVERSE) && kq::tcp_supported(g, dtype, x, tokens) && aligned(signs, 8))
    return dispatch([&] {
      return kq::launch_tcp_rot(x, tokens, g, signs, out, reinterpret_cast<cudaStream_t>(stream));
    });
  return dispatch([&] {
    return kq::launch_rht(x, dtype, tokens, g, signs, out, (flags & KQ_INVERSE) ? 1 : 0,
                          reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API kq_status kq_rht_quant_int4(const void* x, int dtype, int64_t tokens, int dim,
                                   int block, const int8_t* signs, int group, int asym,
                                   uint8_t* codes, void* scales, void* zeros,
                                   kq_stream_t stream) {
  kq::Geometry g;
  kq_status st = check_common(x, dtype, tokens, dim, block, signs, &g);
  if (st != KQ_OK) return st;
  if (tokens > 0 && (!codes || !scales)) return KQ_ERR_INVALID_ARG;
  if (asym != 0 && asym != 1) return KQ_ERR_INVALID_ARG;
  if (asym == 0) {
    if (group != 0) return KQ_ERR_UNSUPPORTED;
    if (zeros) return KQ_ERR_INVALID_ARG;
    if (!aligned(scales, 4)) return KQ_ERR_MISALIGNED;
  } else {
    if (group != 128 || dim % group != 0) return KQ_ERR_UNSUPPORTED;
    if (tokens > 0 && !zeros) return KQ_ERR_INVALID_ARG;
    if (!aligned(scales, 2) || !aligned(zeros, 2)) return KQ_ERR_MISALIGNED;
  }
  if (!aligned(codes, 16)) return KQ_ERR_MISALIGNED;
  if (tokens == 0) return KQ_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (asym == 1 && kq::tcb_supported(g, dtype, x, tokens))
    return dispatch([&] {
      return kq::launch_tcb_asym(x, tokens, g, signs, codes, static_cast<uint16_t*>(scales),
                                 static_cast<uint16_t*>(zeros), nullptr, 0, s);
    });
  if (asym == 1 && kq::blk128_supported(g, dtype) && aligned(signs, 16))
    return dispatch([&] {
      return kq::launch_blk128_asym(x, tokens, g, signs, codes, static_cast<uint16_t*>(scales),
                                    static_cast<uint16_t*>(zeros), nullptr, 0, s);
    });
  if (asym == 0 && kq::tcp_supported(g, dtype, x, tokens) && aligned(signs, 8))
    return dispatch([&] {
      return kq::launch_tcp_int4(x, tokens, g, signs, codes, static_cast<float*>(scales), s);
    });
  if (asym == 0 && kq::rowwarp_supported(g, dtype))
    return dispatch([&] {
      return kq::launch_rowwarp_int4(x, dtype, tokens, g, signs, codes, static_cast<float*>(scales),
                                     s);
    });
  if (asym == 0)
    return dispatch([&] {
      return kq::launch_int4_sym(x, dtype, tokens, g, signs, codes, static_cast<float*>(scales), s);
    });
  return dispatch([&] {
    return kq::launch_int4_asym(x, dtype, tokens, g, signs, group, codes,
                                static_cast<uint16_t*>(scales), static_cast<uint16_t*>(zeros), s);
  });
}

KQ_API kq_status kq_rht_quant_int4_kv(const void* x, int dtype, int64_t tokens, int dim,
                                      int block, const int8_t* signs, int group,
                                      const int64_t* slot_mapping, int64_t num_slots,
                                      uint8_t* codes_cache, uint16_t* scales_cache,
                                      uint16_t* zeros_cache, kq_stream_t stream) {
  kq::Geometry g;
  kq_status st = check_common(x, dtype, tokens, dim, block, signs, &g);
  if (st != KQ_OK) return st;
  if (num_slots < 0) return KQ_ERR_INVALID_ARG;
  if (tokens > 0 && (!slot_mapping || !codes_cache || !scales_cache || !zeros_cache))
    return KQ_ERR_INVALID_ARG;
  if (dtype != KQ_BF16 || group != 128 || g.b != 128 || g.paley) return KQ_ERR_UNSUPPORTED;
  if (!aligned(codes_cache, 16) || !aligned(scales_cache, 2) || !aligned(zeros_cache, 2) ||
      !aligned(slot_mapping, 8) || !aligned(signs, 16))
    return KQ_ERR_MISALIGNED;
  if (tokens == 0) return KQ_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kq::tcb_supported(g, dtype, x, tokens))
    return dispatch([&] {
      return kq::launch_tcb_asym(x, tokens, g, signs, codes_cache, scales_cache, zeros_cache,
                                 slot_mapping, num_slots, s);
    });
  if (kq::blk128_supported(g, dtype))
    return dispatch([&] {
      return kq::launch_blk128_asym(x, tokens, g, signs, codes_cache, scales_cache, zeros_cache,
                                    slot_mapping, num_slots, s);
    });
  return KQ_ERR_UNSUPPORTED;
}

KQ_API kq_status kq_rht_quant_nvfp4(const void* x, int dtype, int64_t tokens, int dim,
                                    int block, const int8_t* signs, uint8_t* codes,
                                    uint8_t* block_scales, float* tensor_scale,
                                    void* workspace, size_t ws_bytes, int flags,
                                    kq_stream_t stream) {
  kq::Geometry g;
  kq_status st = check_common(x, dtype, tokens, dim, block, signs, &g);
  if (st != KQ_OK) return st;
  if (tokens > 0 && (!codes || !block_scales || !tensor_scale)) return KQ_ERR_INVALID_ARG;
  const int mode = flags & (KQ_SCALE_STATIC | KQ_SCALE_DYNAMIC);
  constexpr int kPhases = KQ_DYN_STATS | KQ_DYN_EXACT | KQ_DYN_QUANT;
  if ((flags & ~(KQ_SCALE_STATIC | KQ_SCALE_DYNAMIC | KQ_SCALES_MMA | kPhases)) != 0)
    return KQ_ERR_INVALID_ARG;
  if (mode != KQ_SCALE_STATIC && mode != KQ_SCALE_DYNAMIC) return KQ_ERR_INVALID_ARG;
  if ((flags & kPhases) && mode != KQ_SCALE_DYNAMIC) return KQ_ERR_INVALID_ARG;
  g.dyn = (flags & kPhases) / KQ_DYN_STATS;
  if (!aligned(codes, 16) || !aligned(tensor_scale, 4)) return KQ_ERR_MISALIGNED;
  if (flags & KQ_SCALES_MMA) {
    // tensor-core scale-factor layout: whole 4-block atoms per row
    if (dim % 64 != 0) return KQ_ERR_UNSUPPORTED;
    if (!aligned(block_scales, 16)) return KQ_ERR_MISALIGNED;
    g.sf_kc4 = dim / 64;
  }
  kq::NvWorkspace* ws = nullptr;
  if (mode == KQ_SCALE_DYNAMIC) {
    if ((tokens > 0 && !workspace) || ws_bytes < nv_workspace_bytes(tokens))
      return KQ_ERR_INVALID_ARG;
    if (!aligned(workspace, 16)) return KQ_ERR_MISALIGNED;
    ws = static_cast<kq::NvWorkspace*>(workspace);
  }
  if (tokens == 0) return KQ_OK;
  if (kq::blk128_supported(g, dtype) && aligned(signs, 16) && aligned(block_scales, 8))
    return dispatch([&] {
      return kq::launch_blk128_nvfp4(x, tokens, g, signs, codes, block_scales, tensor_scale, ws,
                                     reinterpret_cast<cudaStream_t>(stream));
    });
  if (kq::tc_row_supported(g, dtype, x, tokens) && aligned(block_scales, 8))
    return dispatch([&] {
      return kq::launch_tc_nvfp4(x, tokens, g, signs, codes, block_scales, tensor_scale, ws,
                                 reinterpret_cast<cudaStream_t>(stream));
    });
  if (kq::rowwarp_supported(g, dtype) && aligned(block_scales, 8))
    return dispatch([&] {
      return kq::launch_rowwarp_nvfp4(x, dtype, tokens, g, signs, codes, block_scales, tensor_scale,
                                      ws, reinterpret_cast<cudaStream_t>(stream));
    });
  return dispatch([&] {
    return kq::launch_nvfp4(x, dtype, tokens, g, signs, codes, block_scales, tensor_scale, ws,
                            reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API kq_status kq_rht_quant_mxfp4(const void* x, int dtype, int64_t tokens, int dim,
                                    int block, const int8_t* signs, uint8_t* codes,
                                    uint8_t* scales, kq_stream_t stream) {
  kq::Geometry g;
  kq_status st = check_common(x, dtype, tokens, dim, block, signs, &g);
  if (st != KQ_OK) return st;
  if (tokens > 0 && (!codes || !scales)) return KQ_ERR_INVALID_ARG;
  if (!aligned(codes, 16)) return KQ_ERR_MISALIGNED;
  if (tokens == 0) return KQ_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (kq::tc_row_supported(g, dtype, x, tokens))
    return dispatch([&] { return kq::launch_tc_mxfp4(x, tokens, g, signs, codes, scales, s); });
  return dispatch([&] { return kq::launch_mxfp4(x, dtype, tokens, g, signs, codes, scales, s); });
}

KQ_API kq_status kq_dequant(int fmt, const uint8_t* codes, const void* scales,
                            const void* zeros, const float* tensor_scale, int64_t tokens,
                            int dim, int group, float* out, kq_stream_t stream) {
  if (tokens < 0 || (tokens > 0 && (!codes || !scales || !out))) return KQ_ERR_INVALID_ARG;
  if (dim <= 0 || dim % 32 != 0) return KQ_ERR_UNSUPPORTED;
  const kq_status st = check_dequant(fmt, codes, scales, zeros, tensor_scale, tokens, dim,
                                     group, out);
  if (st != KQ_OK) return st;
  if (tokens == 0) return KQ_OK;
  return dispatch([&] {
    return kq::launch_dequant(fmt, codes, scales, zeros, tensor_scale, tokens, dim, group, out,
                              reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API kq_status kq_dequant_rht_inverse(int fmt, const uint8_t* codes, const void* scales,
                                        const void* zeros, const float* tensor_scale,
                                        int64_t tokens, int dim, int block, int group,
                                        const int8_t* signs, void* out, int out_dtype,
                                        kq_stream_t stream) {
  if (tokens < 0 || (tokens > 0 && (!codes || !scales || !out))) return KQ_ERR_INVALID_ARG;
  if (out_dtype != KQ_F32 && out_dtype != KQ_BF16) return KQ_ERR_UNSUPPORTED;
  kq::Geometry g;
  kq_status st = make_geometry(dim, block, &g);
  if (st != KQ_OK) return st;
  if (signs && !aligned(signs, 8)) return KQ_ERR_MISALIGNED;
  st = check_dequant(fmt, codes, scales, zeros, tensor_scale, tokens, dim, group, out);
  if (st != KQ_OK) return st;
  if (tokens == 0) return KQ_OK;
  const cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int bf16 = out_dtype == KQ_BF16 ? 1 : 0;
  if (fmt == KQ_FMT_NVFP4 &&
      kq::tci_supported(g, codes, static_cast<const uint8_t*>(scales), signs, out))
    return dispatch([&] {
      return kq::launch_tcinv_nvfp4(codes, static_cast<const uint8_t*>(scales), tensor_scale,
                                    tokens, g, signs, out, bf16, s);
    });
  return dispatch([&] {
    return kq::launch_dequant_rht_inv(fmt, codes, scales, zeros, tensor_scale, tokens, g, group,
                                      signs, out, bf16, s);
  });
}

KQ_API kq_status kq_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                               const float* a_tensor_scale, const uint8_t* b_codes,
                               const uint8_t* b_scales, const float* b_tensor_scale, int64_t m,
                               int64_t n, int64_t k, void* c, int c_dtype, kq_stream_t stream) {
  if (m < 0 || n <= 0 || k <= 0) return KQ_ERR_INVALID_ARG;
  if (c_dtype != KQ_F32 && c_dtype != KQ_BF16) return KQ_ERR_UNSUPPORTED;
  if (n % 128 != 0 || k % 256 != 0) return KQ_ERR_UNSUPPORTED;
  // TMA coordinates are 32-bit: rows and row bytes below 2^31
  if (m >= (int64_t(1) << 31) || n >= (int64_t(1) << 31) || k >= (int64_t(1) << 32))
    return KQ_ERR_UNSUPPORTED;
  if (m == 0) return KQ_OK;
  if (!a_codes || !a_scales || !a_tensor_scale || !b_codes || !b_scales || !b_tensor_scale || !c)
    return KQ_ERR_INVALID_ARG;
  if (!aligned(a_codes, 16) || !aligned(b_codes, 16) || !aligned(a_scales, 16) ||
      !aligned(b_scales, 16) || !aligned(c, 16) || !aligned(a_tensor_scale, 4) ||
      !aligned(b_tensor_scale, 4))
    return KQ_ERR_MISALIGNED;
  return dispatch([&] {
    return kq::launch_gemm_nvfp4(a_codes, a_scales, a_tensor_scale, b_codes, b_scales,
                                 b_tensor_scale, m, n, k, c, c_dtype == KQ_BF16 ? 1 : 0,
                                 reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API kq_status kq_device_errors(unsigned int* flags) {
  if (!flags) return KQ_ERR_INVALID_ARG;
  cudaError_t e = kq::take_tc_errors(&flags[0]);
  if (e == cudaSuccess) e = kq::take_tcp_errors(&flags[1]);
  if (e == cudaSuccess) e = kq::take_tcb_errors(&flags[2]);
  if (e == cudaSuccess) e = kq::take_tci_errors(&flags[3]);
  if (e == cudaSuccess) e = kq::take_diag_errors(&flags[4]);
  if (e == cudaSuccess) e = kq::take_gemm_errors(&flags[5]);
  return finish(e);
}

KQ_API kq_status kq_diag_wait_timeout(long long limit_cycles, kq_stream_t stream) {
  if (limit_cycles <= 0 || limit_cycles > 4000000000ll) return KQ_ERR_INVALID_ARG;
  return dispatch([&] {
    return kq::launch_diag_wait(limit_cycles, reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API size_t kq_workspace_size(int64_t tokens, int dim, int block) {
  kq::Geometry g;
  if (tokens < 0 || make_geometry(dim, block, &g) != KQ_OK) return 0;
  return nv_workspace_bytes(tokens);
}

KQ_API const char* kq_status_str(int status) {
  switch (status) {
    case KQ_OK: return "KQ_OK";
    case KQ_ERR_INVALID_ARG: return "KQ_ERR_INVALID_ARG";
    case KQ_ERR_UNSUPPORTED: return "KQ_ERR_UNSUPPORTED";
    case KQ_ERR_MISALIGNED: return "KQ_ERR_MISALIGNED";
    case KQ_ERR_CUDA: return "KQ_ERR_CUDA";
    default: return "KQ_ERR_UNKNOWN";
  }
}

KQ_API int kq_last_cuda_error(void) { return g_last_cuda_error; }

KQ_API void kq_diag_fail_next_launch(int cuda_error) { g_fail_next_launch = cuda_error; }

KQ_API int kq_version(void) { return (1 << 16) | 1; }

static kq_status diag_tc_steps(const uint16_t* a, const uint16_t* b, float* d1, float* d2,
                               unsigned int* status, int fp16, kq_stream_t stream) {
  if (!a || !b || !d1 || !d2 || !status) return KQ_ERR_INVALID_ARG;
  if (!aligned(a, 2) || !aligned(b, 2) || !aligned(d1, 4) || !aligned(d2, 4) ||
      !aligned(status, 4))
    return KQ_ERR_MISALIGNED;
  return dispatch([&] {
    return kq::launch_diag_tc_steps(a, b, d1, d2, status, fp16,
                                    reinterpret_cast<cudaStream_t>(stream));
  });
}

KQ_API kq_status kq_diag_tc_steps(const uint16_t* a, const uint16_t* b, float* d1, float* d2,
                                  unsigned int* status, kq_stream_t stream) {
  return diag_tc_steps(a, b, d1, d2, status, 0, stream);
}

KQ_API kq_status kq_diag_tc_steps_f16(const uint16_t* a, const uint16_t* b, float* d1,
                                      float* d2, unsigned int* status, kq_stream_t stream) {
  return diag_tc_steps(a, b, d1, d2, status, 1, stream);
}

}  // extern "C"
