// Tensor-core (tcgen05) kernel for the NVFP4 round trip of 4096-wide rows:
// dequantize and apply the inverse rotation in one pass,
//   x'_j = s_j / sqrt(n) * sum_i H[i][j] yq_i,   yq_i = E2M1(code_i) E4M3(s_b) t
// (QuaRot reviews, review 2 Summary: the RHT is invertible; the inverse of
// y = H D x / sqrt(n) is x = D H^T y / sqrt(n), and H^T = H for Sylvester).
//
// yq_i = z_i t with z_i = E2M1(code_i) E4M3(s_b) exact in fp16 (at most six
// significant bits, between 2^-10 and 2688), so the kernel rotates z on the
// tensor cores and scales by t / sqrt(n) afterwards.  The layout is that of
// the forward 4096-wide kernel: a row is 128 rows of 32 (i = a*32 + beta); D =
// H_128 z' over a on the tensor cores (A = H_128, B = z of four tokens,
// MN-major, 64-byte swizzle), then H_32 over beta in the epilogue thread that
// owns TMEM lane o; it holds outputs o*32 .. o*32+31, multiplies by
// t / sqrt(n), applies the signs and stores fp32 or bf16 (rounded to nearest).
//
// Warp roles (14 warps, up to 128 registers a thread): 0 copies (1-D bulk
// copies of the codes and block scales of four tokens), 1 MMA issuer + TMEM
// owner, 2-5 decode (one per token: E2M1 and E4M3 to fp16 with the
// conversion instructions), 6-13 epilogue (two groups of four, alternate
// tiles).  An epilogue warp's outputs of a token are 4 KB of contiguous
// fp32; they pass through a 4 KB shared-memory buffer so that the stores to
// global memory are coalesced.  Every wait is bounded; on timeout the kernel
// records an error code and returns.
#include <cuda.h>

#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_sm100.cuh"

namespace kq {
namespace tci {

using namespace sm100;

constexpr int N = 4096;
constexpr int kTok = 4;                          // tokens per tile
constexpr uint32_t kTokBytes = 128 * 32 * 2;     // z of one token: 128 rows of 32 fp16
constexpr uint32_t kZBytes = kTok * kTokBytes;   // 32 KB
constexpr uint32_t kCodeBytes = N / 2;           // per token
constexpr uint32_t kScaleBytes = N / 16;         // per token
constexpr uint32_t kRawBytes = kTok * (kCodeBytes + kScaleBytes);   // 9 KB
constexpr int kStages = 3;
constexpr int kGroups = 2;
constexpr int kAcc = 4;
constexpr int kAccCols = 32 * kTok;
constexpr int kTmemCols = kAcc * kAccCols;
constexpr int kDecodeWarps = kTok;
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kThreads = 32 * (2 + kDecodeWarps + kEpiWarps);
static_assert((kTmemCols & (kTmemCols - 1)) == 0 && kTmemCols <= 512, "TMEM columns");

__device__ unsigned int g_tci_error = 0;         // nonzero: a wait timed out

struct Params {
  const uint8_t* codes;         // [T, n/2]
  const uint8_t* scales8;       // [T, n/16] E4M3
  const float* tensor_scale;    // device
  const int8_t* signs;          // [n] or null
  void* out;                    // [T, n] fp32 or bf16
  int64_t tokens;
  int64_t tiles;
};

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
  return sm100::mbar_wait(bar, parity, &g_tci_error);
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
// Byte offset of 16-byte chunk c (0..3) of row a of a token's z (64-byte
// swizzle: chunk position c ^ ((a >> 1) & 3)), as the MMA's B operand reads it.
__device__ __forceinline__ uint32_t tok_chunk(int a, int c) {
  return (uint32_t)(a * 64 + ((c ^ ((a >> 1) & 3)) << 4));
}
// fp16x2 of two E2M1 codes (the low nibble to the low half).
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t byte) {
  uint32_t d;
  asm("{\n\t.reg .b8 b;\n\tcvt.u8.u32 b, %1;\n\tcvt.rn.f16x2.e2m1x2 %0, b;\n\t}"
      : "=r"(d) : "r"(byte));
  return d;
}
// fp16x2 (s, s) of one E4M3 code s.
__device__ __forceinline__ uint32_t e4m3_to_f16x2_dup(uint32_t code) {
  uint32_t d;
  const uint16_t two = (uint16_t)(code | (code << 8));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(d) : "h"(two));
  return d;
}
// bf16x2 of (lo, hi), each rounded to nearest even.
__device__ __forceinline__ uint32_t bf16x2_rn(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}
__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// f16 operands: A = H_128 (K-major), B = z (MN-major), M = N = 128.
constexpr uint32_t kIdesc = (1u << 4) | (0u << 7) | (0u << 10) | (1u << 16) |
                            ((uint32_t)(kAccCols >> 3) << 17) | ((128u >> 4) << 24);

template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads, 1) k_tcinv4096(Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // 32 KB: A = H_128 (fp16)
  uint8_t* sZ = smem + 32768;                           // kStages x 32 KB
  uint8_t* sRaw = sZ + kStages * kZBytes;               // kStages x 9 KB: codes, then scales
  uint8_t* sOut = sRaw + kStages * kRawBytes;            // 4 KB per epilogue warp
  uint64_t* bars = reinterpret_cast<uint64_t*>(sOut + kEpiWarps * 4096);
  uint64_t* full = bars;                                // codes and scales landed
  uint64_t* ready = bars + kStages;                     // z written
  uint64_t* empty = bars + 2 * kStages;                 // MMAs done with the stage
  uint64_t* tfull = bars + 3 * kStages;                 // accumulator written (kAcc)
  uint64_t* tempty = tfull + kAcc;                      // accumulator read (kAcc)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kAcc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t my_tiles = (P.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  // ---- set-up: barriers and the first copies, then A and TMEM
  int64_t prefilled = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 32 * kDecodeWarps);
      mbar_init(&empty[s], 1);
    }
    for (int d = 0; d < kAcc; ++d) {
      mbar_init(&tfull[d], 1);
      mbar_init(&tempty[d], 128);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    prefilled = my_tiles < kStages ? my_tiles : kStages;
    for (int64_t k = 0; k < prefilled; ++k) {
      const int64_t tile = blockIdx.x + k * gridDim.x;
      const int64_t t0 = tile * kTok;
      const int64_t nt = P.tokens - t0 < kTok ? P.tokens - t0 : kTok;
      uint8_t* raw = sRaw + k * kRawBytes;
      mbar_expect_tx(&full[k], (uint32_t)nt * (kCodeBytes + kScaleBytes));
      bulk_load(raw, P.codes + t0 * kCodeBytes, (uint32_t)nt * kCodeBytes, &full[k]);
      bulk_load(raw + kTok * kCodeBytes, P.scales8 + t0 * kScaleBytes,
                (uint32_t)nt * kScaleBytes, &full[k]);
    }
  }
  for (int idx = threadIdx.x; idx < 128 * 16; idx += blockDim.x) {
    const int m = idx >> 4, k0 = (idx & 15) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = (__popc(m & (k0 + 2 * e)) & 1) ? 0xBC00u : 0x3C00u;   // -1 / +1
      const uint32_t hi = (__popc(m & (k0 + 2 * e + 1)) & 1) ? 0xBC00u : 0x3C00u;
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(sA + a_off(m, k0)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "n"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ================= copies: codes and block scales of four tokens
    if (lane == 0) {
      int64_t issued = prefilled;
      for (int64_t k = prefilled; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        if (!wait(&empty[s], (uint32_t)(k / kStages - 1) & 1)) break;
        const int64_t tile = blockIdx.x + k * gridDim.x;
        const int64_t t0 = tile * kTok;
        const int64_t nt = P.tokens - t0 < kTok ? P.tokens - t0 : kTok;
        uint8_t* raw = sRaw + s * kRawBytes;
        mbar_expect_tx(&full[s], (uint32_t)nt * (kCodeBytes + kScaleBytes));
        bulk_load(raw, P.codes + t0 * kCodeBytes, (uint32_t)nt * kCodeBytes, &full[s]);
        bulk_load(raw + kTok * kCodeBytes, P.scales8 + t0 * kScaleBytes,
                  (uint32_t)nt * kScaleBytes, &full[s]);
        issued = k + 1;
      }
      for (int64_t k = issued > kStages ? issued - kStages : 0; k < issued; ++k)
        wait(&full[k % kStages], (uint32_t)(k / kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        const int d = (int)(k % kAcc);
        if (!wait(&ready[s], (uint32_t)(k / kStages) & 1)) break;
        if (k >= kAcc && !wait(&tempty[d], (uint32_t)(k / kAcc - 1) & 1)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sZ + s * kZBytes);
        const uint32_t tmem_d = tmem_base + (uint32_t)(d * kAccCols);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint64_t adesc = smem_desc(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2);
          const uint64_t bdesc = smem_desc(b0 + ks * 1024, kTokBytes, 512, 4);
          sm100::mma_bf16(tmem_d, adesc, bdesc, kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[d]);
        issued = k + 1;
      }
      for (int64_t k = issued > kAcc ? issued - kAcc : 0; k < issued; ++k)
        wait(&tfull[k % kAcc], (uint32_t)(k / kAcc) & 1);
    }
  } else if (warp < 2 + kDecodeWarps) {
    // ================= decode: warp t writes token t.  Lane l, step i: row
    // a = (l & 7) + 8 i, chunk column c = l >> 3, so each group of eight lanes
    // stores eight rows of one column (eight distinct 16-byte bank groups
    // under the swizzle) and the warp's 4-byte code reads cover 128
    // contiguous bytes.
    const int t = warp - 2;
    const int c = lane >> 3;
    const int a0 = lane & 7;
    for (int64_t k = 0; k < my_tiles; ++k) {
      const int s = (int)(k % kStages);
      if (!wait(&full[s], (uint32_t)(k / kStages) & 1)) break;
      const uint8_t* raw = sRaw + s * kRawBytes;
      const uint8_t* cr = raw + t * kCodeBytes;
      const uint8_t* sr = raw + kTok * kCodeBytes + t * kScaleBytes;
      uint8_t* zt = sZ + s * kZBytes + t * kTokBytes;
#pragma unroll 4
      for (int i = 0; i < 16; ++i) {
        const int a = a0 + 8 * i;
        // elements a*32 + c*8 .. +7: code bytes a*16 + c*4 .. +3, block 2a + c/2
        const uint32_t w = *reinterpret_cast<const uint32_t*>(cr + a * 16 + c * 4);
        const uint32_t sc = e4m3_to_f16x2_dup(sr[2 * a + (c >> 1)]);
        uint4 z;
        z.x = hmul2(e2m1x2_to_f16x2(w & 0xffu), sc);
        z.y = hmul2(e2m1x2_to_f16x2((w >> 8) & 0xffu), sc);
        z.z = hmul2(e2m1x2_to_f16x2((w >> 16) & 0xffu), sc);
        z.w = hmul2(e2m1x2_to_f16x2(w >> 24), sc);
        *reinterpret_cast<uint4*>(zt + tok_chunk(a, c)) = z;
      }
      fence_async_smem();
      __syncwarp();
      mbar_arrive(&ready[s]);
    }
  } else {
    // ================= epilogue: group g of warps 10+4g .. 13+4g
    const int g = (warp - 2 - kDecodeWarps) >> 2;
    const int q = warp & 3;
    const int o = q * 32 + lane;              // accumulator row: outputs o*32 .. +31
    uint32_t sbits = 0;                       // sign bits of those outputs (bit e: element e)
    if (P.signs) {
      const uint4* sv = reinterpret_cast<const uint4*>(P.signs + o * 32);
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const uint4 v = __ldg(sv + h);
        const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int b = 0; b < 16; ++b)
          sbits |= ((ww[b >> 2] >> (8 * (b & 3) + 7)) & 1u) << (16 * h + b);
      }
    }
    const float scale = *P.tensor_scale * 0x1p-6f;   // t / sqrt(4096)
    uint8_t* wbuf = sOut + (warp - 2 - kDecodeWarps) * 4096;
    for (int64_t k = g; k < my_tiles; k += kGroups) {
      const int d = (int)(k % kAcc);
      const int64_t tile = blockIdx.x + k * gridDim.x;
      if (!wait(&tfull[d], (uint32_t)(k / kAcc) & 1)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(d * kAccCols);
#pragma unroll 1
      for (int t = 0; t < kTok; ++t) {
        float2 v[16];
        {
          uint32_t r[32];
          tmem_ld32(taddr + t * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v[e] = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        }
        if (t == kTok - 1) {
          tc_fence_before();
          mbar_arrive(&tempty[d]);
        }
#pragma unroll
        for (int p = 0; p < 16; ++p) {
          const float a = v[p].x, b = v[p].y;
          v[p] = make_float2(a + b, a - b);
        }
#pragma unroll
        for (int hh = 1; hh < 16; hh <<= 1)
#pragma unroll
          for (int p = 0; p < 16; ++p)
            if (!(p & hh)) bfly2(v[p], v[p | hh]);
        // The warp's 32 lanes hold outputs q*1024 .. q*1024+1023 of the token,
        // 128 (fp32) or 64 (bf16) contiguous bytes per lane: staged through
        // shared memory (16-byte chunk p of lane l at position p ^ (l & 7),
        // or p ^ ((l >> 1) & 3) for bf16), they leave as 512-byte coalesced
        // stores.
        const int64_t token = tile * kTok + t;
        float4 r[8];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          r[p] = make_float4(v[2 * p].x * scale, v[2 * p].y * scale, v[2 * p + 1].x * scale,
                             v[2 * p + 1].y * scale);
          r[p].x = __uint_as_float(__float_as_uint(r[p].x) ^ (((sbits >> (4 * p)) & 1u) << 31));
          r[p].y = __uint_as_float(__float_as_uint(r[p].y) ^ (((sbits >> (4 * p + 1)) & 1u) << 31));
          r[p].z = __uint_as_float(__float_as_uint(r[p].z) ^ (((sbits >> (4 * p + 2)) & 1u) << 31));
          r[p].w = __uint_as_float(__float_as_uint(r[p].w) ^ (((sbits >> (4 * p + 3)) & 1u) << 31));
        }
        if (kBf16Out) {
#pragma unroll
          for (int c = 0; c < 4; ++c)
            *reinterpret_cast<uint4*>(wbuf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(bf16x2_rn(r[2 * c].x, r[2 * c].y), bf16x2_rn(r[2 * c].z, r[2 * c].w),
                           bf16x2_rn(r[2 * c + 1].x, r[2 * c + 1].y),
                           bf16x2_rn(r[2 * c + 1].z, r[2 * c + 1].w));
          __syncwarp();
          if (token < P.tokens) {
            uint4* dst = reinterpret_cast<uint4*>(static_cast<uint16_t*>(P.out) + token * N + q * 1024);
#pragma unroll
            for (int r4 = 0; r4 < 4; ++r4) {
              const int kc = r4 * 32 + lane, l2 = kc >> 2, p2 = kc & 3;
              dst[kc] = *reinterpret_cast<const uint4*>(wbuf + l2 * 64 + ((p2 ^ ((l2 >> 1) & 3)) << 4));
            }
          }
        } else {
#pragma unroll
          for (int p = 0; p < 8; ++p)
            *reinterpret_cast<float4*>(wbuf + lane * 128 + ((p ^ (lane & 7)) << 4)) = r[p];
          __syncwarp();
          if (token < P.tokens) {
            float4* dst = reinterpret_cast<float4*>(static_cast<float*>(P.out) + token * N + q * 1024);
#pragma unroll
            for (int r8 = 0; r8 < 8; ++r8) {
              const int kc = r8 * 32 + lane, l2 = kc >> 3, p2 = kc & 7;
              dst[kc] = *reinterpret_cast<const float4*>(wbuf + l2 * 128 + ((p2 ^ (l2 & 7)) << 4));
            }
          }
        }
        __syncwarp();
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(tmem_base), "n"(kTmemCols));
  }
}

}  // namespace tci

bool tci_supported(const Geometry& g, const uint8_t* codes, const uint8_t* scales,
                   const int8_t* signs, const void* out) {
  return !g.paley && g.b == g.n && g.n == tci::N &&
         (reinterpret_cast<uintptr_t>(codes) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(scales) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(signs) & 15) == 0 &&
         (reinterpret_cast<uintptr_t>(out) & 15) == 0;
}

cudaError_t launch_tcinv_nvfp4(const uint8_t* codes, const uint8_t* scales,
                               const float* tensor_scale, int64_t tokens, const Geometry& g,
                               const int8_t* signs, void* out, int out_bf16, cudaStream_t s) {
  (void)g;
  tci::Params P{};
  P.codes = codes;
  P.scales8 = scales;
  P.tensor_scale = tensor_scale;
  P.signs = signs;
  P.out = out;
  P.tokens = tokens;
  P.tiles = (tokens + tci::kTok - 1) / tci::kTok;
  constexpr size_t kSmem = 1024 + 32768 + tci::kStages * (tci::kZBytes + tci::kRawBytes) +
                           tci::kEpiWarps * 4096 + 256;
  auto k = out_bf16 ? tci::k_tcinv4096<true> : tci::k_tcinv4096<false>;
  cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)kSmem);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = P.tiles < sms ? P.tiles : sms;
  k<<<(int)grid, tci::kThreads, kSmem, s>>>(P);
  return cudaGetLastError();
}

// Reads and clears the error word of the tci kernels (device-synchronous).
cudaError_t take_tci_errors(unsigned int* out) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, tci::g_tci_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tci::g_tci_error, &zero, sizeof(unsigned int));
}

}  // namespace kq
