// The 4-bit GEMM that consumes rotated, NVFP4-quantized activations, on the
// block-scaled tensor cores (tcgen05.mma kind::mxf4nvf4, one E4M3 scale per
// 16 elements of each operand):
//   C[m][n] = t_a t_b sum_k (E2M1(a_mk) E4M3(sa_m,k/16)) (E2M1(b_nk) E4M3(sb_n,k/16)).
// QuaRot reviews, review 2 and review 4 Strengths: the speedup of the rotated
// 4-bit path is the 4-bit GEMM run on quantized activations and weights;
// review 3 Questions: with Y = X H^T applied to both, X W^T is unchanged.
// NVFP4 thread, krylov_schur section 3 table: NVFP4 for weights and activations.
//
// Operands.  A [M, K] and B [N, K] are packed E2M1 codes, K-major (a row's
// codes contiguous, element 2k in the low nibble) -- exactly what
// kq_rht_quant_nvfp4 writes; their block scales are in the tensor-core
// scale-factor layout (KQ_SCALES_MMA: 512-byte atoms of 128 rows x 4
// 16-blocks), so one K = 256 step of a 128-row tile is 2 KB of contiguous
// scales.  t_a, t_b: the fp32 tensor scales, applied in the epilogue.
//
// Tiles of 128 x 128 outputs, K in steps of 256 (128 bytes of codes a row,
// one 128-byte swizzle row): per step a TMA box of A and of B (16 KB each)
// and two 1-D bulk copies of scales (2 KB each) fill one of kStages shared
// stages.  The MMA thread copies the step's scale atoms into tensor memory
// (tcgen05.cp 32x128b, broadcast to the four lane quarters) and issues four
// MMAs of K = 64 (M = 128, N = 128) into one of two TMEM accumulators.  The
// four epilogue warps (one per lane quarter) read the accumulator, multiply
// by t_a t_b, write 32-row x 128-byte pieces to a swizzled staging buffer and
// store them with TMA (coalesced, clipped at row M).  Persistent CTAs walk
// the tiles with M fastest, so the CTAs in flight share their B tiles in L2.
// Every mbarrier wait is bounded; on timeout the kernel records an error and
// returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_sm100.cuh"

namespace kq {
namespace gm {

using namespace sm100;

constexpr int BM = 128, BN = 128;
constexpr int BKB = 128;                         // bytes of codes per row per K step (K = 256)
constexpr uint32_t kTileBytes = 128 * BKB;       // 16 KB: A or B codes of one step
constexpr uint32_t kSfBytes = 4 * 512;           // 2 KB: four scale atoms (K = 256)
constexpr uint32_t kStageBytes = 2 * kTileBytes + 2 * kSfBytes;
constexpr int kStages = 5;
constexpr int kAcc = 2;                          // TMEM accumulators of BN columns
constexpr int kSfCol0 = kAcc * BN;               // TMEM columns of the staged scales
constexpr int kTmemCols = 512;
static_assert(kSfCol0 + kStages * 32 <= kTmemCols, "TMEM columns");
constexpr int kEpiWarps = 4;
constexpr int kThreads = 32 * (2 + kEpiWarps);
constexpr uint32_t kStageOut = 32 * 128;         // one epilogue piece: 32 rows x 128 bytes

__device__ unsigned int g_gemm_error = 0;        // nonzero: a wait timed out

struct Params {
  const uint8_t* sfa;        // A scales, tensor-core layout
  const uint8_t* sfb;
  const float* ta;
  const float* tb;
  int64_t m, n;
  int kc4;                   // K / 64: scale atoms per 128-row block
  int ksteps;                // K / 256
  int mtiles, ntiles;
  int c_bf16;
};

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
  return sm100::mbar_wait(bar, parity, &g_gemm_error);
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void tma_store_2d(const CUtensorMap* map, const void* src, int x,
                                             int y) {
  asm volatile("cp.async.bulk.tensor.2d.global.shared::cta.bulk_group [%0, {%2, %3}], [%1];"
               :: "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(src)), "r"(x), "r"(y)
               : "memory");
}
__device__ __forceinline__ void bulk_commit() {
  asm volatile("cp.async.bulk.commit_group;" ::: "memory");
}
// at most one bulk-store group still reading shared memory
__device__ __forceinline__ void bulk_wait_read1() {
  asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
}
__device__ __forceinline__ void bulk_wait_all() {
  asm volatile("cp.async.bulk.wait_group 0;" ::: "memory");
}
// bf16 pair, rounded to nearest even (lo in bits 0-15)
__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  uint32_t d;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(d) : "f"(hi), "f"(lo));
  return d;
}

// Block-scaled MMA instruction descriptor: A and B E2M1 (format 1 of this
// kind), both K-major, UE4M3 scales (scale format 0), M = 128, N = BN.
constexpr uint32_t kIdesc = (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) |
                            ((uint32_t)(BM >> 4) << 24);

__device__ __forceinline__ void mma_nvfp4(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t sfa, uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.block16 [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate), "r"(sfa), "r"(sfb));
}
// One 512-byte scale atom (32 rows of 16 bytes, no swizzle: 8-row core
// matrices of 128 bytes, 128 bytes apart) into 4 TMEM columns of all four lane
// quarters.
__device__ __forceinline__ void sf_copy(uint32_t tmem_col_addr, uint32_t smem_addr) {
  const uint64_t desc = smem_desc(smem_addr, 128, 128, 0);
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;"
               :: "r"(tmem_col_addr), "l"(desc) : "memory");
}

__global__ void __launch_bounds__(kThreads, 1)
k_gemm_nvfp4(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
             const __grid_constant__ CUtensorMap tmap_c, Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* stages = smem;                                        // kStages x 36 KB
  uint8_t* sout = stages + kStages * kStageBytes;                // 4 warps x 2 x 4 KB
  uint64_t* bars = reinterpret_cast<uint64_t*>(sout + kEpiWarps * 2 * kStageOut);
  uint64_t* full = bars;
  uint64_t* empty = bars + kStages;
  uint64_t* tfull = bars + 2 * kStages;
  uint64_t* tempty = tfull + kAcc;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kAcc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t tiles = (int64_t)P.mtiles * P.ntiles;
  const int64_t my_tiles = (tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int d = 0; d < kAcc; ++d) {
      mbar_init(&tfull[d], 1);
      mbar_init(&tempty[d], 32 * kEpiWarps);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 :: "r"(smem_u32(tmem_slot)), "n"(kTmemCols));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  if (warp == 0) {
    // ================= producer: codes by TMA, scales by 1-D bulk copies
    if (lane == 0) {
      int64_t it = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int64_t t = blockIdx.x + i * gridDim.x;
        const int mt = (int)(t % P.mtiles), nt = (int)(t / P.mtiles);
        for (int ks = 0; ks < P.ksteps; ++ks, ++it) {
          const int s = (int)(it % kStages);
          if (it >= kStages && !wait(&empty[s], (uint32_t)(it / kStages - 1) & 1)) {
            ok = false;
            break;
          }
          uint8_t* st = stages + s * kStageBytes;
          mbar_expect_tx(&full[s], kStageBytes);
          tma_load_2d(st, &tmap_a, ks * BKB, mt * BM, &full[s]);
          tma_load_2d(st + kTileBytes, &tmap_b, ks * BKB, nt * BN, &full[s]);
          bulk_load(st + 2 * kTileBytes, P.sfa + ((int64_t)mt * P.kc4 + 4 * ks) * 512, kSfBytes,
                    &full[s]);
          bulk_load(st + 2 * kTileBytes + kSfBytes, P.sfb + ((int64_t)nt * P.kc4 + 4 * ks) * 512,
                    kSfBytes, &full[s]);
        }
      }
      // no copy may still be in flight when the CTA exits
      for (int64_t j = it > kStages ? it - kStages : 0; j < it; ++j)
        wait(&full[j % kStages], (uint32_t)(j / kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0) {
      int64_t it = 0;
      int64_t done = 0;
      bool ok = true;
      for (int64_t i = 0; i < my_tiles && ok; ++i) {
        const int d = (int)(i % kAcc);
        if (i >= kAcc && !wait(&tempty[d], (uint32_t)(i / kAcc - 1) & 1)) break;
        tc_fence_after();
        const uint32_t tmem_d = tmem_base + (uint32_t)(d * BN);
        for (int ks = 0; ks < P.ksteps; ++ks, ++it) {
          const int s = (int)(it % kStages);
          if (!wait(&full[s], (uint32_t)(it / kStages) & 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t st = smem_u32(stages + s * kStageBytes);
          const uint32_t sfa_col = tmem_base + (uint32_t)(kSfCol0 + 32 * s);
          const uint32_t sfb_col = sfa_col + 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            sf_copy(sfa_col + 4 * j, st + 2 * kTileBytes + 512 * j);
            sf_copy(sfb_col + 4 * j, st + 2 * kTileBytes + kSfBytes + 512 * j);
          }
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // K-major 128-byte swizzle rows, 8-row groups 1 KB apart; K = 64 is 32 bytes
            const uint64_t adesc = smem_desc(st + 32 * j, 16, 1024, 2);
            const uint64_t bdesc = smem_desc(st + kTileBytes + 32 * j, 16, 1024, 2);
            mma_nvfp4(tmem_d, adesc, bdesc, sfa_col + 4 * j, sfb_col + 4 * j,
                      (ks > 0 || j > 0) ? 1u : 0u);
          }
          mma_commit(&empty[s]);
        }
        if (!ok) break;
        mma_commit(&tfull[d]);
        done = i + 1;
      }
      // the accumulators must not be released with MMAs still running
      for (int64_t i = done > kAcc ? done - kAcc : 0; i < done; ++i)
        wait(&tfull[i % kAcc], (uint32_t)(i / kAcc) & 1);
    }
  } else {
    // ================= epilogue: warp w reads TMEM lane quarter w % 4
    const int q = warp & 3;
    const int ew = warp - 2;
    uint8_t* so = sout + ew * 2 * kStageOut;
    const float alpha = *P.ta * *P.tb;
    int piece = 0;
    for (int64_t i = 0; i < my_tiles; ++i) {
      const int d = (int)(i % kAcc);
      const int64_t t = blockIdx.x + i * gridDim.x;
      const int mt = (int)(t % P.mtiles), nt = (int)(t / P.mtiles);
      const bool ok = wait(&tfull[d], (uint32_t)(i / kAcc) & 1);
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(d * BN);
      const int64_t row0 = (int64_t)mt * BM + q * 32;
      const bool rows_in = row0 < P.m;
      // pieces of 128 bytes a row: 32 fp32 or 64 bf16 columns
      const int cols = P.c_bf16 ? 64 : 32;
      for (int c0 = 0; c0 < BN; c0 += cols, ++piece) {
        uint8_t* buf = so + (piece & 1) * kStageOut;
        uint32_t w[32];
        if (P.c_bf16) {
          uint32_t r0[32], r1[32];
          tmem_ld32(taddr + c0, r0);
          tmem_ld32(taddr + c0 + 32, r1);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            w[e] = pack_bf16x2(__uint_as_float(r0[2 * e]) * alpha,
                               __uint_as_float(r0[2 * e + 1]) * alpha);
            w[16 + e] = pack_bf16x2(__uint_as_float(r1[2 * e]) * alpha,
                                    __uint_as_float(r1[2 * e + 1]) * alpha);
          }
        } else {
          uint32_t r0[32];
          tmem_ld32(taddr + c0, r0);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 32; ++e) w[e] = __float_as_uint(__uint_as_float(r0[e]) * alpha);
        }
        // the buffer's previous store has finished reading it
        if (lane == 0) bulk_wait_read1();
        __syncwarp();
        // row `lane` of the piece, 16-byte chunk p at position p ^ (lane & 7)
#pragma unroll
        for (int p = 0; p < 8; ++p)
          *reinterpret_cast<uint4*>(buf + lane * 128 + ((p ^ (lane & 7)) << 4)) =
              make_uint4(w[4 * p], w[4 * p + 1], w[4 * p + 2], w[4 * p + 3]);
        fence_async_smem();
        __syncwarp();
        if (lane == 0) {
          if (ok && rows_in) tma_store_2d(&tmap_c, buf, (int)((int64_t)nt * BN + c0), (int)row0);
          bulk_commit();         // a group per piece (possibly empty): the wait above counts on it
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[d]);
    }
    if (lane == 0) bulk_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;"
                 :: "r"(tmem_base), "n"(kTmemCols));
  }
}

}  // namespace gm

namespace {
constexpr size_t kGemmSmem = 1024 + gm::kStages * gm::kStageBytes +
                             gm::kEpiWarps * 2 * gm::kStageOut +
                             (2 * gm::kStages + 2 * gm::kAcc) * 8 + 16;
}  // namespace

cudaError_t launch_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                              const float* a_tscale, const uint8_t* b_codes,
                              const uint8_t* b_scales, const float* b_tscale, int64_t m,
                              int64_t n, int64_t k, void* c, int c_bf16, cudaStream_t s) {
  CUtensorMap ta, tb, tc;
  // codes: [rows, K/2] bytes, boxes of 128 bytes x 128 rows, 128-byte swizzle
  if (!encode_tmap_2d(&ta, a_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(k / 2),
                      (uint64_t)m, (uint64_t)(k / 2), gm::BKB, gm::BM,
                      CU_TENSOR_MAP_SWIZZLE_128B) ||
      !encode_tmap_2d(&tb, b_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, 1, (uint64_t)(k / 2),
                      (uint64_t)n, (uint64_t)(k / 2), gm::BKB, gm::BN,
                      CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  // C: [M, N] fp32 or bf16, store boxes of 128 bytes x 32 rows, 128-byte swizzle
  const bool ok_c =
      c_bf16 ? encode_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, (uint64_t)n,
                              (uint64_t)m, (uint64_t)n * 2, 64, 32, CU_TENSOR_MAP_SWIZZLE_128B)
             : encode_tmap_2d(&tc, c, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 4, (uint64_t)n,
                              (uint64_t)m, (uint64_t)n * 4, 32, 32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok_c) return cudaErrorNotSupported;
  gm::Params P{};
  P.sfa = a_scales;
  P.sfb = b_scales;
  P.ta = a_tscale;
  P.tb = b_tscale;
  P.m = m;
  P.n = n;
  P.kc4 = (int)(k / 64);
  P.ksteps = (int)(k / 256);
  P.mtiles = (int)((m + gm::BM - 1) / gm::BM);
  P.ntiles = (int)(n / gm::BN);
  P.c_bf16 = c_bf16;
  cudaFuncSetAttribute((const void*)gm::k_gemm_nvfp4, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kGemmSmem);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = (int64_t)P.mtiles * P.ntiles;
  const int grid = (int)(tiles < sms ? tiles : sms);
  gm::k_gemm_nvfp4<<<grid, gm::kThreads, kGemmSmem, s>>>(ta, tb, tc, P);
  return cudaGetLastError();
}

// Reads and clears the error word of the GEMM kernel (device-synchronous).
cudaError_t take_gemm_errors(unsigned int* out) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, gm::g_gemm_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(gm::g_gemm_error, &zero, sizeof(unsigned int));
}

}  // namespace kq
