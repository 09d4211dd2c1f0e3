// Tensor-core (tcgen05) kernel for 12288-wide rows (the intermediate size of
// "Bug: Qwen3-8B integration issue", Model Details: 12288 = 12 x 1024 is
// Hadamard-compatible), rotated by H_12 (Paley) kron H_1024 (Sylvester) and
// quantized to per-token symmetric INT4 (QuaRot reviews, review 2 Summary:
// RTN INT4 of the rotated activations), or written out rotated (fp32).
//
// Index split.  Sylvester's H_1024 in natural order is H_128 kron H_8, so a
// row index is j = i12*1024 + c*8 + d (i12 < 12, c < 128, d < 8) and
//   H[(i12o, co, do)][(i12, c, d)] = H_12[i12o][i12] H_128[co][c] H_8[do][d].
// The transform runs in three stages:
//   (1) the mix over c on the tensor cores: D[co][(i12, d)] = sum_c H_128[co][c]
//       x'[i12*1024 + c*8 + d], D (TMEM, fp32, 128 lanes x 96 columns) = A * B
//       with A = H_128 (bf16 +-1, K-major, 128-byte swizzle, built in shared
//       memory once) and B = the sign-flipped token as the bulk copy left it
//       (K = c, N = i12*8 + d; MN-major without swizzle: a core matrix is the
//       8 values d of 8 consecutive c, 128 contiguous bytes; the next c octet
//       is 128 bytes on, the next i12 2048 bytes on);
//   (2) the H_8 over d, three butterfly stages in registers, by the epilogue
//       thread that owns TMEM lane co;
//   (3) the H_12 over i12 in the same thread, Paley construction I (q = 11):
//       with z_k = x_{1+k}, W_i = sum over r in {0,1,3,4,5,9} of z_{(i+r) mod 11}
//       (zero and the quadratic residues mod 11) and T = sum of all twelve,
//       y_0 = T and y_{1+i} = 2 W_i - T; W_i = q_i + q_{i+3} + v_{i+5} with the
//       pair sums q_k = z_k + z_{k+1}, v_k = z_k + z_{k+4}: 61 operations.
// The thread then holds outputs i12o*1024 + co*8 + do: twelve runs of eight
// contiguous values, one 32-bit word of nibbles each.
//
// Exact scale.  The per-token scale fp32(max|y| / 7), y = S / sqrt(n), needs
// max|S| exactly.  With the accumulation model of tcgen05.mma (see the
// 4096-wide kernel: a K = 16 step adds at most 2.5 u P_k plus the truncation
// of inputs far below the step's largest term, at most 8 u P_k more; P_k =
// partial column sum of |x|) the eight steps err by at most 84 u C_n per
// column n (C_n = its sum of |x'|); the H_8 stages add at most 3 u and the
// H_12 formulas (at most seven roundings on a path, and the doubling) 16 u
// of the sum of |x| over their cone, so |S_hat_i - S_i| <= 103 u sum|x| <=
// 103 u ||S||_2 (Cauchy-Schwarz, ||S||_2 = sqrt(n) ||x||_2) <= E = 108 u
// ||S_hat||_2.  Every output within 2E of the largest |S_hat| is recomputed
// exactly in fp64 by the epilogue group from the staged token, which the
// epilogue holds until then.
//
// Warp roles (12 warps): 0 producer (one bulk copy per token), 1 MMA issuer +
// TMEM owner, 2-3 sign flip, 4-7 and 8-11 two epilogue groups taking
// alternate tokens; warp w reads TMEM lane quarter w % 4, so every group has
// one warp on each scheduler.  A thread keeps its 96 values in registers, so
// the accumulator is handed back to the MMA as soon as it is read.  Every wait
// is bounded; on timeout the kernel records an error code and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_sm100.cuh"

namespace kq {
namespace tcp {

using namespace sm100;

constexpr int N = 12288;
constexpr int kCols = 96;                          // accumulator columns: i12 * 8 + d
constexpr uint32_t kStageBytes = N * 2;            // one token, natural order
constexpr int kStages = 7;
constexpr int kAcc = 4;                            // TMEM accumulators (128 columns apart)
constexpr int kTmemCols = 512;
constexpr int kGroups = 2;
constexpr int kSignWarps = 2;
constexpr int kGroupThreads = 128;                 // one warp per TMEM lane quarter
constexpr int kThreads = 32 * (2 + kSignWarps + 4 * kGroups);
constexpr int kChunks = N / 8;                     // 16-byte chunks per token
constexpr int kSignLanes = 32 * kSignWarps;
constexpr int kSignPer = kChunks / kSignLanes;     // chunks per sign lane
constexpr int kMaxCand = 32;                       // fix-up candidates handled per token
constexpr double kBoundC = 108.0 * 0x1p-24;        // E = kBoundC ||S_hat||_2
static_assert(kChunks % kSignLanes == 0, "sign lanes split the chunks evenly");
static_assert(kAcc % kGroups == 0, "each group owns whole accumulators");

__device__ unsigned int g_tcp_error = 0;           // nonzero: a wait timed out

enum { kInt4 = 0, kRot = 1 };

struct Params {
  const uint16_t* x;     // bf16 [T, n]
  uint8_t* codes;        // kInt4: [T, n/2]
  float* scales;         // kInt4: [T]
  float* out;            // kRot: fp32 [T, n]
  int64_t tokens;
  double sqrt_n;         // IEEE sqrt(12288)
  double rcp_sqrt_n;     // fp64 1 / sqrt_n, correctly rounded
};


// Per-group scratch for the token reductions.
struct GroupScratch {
  float wmax[4];
  float wsq[4];
  double part[2][4];     // per candidate parity
  int wcnt[4];
  int ncand;
  int cand[kMaxCand];
};

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
  return sm100::mbar_wait(bar, parity, &g_tcp_error);
}
__device__ __forceinline__ void group_sync(int g) {
  asm volatile("bar.sync %0, %1;" :: "r"(1 + g), "n"(kGroupThreads) : "memory");
}
__device__ __forceinline__ void bulk_load(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               :: "r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

// x 2^-896 as a double for the bf16 x in the top half of w: sign, exponent and
// mantissa move into the double's high word as they are (an arithmetic shift
// by 3 and a mask), so zero and subnormals map exactly too; integer pipes only.
__device__ __forceinline__ double bf16_hi_scaled(uint32_t w) {
  return __hiloint2double((int)((uint32_t)((int32_t)w >> 3) & 0x8FFFE000u), 0);
}
constexpr double kUnscale = 0x1p896;

// Exact S_i (fp64) of a staged, sign-flipped token, i = (i12o, co, do),
// computed by the kGroupThreads threads of an epilogue group: thread tau sums
// the 96 terms with c = tau, held in the chunks k = i12 (k = 0..11) at byte
// k*2048 + tau*16 of the stage (x'[k*1024 + tau*8 + d], d = 0..7).  The sign
// of a term is H_12[i12o][k] H_128[co][tau] H_8[do][d]; bit k of row12 is
// H_12[i12o][k] < 0.  Values enter fp64 exactly, scaled by 2^-896
// (bf16_hi_scaled), and the partial sum is scaled back at the end.  Returns
// this thread's partial sum.
__device__ __forceinline__ double exact_partial(const uint8_t* tok, int i, uint32_t row12,
                                                int tau) {
  const int co = (i >> 3) & 127, dd = i & 7;
  // row dd of H_8 as bits: bit d = popc(dd & d) & 1
  const uint32_t h8 = (uint32_t)(0x963C5AF066CCAA00ull >> (8 * dd));
  uint32_t em[4];
#pragma unroll
  for (int w = 0; w < 4; ++w)
    em[w] = (((h8 >> (2 * w)) & 1u) << 15) | (((h8 >> (2 * w + 1)) & 1u) << 31);
  const uint32_t fc = (__popc(co & tau) & 1) ? 0x80008000u : 0u;
  const uint8_t* p = tok + tau * 16;
  double acc[4] = {0.0, 0.0, 0.0, 0.0};
#pragma unroll
  for (int k = 0; k < 12; ++k) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + k * 2048);
    const uint32_t flip = fc ^ ((0u - ((row12 >> k) & 1u)) & 0x80008000u);
    const uint32_t ww[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const uint32_t x2 = ww[w] ^ em[w] ^ flip;   // the two terms' signed bf16 bits
      acc[w] += bf16_hi_scaled(x2 << 16);
      acc[(w + 2) & 3] += bf16_hi_scaled(x2);
    }
  }
  return ((acc[0] + acc[1]) + (acc[2] + acc[3])) * kUnscale;
}

// H_8 over d on f[0..3] (f[e] holds d = 2e, 2e + 1), natural order.
__device__ __forceinline__ void h8(float2* f) {
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float a = f[e].x, b = f[e].y;
    f[e] = make_float2(a + b, a - b);
  }
  bfly2(f[0], f[1]);
  bfly2(f[2], f[3]);
  bfly2(f[0], f[2]);
  bfly2(f[1], f[3]);
}

// H_12 (Paley I, q = 11) over i12 on the twelve vectors f[0], f[4], ..., f[44]
// (two independent transforms, one per f32x2 half), in place.
__device__ __forceinline__ void h12(float2* f) {
  float2 q[11], v[11];
#pragma unroll
  for (int k = 0; k < 11; ++k) {
    q[k] = add2(f[4 * (1 + k)], f[4 * (1 + (k + 1) % 11)]);
    v[k] = add2(f[4 * (1 + k)], f[4 * (1 + (k + 4) % 11)]);
  }
  const float2 t = add2(f[0], add2(add2(add2(add2(add2(q[0], q[2]), q[4]), q[6]), q[8]), f[44]));
  const float2 two = make_float2(2.0f, 2.0f), negt = make_float2(-t.x, -t.y);
#pragma unroll
  for (int i = 0; i < 11; ++i)
    f[4 * (1 + i)] = fma2(two, add2(add2(q[i], q[(i + 3) % 11]), v[(i + 5) % 11]), negt);
  f[0] = t;
}

// Two's-complement INT4 nibble in the low 4 bits of the fp32 value
// t = v * c + 1.5 * 2^23 (one rounding: the integer nearest v * c, ties to
// even, for |v * c| < 2^22).
constexpr float kRneMagic = 12582912.0f;

// Eight values (4 pairs) -> 8 nibbles, element k in bits 4k .. 4k + 3.
__device__ __forceinline__ uint32_t int4x8(const float2* f, float2 c2) {
  const float2 m2 = make_float2(kRneMagic, kRneMagic);
  uint32_t byte[4];
#pragma unroll
  for (int p = 0; p < 4; ++p) {
    const float2 t = fma2(f[p], c2, m2);
    byte[p] = (__float_as_uint(t.x) & 0xFu) | ((__float_as_uint(t.y) & 0xFu) << 4);
  }
  return __byte_perm(__byte_perm(byte[0], byte[1], 0x0040), __byte_perm(byte[2], byte[3], 0x0040),
                     0x5410);
}

template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
k_tc12288(const int8_t* __restrict__ signs, Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                    // 32 KB: A = H_128
  uint8_t* sB = smem + 32768;                            // kStages x 24 KB
  GroupScratch* gs = reinterpret_cast<GroupScratch*>(sB + kStages * kStageBytes);   // 2 x 2
  uint32_t* prow = reinterpret_cast<uint32_t*>(gs + 2 * kGroups);   // 12 rows of H_12 as bits
  uint64_t* bars = reinterpret_cast<uint64_t*>(prow + 16);
  uint64_t* full = bars;                                 // bulk copy landed
  uint64_t* ready = bars + kStages;                      // signs applied
  uint64_t* empty = bars + 2 * kStages;                  // MMAs and fix-ups done with the stage
  uint64_t* tfull = bars + 3 * kStages;                  // accumulator written (kAcc)
  uint64_t* tempty = tfull + kAcc;                       // accumulator read (kAcc)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kAcc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  const int64_t my_tiles = (P.tokens - blockIdx.x + gridDim.x - 1) / gridDim.x;

  // ---- set-up.  The producer thread initialises the barriers and starts the
  // first copies before the rest of the set-up, so they overlap it.
  int64_t prefilled = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], kSignLanes);
      mbar_init(&empty[s], kMode == kInt4 ? 2 : 1);   // MMA commit [+ epilogue]
    }
    for (int d = 0; d < kAcc; ++d) {
      mbar_init(&tfull[d], 1);
      mbar_init(&tempty[d], kGroupThreads);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefilled = my_tiles < kStages ? my_tiles : kStages;
    for (int64_t k = 0; k < prefilled; ++k) {
      const int64_t token = blockIdx.x + k * gridDim.x;
      mbar_expect_tx(&full[k], kStageBytes);
      bulk_load(sB + k * kStageBytes, P.x + token * N, kStageBytes, &full[k]);
    }
  }
  // A = H_128, one 16-byte chunk (8 columns) per step
  for (int idx = threadIdx.x; idx < 128 * 16; idx += blockDim.x) {
    const int m = idx >> 4, k0 = (idx & 15) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = (__popc(m & (k0 + 2 * e)) & 1) ? 0xBF80u : 0x3F80u;   // -1 / +1
      const uint32_t hi = (__popc(m & (k0 + 2 * e + 1)) & 1) ? 0xBF80u : 0x3F80u;
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(sA + a_off(m, k0)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (threadIdx.x < 12) {
    uint32_t bits = 0;
    for (int c = 0; c < 12; ++c) bits |= (uint32_t)paley_negative(threadIdx.x, c) << c;
    prow[threadIdx.x] = bits;
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
    // ================= producer: one 24 KB bulk copy per token
    if (lane == 0) {
      int64_t issued = prefilled;
      for (int64_t k = prefilled; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        if (k >= kStages && !wait(&empty[s], (uint32_t)(k / kStages - 1) & 1)) break;
        const int64_t token = blockIdx.x + k * gridDim.x;
        mbar_expect_tx(&full[s], kStageBytes);
        bulk_load(sB + s * kStageBytes, P.x + token * N, kStageBytes, &full[s]);
        issued = k + 1;
      }
      // no copy may still be in flight when the CTA exits
      for (int64_t k = issued > kStages ? issued - kStages : 0; k < issued; ++k)
        wait(&full[k % kStages], (uint32_t)(k / kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16(128, kCols, 1);
      int64_t issued = 0;
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        const int d = (int)(k % kAcc);
        if (!wait(&ready[s], (uint32_t)(k / kStages) & 1)) break;
        if (k >= kAcc && !wait(&tempty[d], (uint32_t)(k / kAcc - 1) & 1)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB + s * kStageBytes);
        const uint32_t tmem_d = tmem_base + (uint32_t)(d * 128);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // A: K-major, K step of 16 = 32 bytes inside a 128-byte swizzle row
          const uint64_t adesc = smem_desc(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024, 2);
          // B: MN-major, no swizzle: c octets 128 bytes apart (leading), i12
          // blocks 2048 bytes apart (stride); a K step of 16 is two c octets
          const uint64_t bdesc = smem_desc(b0 + ks * 256, 128, 2048, 0);
          mma_bf16(tmem_d, adesc, bdesc, idesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&empty[s]);
        mma_commit(&tfull[d]);
        issued = k + 1;
      }
      for (int64_t k = issued > kAcc ? issued - kAcc : 0; k < issued; ++k)
        wait(&tfull[k % kAcc], (uint32_t)(k / kAcc) & 1);
    }
  } else if (warp < 2 + kSignWarps) {
    // ================= sign flip: lane t0 takes the chunks t0 + 64 i
    // (consecutive lanes, consecutive 16-byte chunks); its masks stay in
    // registers.
    const int t0 = (warp - 2) * 32 + lane;
    uint4 msk[kSignPer];
#pragma unroll
    for (int i = 0; i < kSignPer; ++i) {
      msk[i] = make_uint4(0, 0, 0, 0);
      if (signs) {
        const uint2 sv = __ldg(reinterpret_cast<const uint2*>(signs) + t0 + kSignLanes * i);
        msk[i] = make_uint4(__byte_perm(sv.x, 0, 0x1404) & 0x80008000u,
                            __byte_perm(sv.x, 0, 0x3424) & 0x80008000u,
                            __byte_perm(sv.y, 0, 0x1404) & 0x80008000u,
                            __byte_perm(sv.y, 0, 0x3424) & 0x80008000u);
      }
    }
    for (int64_t k = 0; k < my_tiles; ++k) {
      const int s = (int)(k % kStages);
      if (!wait(&full[s], (uint32_t)(k / kStages) & 1)) break;
      if (signs) {
        uint4* st = reinterpret_cast<uint4*>(sB + s * kStageBytes) + t0;
#pragma unroll
        for (int i = 0; i < kSignPer; ++i) {
          uint4 w = st[kSignLanes * i];
          w.x ^= msk[i].x;
          w.y ^= msk[i].y;
          w.z ^= msk[i].z;
          w.w ^= msk[i].w;
          st[kSignLanes * i] = w;
        }
        fence_async_smem();
      }
      __syncwarp();
      mbar_arrive(&ready[s]);
    }
  } else {
    // ================= epilogue: group g of warps 4 + 4g .. 7 + 4g; warp w
    // reads TMEM lane quarter q = w % 4, lane co = 32 q + lane.
    const int g = (warp - 4) >> 2;
    const int q = warp & 3;
    const int co = q * 32 + lane;             // also the thread's index in the group
    const int ntiles = (int)my_tiles;         // tokens < 2^31
    for (int k = g; k < ntiles; k += kGroups) {
      const int d = k % kAcc;
      const int st = k % kStages;
      const int64_t token = blockIdx.x + (int64_t)k * gridDim.x;
      // scratch alternates between the group's consecutive tokens, so a token
      // never overwrites one that a slower warp may still be reading
      GroupScratch& S = gs[2 * g + ((k / kGroups) & 1)];
      // A timed-out wait does not leave the loop: the failure is recorded and
      // the token's outputs are not written.
      const bool ok = wait(&tfull[d], (uint32_t)(k / kAcc) & 1);
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(d * 128);
      float2 f[48];                           // f[4 i12 + e] holds d = 2e, 2e + 1
      {
        uint32_t r[3][32];
#pragma unroll
        for (int c = 0; c < 3; ++c) tmem_ld32(taddr + c * 32, r[c]);
        tmem_wait_ld();
#pragma unroll
        for (int c = 0; c < 3; ++c)
#pragma unroll
          for (int p = 0; p < 16; ++p)
            f[16 * c + p] =
                make_float2(__uint_as_float(r[c][2 * p]), __uint_as_float(r[c][2 * p + 1]));
      }
      tc_fence_before();
      mbar_arrive(&tempty[d]);                // the values live in registers from here on
#pragma unroll
      for (int i12 = 0; i12 < 12; ++i12) h8(f + 4 * i12);
#pragma unroll
      for (int e = 0; e < 4; ++e) h12(f + e);

      if (kMode == kRot) {
        if (ok) {
          const float inv = (float)(1.0 / P.sqrt_n);
          float* dst = P.out + token * N + co * 8;
#pragma unroll
          for (int i12 = 0; i12 < 12; ++i12) {
            const float2* h = f + 4 * i12;
            reinterpret_cast<float4*>(dst + i12 * 1024)[0] =
                make_float4(h[0].x * inv, h[0].y * inv, h[1].x * inv, h[1].y * inv);
            reinterpret_cast<float4*>(dst + i12 * 1024)[1] =
                make_float4(h[2].x * inv, h[2].y * inv, h[3].x * inv, h[3].y * inv);
          }
        }
        continue;
      }

      // ---- token maximum and ||S_hat||_2^2 over the group
      // four independent chains each
      float mj[4] = {0.0f, 0.0f, 0.0f, 0.0f};
      float2 sj[4] = {make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f), make_float2(0.0f, 0.0f),
                      make_float2(0.0f, 0.0f)};
#pragma unroll
      for (int p = 0; p < 48; ++p) {
        mj[p & 3] = fmax3(mj[p & 3], fabsf(f[p].x), fabsf(f[p].y));
        sj[p & 3] = fma2(f[p], f[p], sj[p & 3]);
      }
      float mx = fmaxf(fmaxf(mj[0], mj[1]), fmaxf(mj[2], mj[3]));
      const float2 sq2 = add2(add2(sj[0], sj[1]), add2(sj[2], sj[3]));
      float sq = sq2.x + sq2.y;
      const float own_mx = mx;
      mx = __uint_as_float(redux_max(__float_as_uint(mx)));   // non-negative: integer order
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sq += __shfl_xor_sync(0xffffffffu, sq, off);
      if (lane == 0) {
        S.wmax[q] = mx;
        S.wsq[q] = sq;
      }
      if (co == 0) S.ncand = 0;
      group_sync(g);
      float M = 0.0f, Q = 0.0f;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        M = fmaxf(M, S.wmax[w]);
        Q += S.wsq[w];
      }
      const bool finite = isfinite(M) && isfinite(Q);
      // E rounded up (fp32 sums of 12288 squares err by far less than 2^-10; a
      // correctly rounded square root is within 2^-24 of the true one)
      const float E = __fmul_ru(__fmul_ru((float)kBoundC, 1.0f + 0x1p-22f),
                                sqrtf(__fmul_ru(Q, 1.0f + 0x1p-10f)));
      const float thr = __fsub_rd(M, __fmul_ru(2.0f, E));
      // ---- candidates: every output within 2E of the maximum
      uint32_t cm[3] = {0u, 0u, 0u};
      if (finite && M > 0.0f && own_mx >= thr) {
#pragma unroll
        for (int p = 0; p < 48; ++p) {
          if (fabsf(f[p].x) >= thr) cm[p >> 4] |= 1u << (2 * (p & 15));
          if (fabsf(f[p].y) >= thr) cm[p >> 4] |= 1u << (2 * (p & 15) + 1);
        }
      }
      // value 2p + h of this thread is output (p / 4) * 1024 + co * 8 + (p % 4) * 2 + h
      const int myc = __popc(cm[0]) + __popc(cm[1]) + __popc(cm[2]);
      if (myc > 0) {
        int slot = atomicAdd(&S.ncand, myc);
#pragma unroll
        for (int w = 0; w < 3; ++w) {
          uint32_t bits = cm[w];
          while (bits) {
            const int b = __ffs(bits) - 1;
            bits &= bits - 1;
            const int v = 32 * w + b, p = v >> 1;
            if (slot < kMaxCand) S.cand[slot] = (p >> 2) * 1024 + co * 8 + (p & 3) * 2 + (v & 1);
            ++slot;
          }
        }
      }
      group_sync(g);
      const int total = S.ncand;

      // ---- exact maximum over the candidates
      double best = 0.0;
      const uint8_t* tok = sB + st * kStageBytes;   // held until the fix-ups are done
      auto exact_at = [&](int ci) { return exact_partial(tok, ci, prow[ci >> 10], co); };
      if (total > 0) wait(&ready[st], (uint32_t)(k / kStages) & 1);   // sign flips visible
      if (total <= kMaxCand) {
        for (int c = 0; c < total; ++c) {
          double part = warp_sum_d(exact_at(S.cand[c]));
          if (lane == 0) S.part[c & 1][q] = part;
          group_sync(g);
          const double sum = (S.part[c & 1][0] + S.part[c & 1][1]) +
                             (S.part[c & 1][2] + S.part[c & 1][3]);
          best = fmax(best, fabs(sum));
        }
      } else {
        // many candidates (degenerate rows): rank them and take kMaxCand at a time
        int incl = myc;
#pragma unroll
        for (int off = 1; off < 32; off <<= 1) {
          const int v = __shfl_up_sync(0xffffffffu, incl, off);
          if (lane >= off) incl += v;
        }
        if (lane == 31) S.wcnt[q] = incl;
        group_sync(g);
        int base = 0;
#pragma unroll
        for (int w = 0; w < 4; ++w) base += (w < q) ? S.wcnt[w] : 0;
        const int rank0 = base + incl - myc;
        for (int r0 = 0; r0 < total; r0 += kMaxCand) {
          group_sync(g);                        // the previous round's reads are done
          if (myc > 0 && rank0 < r0 + kMaxCand && rank0 + myc > r0) {
            int rk = rank0;
#pragma unroll
            for (int w = 0; w < 3; ++w) {
              uint32_t bits = cm[w];
              while (bits) {
                const int b = __ffs(bits) - 1;
                bits &= bits - 1;
                const int v = 32 * w + b, p = v >> 1;
                if (rk >= r0 && rk < r0 + kMaxCand)
                  S.cand[rk - r0] = (p >> 2) * 1024 + co * 8 + (p & 3) * 2 + (v & 1);
                ++rk;
              }
            }
          }
          group_sync(g);
          const int nc = min(kMaxCand, total - r0);
          for (int c = 0; c < nc; ++c) {
            double part = warp_sum_d(exact_at(S.cand[c]));
            if (lane == 0) S.part[c & 1][q] = part;
            group_sync(g);
            const double sum = (S.part[c & 1][0] + S.part[c & 1][1]) +
                               (S.part[c & 1][2] + S.part[c & 1][3]);
            best = fmax(best, fabs(sum));
          }
        }
      }
      if (co == 0) mbar_arrive(&empty[st]);   // every read of the stage is behind a group sync

      // ---- scale and codes: one 32-bit word per i12.  A row holding an
      // infinity or NaN gets the scale of its computed maximum (not exact).
      float scale = 0.0f;
      if (!finite)
        scale = __double2float_rn(((double)M / P.sqrt_n) / 7.0);
      else if (M > 0.0f)
        scale = __double2float_rn(div_rn(div_rn(best, P.sqrt_n, P.rcp_sqrt_n), 7.0, 1.0 / 7.0));
      if (ok) {
        // 1 / (sqrt(n) scale) in fp32 (an error of a few ulp moves only codes
        // within far less than 1e-5 of a rounding boundary)
        const float cq = scale > 0.0f ? __frcp_rn((float)P.sqrt_n * scale) : 0.0f;
        const float2 c2 = make_float2(cq, cq);
        uint32_t* dst = reinterpret_cast<uint32_t*>(P.codes + token * (N / 2)) + co;
#pragma unroll
        for (int i12 = 0; i12 < 12; ++i12) dst[i12 * 128] = int4x8(f + 4 * i12, c2);
        if (co == 0) P.scales[token] = scale;
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

}  // namespace tcp

// ------------------------------------------------------------- launchers
namespace {

constexpr size_t kTcpSmem = 1024 + 32768 + tcp::kStages * tcp::kStageBytes +
                            2 * tcp::kGroups * sizeof(tcp::GroupScratch) + 64 + 256;

template <int kMode>
cudaError_t launch_tcp(const void* x, const int8_t* signs, tcp::Params& P, const Geometry& g,
                       cudaStream_t s) {
  P.x = static_cast<const uint16_t*>(x);
  P.sqrt_n = g.sqrt_b;
  P.rcp_sqrt_n = 1.0 / g.sqrt_b;
  auto k = tcp::k_tc12288<kMode>;
  cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kTcpSmem);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = P.tokens < sms ? P.tokens : sms;
  k<<<(int)grid, tcp::kThreads, kTcpSmem, s>>>(signs, P);
  return cudaGetLastError();
}

}  // namespace

bool tcp_supported(const Geometry& g, int dtype, const void* x, int64_t tokens) {
  // bulk copies: a 16-byte aligned base (each row is 24 KB, so every row is
  // aligned); 32-bit token counters in the epilogue
  return dtype == 1 && g.paley && g.b == g.n && g.n == tcp::N &&
         (reinterpret_cast<uintptr_t>(x) & 15) == 0 && tokens < (int64_t(1) << 31);
}

cudaError_t launch_tcp_int4(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, float* scales, cudaStream_t s) {
  tcp::Params P{};
  P.codes = codes;
  P.scales = scales;
  P.tokens = tokens;
  return launch_tcp<tcp::kInt4>(x, signs, P, g, s);
}

cudaError_t launch_tcp_rot(const void* x, int64_t tokens, const Geometry& g,
                           const int8_t* signs, float* out, cudaStream_t s) {
  tcp::Params P{};
  P.out = out;
  P.tokens = tokens;
  return launch_tcp<tcp::kRot>(x, signs, P, g, s);
}

// Reads and clears the error word of the tcp kernels (device-synchronous).
cudaError_t take_tcp_errors(unsigned int* out) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, tcp::g_tcp_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tcp::g_tcp_error, &zero, sizeof(unsigned int));
}

}  // namespace kq
