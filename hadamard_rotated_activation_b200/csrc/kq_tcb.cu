// Tensor-core (tcgen05) kernel for 128-wide Hadamard blocks with asymmetric
// INT4 per 128-group: the KV-cache layout (QuaRot reviews, final comments: a
// 128-point Hadamard per head; NVFP4 thread, discrete_descent's INT4-g128
// note).
//
// A row of n values is n/128 independent units of 128 (unit u = token * n/128
// + column block), and the input viewed as [units, 128] is row-major with
// 256-byte rows.  The transform of every unit is one dense +-1 contraction:
//   S[u][j] = sum_k x'[u][k] H_128[k][j]      (x' = sign-flipped input)
// so a tile of 128 consecutive units (32 KB, contiguous in HBM) is the A
// operand of one tcgen05.mma chain (M = 128 units, K = 128, bf16, K-major,
// 128-byte swizzle, two TMA boxes of 64 columns) and B = H_128 (N = 128,
// K-major, built in shared memory once).  The accumulator row of unit m sits
// in TMEM lane m: the epilogue thread of that lane owns the unit's 128
// outputs, which are exactly one INT4 group, so extrema, scale, zero point,
// rounding and nibble packing need no communication.
//
// Error bound.  One tcgen05.mma kind::f16 step (K = 16) behaves per output as:
// the 16 products and the incoming accumulator are truncated toward zero to a
// multiple of g = 2^(emax - 25) (emax = exponent of the largest of them),
// added exactly, and the sum is truncated to fp32 (the tensor-core rounding
// test reproduces this bit for bit).  With P_k = sum of |x'| over the inputs
// of steps 0..k, step k loses less than 2^-25 P_k on the accumulator and less
// than 2^-23 P_k in the final truncation.  A bf16 input with |x| >= 2^-17
// sum|x'| lies on the grid and loses nothing; a smaller one loses less than
// g <= 2^-25 P_k.  So, with W = sum_k P_k = sum_i (8 - i/16) |x'_i|,
//   |S_hat - S| <= 5 * 2^-25 W          (no input below 2^-17 sum|x'|),
//   |S_hat - S| <= 21 * 2^-25 W         (otherwise: 16 inputs per step),
// for every output of the unit.  The statistics warps compute W and sum|x'|
// per unit while they touch the staged tile (bf16 sums of |x'| in three
// levels, made upper bounds by a 2^-5 relative margin) and pass E to the epilogue.  The
// scale and zero point are decided from the fp32 values when the interval of
// each rounds to one value; otherwise the warp recomputes the unit's extrema
// exactly in fp64 from the staged input (about 1 % of units).
//
// Warp roles (12 warps, up to 168 registers a thread): 0 TMA producer, 1 MMA
// issuer + TMEM owner, 2-3 statistics (bound E per unit; with signs they
// first XOR the sign bits into the staged tile), 4-11 epilogue in two groups of four (alternate
// tiles; warp w reads TMEM lane quarter w % 4).  A stage is released by the
// epilogue once its fix-ups no longer need the input.  The codes of a warp's
// 32 units (2 KB, contiguous) pass through shared memory and leave as
// coalesced 16-byte stores.  Every wait is bounded; on timeout the kernel
// records an error code and returns.
#include <cuda.h>

#include <cfloat>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"
#include "kq_sm100.cuh"

namespace kq {
namespace tcb {

using namespace sm100;

constexpr int B = 128;
constexpr uint32_t kTileBytes = 128 * B * 2;   // 32 KB
constexpr int kStages = 5;
constexpr int kAcc = 4;
constexpr int kGroups = 2;
constexpr int kStatWarps = 2;
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kEpi0 = 2 + kStatWarps;          // first epilogue warp
constexpr int kThreads = 32 * (kEpi0 + kEpiWarps);
constexpr int kTmemCols = kAcc * B;
constexpr uint32_t kIdesc = idesc_bf16(128, B, 0);
static_assert(kAcc >= kGroups && kTmemCols <= 512, "TMEM");
static_assert(kEpi0 % 4 == 0, "epilogue groups must start on a lane quarter");

__device__ unsigned int g_tcb_error = 0;       // nonzero: a wait timed out

struct Params {
  const int8_t* signs;          // [n] or null
  uint8_t* codes;               // [units, 64]
  uint16_t* scales16;           // fp16 [units]
  uint16_t* zeros16;            // fp16 [units]
  int64_t units;                // tokens * n / 128 (>= 128)
  const int64_t* slots;         // cache row of each input row, or null
  int64_t num_slots;
  int64_t tiles;
  int kpr;                      // column blocks per row, n / 128
};

constexpr size_t kSmemBytes = 1024 + 32768 + kStages * kTileBytes + 4096 /* mask table */ +
                              2048 /* sign bits, n <= 16384 */ + kEpiWarps * 2048 +
                              kStages * 128 * 4 /* bounds */ + 256;

__device__ __forceinline__ bool wait(uint64_t* bar, uint32_t parity) {
  return sm100::mbar_wait(bar, parity, &g_tcb_error);
}

__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t f16x2_pair(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;   // bits 0-15: fp16(lo), bits 16-31: fp16(hi)
}
// Eight integers -> eight nibbles (element k in bits 4k .. 4k+3), each
// saturated to 0..15 by the packing conversion.
__device__ __forceinline__ uint32_t pack_u4x8(const int (&q)[8]) {
  uint32_t d = 0;
#pragma unroll
  for (int k = 3; k >= 0; --k)
    asm("cvt.pack.sat.u4.s32.b32 %0, %1, %2, %3;" : "=r"(d) : "r"(q[2 * k + 1]), "r"(q[2 * k]), "r"(d));
  return d;
}

// Exact extremes of the outputs of tile row m: the whole warp transforms the
// staged, sign-flipped unit in fp64 (lane l holds inputs 4l .. 4l+3; index
// bits 0-1 in the lane, bits 2-6 across lanes by shuffles; Sylvester order is
// natural) and reduces.  Every lane gets max_j S_j and min_j S_j.
__device__ __noinline__ void tile_exact_minmax(const uint8_t* tile, int m, double& smax,
                                               double& smin) {
  const int lane = threadIdx.x & 31;
  const uint2 w = *reinterpret_cast<const uint2*>(tile + a_off(m, (lane >> 1) * 8) + (lane & 1) * 8);
  const double x0 = (double)__uint_as_float(w.x << 16);
  const double x1 = (double)__uint_as_float(w.x & 0xffff0000u);
  const double x2 = (double)__uint_as_float(w.y << 16);
  const double x3 = (double)__uint_as_float(w.y & 0xffff0000u);
  const double a0 = x0 + x1, a1 = x0 - x1, a2 = x2 + x3, a3 = x2 - x3;
  double v[4] = {a0 + a2, a1 + a3, a0 - a2, a1 - a3};
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const bool upper = (lane & o) != 0;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const double p = __shfl_xor_sync(0xffffffffu, v[q], o);
      v[q] = upper ? p - v[q] : v[q] + p;
    }
  }
  double hi = fmax(fmax(v[0], v[1]), fmax(v[2], v[3]));
  double lo = fmin(fmin(v[0], v[1]), fmin(v[2], v[3]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    hi = fmax(hi, __shfl_xor_sync(0xffffffffu, hi, o));
    lo = fmin(lo, __shfl_xor_sync(0xffffffffu, lo, o));
  }
  smax = hi;
  smin = lo;
}

template <bool kKv>
__global__ void __launch_bounds__(kThreads, 1)
k_tcb128_asym(const __grid_constant__ CUtensorMap tmap, Params P) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sB = smem;                                        // 32 KB: H_128 (bf16)
  uint8_t* sX = smem + 32768;                                // kStages x 32 KB
  uint4* stbl = reinterpret_cast<uint4*>(sX + kStages * kTileBytes);   // byte -> XOR masks
  uint8_t* sbits = reinterpret_cast<uint8_t*>(stbl + 256);   // sign bits, n / 8 bytes
  uint8_t* sOut = sbits + 2048;                              // 2 KB per epilogue warp
  float* sE = reinterpret_cast<float*>(sOut + kEpiWarps * 2048);   // bound per (stage, unit)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sE + kStages * 128);
  uint64_t* full = bars;                                     // tile landed
  uint64_t* ready = bars + kStages;                          // flipped, bounds written
  uint64_t* empty = bars + 2 * kStages;                      // epilogue done with the tile
  uint64_t* tfull = bars + 3 * kStages;                      // accumulator written (kAcc)
  uint64_t* tempty = tfull + kAcc;                           // accumulator read (kAcc)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kAcc);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t my_tiles = (P.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;
  const bool has_signs = P.signs != nullptr;
  const int64_t last_y = P.units - 128;   // the last tile starts here (it may overlap)

  // ---- set-up: barriers and the first copies, then B, the sign tables, TMEM
  int64_t prefilled = 0;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 32 * kStatWarps);
      mbar_init(&empty[s], 4);
    }
    for (int d = 0; d < kAcc; ++d) {
      mbar_init(&tfull[d], 1);
      mbar_init(&tempty[d], 128);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    prefilled = my_tiles < kStages ? my_tiles : kStages;
    for (int64_t k = 0; k < prefilled; ++k) {
      const int64_t tile = blockIdx.x + k * gridDim.x;
      const int64_t y0 = tile * 128 < last_y ? tile * 128 : last_y;
      mbar_expect_tx(&full[k], kTileBytes);
      tma_load_2d(sX + k * kTileBytes, &tmap, 0, (int)y0, &full[k]);
      tma_load_2d(sX + k * kTileBytes + 16384, &tmap, 64, (int)y0, &full[k]);
    }
  }
  for (int idx = threadIdx.x; idx < 128 * 16; idx += blockDim.x) {
    const int r = idx >> 4, k0 = (idx & 15) * 8;
    uint32_t w[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      const uint32_t lo = (__popc(r & (k0 + 2 * e)) & 1) ? 0xBF80u : 0x3F80u;   // -1 / +1
      const uint32_t hi = (__popc(r & (k0 + 2 * e + 1)) & 1) ? 0xBF80u : 0x3F80u;
      w[e] = lo | (hi << 16);
    }
    *reinterpret_cast<uint4*>(sB + a_off(r, k0)) = make_uint4(w[0], w[1], w[2], w[3]);
  }
  if (has_signs) {
    for (int i = threadIdx.x; i < 256; i += blockDim.x) {
      uint32_t w[4];
#pragma unroll
      for (int e = 0; e < 4; ++e)
        w[e] = (((uint32_t)i >> (2 * e)) & 1u) << 15 | (((uint32_t)i >> (2 * e + 1)) & 1u) << 31;
      stbl[i] = make_uint4(w[0], w[1], w[2], w[3]);
    }
    for (int i = threadIdx.x; i < P.kpr * 16; i += blockDim.x) {
      const uint2 sv = __ldg(reinterpret_cast<const uint2*>(P.signs) + i);
      uint32_t b = 0;
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        b |= ((sv.x >> (8 * e + 7)) & 1u) << e;
        b |= ((sv.y >> (8 * e + 7)) & 1u) << (e + 4);
      }
      sbits[i] = (uint8_t)b;
    }
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
    // ================= TMA producer
    if (lane == 0) {
      int64_t issued = prefilled;
      for (int64_t k = prefilled; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        if (!wait(&empty[s], (uint32_t)(k / kStages - 1) & 1)) break;
        const int64_t tile = blockIdx.x + k * gridDim.x;
        const int64_t y0 = tile * 128 < last_y ? tile * 128 : last_y;
        mbar_expect_tx(&full[s], kTileBytes);
        tma_load_2d(sX + s * kTileBytes, &tmap, 0, (int)y0, &full[s]);
        tma_load_2d(sX + s * kTileBytes + 16384, &tmap, 64, (int)y0, &full[s]);
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
        if (!wait(has_signs ? &ready[s] : &full[s], (uint32_t)(k / kStages) & 1)) break;
        if (k >= kAcc && !wait(&tempty[d], (uint32_t)(k / kAcc - 1) & 1)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sX + s * kTileBytes), b0 = smem_u32(sB);
        const uint32_t tmem_d = tmem_base + (uint32_t)(d * B);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          const uint32_t off = (ks >> 2) * 16384 + (ks & 3) * 32;
          mma_bf16(tmem_d, smem_desc(a0 + off, 16, 1024, 2), smem_desc(b0 + off, 16, 1024, 2),
                   kIdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&tfull[d]);
        issued = k + 1;
      }
      for (int64_t k = issued > kAcc ? issued - kAcc : 0; k < issued; ++k)
        wait(&tfull[k % kAcc], (uint32_t)(k / kAcc) & 1);
    }
  } else if (warp < kEpi0) {
    // ================= statistics (+ sign flips): lane l of warp w owns tile
    // rows 64 w + l and 64 w + l + 32 (eight consecutive rows per bank phase:
    // eight distinct 16-byte bank groups under the swizzle)
    const int w = warp - 2;
    for (int64_t k = 0; k < my_tiles; ++k) {
      const int s = (int)(k % kStages);
      if (!wait(&full[s], (uint32_t)(k / kStages) & 1)) break;
      const int64_t tile = blockIdx.x + k * gridDim.x;
      const int64_t y0 = tile * 128 < last_y ? tile * 128 : last_y;
      uint8_t* t = sX + s * kTileBytes;
      // both rows at once, every chunk unrolled: the loads are independent
      const int m0 = 64 * w + lane, m1 = m0 + 32;
      int kk[2] = {0, 0};
      if (has_signs) {
        kk[0] = (int)((y0 + m0) % P.kpr);
        kk[1] = (int)((y0 + m1) % P.kpr);
      }
      float a1[2] = {0.0f, 0.0f}, wsum[2] = {0.0f, 0.0f};
      uint32_t mn[2] = {0x7f807f80u, 0x7f807f80u};   // bf16x2 (+inf, +inf)
#pragma unroll
      for (int st = 0; st < 8; ++st) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          const int m = h ? m1 : m0;
          uint32_t b[8];
#pragma unroll
          for (int cc = 0; cc < 2; ++cc) {
            const int c = 2 * st + cc;
            uint4* p = reinterpret_cast<uint4*>(t + a_off(m, c * 8));
            uint4 v = *p;
            if (has_signs) {
              const uint4 mk = stbl[sbits[kk[h] * 16 + c]];
              v.x ^= mk.x;
              v.y ^= mk.y;
              v.z ^= mk.z;
              v.w ^= mk.w;
              *p = v;
            }
            b[4 * cc + 0] = v.x & 0x7fff7fffu;
            b[4 * cc + 1] = v.y & 0x7fff7fffu;
            b[4 * cc + 2] = v.z & 0x7fff7fffu;
            b[4 * cc + 3] = v.w & 0x7fff7fffu;
          }
          const uint32_t n01 = min_bf16x2(min_bf16x2(b[0], b[1]), min_bf16x2(b[2], b[3]));
          const uint32_t n23 = min_bf16x2(min_bf16x2(b[4], b[5]), min_bf16x2(b[6], b[7]));
          mn[h] = min_bf16x2(mn[h], min_bf16x2(n01, n23));
          const uint32_t s01 = add_bf16x2(add_bf16x2(b[0], b[1]), add_bf16x2(b[2], b[3]));
          const uint32_t s23 = add_bf16x2(add_bf16x2(b[4], b[5]), add_bf16x2(b[6], b[7]));
          const uint32_t sm = add_bf16x2(s01, s23);
          const float ps = __uint_as_float(sm << 16) + __uint_as_float(sm & 0xffff0000u);
          a1[h] += ps;
          wsum[h] = fmaf(ps, (float)(8 - st), wsum[h]);
        }
      }
      // three levels of bf16 sums lose at most (1 + 2^-8)^3: 2^-5 covers them
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        const float mnf =
            fminf(__uint_as_float(mn[h] << 16), __uint_as_float(mn[h] & 0xffff0000u));
        const bool tiny = mnf < (a1[h] * 1.03125f) * 0x1p-17f;
        sE[s * 128 + (h ? m1 : m0)] =
            __fmul_ru(__fmul_ru(wsum[h], 1.03125f), tiny ? 21.0f * 0x1p-25f : 5.0f * 0x1p-25f) +
            1e-37f;
      }
      if (has_signs) fence_async_smem();
      __syncwarp();
      mbar_arrive(&ready[s]);
    }
  } else {
    // ================= epilogue: group g of warps kEpi0+4g .. kEpi0+4g+3;
    // thread of TMEM lane m owns unit y0 + m of the tile
    const int g = (warp - kEpi0) >> 2;
    const int q = warp & 3;
    const int m = q * 32 + lane;
    uint8_t* wbuf = sOut + (warp - kEpi0) * 2048;
    const float k15 = (float)(1.0 / (15.0 * 11.313708498984761));
    for (int64_t k = g; k < my_tiles; k += kGroups) {
      const int d = (int)(k % kAcc), s = (int)(k % kStages);
      const int64_t tile = blockIdx.x + k * gridDim.x;
      const int64_t y0 = tile * 128 < last_y ? tile * 128 : last_y;
      if (!wait(&tfull[d], (uint32_t)(k / kAcc) & 1)) break;
      if (!wait(&ready[s], (uint32_t)(k / kStages) & 1)) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(d * B);
      const float E = sE[s * 128 + m];   // |S_hat - S| <= E for the unit's outputs

      // ---- extrema of the unit
      float mx = -FLT_MAX, mn = FLT_MAX;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t r[32];
        tmem_ld32(taddr + cb * 32, r);
        tmem_wait_ld();
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = __uint_as_float(r[2 * e]), b = __uint_as_float(r[2 * e + 1]);
          mx = fmax3(mx, a, b);
          mn = fmin3(mn, a, b);
        }
      }

      // ---- scale16 = fp16((max - min) / (15 sqrt(b))), zero = rint(-min /
      // (sqrt(b) scale16)), each decided when its interval rounds to one value
      const float r_lo = fmaxf(mx - mn - 2.0f * E, 0.0f) * k15 * (1.0f - 0x1p-20f);
      const float r_hi = (mx - mn + 2.0f * E) * k15 * (1.0f + 0x1p-20f);
      const uint32_t hh = f16x2_pair(r_lo, r_hi);
      uint32_t s16 = hh & 0xffffu;
      bool decided = s16 == (hh >> 16);
      float zf = 0.0f;
      if (decided && s16 != 0) {
        const float inv = 1.0f / (11.313708498984761f * f16_bits_to_f32((uint16_t)s16));
        const float z_hi = rintf(-(mn - E) * inv * (1.0f + 0x1p-20f * (mn - E < 0 ? 1.f : -1.f)));
        const float z_lo = rintf(-(mn + E) * inv * (1.0f - 0x1p-20f * (mn + E < 0 ? 1.f : -1.f)));
        decided = z_hi == z_lo;
        zf = z_lo;
      }

      // ---- exact extremes (fp64) for the undecided units of the warp
      unsigned todo = __ballot_sync(0xffffffffu, !decided);
      const uint8_t* stile = sX + s * kTileBytes;
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        double smax, smin;
        tile_exact_minmax(stile, q * 32 + src, smax, smin);
        if (lane == src) {
          constexpr double kSqrt128 = 11.313708498984761;   // IEEE sqrt(128)
          const bool fin = isfinite(smax) && isfinite(smin);
          const double ymx = fin ? div_rn(smax, kSqrt128, 1.0 / kSqrt128) : smax / kSqrt128;
          const double ymn = fin ? div_rn(smin, kSqrt128, 1.0 / kSqrt128) : smin / kSqrt128;
          const double rng = ymx - ymn;
          s16 = f64_to_f16_bits(isfinite(rng) ? div_rn(rng, 15.0, 1.0 / 15.0) : rng / 15.0);
          const double sd = f16_bits_to_f64((uint16_t)s16);
          zf = sd > 0.0 ? (float)rint(-ymn / sd) : 0.0f;
        }
      }

      // ---- codes: (S c) + (1.5 2^23 + z) rounds S c + z to an integer in the
      // low bits; 16 bytes per 32 outputs into the warp's staging buffer
      // (chunk cb of lane l at position cb ^ ((l >> 1) & 3))
      const float c = (s16 != 0) ? 1.0f / (11.313708498984761f * f16_bits_to_f32((uint16_t)s16))
                                 : 0.0f;
      if (s16 == 0) zf = 0.0f;
      const float magic = 12582912.0f + zf;
#pragma unroll 1
      for (int cb = 0; cb < 4; ++cb) {
        uint32_t r[32];
        tmem_ld32(taddr + cb * 32, r);
        tmem_wait_ld();
        uint32_t words[4];
#pragma unroll
        for (int w4 = 0; w4 < 4; ++w4) {
          int qv[8];
#pragma unroll
          for (int p = 0; p < 8; ++p)
            qv[p] = __float_as_int(fmaf(__uint_as_float(r[8 * w4 + p]), c, magic)) - 0x4B400000;
          words[w4] = pack_u4x8(qv);
        }
        *reinterpret_cast<uint4*>(wbuf + lane * 64 + ((cb ^ ((lane >> 1) & 3)) << 4)) =
            make_uint4(words[0], words[1], words[2], words[3]);
      }
      tc_fence_before();
      mbar_arrive(&tempty[d]);
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // the fix-ups are done with the tile

      // ---- stores: the warp's 32 units are 2 KB of contiguous codes
      const int64_t u_lo = tile * 128;   // units below belong to the previous tile
      const int64_t ub = y0 + q * 32;
#pragma unroll
      for (int r4 = 0; r4 < 4; ++r4) {
        const int kc = r4 * 32 + lane, l2 = kc >> 2, p2 = kc & 3;
        const uint4 val =
            *reinterpret_cast<const uint4*>(wbuf + l2 * 64 + ((p2 ^ ((l2 >> 1) & 3)) << 4));
        const int64_t ou =
            ub + l2 < u_lo ? -1 : (kKv ? kv_unit(P.slots, P.num_slots, P.kpr, ub + l2) : ub + l2);
        if (ou >= 0) *reinterpret_cast<uint4*>(P.codes + ou * 64 + p2 * 16) = val;
      }
      const int64_t om =
          y0 + m < u_lo ? -1 : (kKv ? kv_unit(P.slots, P.num_slots, P.kpr, y0 + m) : y0 + m);
      if (om >= 0) {
        uint16_t zh;
        asm("cvt.rn.f16.f32 %0, %1;" : "=h"(zh) : "f"(zf));
        P.scales16[om] = (uint16_t)s16;
        P.zeros16[om] = zh;
      }
      __syncwarp();
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

}  // namespace tcb

bool tcb_supported(const Geometry& g, int dtype, const void* x, int64_t tokens) {
  const int64_t units = tokens * (g.n / tcb::B);
  return dtype == 1 && !g.paley && g.b == tcb::B && g.n <= 16384 &&
         (reinterpret_cast<uintptr_t>(x) & 15) == 0 && units >= 128 &&
         units < (int64_t(1) << 31);
}

cudaError_t launch_tcb_asym(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, uint16_t* scales,
                            uint16_t* zeros, const int64_t* slots, int64_t num_slots,
                            cudaStream_t s) {
  tcb::Params P{};
  P.signs = signs;
  P.codes = codes;
  P.scales16 = scales;
  P.zeros16 = zeros;
  P.slots = slots;
  P.num_slots = num_slots;
  P.units = tokens * (g.n / tcb::B);
  P.tiles = (P.units + 127) / 128;
  P.kpr = g.n / tcb::B;
  // [units, 128] bf16 view of the input, 64 x 128 boxes, 128-byte swizzle
  CUtensorMap map;
  if (!encode_tmap_bf16_2d(&map, x, 128, (uint64_t)P.units, 64, 128,
                           CU_TENSOR_MAP_SWIZZLE_128B))
    return cudaErrorNotSupported;
  auto k = slots ? tcb::k_tcb128_asym<true> : tcb::k_tcb128_asym<false>;
  cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)tcb::kSmemBytes);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t grid = P.tiles < sms ? P.tiles : sms;
  k<<<(int)grid, tcb::kThreads, tcb::kSmemBytes, s>>>(map, P);
  return cudaGetLastError();
}

// Reads and clears the error word of the tcb kernels (device-synchronous).
cudaError_t take_tcb_errors(unsigned int* out) {
  const unsigned int zero = 0;
  cudaError_t e = cudaMemcpyFromSymbol(out, tcb::g_tcb_error, sizeof(unsigned int));
  if (e != cudaSuccess) return e;
  return cudaMemcpyToSymbol(tcb::g_tcb_error, &zero, sizeof(unsigned int));
}

}  // namespace kq
