// Tensor-core (tcgen05) kernels for full-row Hadamard transforms of 4096-wide
// rows (the hidden size of "Bug: Qwen3-8B integration issue", Model Details).
//
// A row of n = 4096 values is viewed as 64 blocks of 64 (index i = o*64 + beta).
// Sylvester H_4096 = H_64 kron H_64 in natural order, so the transform splits
// into
//   (1) a cross-block mix  D[o][beta] = sum_a H_64[o][a] x'[a*64 + beta]
//       -- a dense +-1 contraction over the block index, run on the tensor
//       cores: D (TMEM, fp32) = A * B with A = I_2 kron H_64 (bf16 +-1,
//       K-major, built in shared memory once) and B = 128 consecutive
//       64-element blocks of x' (the sign-flipped input, MN-major, one TMA box
//       per tile), i.e. two tokens per tile;
//   (2) the in-block H_64 over beta, run by the epilogue thread that owns TMEM
//       lane (token, o): it reads the 64 columns of its lane and finishes the
//       transform with six butterfly stages in fp32 (five on f32x2 pairs).
// The thread then holds the 64 contiguous outputs o*64 .. o*64+63 of its
// token: four NVFP4 16-blocks, quantized in registers.  (QuaRot reviews,
// review 1 Summary: Walsh-Hadamard algorithm; NVFP4 thread: NVFP4 format.)
//
// Products of bf16 inputs with +-1 are exact; the tensor core accumulates in
// fp32.  The error of S_hat is bounded by E = 16 u sum|x| per token: four
// k-steps with non-zero products, each rounding its sum into the fp32
// accumulator once (at most 2u relative each), then six fp32 butterfly stages
// (6u).  sum|x| is accumulated by the sign-flip warps while they touch the
// tile.  (Measured on B200: the largest error seen was 0.94 u sum|x|, on
// inputs spanning 2^40 in magnitude.)  Scales undecided under the bound are
// recomputed exactly (fp64) from the staged input, which stays in shared
// memory until the epilogue releases its stage.
//
// Warp roles (14 warps): 0 TMA producer, 1 MMA issuer + TMEM owner, 2-5 sign
// flip and sum|x| in shared memory (two warps per token), 6-13 epilogue (two
// groups of four warps, one per TMEM accumulator; warp w reads TMEM lane
// quarter w % 4).  Every wait on an mbarrier is bounded; on timeout the kernel
// records an error code and returns.
#include <cuda.h>
#include <cudaTypedefs.h>

#include <cfloat>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace tc {

constexpr int kStages = 8;
constexpr int kGroups = 2;                     // epilogue groups = TMEM accumulators
constexpr int kSignWarps = 4;                  // two per token
constexpr int kEpiWarps = 4 * kGroups;
constexpr int kThreads = 32 * (2 + kSignWarps + kEpiWarps);   // 14 warps
constexpr int kTileRows = 128;                 // rows of the [T*64, 64] view per tile
constexpr uint32_t kTileBytes = kTileRows * 64 * 2;    // 16 KB
constexpr long long kWaitCycles = 4000000000ll;   // about 2 s at 2 GHz

__device__ unsigned int g_tc_error = 0;        // nonzero: a wait timed out

enum { kNvfp4 = 0, kNvStats = 1, kRot = 2 };

struct Params {
  uint8_t* codes;               // [T, n/2]
  uint8_t* scales8;             // [T, n/16]
  float* tensor_scale;
  NvWorkspace* ws;
  float* out;                   // kRot: fp32 [T, n]
  const uint16_t* x;            // for exact fix-ups from global (unused) / debug
  int64_t tokens;
  int64_t tiles;
  float e_coef;                 // E = e_coef * sum|x| of the token (rounded up)
};

// --------------------------------------------------------------- helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" :: "r"(smem_u32(bar)), "r"(count));
}
__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];" :: "r"(smem_u32(bar))
               : "memory");
}
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;"
               :: "r"(smem_u32(bar)), "r"(bytes) : "memory");
}
// Bounded wait for the phase with the given parity; false on timeout (about
// two seconds).  try_wait suspends the thread for up to the hint (ns) instead
// of spinning.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  const long long start = clock64();
  for (;;) {
    uint32_t ok;
    asm volatile("{\n\t.reg .pred p;\n\t"
                 "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
                 "selp.u32 %0, 1, 0, p;\n\t}"
                 : "=r"(ok) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    if (ok) return true;
    if (clock64() - start > kWaitCycles) break;
  }
  atomicOr(&g_tc_error, 1u);
  return false;
}
__device__ __forceinline__ void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y,
                                            uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];"
      :: "r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
         "r"(smem_u32(bar)) : "memory");
}
__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor (tcgen05): start >> 4, leading and stride
// byte offsets >> 4, version 1, layout type 2 (128-byte swizzle).
__device__ __forceinline__ uint64_t smem_desc(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  uint64_t d = 0;
  d |= (uint64_t)((addr >> 4) & 0x3FFFu);
  d |= (uint64_t)((lbo >> 4) & 0x3FFFu) << 16;
  d |= (uint64_t)((sbo >> 4) & 0x3FFFu) << 32;
  d |= (uint64_t)1 << 46;           // version
  d |= (uint64_t)2 << 61;           // SWIZZLE_128B
  return d;
}

// kind::f16 instruction descriptor: D fp32, A and B bf16, A K-major,
// B MN-major, N = 64, M = 128.
constexpr uint32_t kIdesc = (1u << 4) | (1u << 7) | (1u << 10) | (0u << 15) | (1u << 16) |
                            ((64u >> 3) << 17) | ((128u >> 4) << 24);

__device__ __forceinline__ void mma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %6, %7, %8}, p;\n\t}"
      :: "r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(kIdesc), "r"(accumulate),
         "r"(0u), "r"(0u), "r"(0u), "r"(0u));
}
__device__ __forceinline__ void mma_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];"
               :: "r"(smem_u32(bar)) : "memory");
}

// 32 consecutive TMEM columns of this thread's lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
      "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}
__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void bfly2(float2& a, float2& b) {
  uint64_t ua = *reinterpret_cast<uint64_t*>(&a), ub = *reinterpret_cast<uint64_t*>(&b), s, d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s) : "l"(ua), "l"(ub));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(ua), "l"(ub));
  a = *reinterpret_cast<float2*>(&s);
  b = *reinterpret_cast<float2*>(&d);
}
__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t ua = *reinterpret_cast<uint64_t*>(&a), ub = *reinterpret_cast<uint64_t*>(&b),
           uc = *reinterpret_cast<uint64_t*>(&c), r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ua), "l"(ub), "l"(uc));
  return *reinterpret_cast<float2*>(&r);
}
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ uint32_t e4m3_pair(float r_lo, float r_hi) {
  uint32_t out;
  asm("{.reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %2; cvt.u32.u16 %0, t;}"
      : "=r"(out) : "f"(r_hi), "f"(r_lo));
  return out;
}
// 1 / value of a non-zero E4M3 code: a rounded reciprocal of the significand
// (table folded at compile time) scaled by an exact power of two.
__device__ __forceinline__ float e4m3_recip(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return 512.0f / (float)m;                 // subnormal: m * 2^-9
  constexpr float kR0 = 1.0f / 1.0f, kR1 = 1.0f / 1.125f, kR2 = 1.0f / 1.25f,
                  kR3 = 1.0f / 1.375f, kR4 = 1.0f / 1.5f, kR5 = 1.0f / 1.625f,
                  kR6 = 1.0f / 1.75f, kR7 = 1.0f / 1.875f;
  const float r = m < 4 ? (m < 2 ? (m == 0 ? kR0 : kR1) : (m == 2 ? kR2 : kR3))
                        : (m < 6 ? (m == 4 ? kR4 : kR5) : (m == 6 ? kR6 : kR7));
  return __uint_as_float(__float_as_uint(r) + ((7u - e) << 23));   // r * 2^(7-e)
}

// Byte offset of element (row r, column col) of a 128-byte-swizzled matrix
// stored as 16 KB halves of 128 rows x 64 columns (bf16): 16-byte chunk c of
// row r sits at chunk position c ^ (r & 7).  The input tiles are one half; the
// 128 x 128 A operand is two.
__device__ __forceinline__ uint32_t tile_off(int r, int col) {
  const int h = col >> 6, c = (col >> 3) & 7, e = col & 7;
  return (uint32_t)(h * 16384 + r * 128 + ((c ^ (r & 7)) << 4) + e * 2);
}

// Exact S_i of token row `tr` of a staged tile (rows tr*64 .. tr*64+63, sign-
// flipped), warp-cooperative fp64: lane l sums columns l and l + 32 of every
// block.  Every lane gets the result.
__device__ __noinline__ double warp_exact_S(const uint8_t* stage, int tr, int i) {
  const int lane = threadIdx.x & 31;
  double acc = 0.0;
  for (int a = 0; a < 64; ++a) {
    const int r = tr * 64 + a;
#pragma unroll
    for (int q = 0; q < 2; ++q) {
      const int beta = lane + 32 * q;
      const uint16_t b = *reinterpret_cast<const uint16_t*>(stage + tile_off(r, beta));
      const double xv = (double)__uint_as_float((uint32_t)b << 16);
      const int j = a * 64 + beta;
      acc += (__popc(i & j) & 1) ? -xv : xv;
    }
  }
  return warp_sum_d(acc);
}

// ---------------------------------------------------------------- kernel
template <int kMode>
__global__ void __launch_bounds__(kThreads, 1)
k_tc4096(const __grid_constant__ CUtensorMap tmap, const int8_t* __restrict__ signs, Params P) {
  constexpr int N = 4096;
  constexpr double kSqrtN = 64.0;
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  uint8_t* sA = smem;                                   // 32 KB: A = I_2 kron H_64
  uint8_t* sB = smem + 32768;                           // kStages x 16 KB
  uint4* smask = reinterpret_cast<uint4*>(sB + kStages * kTileBytes);   // 512 chunks
  uint4* scode = smask + 512;                           // epilogue warps x 1 KB code staging
  float* sabs = reinterpret_cast<float*>(scode + kEpiWarps * 64);   // sum|x| per (stage, sign warp)
  uint64_t* bars = reinterpret_cast<uint64_t*>(sabs + kSignWarps * kStages);
  uint64_t* full = bars;                                // TMA landed
  uint64_t* ready = bars + kStages;                     // signs applied
  uint64_t* empty = bars + 2 * kStages;                 // epilogue done with the stage
  uint64_t* tfull = bars + 3 * kStages;                 // accumulator written (kGroups)
  uint64_t* tempty = tfull + kGroups;                   // accumulator read (kGroups)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + kGroups);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  // ---- set-up: A operand, sign masks, barriers, TMEM
  for (int idx = threadIdx.x; idx < 128 * 128; idx += blockDim.x) {
    const int m = idx >> 7, k = idx & 127;
    const int tm = m >> 6, o = m & 63, tk = k >> 6, a = k & 63;
    uint16_t v = 0;
    if (tm == tk) v = (__popc(o & a) & 1) ? 0xBF80 : 0x3F80;    // -1 / +1 in bf16
    *reinterpret_cast<uint16_t*>(sA + tile_off(m, k)) = v;
  }
  for (int i = threadIdx.x; i < 512; i += blockDim.x) {
    // chunk (a, c): columns c*8 .. c*8+7 of 64-block a = sign bytes 8 i .. 8 i + 7
    uint4 m4 = make_uint4(0, 0, 0, 0);
    if (signs) {
      const uint2 sv = __ldg(reinterpret_cast<const uint2*>(signs) + i);
      m4 = make_uint4(__byte_perm(sv.x, 0, 0x1404) & 0x80008000u,
                      __byte_perm(sv.x, 0, 0x3424) & 0x80008000u,
                      __byte_perm(sv.y, 0, 0x1404) & 0x80008000u,
                      __byte_perm(sv.y, 0, 0x3424) & 0x80008000u);
    }
    smask[i] = m4;
  }
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&ready[s], 32 * kSignWarps);
      mbar_init(&empty[s], 128);
    }
    for (int d = 0; d < kGroups; ++d) {
      mbar_init(&tfull[d], 1);
      mbar_init(&tempty[d], 128);
    }
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], 256;"
                 :: "r"(smem_u32(tmem_slot)));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  fence_async_smem();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  const int64_t my_tiles = (P.tiles - blockIdx.x + gridDim.x - 1) / gridDim.x;

  if (warp == 0) {
    // ================= TMA producer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        const uint32_t use = (uint32_t)(k / kStages);
        if (k >= kStages && !mbar_wait(&empty[s], (use - 1) & 1)) break;
        const int64_t tile = blockIdx.x + k * gridDim.x;
        mbar_expect_tx(&full[s], kTileBytes);
        tma_load_2d(sB + s * kTileBytes, &tmap, 0, (int)(tile * kTileRows), &full[s]);
        issued = k + 1;
      }
      // no copy may still be in flight when the CTA exits (matters only after
      // a timeout; in normal operation these phases have completed)
      for (int64_t k = issued > kStages ? issued - kStages : 0; k < issued; ++k)
        mbar_wait(&full[k % kStages], (uint32_t)(k / kStages) & 1);
    }
  } else if (warp == 1) {
    // ================= MMA issuer
    if (lane == 0) {
      int64_t issued = 0;
      for (int64_t k = 0; k < my_tiles; ++k) {
        const int s = (int)(k % kStages);
        const int d = (int)(k % kGroups);
        if (!mbar_wait(&ready[s], (uint32_t)(k / kStages) & 1)) break;
        if (k >= kGroups && !mbar_wait(&tempty[d], (uint32_t)(k / kGroups - 1) & 1)) break;
        tc_fence_after();
        const uint32_t a0 = smem_u32(sA), b0 = smem_u32(sB + s * kTileBytes);
        const uint32_t tmem_d = tmem_base + (uint32_t)(d * 64);
#pragma unroll
        for (int ks = 0; ks < 8; ++ks) {
          // A: K-major, K step of 16 = 32 bytes inside a 128-byte swizzle row
          const uint64_t adesc = smem_desc(a0 + (ks >> 2) * 16384 + (ks & 3) * 32, 16, 1024);
          // B: MN-major (one 64-wide atom), K step of 16 rows = two 1 KB atoms
          const uint64_t bdesc = smem_desc(b0 + ks * 2048, 16384, 1024);
          mma_bf16(tmem_d, adesc, bdesc, ks > 0 ? 1u : 0u);
        }
        mma_commit(&tfull[d]);
        issued = k + 1;
      }
      // the accumulators must not be released with MMAs still running
      for (int64_t k = issued > kGroups ? issued - kGroups : 0; k < issued; ++k)
        mbar_wait(&tfull[k % kGroups], (uint32_t)(k / kGroups) & 1);
    }
  } else if (warp < 2 + kSignWarps) {
    // ================= sign flip + sum|x|: warps 2-3 token 0, warps 4-5 token 1
    const int sw = warp - 2;                 // 0..3: token sw/2, half sw%2
    for (int64_t k = 0; k < my_tiles; ++k) {
      const int s = (int)(k % kStages);
      if (!mbar_wait(&full[s], (uint32_t)(k / kStages) & 1)) break;
      uint8_t* st = sB + s * kTileBytes;
      float2 acc = make_float2(0.0f, 0.0f);
#pragma unroll 4
      for (int j = 0; j < 8; ++j) {
        // physical chunk idx of this token half: row r, swizzled chunk pc
        const int idx = sw * 256 + lane + 32 * j;
        const int r = idx >> 3, pc = idx & 7;
        const int c = pc ^ (r & 7);
        uint4* p = reinterpret_cast<uint4*>(st + idx * 16);
        uint4 w = *p;
        if (signs) {
          const uint4 m = smask[(r & 63) * 8 + c];
          w.x ^= m.x;
          w.y ^= m.y;
          w.z ^= m.z;
          w.w ^= m.w;
          *p = w;
        }
        const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const uint32_t wa = ww[e] & 0x7fff7fffu;      // |x| of both halves
          const float2 ab = make_float2(__uint_as_float(wa << 16), __uint_as_float(wa & 0xffff0000u));
          uint64_t ua = *reinterpret_cast<const uint64_t*>(&ab),
                   uc = *reinterpret_cast<uint64_t*>(&acc), rr;
          asm("add.rn.f32x2 %0, %1, %2;" : "=l"(rr) : "l"(uc), "l"(ua));
          acc = *reinterpret_cast<float2*>(&rr);
        }
      }
      float sum = acc.x + acc.y;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
      if (lane == 0) sabs[s * kSignWarps + sw] = sum;
      if (signs) fence_async_smem();
      __syncwarp();
      mbar_arrive(&ready[s]);
    }
  } else {
    // ================= epilogue: group g of warps 6+4g .. 9+4g
    const int g = (warp - 2 - kSignWarps) >> 2;
    const int q = warp & 3;                   // TMEM lane quarter
    const int m = q * 32 + lane;              // accumulator row = (token in tile, block o)
    const int tr = m >> 6, o = m & 63;
    const int ew = warp - 2 - kSignWarps;     // epilogue warp index
    uint4* wcode = scode + ew * 64;
    float t = 0.0f, c6 = 0.0f, inv_bt = 0.0f;
    if (kMode == kNvfp4) {
      if (P.ws) {
        const double gm = __longlong_as_double((long long)P.ws->gmax_bits);
        t = __double2float_rn((gm / kSqrtN) / 2688.0);
        if (blockIdx.x == 0 && ew == 0 && lane == 0) *P.tensor_scale = t;
      } else {
        t = *P.tensor_scale;
      }
      c6 = (t > 0.0f) ? (float)(1.0 / (kSqrtN * 6.0 * (double)t)) : 0.0f;
      inv_bt = (t > 0.0f) ? (float)(1.0 / (kSqrtN * (double)t)) : 0.0f;
    }
    for (int64_t k = g; k < my_tiles; k += kGroups) {
      const int s = (int)(k % kStages);
      const int64_t tile = blockIdx.x + k * gridDim.x;
      // Both warps of a token pass the same named barriers below, so a timed-out
      // wait does not leave the loop: the failure is recorded (g_tc_error) and
      // the tile's outputs are not written.
      bool ok = mbar_wait(&tfull[g], (uint32_t)(k / kGroups) & 1);
      // the staged input (read by the fix-ups) is final once its signs are applied
      ok = mbar_wait(&ready[s], (uint32_t)(k / kStages) & 1) && ok;
      tc_fence_after();
      float2 v[32];
      {
        uint32_t r[32];
        const uint32_t taddr = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)(g * 64);
#pragma unroll
        for (int cb = 0; cb < 2; ++cb) {
          tmem_ld32(taddr + cb * 32, r);
          tmem_wait_ld();
#pragma unroll
          for (int e = 0; e < 16; ++e)
            v[cb * 16 + e] = make_float2(__uint_as_float(r[2 * e]), __uint_as_float(r[2 * e + 1]));
        }
      }
      tc_fence_before();
      mbar_arrive(&tempty[g]);
      // in-block H_64 over beta
#pragma unroll
      for (int p = 0; p < 32; ++p) {
        const float a = v[p].x, b = v[p].y;
        v[p] = make_float2(a + b, a - b);
      }
#pragma unroll
      for (int hh = 1; hh < 32; hh <<= 1)
#pragma unroll
        for (int p = 0; p < 32; ++p)
          if (!(p & hh)) bfly2(v[p], v[p | hh]);

      const int64_t token = tile * 2 + tr;
      const bool valid = ok && token < P.tokens;
      float bm[4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        float mm = 0.0f;
#pragma unroll
        for (int p = 8 * j; p < 8 * j + 8; ++p) mm = fmax3(mm, fabsf(v[p].x), fabsf(v[p].y));
        bm[j] = mm;
      }
      // |S_hat - S| <= E for every output of the token (sum|x| rounded up)
      const float E =
          __fmul_ru(P.e_coef, (sabs[s * kSignWarps + 2 * tr] + sabs[s * kSignWarps + 2 * tr + 1]) *
                                  1.001f);

      if (kMode == kRot) {
        if (valid) {
          const float inv = (float)(1.0 / kSqrtN);
          float4* dst = reinterpret_cast<float4*>(P.out + token * N + o * 64);
#pragma unroll
          for (int p = 0; p < 16; ++p)
            dst[p] = make_float4(v[2 * p].x * inv, v[2 * p].y * inv, v[2 * p + 1].x * inv,
                                 v[2 * p + 1].y * inv);
        }
        mbar_arrive(&empty[s]);
        continue;
      }
      if (kMode == kNvStats) {
        float mh = fmaxf(fmaxf(bm[0], bm[1]), fmaxf(bm[2], bm[3]));
#pragma unroll
        for (int off = 16; off > 0; off >>= 1)
          mh = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, off));
        if (valid && lane == 0) {   // two warps per token: max through atomics
          atomicMax(reinterpret_cast<unsigned int*>(&P.ws->rows[token].x), __float_as_uint(mh));
          atomicMax(reinterpret_cast<unsigned int*>(&P.ws->rows[token].y), __float_as_uint(E));
          atomicMax(&P.ws->lower_bits, __float_as_uint(fmaxf(__fsub_rd(mh, E), 0.0f)));
        }
        mbar_arrive(&empty[s]);
        continue;
      }

      // ---- NVFP4 block scales, exact where undecided
      uint32_t sc = 0;
      uint32_t undecided = 0;
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const float lo = fmaxf(bm[j] - E, 0.0f) * c6 * (1.0f - 0x1p-20f);
        const float hi = (bm[j] + E) * c6 * (1.0f + 0x1p-20f);
        const uint32_t cc = e4m3_pair(lo, hi);
        sc |= (cc & 0xffu) << (8 * j);
        if ((cc & 0xffu) != (cc >> 8)) undecided |= 1u << j;
      }
      if (t <= 0.0f || !valid) undecided = 0;
      unsigned todo = __ballot_sync(0xffffffffu, undecided != 0);
      const uint8_t* stage = sB + s * kTileBytes;
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        const uint32_t und = __shfl_sync(0xffffffffu, undecided, src);
        const int src_o = (q * 32 + src) & 63;
        for (int j = 0; j < 4; ++j) {
          if (!((und >> j) & 1u)) continue;
          uint32_t cand = 0;
          if (lane == src) {
            float bmj = 0.0f;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq)
              if (qq == j) bmj = bm[qq];
            const float thr = bmj - 2.0f * E;
#pragma unroll
            for (int qq = 0; qq < 4; ++qq) {
              if (qq != j) continue;
#pragma unroll
              for (int p = 0; p < 8; ++p) {
                const float2 a = v[8 * qq + p];
                if (fabsf(a.x) >= thr) cand |= 1u << (2 * p);
                if (fabsf(a.y) >= thr) cand |= 1u << (2 * p + 1);
              }
            }
          }
          cand = __shfl_sync(0xffffffffu, cand, src);
          double best = 0.0;
          while (cand) {
            const int e = __ffs(cand) - 1;
            cand &= cand - 1;
            best = fmax(best, fabs(warp_exact_S(stage, tr, src_o * 64 + 16 * j + e)));
          }
          const float r = __double2float_rn((best / kSqrtN) / (6.0 * (double)t));
          const uint32_t code = e4m3_pair(r, r) & 0xffu;
          if (lane == src) sc = (sc & ~(0xffu << (8 * j))) | (code << (8 * j));
        }
      }
      __syncwarp();
      mbar_arrive(&empty[s]);        // staged input no longer needed

      // ---- codes: 32 bytes (two 16-byte chunks) per lane
      const float2 zero2 = make_float2(0.0f, 0.0f);
      uint4 cw[2];
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        uint32_t words[4];
#pragma unroll
        for (int jj = 0; jj < 2; ++jj) {
          const int j = 2 * kk + jj;
          const uint32_t code = (sc >> (8 * j)) & 0xffu;
          if (code != 0 && t > 0.0f) {
            const float c = inv_bt * e4m3_recip(code);
            const float2 c2 = make_float2(c, c);
            float qv[16];
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const float2 a = fma2(v[8 * j + p], c2, zero2);   // + 0 turns -0 into +0
              qv[2 * p] = a.x;
              qv[2 * p + 1] = a.y;
            }
            words[2 * jj] = e2m1x8_hw(qv);
            words[2 * jj + 1] = e2m1x8_hw(qv + 8);
          } else {
            uint32_t w0 = 0, w1 = 0;
#pragma unroll
            for (int p = 0; p < 4; ++p) {
              w0 |= (v[8 * j + p].x < 0.0f ? 8u : 0u) << (8 * p);
              w0 |= (v[8 * j + p].y < 0.0f ? 8u : 0u) << (8 * p + 4);
              w1 |= (v[8 * j + 4 + p].x < 0.0f ? 8u : 0u) << (8 * p);
              w1 |= (v[8 * j + 4 + p].y < 0.0f ? 8u : 0u) << (8 * p + 4);
            }
            words[2 * jj] = w0;
            words[2 * jj + 1] = w1;
          }
        }
        cw[kk] = make_uint4(words[0], words[1], words[2], words[3]);
      }
      // the warp's 32 lanes own 1 KB of consecutive code bytes of its token;
      // stage through shared memory so the warp stores whole 16-byte chunks
      __syncwarp();
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) wcode[lane * 2 + (kk ^ (lane & 1))] = cw[kk];
      __syncwarp();
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(P.codes + token * (N / 2) + (o - lane) * 32);
#pragma unroll
        for (int jx = 0; jx < 2; ++jx) {
          const int idx = lane + 32 * jx;
          const int src = idx >> 1, kk = idx & 1;
          dst[idx] = wcode[src * 2 + (kk ^ (src & 1))];
        }
        *reinterpret_cast<uint32_t*>(P.scales8 + token * (N / 16) + o * 4) = sc;
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, 256;" :: "r"(tmem_base));
  }
}

}  // namespace tc

// ------------------------------------------------------------- launchers
namespace {

PFN_cuTensorMapEncodeTiled_v12000 get_encode() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// [rows, 64] bf16 view of the input (rows of 128 bytes), 64 x 128 boxes,
// 128-byte swizzle.
bool make_tmap(CUtensorMap* map, const void* x, int64_t rows) {
  auto enc = get_encode();
  if (!enc) return false;
  cuuint64_t gdim[2] = {64, (cuuint64_t)rows};
  cuuint64_t gstride[1] = {128};
  cuuint32_t box[2] = {64, 128};
  cuuint32_t estride[2] = {1, 1};
  CUresult r = enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(x), gdim, gstride,
                   box, estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                   CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

constexpr size_t kSmemBytes = 1024 + 32768 + tc::kStages * tc::kTileBytes + 512 * 16 +
                              tc::kEpiWarps * 64 * 16 + tc::kSignWarps * tc::kStages * 4 + 512;

template <int kMode>
cudaError_t launch_tc(const void* x, const int8_t* signs, tc::Params& P, cudaStream_t s) {
  CUtensorMap map;
  if (!make_tmap(&map, x, P.tokens * 64)) return cudaErrorNotSupported;
  auto k = tc::k_tc4096<kMode>;
  cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       (int)kSmemBytes);
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  P.tiles = (P.tokens * 64 + tc::kTileRows - 1) / tc::kTileRows;
  const int64_t grid = P.tiles < sms ? P.tiles : sms;
  k<<<(int)grid, tc::kThreads, kSmemBytes, s>>>(map, signs, P);
  return cudaGetLastError();
}

float e_coef_tc() {
  // 4 accumulation steps x 2u + 6 fp32 stages = 14u, rounded up to 16u
  return (float)(16.0 * 0x1p-24);
}

}  // namespace

bool tc_row_supported(const Geometry& g, int dtype) {
  return dtype == 1 && !g.paley && g.b == g.n && g.n == 4096;
}

cudaError_t launch_tc_nvfp4(const void* x, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                            float* tensor_scale, NvWorkspace* ws, cudaStream_t s) {
  tc::Params P{};
  P.codes = codes;
  P.scales8 = bscales;
  P.tensor_scale = tensor_scale;
  P.ws = ws;
  P.tokens = tokens;
  P.x = static_cast<const uint16_t*>(x);
  P.e_coef = e_coef_tc();
  cudaError_t e;
  if (ws) {
    e = cudaMemsetAsync(ws, 0, kNvWorkspaceHeader + (size_t)tokens * sizeof(float2), s);
    if (e != cudaSuccess) return e;
    e = launch_tc<tc::kNvStats>(x, signs, P, s);
    if (e != cudaSuccess) return e;
    e = launch_nvfp4_global(x, 1, tokens, g, signs, ws, s);
    if (e != cudaSuccess) return e;
  }
  return launch_tc<tc::kNvfp4>(x, signs, P, s);
}

cudaError_t launch_tc_rot(const void* x, int64_t tokens, const Geometry& g, const int8_t* signs,
                          float* out, cudaStream_t s) {
  tc::Params P{};
  P.out = out;
  P.tokens = tokens;
  P.x = static_cast<const uint16_t*>(x);
  P.e_coef = e_coef_tc();
  (void)g;
  return launch_tc<tc::kRot>(x, signs, P, s);
}

int tc_error_flag() {
  unsigned int v = 0;
  cudaMemcpyFromSymbol(&v, tc::g_tc_error, sizeof(v));
  return (int)v;
}

}  // namespace kq
