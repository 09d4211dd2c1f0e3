// SIMT kernels for 128-wide Hadamard blocks (block = 128).
//
// "Block-Hadamard-128" (NVFP4 thread, discrete_descent's note) and the
// per-head 128-point Hadamard of the KV cache (QuaRot reviews, final comments)
// apply an independent H_128 to every 128 consecutive columns.
//   * Asymmetric INT4: one thread owns one (row, block) unit: its 128 inputs
//     arrive from a per-warp shared-memory stage, the sign flips are XORs on
//     the bf16 sign bits, and the seven butterfly stages run in registers
//     (stage 0 in scalar fp32, stages 1..6 on packed f32x2 pairs).  The
//     128-element group lies inside the thread, so extrema, scale, zero
//     point, rounding and nibble packing need no communication.
//   * NVFP4: four lanes share a unit (five stages in registers, two across
//     the quad by shuffles); each lane then owns two whole 16-blocks.
//
// Exact scales.  The fp32 transform of one 128-block is within
// E = gamma_7 sqrt(128) max|S_hat| of the exact sums (see error_bound in
// kq_device.cuh).  A scale is decided from the fp32 values when both ends of
// its interval round to the same stored value; the rare undecided ones are
// recomputed by the whole warp as exact fp64 dot products with the input.
//
// Dynamic NVFP4 tensor scale: a statistics pass (row maxima and bounds), then
// the quantisation pass, which on up to kFusedExactRows rows finds the exact
// global maximum itself (each CTA screens every row's statistics and
// transforms the candidate rows in fp64) and is launched as a programmatic
// dependent of the statistics pass.
#include <cfloat>
#include <climits>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace blk {

constexpr int B = 128;          // Hadamard block width
constexpr int kThreads = 128;

struct Params {
  const uint16_t* x;            // bf16 bits [T, n]
  const int8_t* signs;          // [n] or null
  uint8_t* codes;               // [T, n/2]
  uint8_t* scales8;             // NVFP4 E4M3 [T, n/16]
  uint16_t* scales16;           // asym fp16 [T, n/128]
  uint16_t* zeros16;            // asym fp16 [T, n/128]
  float* tensor_scale;          // NVFP4 t (device): read if static, written if dynamic
  NvWorkspace* ws;              // NVFP4 dynamic: gmax (read) / row stats (written)
  int64_t units;                // T * n / 128
  const int64_t* slots;         // asym: cache row of each input row, or null
  int64_t num_slots;
  int n;
  float e_coef;                 // E = e_coef * max|S_hat| (rounded up)
  int sf_kc4;                   // NVFP4 scale layout (Geometry::sf_kc4)
  int fuse_exact;               // NVFP4 dynamic quantisation: compute the exact maximum first
};

__device__ __forceinline__ int stage_chunk(int unit, int c);

// packed f32x2 butterfly: (a, b) <- (a + b, a - b) on two lanes at once
__device__ __forceinline__ void bfly2(float2& a, float2& b) {
  uint64_t ua = *reinterpret_cast<uint64_t*>(&a), ub = *reinterpret_cast<uint64_t*>(&b), s, d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(s) : "l"(ua), "l"(ub));
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(ua), "l"(ub));
  a = *reinterpret_cast<float2*>(&s);
  b = *reinterpret_cast<float2*>(&d);
}

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}
__device__ __forceinline__ float fmin3(float a, float b, float c) {
  float d;
  asm("min.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
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

__device__ __forceinline__ float2 fma2(float2 a, float2 b, float2 c) {
  uint64_t ua = *reinterpret_cast<uint64_t*>(&a), ub = *reinterpret_cast<uint64_t*>(&b),
           uc = *reinterpret_cast<uint64_t*>(&c), r;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(r) : "l"(ua), "l"(ub), "l"(uc));
  return *reinterpret_cast<float2*>(&r);
}

// Shared-memory stage of one warp: 32 units x 256 bytes, 16-byte chunk c of
// unit t stored at chunk position c ^ (t & 15) of its row.  Warp-wide
// coalesced writes (lane l -> chunk l + 32 j) and per-thread row reads are
// both bank-conflict-free.
__device__ __forceinline__ int stage_chunk(int unit, int c) { return unit * 16 + (c ^ (unit & 15)); }


// Starts copying the warp's 32 consecutive units (8 KB, contiguous in memory)
// into the stage with coalesced 16-byte asynchronous copies, as one commit
// group.  Units at or beyond `units` are skipped.
__device__ __forceinline__ void prefetch_units(const uint16_t* __restrict__ x, int64_t ub,
                                               int64_t units, uint4* stage) {
  const int lane = threadIdx.x & 31;
  const uint4* src = reinterpret_cast<const uint4*>(x + ub * B);
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(stage);
#pragma unroll
  for (int j = 0; j < 16; ++j) {
    const int idx = lane + 32 * j;
    if (ub + (idx >> 4) < units) {
      const uint32_t dst = base + 16u * (uint32_t)stage_chunk(idx >> 4, idx & 15);
      asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(dst), "l"(src + idx)
                   : "memory");
    }
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

__device__ __forceinline__ void wait_prefetch(bool newer_pending) {
  if (newer_pending)
    asm volatile("cp.async.wait_group 1;" ::: "memory");
  else
    asm volatile("cp.async.wait_group 0;" ::: "memory");
  __syncwarp();
}

// Sign masks of every 128-column block, staged per CTA: 16-byte chunk c of
// column block k (four bf16-pair masks: bit 15 even, bit 31 odd element) at
// chunk position c ^ (k & 15).
__device__ __forceinline__ void stage_signs(const int8_t* __restrict__ signs, int n,
                                            uint4* smask) {
  for (int i = threadIdx.x; i < n / 8; i += blockDim.x) {
    const uint2 sv = __ldg(reinterpret_cast<const uint2*>(signs) + i);
    const int k = i >> 4, c = i & 15;
    smask[k * 16 + (c ^ (k & 15))] =
        make_uint4(__byte_perm(sv.x, 0, 0x1404) & 0x80008000u,
                   __byte_perm(sv.x, 0, 0x3424) & 0x80008000u,
                   __byte_perm(sv.y, 0, 0x1404) & 0x80008000u,
                   __byte_perm(sv.y, 0, 0x3424) & 0x80008000u);
  }
}

// Transforms this thread's unit from the stage: applies the signs of column
// block k (if smask) and runs the unnormalised H_128; v[p] = {S[2p], S[2p+1]}.
__device__ __forceinline__ void load_transform(const uint4* stage, int t, const uint4* smask,
                                               int k, float2 (&v)[64]) {
#pragma unroll
  for (int c = 0; c < 16; ++c) {
    const uint4 w = stage[stage_chunk(t, c)];
    uint32_t ww[4] = {w.x, w.y, w.z, w.w};
    if (smask) {
      const uint4 m = smask[k * 16 + (c ^ (k & 15))];
      ww[0] ^= m.x;
      ww[1] ^= m.y;
      ww[2] ^= m.z;
      ww[3] ^= m.w;
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const float lo = __uint_as_float(ww[q] << 16);
      const float hi = __uint_as_float(ww[q] & 0xffff0000u);
      v[4 * c + q] = make_float2(lo + hi, lo - hi);   // stage on bit 0
    }
  }
#pragma unroll
  for (int h = 1; h < 64; h <<= 1)
#pragma unroll
    for (int p = 0; p < 64; ++p)
      if (!(p & h)) bfly2(v[p], v[p | h]);
}

// Exact S of element `e` (0..127) of the warp's unit `t`, computed by the
// whole warp in fp64 from the staged input (lane l sums inputs 4l..4l+3) and
// the staged sign masks of column block k; every lane gets the result.
__device__ __noinline__ double warp_exact_S(const uint4* stage, const uint4* smask, int t,
                                            int k, int e) {
  const int lane = threadIdx.x & 31;
  const uint4 w = stage[stage_chunk(t, lane >> 1)];
  const uint32_t a = (lane & 1) ? w.z : w.x, b = (lane & 1) ? w.w : w.y;
  uint32_t ma = 0, mb = 0;
  if (smask) {
    const uint4 m = smask[k * 16 + ((lane >> 1) ^ (k & 15))];
    ma = (lane & 1) ? m.z : m.x;
    mb = (lane & 1) ? m.w : m.y;
  }
  const uint32_t pr[2] = {a ^ ma, b ^ mb};
  double acc = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = 4 * lane + q;
    const uint32_t bits = (q & 1) ? (pr[q >> 1] & 0xffff0000u) : (pr[q >> 1] << 16);
    const double xv = (double)__uint_as_float(bits);
    acc += (__popc(e & j) & 1) ? -xv : xv;
  }
  return warp_sum_d(acc);
}

// E4M3 code of r (>= 0) with the conversion instruction, nearest-even, satfinite.
__device__ __forceinline__ uint32_t e4m3_pair(float r_lo, float r_hi) {
  uint32_t out;
  asm("{.reg .b16 t; cvt.rn.satfinite.e4m3x2.f32 t, %1, %2; cvt.u32.u16 %0, t;}"
      : "=r"(out) : "f"(r_hi), "f"(r_lo));
  return out;   // bits 0-7: code(r_lo), bits 8-15: code(r_hi)
}

// 1 / value(E4M3 code) for a non-zero code (exact power-of-two scaling of a
// rounded reciprocal of the significand).
__device__ __forceinline__ float e4m3_recip(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return 512.0f / (float)m;                  // m * 2^-9
  const float r = 1.0f / (1.0f + 0.125f * (float)m);     // (1 + m/8)^-1
  return ldexpf(r, 7 - (int)e);
}

// ------------------------------------------------ NVFP4, four lanes a block
// Four lanes (a quad) share one 128-block: lane j of the quad loads the 64
// contiguous bytes of elements 32j .. 32j+31 (a warp reads 2 KB contiguous),
// runs the five in-lane butterfly stages (bit 0 in scalar fp32, bits 1-4 on
// f32x2 pairs) and the two stages across the quad (bits 5 and 6, shuffles),
// and then holds the outputs 32j .. 32j+31: its two NVFP4 16-blocks.  Same
// seven fp32 stages as a thread-per-block transform, so the same bound
// E = e_coef max|S_hat| over the block.  A quad per block gives four times the
// warps of a thread per block, which the short c2-sized inputs need (12.5
// against 14.4 us on 2048 x 4096; 55.2 against 56.0 us on 16384 x 4096).
constexpr int kQThreads = 256;
constexpr int kQLanes = 4;        // quantisation pass
constexpr int kQLanesStats = 8;   // statistics pass of the dynamic tensor scale, and the
                                  // quantisation pass that computes the exact maximum

// Exact S of element e (0..127) of 128-block u, computed by the whole warp in
// fp64 from global memory (lane l sums inputs 4l .. 4l+3, with the staged sign
// masks of column block k); every lane gets the result.
__device__ __noinline__ double warp_exact_S_global(const uint16_t* __restrict__ x,
                                                   const uint4* smask, int64_t u, int k, int e) {
  const int lane = threadIdx.x & 31;
  const uint2 w = __ldg(reinterpret_cast<const uint2*>(x + u * B) + lane);
  uint32_t ma = 0, mb = 0;
  if (smask) {
    const uint4 m = smask[k * 16 + ((lane >> 1) ^ (k & 15))];
    ma = (lane & 1) ? m.z : m.x;
    mb = (lane & 1) ? m.w : m.y;
  }
  const uint32_t pr[2] = {w.x ^ ma, w.y ^ mb};
  double acc = 0.0;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    const int j = 4 * lane + q;
    const uint32_t bits = (q & 1) ? (pr[q >> 1] & 0xffff0000u) : (pr[q >> 1] << 16);
    const double xv = (double)__uint_as_float(bits);
    acc += (__popc(e & j) & 1) ? -xv : xv;
  }
  return warp_sum_d(acc);
}

// max |S| over the outputs of up to four 128-blocks at once, in fp64: eight
// lanes a block (lanes 8i .. 8i+7 take block u_i of column block k_i, or
// nothing if u_i < 0); lane j of the eight holds inputs 16j .. 16j+15 (signs
// applied, exact in fp64), runs index bits 0 .. 3 as butterflies in the lane
// and bits 4 .. 6 across the eight.  Every lane gets the maximum over the
// four blocks.
__device__ __noinline__ double warp_blocks_absmax_f64(const uint16_t* __restrict__ x,
                                                      const uint4* smask, int64_t u, int k) {
  const int lane = threadIdx.x & 31, j = lane & 7;
  double v[16];
  if (u >= 0) {
    const uint4* src = reinterpret_cast<const uint4*>(x + u * B) + 2 * j;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const uint4 w = __ldg(src + h);
      uint4 m = make_uint4(0, 0, 0, 0);
      if (smask) m = smask[k * 16 + ((2 * j + h) ^ (k & 15))];
      const uint32_t ww[4] = {w.x ^ m.x, w.y ^ m.y, w.z ^ m.z, w.w ^ m.w};
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        v[8 * h + 2 * q] = (double)__uint_as_float(ww[q] << 16);
        v[8 * h + 2 * q + 1] = (double)__uint_as_float(ww[q] & 0xffff0000u);
      }
    }
  } else {
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = 0.0;
  }
#pragma unroll
  for (int st = 1; st < 16; st <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e)
      if (!(e & st)) {
        const double a = v[e], b = v[e | st];
        v[e] = a + b;
        v[e | st] = a - b;
      }
#pragma unroll
  for (int o = 1; o < 8; o <<= 1)
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const double p = __shfl_xor_sync(0xffffffffu, v[e], o);
      v[e] = (lane & o) ? p - v[e] : v[e] + p;
    }
  double m = 0.0;
#pragma unroll
  for (int e = 0; e < 16; ++e) m = fmax(m, fabs(v[e]));
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmax(m, __shfl_xor_sync(0xffffffffu, m, o));
  return m;
}

// The exact maximum of the dynamic tensor scale, computed by one whole CTA
// from the row statistics of the workspace: rows whose bound reaches the
// global lower bound are candidates, and every 128-block of a candidate row
// is transformed in fp64 (eight lanes a block, four blocks a warp).  A row
// whose computed maximum is zero has E = 0 and is exactly zero.  The row
// statistics are read eight rows a thread at a time into one candidate list;
// if more rows qualify than the list holds (many rows tied), each warp screens
// and finishes rows on its own instead, which costs one fp64 transform per
// tied row.  Every thread of the CTA must call it; all get max |S| (fp64,
// unnormalised).
constexpr int kTailCand = 512;
__device__ __forceinline__ bool tail_candidate(float2 st, float L) {
  return st.x > 0.0f && (double)st.x + (double)st.y >= (double)L;
}
__device__ __noinline__ double cta_exact_max(const uint16_t* __restrict__ x, const NvWorkspace* ws,
                                             int64_t units, const uint4* smask, int kpr_log2) {
  __shared__ int64_t s_cand[kTailCand];
  __shared__ int s_nc;
  __shared__ double s_m[kQThreads / 32];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float L = __uint_as_float(__ldcg(&ws->lower_bits));
  const int64_t tokens = units >> kpr_log2;
  const int kpr = 1 << kpr_log2;
  if (threadIdx.x == 0) s_nc = 0;
  __syncthreads();
  for (int64_t base = 0; base < tokens; base += 8 * (int64_t)blockDim.x) {
    float2 st[8];
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const int64_t r = base + i * (int64_t)blockDim.x + threadIdx.x;
      st[i] = r < tokens ? __ldcg(&ws->rows[r]) : make_float2(0.0f, 0.0f);
    }
#pragma unroll
    for (int i = 0; i < 8; ++i)
      if (tail_candidate(st[i], L)) {
        const int slot = atomicAdd(&s_nc, 1);
        if (slot < kTailCand) s_cand[slot] = base + i * (int64_t)blockDim.x + threadIdx.x;
      }
  }
  __syncthreads();
  const int nc = s_nc;
  double m = 0.0;
  if (nc <= kTailCand) {
    // (row, block) pairs, four a warp at a time
    const int npairs = nc << kpr_log2;
    for (int p0 = 4 * warp; p0 < npairs; p0 += 4 * nw) {
      const int p = p0 + (lane >> 3);
      const int kb = p & (kpr - 1);
      const int64_t u = p < npairs ? (s_cand[p >> kpr_log2] << kpr_log2) + kb : -1;
      m = fmax(m, warp_blocks_absmax_f64(x, smask, u, kb));
    }
  } else {
    for (int64_t r0 = (int64_t)warp * 32; r0 < tokens; r0 += (int64_t)nw * 32) {
      const int64_t r = r0 + lane;
      const bool c = r < tokens && tail_candidate(__ldcg(&ws->rows[r]), L);
      unsigned todo = __ballot_sync(0xffffffffu, c);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        for (int kb0 = 0; kb0 < kpr; kb0 += 4) {
          const int kb = kb0 + (lane >> 3);
          const int64_t u = kb < kpr ? ((r0 + src) << kpr_log2) + kb : -1;
          m = fmax(m, warp_blocks_absmax_f64(x, smask, u, kb));
        }
      }
    }
  }
  if (lane == 0) s_m[warp] = m;
  __syncthreads();
  double t = s_m[0];
  for (int w = 1; w < nw; ++w) t = fmax(t, s_m[w]);
  return t;
}

// The 64 input bytes of lane qj of block u (zeros past the last block).
template <int kCpl>
__device__ __forceinline__ void load_step(const uint16_t* __restrict__ x, int64_t u, int64_t units,
                                          int qj, uint4 (&w)[kCpl]) {
#pragma unroll
  for (int c = 0; c < kCpl; ++c)
    w[c] = u < units ? __ldg(reinterpret_cast<const uint4*>(x + u * B + qj * (kCpl * 8)) + c)
                     : make_uint4(0, 0, 0, 0);
}

// Inputs of the largest row count whose quantisation pass computes the exact
// maximum itself (every CTA reads all row statistics in its prologue); larger
// inputs run the exact-maximum step as a launch of its own.
constexpr int64_t kFusedExactRows = 8192;

// kMode 0: quantize with the static/dynamic tensor scale.
// kMode 1: dynamic-scale statistics (row max and bound), no outputs.
// Four lanes share a block: each holds 32 consecutive elements, runs five
// butterfly stages in registers and two across its quad, and owns two NVFP4
// blocks of the outputs.  Dynamic quantisation takes t from the workspace's
// exact maximum, or (P.fuse_exact) computes that maximum itself first; it
// waits for the statistics launch (programmatic dependent launch) only after
// the signs are staged and its first inputs are on their way into L2.
template <int kMode, int kLanes>
__global__ void __launch_bounds__(kQThreads, kLanes >= 4 ? 3 : 2)
k_blk128_nvfp4_q(Params P) {
  constexpr int kEpl = B / kLanes;          // elements a lane
  constexpr int kPpl = kEpl / 2;            // f32x2 pairs a lane
  constexpr int kCpl = kEpl / 8;            // 16-byte chunks a lane
  constexpr int kBpl = kEpl / 16;           // NVFP4 blocks a lane
  constexpr int kUpw = 32 / kLanes;         // blocks a warp per step
  const int lane = threadIdx.x & 31, qj = lane & (kLanes - 1);
  extern __shared__ __align__(16) uint4 smem4[];
  uint4* smask = P.signs ? smem4 : nullptr;
  float* rcp = reinterpret_cast<float*>(smem4 + (P.signs ? P.n / 8 : 0));
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  const int64_t ub0 = ((int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5)) * kUpw;
  if (kMode == 1) asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
  // the lane's inputs of the first step are loaded before the prologue (sign
  // table, tensor scale), the next step's at the end of each step
  uint4 w[kCpl];
  load_step(P.x, ub0 + lane / kLanes, P.units, qj, w);
  if (smask) stage_signs(P.signs, P.n, smask);
  if (kMode == 0)
    for (int i = threadIdx.x; i < 128; i += blockDim.x)
      rcp[i] = (i >= 1 && i <= 126) ? e4m3_recip((uint32_t)i) : 0.0f;
  __syncthreads();
  const int kpr = P.n / B;
  const int kpr_log2 = __ffs(kpr) - 1;
  float t = 0.0f, c6 = 0.0f, inv_bt = 0.0f;
  if (kMode == 0) {
    // the statistics launch (if any) is complete past this point
    asm volatile("griddepcontrol.wait;" ::: "memory");
    if (P.ws) {
      const double g = P.fuse_exact ? cta_exact_max(P.x, P.ws, P.units, smask, kpr_log2)
                                    : __longlong_as_double((long long)__ldcg(&P.ws->gmax_bits));
      t = __double2float_rn((g / 11.313708498984761) / 2688.0);
      if (blockIdx.x == 0 && threadIdx.x == 0) {
        *P.tensor_scale = t;
        if (P.fuse_exact) P.ws->gmax_bits = (unsigned long long)__double_as_longlong(g);
      }
    } else {
      t = *P.tensor_scale;
    }
    c6 = (t > 0.0f) ? (float)(1.0 / (11.313708498984761 * 6.0 * (double)t)) : 0.0f;
    inv_bt = (t > 0.0f) ? (float)(1.0 / (11.313708498984761 * (double)t)) : 0.0f;
  }
  // lanes whose blocks share a row in one step (a power of two <= 32)
  const int seg = kLanes * kpr < 32 ? kLanes * kpr : 32;
  float lower = 0.0f;   // statistics: this lane's largest lower bound
  // uniform trip count across the warp
  for (int64_t ub = ub0; ub < P.units; ub += nwarps * kUpw) {
    const int64_t u = ub + lane / kLanes;
    const bool active = u < P.units;
    const int k = (int)(u & (kpr - 1));
    float2 v[kPpl];
#pragma unroll
    for (int c = 0; c < kCpl; ++c) {
      uint32_t ww[4] = {w[c].x, w[c].y, w[c].z, w[c].w};
      if (smask) {
        const uint4 m = smask[k * 16 + ((qj * kCpl + c) ^ (k & 15))];
        ww[0] ^= m.x;
        ww[1] ^= m.y;
        ww[2] ^= m.z;
        ww[3] ^= m.w;
      }
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const float lo = __uint_as_float(ww[q] << 16);
        const float hi = __uint_as_float(ww[q] & 0xffff0000u);
        v[4 * c + q] = make_float2(lo + hi, lo - hi);   // stage on bit 0
      }
    }
    // the next step's inputs: here in the statistics pass (they load during
    // the butterflies), after the stores in the quantisation pass (whose
    // registers are all in use until then)
    if (kMode == 1) load_step(P.x, u + nwarps * kUpw, P.units, qj, w);
#pragma unroll
    for (int h = 1; h < kPpl; h <<= 1)
#pragma unroll
      for (int p = 0; p < kPpl; ++p)
        if (!(p & h)) bfly2(v[p], v[p | h]);
    // the high index bits: across the lane group (the lane with the bit set
    // keeps a - b)
#pragma unroll
    for (int o = 1; o < kLanes; o <<= 1) {
      const float2 sg = (qj & o) ? make_float2(-1.0f, -1.0f) : make_float2(1.0f, 1.0f);
#pragma unroll
      for (int p = 0; p < kPpl; ++p) {
        const float2 pv = make_float2(__shfl_xor_sync(0xffffffffu, v[p].x, o),
                                      __shfl_xor_sync(0xffffffffu, v[p].y, o));
        v[p] = fma2(v[p], sg, pv);
      }
    }
    // the lane's blocks: outputs kEpl qj + 16 j .. +15
    float bm[kBpl];
#pragma unroll
    for (int j = 0; j < kBpl; ++j) {
      float m = 0.0f;
#pragma unroll
      for (int p = 8 * j; p < 8 * j + 8; ++p) m = fmax3(m, fabsf(v[p].x), fabsf(v[p].y));
      bm[j] = m;
    }
    float mh = bm[0];
#pragma unroll
    for (int j = 1; j < kBpl; ++j) mh = fmaxf(mh, bm[j]);
#pragma unroll
    for (int o = 1; o < kLanes; o <<= 1) mh = fmaxf(mh, __shfl_xor_sync(0xffffffffu, mh, o));
    const float E = __fmul_ru(P.e_coef, mh);
    const int64_t row = active ? (u >> kpr_log2) : 0;

    if (kMode == 1) {
      // one atomic pair a row and step (the row's E is e_coef times its
      // maximum, rounded up, like every block's); one lower-bound atomic a warp
      if (active) lower = fmaxf(lower, __fsub_rd(mh, E));
      float rm = mh;
#pragma unroll
      for (int o = kLanes; o < 32; o <<= 1)
        if (o < seg) rm = fmaxf(rm, __shfl_xor_sync(0xffffffffu, rm, o));
      if (active && (lane & (seg - 1)) == 0) {
        atomicMax(reinterpret_cast<unsigned int*>(&P.ws->rows[row].x), __float_as_uint(rm));
        atomicMax(reinterpret_cast<unsigned int*>(&P.ws->rows[row].y),
                  __float_as_uint(__fmul_ru(P.e_coef, rm)));
      }
      continue;
    }
    // E4M3 block scales from [m - E, m + E] (scaled by c6 with a relative
    // margin covering every fp32 rounding on the way)
    uint32_t sc = 0, undecided = 0;
#pragma unroll
    for (int j = 0; j < kBpl; ++j) {
      const float lo = fmaxf(bm[j] - E, 0.0f) * c6 * (1.0f - 0x1p-20f);
      const float hi = (bm[j] + E) * c6 * (1.0f + 0x1p-20f);
      const uint32_t cc = e4m3_pair(lo, hi);
      sc |= (cc & 0xffu) << (8 * j);
      if ((cc & 0xffu) != (cc >> 8)) undecided |= 1u << j;
    }
    if (t <= 0.0f || !active) undecided = 0;
    // warp-cooperative exact fix-up of undecided block scales
    unsigned todo = __ballot_sync(0xffffffffu, undecided != 0);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const uint32_t und = __shfl_sync(0xffffffffu, undecided, src);
      const int64_t usrc = __shfl_sync(0xffffffffu, u, src);
      const int ksrc = __shfl_sync(0xffffffffu, k, src);
#pragma unroll 1
      for (int j = 0; j < kBpl; ++j) {
        if (!((und >> j) & 1u)) continue;
        // candidates: |S_hat| >= bm[j] - 2E inside block j of lane src
        uint32_t cand = 0;
        if (lane == src) {
          float bmj = bm[0];
#pragma unroll
          for (int q = 1; q < kBpl; ++q)
            if (q == j) bmj = bm[q];
          const float thr = bmj - 2.0f * E;
#pragma unroll
          for (int q = 0; q < kBpl; ++q) {
            if (q != j) continue;
#pragma unroll
            for (int p = 0; p < 8; ++p) {
              const float2 a = v[8 * q + p];
              if (fabsf(a.x) >= thr) cand |= 1u << (2 * p);
              if (fabsf(a.y) >= thr) cand |= 1u << (2 * p + 1);
            }
          }
        }
        cand = __shfl_sync(0xffffffffu, cand, src);
        const int e0 = kEpl * (src & (kLanes - 1)) + 16 * j;
        double best = 0.0;
        while (cand) {
          const int e = __ffs(cand) - 1;
          cand &= cand - 1;
          best = fmax(best, fabs(warp_exact_S_global(P.x, smask, usrc, ksrc, e0 + e)));
        }
        const double y = best / 11.313708498984761;
        const float r = __double2float_rn(y / (6.0 * (double)t));
        const uint32_t code = e4m3_pair(r, r) & 0xffu;
        if (lane == src) sc = (sc & ~(0xffu << (8 * j))) | (code << (8 * j));
      }
    }
    // codes: the lane's kEpl outputs are kEpl / 2 bytes
    uint32_t words[2 * kBpl];
    const float2 zero2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int j = 0; j < kBpl; ++j) {
      const uint32_t code = (sc >> (8 * j)) & 0xffu;
      if (code != 0 && t > 0.0f) {
        const float c = inv_bt * rcp[code];
        const float2 c2 = make_float2(c, c);
        float q[16];
#pragma unroll
        for (int p = 0; p < 8; ++p) {
          const float2 a = fma2(v[8 * j + p], c2, zero2);   // + 0 turns -0 into +0
          q[2 * p] = a.x;
          q[2 * p + 1] = a.y;
        }
        words[2 * j] = e2m1x8_hw(q);
        words[2 * j + 1] = e2m1x8_hw(q + 8);
      } else {
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          w0 |= (v[8 * j + p].x < 0.0f ? 8u : 0u) << (8 * p);
          w0 |= (v[8 * j + p].y < 0.0f ? 8u : 0u) << (8 * p + 4);
          w1 |= (v[8 * j + 4 + p].x < 0.0f ? 8u : 0u) << (8 * p);
          w1 |= (v[8 * j + 4 + p].y < 0.0f ? 8u : 0u) << (8 * p + 4);
        }
        words[2 * j] = w0;
        words[2 * j + 1] = w1;
      }
    }
    if (active) {
      uint8_t* cdst = P.codes + u * (B / 2) + qj * (kEpl / 2);
#pragma unroll
      for (int h = 0; h < kBpl / 2; ++h)
        reinterpret_cast<uint4*>(cdst)[h] =
            make_uint4(words[4 * h], words[4 * h + 1], words[4 * h + 2], words[4 * h + 3]);
      if (kBpl == 1) *reinterpret_cast<uint2*>(cdst) = make_uint2(words[0], words[1]);
      // the lane's blocks start at an index that is a multiple of kBpl: they are
      // consecutive bytes in either layout
      const int c0 = k * (B / 16) + kBpl * qj;
      const int64_t off = P.sf_kc4 == 0 ? u * (B / 16) + kBpl * qj
                                        : sf_offset(row, c0, P.n / 16, P.sf_kc4);
      if (kBpl == 4)
        *reinterpret_cast<uint32_t*>(P.scales8 + off) = sc;
      else if (kBpl == 2)
        *reinterpret_cast<uint16_t*>(P.scales8 + off) = (uint16_t)sc;
      else
        P.scales8[off] = (uint8_t)sc;
    }
    load_step(P.x, u + nwarps * kUpw, P.units, qj, w);
  }
  if (kMode == 1) {
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) lower = fmaxf(lower, __shfl_xor_sync(0xffffffffu, lower, o));
    if (lane == 0 && lower > 0.0f) atomicMax(&P.ws->lower_bits, __float_as_uint(lower));
  }
}

// ------------------------------------------------------- INT4 asym, g128
__device__ __forceinline__ uint32_t f16x2_pair(float lo, float hi) {
  uint32_t out;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(out) : "f"(hi), "f"(lo));
  return out;   // bits 0-15: fp16(lo), bits 16-31: fp16(hi)
}

__global__ void __launch_bounds__(kThreads, 3)
k_blk128_asym(Params P) {
  const int lane = threadIdx.x & 31;
  const float k15 = (float)(1.0 / (15.0 * 11.313708498984761));
  extern __shared__ __align__(16) uint4 smem4[];
  uint4* stages = smem4 + (threadIdx.x >> 5) * 1024;
  uint4* smask = P.signs ? smem4 + (blockDim.x >> 5) * 1024 : nullptr;
  if (smask) stage_signs(P.signs, P.n, smask);
  __syncthreads();
  const int kpr = P.n / B;
  const int64_t stride = (int64_t)gridDim.x * blockDim.x;
  const int64_t base0 = (int64_t)blockIdx.x * blockDim.x + (threadIdx.x & ~31);
  if (base0 < P.units) prefetch_units(P.x, base0, P.units, stages);
  int it = 0;
  for (int64_t ub = base0; ub < P.units; ub += stride, ++it) {
    const int64_t u = ub + lane;
    const bool active = u < P.units;
    float2 v[64];
    uint4* stage = stages + (it & 1) * 512;
    __syncwarp();
    const bool more = ub + stride < P.units;
    if (more) prefetch_units(P.x, ub + stride, P.units, stages + ((it + 1) & 1) * 512);
    wait_prefetch(more);
    load_transform(stage, lane, smask, (int)(u & (kpr - 1)), v);
    if (!active) {
#pragma unroll
      for (int p = 0; p < 64; ++p) v[p] = make_float2(0.f, 0.f);
    }
    float mx = -FLT_MAX, mn = FLT_MAX;
#pragma unroll
    for (int p = 0; p < 64; ++p) {
      mx = fmax3(mx, v[p].x, v[p].y);
      mn = fmin3(mn, v[p].x, v[p].y);
    }
    const float E = __fmul_ru(P.e_coef, fmaxf(fabsf(mx), fabsf(mn)));
    // scale16 = fp16((mx - mn) / (15 sqrt(b))) over the interval of (mx, mn)
    const float r_lo = fmaxf(mx - mn - 2.0f * E, 0.0f) * k15 * (1.0f - 0x1p-20f);
    const float r_hi = (mx - mn + 2.0f * E) * k15 * (1.0f + 0x1p-20f);
    const uint32_t hh = f16x2_pair(r_lo, r_hi);
    uint32_t s16 = hh & 0xffffu;
    bool decided = s16 == (hh >> 16);
    float zf = 0.0f;
    if (decided && s16 != 0) {
      // z = rint(-mn / (sqrt(b) s16)) over the interval of mn
      const float inv = 1.0f / (11.313708498984761f * f16_bits_to_f32((uint16_t)s16));
      const float z_hi = rintf(-(mn - E) * inv * (1.0f + 0x1p-20f * (mn - E < 0 ? 1.f : -1.f)));
      const float z_lo = rintf(-(mn + E) * inv * (1.0f - 0x1p-20f * (mn + E < 0 ? 1.f : -1.f)));
      decided = z_hi == z_lo;
      zf = z_lo;
    }
    // warp-cooperative exact extremes for undecided groups
    unsigned todo = __ballot_sync(0xffffffffu, active && !decided);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const int kk = (int)((ub + src) & (kpr - 1));
      uint32_t cmax[4] = {0, 0, 0, 0}, cmin[4] = {0, 0, 0, 0};
      if (lane == src) {
        const float th = mx - 2.0f * E, tl = mn + 2.0f * E;
#pragma unroll
        for (int p = 0; p < 64; ++p) {
          if (v[p].x >= th) cmax[p >> 4] |= 1u << (2 * (p & 15));
          if (v[p].y >= th) cmax[p >> 4] |= 1u << (2 * (p & 15) + 1);
          if (v[p].x <= tl) cmin[p >> 4] |= 1u << (2 * (p & 15));
          if (v[p].y <= tl) cmin[p >> 4] |= 1u << (2 * (p & 15) + 1);
        }
      }
      double smax = -DBL_MAX, smin = DBL_MAX;
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        uint32_t a = __shfl_sync(0xffffffffu, cmax[w], src);
        uint32_t b = __shfl_sync(0xffffffffu, cmin[w], src);
        uint32_t any = a | b;
        while (any) {
          const int e = __ffs(any) - 1;
          any &= any - 1;
          const double s = warp_exact_S(stage, smask, src, kk, 32 * w + e);
          if ((a >> e) & 1u) smax = fmax(smax, s);
          if ((b >> e) & 1u) smin = fmin(smin, s);
        }
      }
      if (lane == src) {
        const double ymx = smax / 11.313708498984761, ymn = smin / 11.313708498984761;
        s16 = f64_to_f16_bits((ymx - ymn) / 15.0);
        const double sd = f16_bits_to_f64((uint16_t)s16);
        zf = sd > 0.0 ? (float)rint(-ymn / sd) : 0.0f;
        decided = true;
      }
    }
    // codes, 16 bytes (32 elements) at a time, straight to global memory
    const float c = (s16 != 0) ? 1.0f / (11.313708498984761f * f16_bits_to_f32((uint16_t)s16))
                               : 0.0f;
    if (s16 == 0) zf = 0.0f;
    const float2 c2 = make_float2(c, c);
    // (S c) + (1.5 2^23 + z) rounds S c + z to an integer in the low bits
    const float magic = 12582912.0f + zf;
    const float2 m2 = make_float2(magic, magic);
    const int64_t ou = active ? kv_unit(P.slots, P.num_slots, kpr, u) : -1;
    uint4* dst = reinterpret_cast<uint4*>(P.codes + ou * (B / 2));
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      uint32_t words[4];
#pragma unroll
      for (int w = 0; w < 4; ++w) {
        int q[8];
#pragma unroll
        for (int p = 0; p < 4; ++p) {
          const float2 a = fma2(v[16 * k + 4 * w + p], c2, m2);
          q[2 * p] = __float_as_int(a.x) - 0x4B400000;
          q[2 * p + 1] = __float_as_int(a.y) - 0x4B400000;
        }
        words[w] = pack_u4x8(q);
      }
      if (ou >= 0) dst[k] = make_uint4(words[0], words[1], words[2], words[3]);
    }
    if (ou >= 0) {
      uint16_t zh;
      asm("cvt.rn.f16.f32 %0, %1;" : "=h"(zh) : "f"(zf));
      P.scales16[ou] = (uint16_t)s16;
      P.zeros16[ou] = zh;
    }
  }
}

}  // namespace blk

// ------------------------------------------------------------- launchers
namespace {
size_t blk_smem(int n, bool signs) {
  return (size_t)(blk::kThreads / 32) * 1024 * 16 + (signs ? (size_t)n / 8 * 16 : 0) + 128 * 4;
}

int blk_grid(const void* kernel, int64_t units, size_t smem) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, blk::kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t need = (units + blk::kThreads - 1) / blk::kThreads;
  const int64_t cap = (int64_t)sms * per_sm;
  return (int)(need < cap ? need : cap);
}

float e_coef_128() {
  const double u = 0x1p-24, L = 7.0;
  const double gam = L * u / (1.0 - L * u);
  const double c = gam * std::sqrt(128.0);
  return (float)((c / (1.0 - c)) * 1.001);
}
}  // namespace

bool blk128_supported(const Geometry& g, int dtype) {
  const int kpr = g.n / 128;
  return dtype == 1 && g.b == 128 && !g.paley && g.n % 128 == 0 && (kpr & (kpr - 1)) == 0;
}

int qblk_grid(const void* kernel, int64_t units, size_t smem, int lanes) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, blk::kQThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t per_cta = (blk::kQThreads / 32) * (32 / lanes);   // blocks per step
  const int64_t need = (units + per_cta - 1) / per_cta;
  const int64_t cap = (int64_t)sms * per_sm;
  return (int)(need < cap ? need : cap);
}

cudaError_t launch_blk128_nvfp4(const void* x, int64_t tokens, const Geometry& g,
                                const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                                float* tensor_scale, NvWorkspace* ws, cudaStream_t s) {
  blk::Params P{};
  P.x = static_cast<const uint16_t*>(x);
  P.signs = signs;
  P.codes = codes;
  P.scales8 = bscales;
  P.tensor_scale = tensor_scale;
  P.ws = ws;
  P.units = tokens * (g.n / blk::B);
  P.n = g.n;
  P.e_coef = e_coef_128();
  P.sf_kc4 = g.sf_kc4;
  const size_t smq = (signs ? (size_t)g.n / 8 * 16 : 0) + 128 * 4;
  auto k0 = blk::k_blk128_nvfp4_q<0, blk::kQLanes>;
  const int grid0 = qblk_grid((const void*)k0, P.units, smq, blk::kQLanes);
  if (!ws) {
    k0<<<grid0, blk::kQThreads, smq, s>>>(P);
    return cudaGetLastError();
  }
  const int ph = g.dyn ? g.dyn : 7;
  // the whole dynamic call on a modest row count: statistics, then the
  // quantisation pass computing the exact maximum itself, launched as a
  // programmatic dependent of the statistics (it reads only the input before
  // waiting for them)
  const bool fused = ph == 7 && tokens <= blk::kFusedExactRows;
  if (ph & 1) {
    cudaError_t e =
        cudaMemsetAsync(ws, 0, kNvWorkspaceHeader + (size_t)tokens * sizeof(float2), s);
    if (e != cudaSuccess) return e;
    auto k1 = blk::k_blk128_nvfp4_q<1, blk::kQLanesStats>;
    k1<<<qblk_grid((const void*)k1, P.units, smq, blk::kQLanesStats), blk::kQThreads, smq, s>>>(P);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  if ((ph & 2) && !fused) {
    cudaError_t e = launch_nvfp4_global(x, 1, tokens, g, signs, ws, s);
    if (e != cudaSuccess) return e;
  }
  if (!(ph & 4)) return cudaSuccess;
  if (!fused) {
    k0<<<grid0, blk::kQThreads, smq, s>>>(P);
    return cudaGetLastError();
  }
  P.fuse_exact = 1;
  auto kf = blk::k_blk128_nvfp4_q<0, blk::kQLanesStats>;
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = dim3((unsigned)qblk_grid((const void*)kf, P.units, smq, blk::kQLanesStats));
  cfg.blockDim = dim3(blk::kQThreads);
  cfg.dynamicSmemBytes = smq;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kf, P);
}

cudaError_t launch_blk128_asym(const void* x, int64_t tokens, const Geometry& g,
                               const int8_t* signs, uint8_t* codes, uint16_t* scales,
                               uint16_t* zeros, const int64_t* slots, int64_t num_slots,
                               cudaStream_t s) {
  blk::Params P{};
  P.x = static_cast<const uint16_t*>(x);
  P.signs = signs;
  P.codes = codes;
  P.scales16 = scales;
  P.zeros16 = zeros;
  P.slots = slots;
  P.num_slots = num_slots;
  P.units = tokens * (g.n / blk::B);
  P.n = g.n;
  P.e_coef = e_coef_128();
  auto k = blk::k_blk128_asym;
  const size_t sm = blk_smem(g.n, signs != nullptr);
  k<<<blk_grid((const void*)k, P.units, sm), blk::kThreads, sm, s>>>(P);
  return cudaGetLastError();
}

}  // namespace kq
