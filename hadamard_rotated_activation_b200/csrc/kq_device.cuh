// Device-side helpers shared by the kq kernels (sm_100a).
//
// Hadamard factors:
//   * Sylvester, natural order: H[i][j] = (-1)^popcount(i & j) -- the matrix the
//     in-place fast Walsh-Hadamard butterfly produces (QuaRot reviews, review 1
//     Summary: the online Hadamard runs with the Walsh-Hadamard algorithm).
//   * Paley-12 for 12 * 2^k rows ("Bug: Qwen3-8B integration issue", Model
//     Details: 12288 = 12 x 1024 is Hadamard-compatible): Paley construction I
//     with q = 11, built here at compile time from the quadratic-residue rule.
//
// Number formats, written from their public definitions:
//   * E4M3 (OCP OFP8): bias 7, max 448, subnormal step 2^-9, no Inf.
//   * E2M1 (OCP MX FP4): values 0, .5, 1, 1.5, 2, 3, 4, 6.
#pragma once

#include <cstdint>
#include <cuda_runtime.h>

namespace kq {

// ----------------------------------------------------------------- Paley-12
__host__ __device__ constexpr int quadratic_residue_mask11() {
  int m = 0;
  for (int k = 1; k < 11; ++k) m |= 1 << ((k * k) % 11);
  return m;
}

// Legendre symbol chi(d) mod 11 (0 for d == 0).
__host__ __device__ constexpr int paley_chi(int d) {
  d %= 11;
  if (d < 0) d += 11;
  return d == 0 ? 0 : (((quadratic_residue_mask11() >> d) & 1) ? 1 : -1);
}

// Entry (a, c) of H12 = I + S, S = [[0, 1^T], [-1, Q]], Q[i][j] = chi(j - i).
__host__ __device__ constexpr int paley12_entry(int a, int c) {
  int s = 0;
  if (a == 0 && c == 0)
    s = 0;
  else if (a == 0)
    s = 1;
  else if (c == 0)
    s = -1;
  else
    s = paley_chi((c - 1) - (a - 1));
  return (a == c ? 1 : 0) + s;
}

// 12 x 12 sign bits: bit (a * 12 + c) set <=> H12[a][c] == -1.
struct PaleyBits {
  uint32_t w[5];
};
__host__ __device__ constexpr PaleyBits paley12_bits() {
  PaleyBits p{{0, 0, 0, 0, 0}};
  for (int a = 0; a < 12; ++a)
    for (int c = 0; c < 12; ++c)
      if (paley12_entry(a, c) < 0) {
        int k = a * 12 + c;
        p.w[k >> 5] |= 1u << (k & 31);
      }
  return p;
}

__device__ __forceinline__ bool paley_negative(int a, int c) {
  constexpr PaleyBits p = paley12_bits();
  const int k = a * 12 + c;
  const uint32_t w = k < 32 ? p.w[0] : k < 64 ? p.w[1] : k < 96 ? p.w[2]
                   : k < 128 ? p.w[3] : p.w[4];
  return (w >> (k & 31)) & 1u;
}

// a / b correctly rounded for finite a and a constant b, from rb = RN(1 / b):
// q0 = RN(a rb) is within an ulp, its residual a - q0 b is exact under an
// FMA, and one correction step gives the rounded quotient (Markstein's
// theorem for fused multiply-add); a short dependent chain instead of a
// division routine.
__device__ __forceinline__ double div_rn(double a, double b, double rb) {
  const double q0 = a * rb;
  return fma(fma(-q0, b, a), rb, q0);
}

// ------------------------------------------------------------ KV-cache rows
// Output unit of input unit u (kpr units of 128 per row) when rows go to the
// cache rows a slot mapping names: slot[u / kpr] * kpr + u % kpr, or -1 when
// the row's slot is negative (padding) or not below num_slots; u itself
// without a mapping.
__device__ __forceinline__ int64_t kv_unit(const int64_t* slots, int64_t num_slots, int kpr,
                                           int64_t u) {
  if (!slots) return u;
  const int64_t t = u / kpr;
  const int64_t sl = __ldg(slots + t);
  return (sl >= 0 && sl < num_slots) ? sl * kpr + (u - t * kpr) : -1;
}

// ------------------------------------------------------------ transform spec
struct Geometry {
  int n;          // row length (dim)
  int b;          // Hadamard block width (n when the whole row is one block)
  int m;          // Sylvester factor width: b, or b / 12 with the Paley factor
  int paley;      // 1 when b = 12 m
  int depth;      // roundings along any input -> output path of the fp32 transform
  float inv_sqrt_b;
  double sqrt_b;
  int sf_kc4;     // NVFP4 block scales: 0 = row-major [T, n/16]; else the tensor-core
                  // scale-factor layout with sf_kc4 = n/64 atoms per 128-row block
  int dyn;        // dynamic NVFP4 phases to run (bit 0 statistics, 1 exact maximum,
                  // 2 quantization); 0 = all three
};

// Byte offset of the NVFP4 block scale of 16-block c in row `row` (nb blocks a
// row).  Row-major when kc4 == 0.  Otherwise the layout a tcgen05 block-scaled
// MMA takes from tensor memory: 512-byte atoms of 128 rows x 4 blocks, lane
// row % 32 holding 16 bytes, byte 4 ((row / 32) % 4) + c % 4; atoms ordered by
// c / 4 within a 128-row block, then by row block.  Four blocks 4j .. 4j+3 of
// a row are one aligned 32-bit word in both layouts.
__device__ __forceinline__ int64_t sf_offset(int64_t row, int c, int nb, int kc4) {
  if (kc4 == 0) return row * nb + c;
  return (((row >> 7) * kc4 + (c >> 2)) << 9) + ((row & 31) << 4) + (((row >> 5) & 3) << 2) +
         (c & 3);
}

// Rigorous bound on |S_hat - S| for every output of one Hadamard block, from
// the computed maximum |S_hat| of that block (or any larger value).
//   |S_hat_i - S_i| <= gamma_L * sum_j |x_j|,   gamma_L = L u / (1 - L u)
//   sum_j |x_j| <= sqrt(b) ||x||_2 = ||S||_2 <= sqrt(b) max|S| <= sqrt(b)(M + E)
// so E <= gamma_L sqrt(b) M / (1 - gamma_L sqrt(b)).  A tiny absolute term
// covers subnormal intermediates.
__device__ __forceinline__ double error_bound(const Geometry& g, float m_hat) {
  const double u = 0x1p-24;
  const double L = g.depth;
  const double gam = L * u / (1.0 - L * u);
  const double c = gam * g.sqrt_b;
  return (c * (double)m_hat / (1.0 - c)) * 1.0001 + 1e-36;
}

// ----------------------------------------------------------- E4M3 (scales)
// Round a non-negative fp32 value to E4M3, nearest-even, saturating at 448.
__device__ __forceinline__ uint32_t e4m3_encode_rne_sat(float r) {
  if (!(r > 0.0f)) return 0u;
  if (r >= 448.0f) return 0x7Eu;
  if (r < 0x1p-6f) {
    // subnormal range: value = q * 2^-9, q = 0..8 (q = 8 is the min normal)
    const float q = rintf(r * 512.0f);
    return (uint32_t)q;
  }
  int e;
  const float fr = frexpf(r, &e);      // r = fr * 2^e, fr in [0.5, 1)
  const float mant = fr * 2.0f;        // [1, 2), exponent e - 1
  int ex = e - 1;
  int q = (int)rintf((mant - 1.0f) * 8.0f);   // exact scaling, RNE
  if (q == 8) { q = 0; ++ex; }
  uint32_t code = (uint32_t)((ex + 7) << 3) | (uint32_t)q;
  return code > 0x7Eu ? 0x7Eu : code;
}

__device__ __forceinline__ float e4m3_decode(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  float v = (e == 0) ? (float)m * 0x1p-9f : ldexpf(1.0f + (float)m * 0.125f, (int)e - 7);
  return (c & 0x80u) ? -v : v;
}

// E2M1 value of a 4-bit code.
__device__ __forceinline__ float e2m1_decode(uint32_t c) {
  const uint32_t i = c & 7u;
  const float mag = (i < 2) ? 0.5f * (float)i
                  : ldexpf(1.0f + 0.5f * (float)(i & 1u), (int)(i >> 1) - 1);
  return (c & 8u) ? -mag : mag;
}

// Eight fp32 values -> 32 bits of E2M1 codes (element k in bits 4k..4k+3),
// nearest-even, saturating at +-6, with the sm_100a conversion instruction.
// The instruction writes its first source operand to the upper nibble.
__device__ __forceinline__ uint32_t e2m1x8_hw(const float* v) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(v[0]), "f"(v[1]), "f"(v[2]), "f"(v[3]),
        "f"(v[4]), "f"(v[5]), "f"(v[6]), "f"(v[7]));
  return out;
}

// ----------------------------------------------------------------- fp16
__device__ __forceinline__ uint16_t f64_to_f16_bits(double v) {
  uint16_t h;
  asm("cvt.rn.f16.f64 %0, %1;" : "=h"(h) : "d"(v));
  return h;
}
__device__ __forceinline__ double f16_bits_to_f64(uint16_t h) {
  double d;
  asm("cvt.f64.f16 %0, %1;" : "=d"(d) : "h"(h));
  return d;
}
__device__ __forceinline__ float f16_bits_to_f32(uint16_t h) {
  float f;
  asm("cvt.f32.f16 %0, %1;" : "=f"(f) : "h"(h));
  return f;
}

// ------------------------------------------------------------ reductions
// All reductions use a fixed order (xor-shuffle tree, then warp 0 in order),
// so results are reproducible run to run.
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ float warp_min(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fminf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
__device__ __forceinline__ int warp_min_i(int v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = min(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}
// Exact fp64 images of the two bf16 values packed in `w` (low half first),
// scaled by 2^-896: the bf16 bit pattern is placed in the high word of a
// double so that its 8-bit exponent field becomes the double's (biased 1023
// instead of 127).  Zeros and bf16 subnormals land on double zeros and
// subnormals with the same 2^-896 factor, so the mapping is exact for every
// finite bf16; infinities and NaNs are NOT preserved (callers route non-finite
// rows elsewhere).  Three integer operations per value, no conversion unit.
__device__ __forceinline__ void bf16x2_to_f64_scaled(uint32_t w, double& lo, double& hi) {
  const uint32_t flo = w << 16, fhi = w & 0xffff0000u;     // the fp32 images
  const uint32_t hlo = (flo & 0x80000000u) | ((flo >> 3) & 0x0fffffffu);
  const uint32_t hhi = (fhi & 0x80000000u) | ((fhi >> 3) & 0x0fffffffu);
  lo = __hiloint2double((int)hlo, 0);
  hi = __hiloint2double((int)hhi, 0);
}
// Undoes the 2^-896 scaling of bf16x2_to_f64_scaled (exact).
constexpr double kF64Unscale = 0x1p+896;

__device__ __forceinline__ double warp_sum_d(double v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

// Block-wide reductions; `red` is shared scratch of >= 33 doubles.  Every
// thread of the block must call them; all threads get the result.
__device__ __forceinline__ float block_max(float v, double* red) {
  float* r = reinterpret_cast<float*>(red);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_max(v);
  __syncthreads();
  if (lane == 0) r[wid] = v;
  __syncthreads();
  float t = r[0];
  for (int i = 1; i < nw; ++i) t = fmaxf(t, r[i]);
  return t;
}
__device__ __forceinline__ int block_min_i(int v, double* red) {
  int* r = reinterpret_cast<int*>(red);
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_min_i(v);
  __syncthreads();
  if (lane == 0) r[wid] = v;
  __syncthreads();
  int t = r[0];
  for (int i = 1; i < nw; ++i) t = min(t, r[i]);
  return t;
}
__device__ __forceinline__ double block_sum_d(double v, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
  v = warp_sum_d(v);
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  double t = red[0];
  for (int i = 1; i < nw; ++i) t += red[i];
  return t;
}

// ------------------------------------------------------------ input access
__device__ __forceinline__ double load_x_f64(const float* x, int j) { return (double)x[j]; }
__device__ __forceinline__ double load_x_f64(const uint16_t* x, int j) {
  return (double)__uint_as_float((uint32_t)x[j] << 16);
}

}  // namespace kq
