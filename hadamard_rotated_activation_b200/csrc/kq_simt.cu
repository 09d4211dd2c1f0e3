// Row-per-CTA kernels: randomized Hadamard transform + 4-bit quantizers.
//
// One CTA owns one activation row at a time (grid-stride over rows).  The row
// is loaded with 16-byte vector loads, the sign vector D is applied, and the
// unnormalised transform S = (x . D) . H^T runs in shared memory as radix-8
// butterfly passes (Sylvester factor) plus, for 12 * 2^k rows, one dense pass
// of the Paley-12 factor across the 12 segments.  This is the general path:
// every shape, both input types, every output format.
//
// Exact scales.  The fp32 transform is within a rigorous bound E of the exact
// sums (error_bound in kq_device.cuh).  Each scale depends on a maximum (or a
// minimum) through a monotone rounding chain, so it is decided by the fp32
// values whenever both ends of the interval [M - E, M + E] round to the same
// scale.  Otherwise every element that can be the extremum (|S_hat| within 2E
// of it) is recomputed exactly as an fp64 dot product with the input row, and
// the scale follows the fp64 formula.  Codes come from the fp32 values with the
// exact scales.
//
// Sources: QuaRot reviews (RHT on activations, Walsh-Hadamard algorithm,
// Y = X H^T, INT4 RTN), "Bug: Qwen3-8B integration issue" (12288 = 12 x 1024),
// NVFP4 thread (block-Hadamard-128, NVFP4 4.50 bits).
#include <cfloat>
#include <climits>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {

constexpr int kThreads = 256;

// ------------------------------------------------------------- row loading
// buf[j] = s_j * x_j as fp32 or fp64 (exact for bf16 and fp32 inputs), in
// 16-byte chunks so that every thread has few loads in flight in sequence.
template <typename F>
__device__ __forceinline__ void load_row(const uint16_t* __restrict__ xr,
                                         const int8_t* __restrict__ signs,
                                         F* buf, int n) {
  const uint4* xv = reinterpret_cast<const uint4*>(xr);
#pragma unroll 2
  for (int c = threadIdx.x; c < n / 8; c += blockDim.x) {
    const uint4 w = __ldg(xv + c);
    uint32_t s0 = 0, s1 = 0;
    if (signs) {
      const uint2 sv = __ldg(reinterpret_cast<const uint2*>(signs) + c);
      s0 = sv.x;
      s1 = sv.y;
    }
    const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t sw = k < 2 ? s0 : s1;
      const uint32_t sb0 = (sw >> (16 * (k & 1) + 7)) & 1u;   // sign byte 2k
      const uint32_t sb1 = (sw >> (16 * (k & 1) + 15)) & 1u;  // sign byte 2k+1
      const uint32_t lo = (ww[k] << 16) ^ (sb0 << 31);
      const uint32_t hi = (ww[k] & 0xffff0000u) ^ (sb1 << 31);
      buf[8 * c + 2 * k] = __uint_as_float(lo);
      buf[8 * c + 2 * k + 1] = __uint_as_float(hi);
    }
  }
}

template <typename F>
__device__ __forceinline__ void load_row(const float* __restrict__ xr,
                                         const int8_t* __restrict__ signs,
                                         F* buf, int n) {
  const float4* xv = reinterpret_cast<const float4*>(xr);
#pragma unroll 4
  for (int c = threadIdx.x; c < n / 4; c += blockDim.x) {
    float4 v = __ldg(xv + c);
    if (signs) {
      const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(signs) + c);
      v.x = __uint_as_float(__float_as_uint(v.x) ^ (((sw >> 7) & 1u) << 31));
      v.y = __uint_as_float(__float_as_uint(v.y) ^ (((sw >> 15) & 1u) << 31));
      v.z = __uint_as_float(__float_as_uint(v.z) ^ (((sw >> 23) & 1u) << 31));
      v.w = __uint_as_float(__float_as_uint(v.w) ^ (((sw >> 31) & 1u) << 31));
    }
    if constexpr (sizeof(F) == 4) {
      reinterpret_cast<float4*>(buf)[c] = v;
    } else {
      buf[4 * c] = v.x;
      buf[4 * c + 1] = v.y;
      buf[4 * c + 2] = v.z;
      buf[4 * c + 3] = v.w;
    }
  }
}

// -------------------------------------------------------- butterfly passes
// One radix-R pass over strides h, 2h, ..., (R/2)h inside every m-segment.
template <int R, typename F>
__device__ __forceinline__ void fwht_pass(F* buf, int n, int h) {
  const int groups = n / R;
  for (int gi = threadIdx.x; gi < groups; gi += blockDim.x) {
    const int lo = gi % h, hi = gi / h;
    const int base = hi * h * R + lo;
    F v[R];
#pragma unroll
    for (int k = 0; k < R; ++k) v[k] = buf[base + k * h];
#pragma unroll
    for (int s = 1; s < R; s <<= 1)
#pragma unroll
      for (int k = 0; k < R; ++k)
        if (!(k & s)) {
          const F a = v[k], b = v[k | s];
          v[k] = a + b;
          v[k | s] = a - b;
        }
#pragma unroll
    for (int k = 0; k < R; ++k) buf[base + k * h] = v[k];
  }
  __syncthreads();
}

// Unnormalised Sylvester transform of every m-segment of buf (m | n), in
// fp32 or fp64; h0 > 1 skips the strides below h0 (already applied).
template <typename F>
__device__ void fwht_smem(F* buf, int n, int m, int h0 = 1) {
  int h = h0;
  while (h < m) {
    const int left = m / h;
    if (left >= 8) {
      fwht_pass<8>(buf, n, h);
      h *= 8;
    } else if (left >= 4) {
      fwht_pass<4>(buf, n, h);
      h *= 4;
    } else {
      fwht_pass<2>(buf, n, h);
      h *= 2;
    }
  }
}

// Paley-12 factor across the 12 segments of width m:
// z[a m + beta] = sum_c P[a][c] w[c m + beta] (P = H12, or H12^T when
// kTranspose), summed in the order c = 0..11.
template <bool kTranspose, typename F>
__device__ void paley_smem(F* buf, int m) {
  for (int beta = threadIdx.x; beta < m; beta += blockDim.x) {
    F w[12], z[12];
#pragma unroll
    for (int c = 0; c < 12; ++c) w[c] = buf[c * m + beta];
#pragma unroll
    for (int a = 0; a < 12; ++a) {
      F acc = (kTranspose ? paley_negative(0, a) : paley_negative(a, 0)) ? -w[0] : w[0];
#pragma unroll
      for (int c = 1; c < 12; ++c) {
        const bool neg = kTranspose ? paley_negative(c, a) : paley_negative(a, c);
        acc = neg ? acc - w[c] : acc + w[c];
      }
      z[a] = acc;
    }
#pragma unroll
    for (int a = 0; a < 12; ++a) buf[a * m + beta] = z[a];
  }
  __syncthreads();
}

template <typename T>
__device__ __forceinline__ void transform_row(const T* xr, const int8_t* signs,
                                              float* buf, const Geometry& g,
                                              bool transpose) {
  load_row(xr, signs, buf, g.n);
  __syncthreads();
  fwht_smem(buf, g.n, g.m);
  if (g.paley) {
    if (transpose)
      paley_smem<true>(buf, g.m);
    else
      paley_smem<false>(buf, g.m);
  }
}

// --------------------------------------------------------- exact fix-up
// Exact S_i = sum_j H_b[i_loc][j] s_j x_j (fp64, fixed order), block-wide.
template <typename T>
__device__ double exact_S(const T* __restrict__ xr, const int8_t* __restrict__ signs,
                          const Geometry& g, int i, double* red) {
  const int blk = i / g.b;
  const int off = blk * g.b;
  const int il = i - off;
  const int ia = g.paley ? il / g.m : 0;
  const int ib = g.paley ? il - ia * g.m : il;
  double acc = 0.0;
#pragma unroll 4
  for (int j = threadIdx.x; j < g.b; j += blockDim.x) {
    int ja = 0, jb = j;
    if (g.paley) {
      ja = j / g.m;
      jb = j - ja * g.m;
    }
    bool neg = (__popc(ib & jb) & 1) != 0;
    if (g.paley) neg ^= paley_negative(ia, ja);
    if (signs && signs[off + j] < 0) neg = !neg;
    const double xv = load_x_f64(xr, off + j);
    acc += neg ? -xv : xv;
  }
  return block_sum_d(acc, red);
}

// Next index > prev whose |buf| >= thr (INT_MAX if none), block-wide.
__device__ __forceinline__ int next_candidate(const float* buf, int lo, int hi,
                                              int prev, float thr, double* red) {
  int best = INT_MAX;
  for (int i = lo + threadIdx.x; i < hi; i += blockDim.x)
    if (i > prev && fabsf(buf[i]) >= thr) {
      best = i;
      break;
    }
  return block_min_i(best, red);
}

// Exact max |S| over candidates in buf[lo, hi) with |S_hat| >= thr.
template <typename T>
__device__ double exact_max_abs(const T* xr, const int8_t* signs, const Geometry& g,
                                const float* buf, int lo, int hi, float thr,
                                double* red) {
  double best = 0.0;
  int prev = lo - 1;
  for (;;) {
    const int c = next_candidate(buf, lo, hi, prev, thr, red);
    if (c == INT_MAX) break;
    best = fmax(best, fabs(exact_S(xr, signs, g, c, red)));
    prev = c;
  }
  return best;
}

// exact_S from a shared-memory copy xs of the sign-flipped row (fp32 holds
// every bf16 or fp32 input exactly): the same terms in the same order.
__device__ double exact_S_smem(const float* xs, const Geometry& g, int i, double* red) {
  const int blk = i / g.b;
  const int off = blk * g.b;
  const int il = i - off;
  const int ia = g.paley ? il / g.m : 0;
  const int ib = g.paley ? il - ia * g.m : il;
  double acc = 0.0;
  for (int j = threadIdx.x; j < g.b; j += blockDim.x) {
    int ja = 0, jb = j;
    if (g.paley) {
      ja = j / g.m;
      jb = j - ja * g.m;
    }
    bool neg = (__popc(ib & jb) & 1) != 0;
    if (g.paley) neg ^= paley_negative(ia, ja);
    const double xv = (double)xs[off + j];
    acc += neg ? -xv : xv;
  }
  return block_sum_d(acc, red);
}

__device__ double exact_max_abs_smem(const float* xs, const Geometry& g, const float* buf,
                                     int lo, int hi, float thr, double* red) {
  double best = 0.0;
  int prev = lo - 1;
  for (;;) {
    const int c = next_candidate(buf, lo, hi, prev, thr, red);
    if (c == INT_MAX) break;
    best = fmax(best, fabs(exact_S_smem(xs, g, c, red)));
    prev = c;
  }
  return best;
}

__device__ __forceinline__ float thr_down(double v) {
  return v > 0.0 ? __double2float_rd(v) : 0.0f;
}

// Row max of |buf| (block-wide).
__device__ __forceinline__ float row_absmax(const float* buf, int n, double* red) {
  float m = 0.0f;
  for (int i = threadIdx.x; i < n; i += blockDim.x) m = fmaxf(m, fabsf(buf[i]));
  return block_max(m, red);
}

// ============================================================== kq_rht
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_rht(const T* __restrict__ x, const int8_t* __restrict__ signs, float* __restrict__ out,
      int64_t tokens, Geometry g, int inverse) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const T* xr = x + row * g.n;
    transform_row(xr, inverse ? nullptr : signs, buf, g, inverse != 0);
    float* orow = out + row * g.n;
    for (int c = threadIdx.x; c < g.n / 4; c += blockDim.x) {
      float4 v = reinterpret_cast<const float4*>(buf)[c];
      v.x *= g.inv_sqrt_b;
      v.y *= g.inv_sqrt_b;
      v.z *= g.inv_sqrt_b;
      v.w *= g.inv_sqrt_b;
      if (inverse && signs) {
        const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(signs) + c);
        v.x = __uint_as_float(__float_as_uint(v.x) ^ (((sw >> 7) & 1u) << 31));
        v.y = __uint_as_float(__float_as_uint(v.y) ^ (((sw >> 15) & 1u) << 31));
        v.z = __uint_as_float(__float_as_uint(v.z) ^ (((sw >> 23) & 1u) << 31));
        v.w = __uint_as_float(__float_as_uint(v.w) ^ (((sw >> 31) & 1u) << 31));
      }
      reinterpret_cast<float4*>(orow)[c] = v;
    }
    __syncthreads();
  }
}

// ======================================================= INT4 per token
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_int4_sym(const T* __restrict__ x, const int8_t* __restrict__ signs,
           uint8_t* __restrict__ codes, float* __restrict__ scales, int64_t tokens,
           Geometry g) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  double* red = reinterpret_cast<double*>(buf + g.n);
  float* xs = reinterpret_cast<float*>(red + 64);   // the sign-flipped row, for fix-ups
  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const T* xr = x + row * g.n;
    load_row(xr, signs, buf, g.n);
    __syncthreads();
    for (int c = threadIdx.x; c < g.n / 4; c += blockDim.x)
      reinterpret_cast<float4*>(xs)[c] = reinterpret_cast<const float4*>(buf)[c];
    __syncthreads();
    fwht_smem(buf, g.n, g.m);
    if (g.paley) paley_smem<false>(buf, g.m);
    const float mh = row_absmax(buf, g.n, red);
    const double E = error_bound(g, mh);
    // scale32 = fp32(fp64(max|S| / sqrt(b)) / 7): decided by fp32 values only
    // when both interval ends give the same fp32; otherwise recompute exactly.
    const float lo_s = __double2float_rn((fmax((double)mh - E, 0.0) / g.sqrt_b) / 7.0);
    const float hi_s = __double2float_rn((((double)mh + E) / g.sqrt_b) / 7.0);
    float scale;
    if (lo_s == hi_s) {
      scale = lo_s;
    } else {
      const double smax = exact_max_abs_smem(xs, g, buf, 0, g.n,
                                             thr_down((double)mh - 2.0 * E), red);
      scale = __double2float_rn((smax / g.sqrt_b) / 7.0);
    }
    if (threadIdx.x == 0) scales[row] = scale;
    const float c = scale > 0.0f ? __double2float_rn(1.0 / (g.sqrt_b * (double)scale)) : 0.0f;
    uint32_t* crow = reinterpret_cast<uint32_t*>(codes + row * (g.n / 2));
    for (int q = threadIdx.x; q < g.n / 8; q += blockDim.x) {
      uint32_t word = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        int v = __float2int_rn(buf[8 * q + k] * c);
        v = max(-8, min(7, v));
        word |= (uint32_t)(v & 15) << (4 * k);
      }
      crow[q] = word;
    }
    __syncthreads();
  }
}

// ================================================ INT4 asymmetric, grouped
// fp16((mx - mn) / 15) from unnormalised extremes, as the fp64 formula.
__device__ __forceinline__ uint16_t asym_scale16(double smax, double smin, double sqrt_b) {
  const double mx = smax / sqrt_b, mn = smin / sqrt_b;
  return f64_to_f16_bits((mx - mn) / 15.0);
}
__device__ __forceinline__ double asym_zero(double smin, double sqrt_b, uint16_t s16) {
  const double s = f16_bits_to_f64(s16);
  if (!(s > 0.0)) return 0.0;
  return rint(-(smin / sqrt_b) / s);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
k_int4_asym(const T* __restrict__ x, const int8_t* __restrict__ signs,
            uint8_t* __restrict__ codes, uint16_t* __restrict__ scales,
            uint16_t* __restrict__ zeros, int64_t tokens, Geometry g, int group) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  const int ngroups = g.n / group;
  float* gmx = buf + g.n;                       // per group: computed max
  float* gmn = gmx + ngroups;                   //            computed min
  uint16_t* gs = reinterpret_cast<uint16_t*>(gmn + ngroups);   // scale16 bits
  uint16_t* gz = gs + ngroups;                  // zero16 bits
  int* gflag = reinterpret_cast<int*>(gz + ngroups + (ngroups & 1));
  double* red = reinterpret_cast<double*>(
      (reinterpret_cast<uintptr_t>(gflag + ngroups) + 15) & ~uintptr_t(15));
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;

  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const T* xr = x + row * g.n;
    transform_row(xr, signs, buf, g, false);
    const float mh = row_absmax(buf, g.n, red);
    const double E = error_bound(g, mh);
    // per-group extremes, one warp per group
    for (int grp = wid; grp < ngroups; grp += nw) {
      float mx = -FLT_MAX, mn = FLT_MAX;
      for (int i = lane; i < group; i += 32) {
        const float v = buf[grp * group + i];
        mx = fmaxf(mx, v);
        mn = fminf(mn, v);
      }
      mx = warp_max(mx);
      mn = warp_min(mn);
      if (lane == 0) {
        gmx[grp] = mx;
        gmn[grp] = mn;
        const uint16_t s_lo = asym_scale16((double)mx - E, (double)mn + E, g.sqrt_b);
        const uint16_t s_hi = asym_scale16((double)mx + E, (double)mn - E, g.sqrt_b);
        int flag = 1;
        if (s_lo == s_hi) {
          const double z_lo = asym_zero((double)mn + E, g.sqrt_b, s_lo);
          const double z_hi = asym_zero((double)mn - E, g.sqrt_b, s_lo);
          if (z_lo == z_hi) {
            flag = 0;
            gs[grp] = s_lo;
            gz[grp] = f64_to_f16_bits(z_lo);
          }
        }
        gflag[grp] = flag;
      }
    }
    __syncthreads();
    // exact extremes for undecided groups, in group order
    for (int grp = 0; grp < ngroups; ++grp) {
      if (!gflag[grp]) continue;             // uniform: shared flag
      const int lo = grp * group, hi = lo + group;
      const float mx = gmx[grp], mn = gmn[grp];
      double smax = -DBL_MAX, smin = DBL_MAX;
      const float thr_hi = __double2float_rd((double)mx - 2.0 * E);
      const float thr_lo = __double2float_ru((double)mn + 2.0 * E);
      for (int prev = lo - 1;;) {
        int best = INT_MAX;
        for (int i = lo + threadIdx.x; i < hi; i += blockDim.x)
          if (i > prev && (buf[i] >= thr_hi || buf[i] <= thr_lo)) { best = i; break; }
        const int cnd = block_min_i(best, red);
        if (cnd == INT_MAX) break;
        const double s = exact_S(xr, signs, g, cnd, red);
        if (buf[cnd] >= thr_hi) smax = fmax(smax, s);
        if (buf[cnd] <= thr_lo) smin = fmin(smin, s);
        prev = cnd;
      }
      if (threadIdx.x == 0) {
        const uint16_t s16 = asym_scale16(smax, smin, g.sqrt_b);
        gs[grp] = s16;
        gz[grp] = f64_to_f16_bits(asym_zero(smin, g.sqrt_b, s16));
      }
    }
    __syncthreads();
    // quantize and store
    uint32_t* crow = reinterpret_cast<uint32_t*>(codes + row * (g.n / 2));
    for (int q = threadIdx.x; q < g.n / 8; q += blockDim.x) {
      const int grp = (8 * q) / group;
      const float s = f16_bits_to_f32(gs[grp]);
      const float z = f16_bits_to_f32(gz[grp]);
      uint32_t word = 0;
      if (s > 0.0f) {
        const float c = __double2float_rn(1.0 / (g.sqrt_b * (double)s));
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          float u = rintf(buf[8 * q + k] * c) + z;
          u = fminf(fmaxf(u, 0.0f), 15.0f);
          word |= (uint32_t)u << (4 * k);
        }
      }
      crow[q] = word;
    }
    for (int grp = threadIdx.x; grp < ngroups; grp += blockDim.x) {
      const bool zs = !(f16_bits_to_f32(gs[grp]) > 0.0f);
      scales[row * ngroups + grp] = gs[grp];
      zeros[row * ngroups + grp] = zs ? (uint16_t)0 : gz[grp];
    }
    __syncthreads();
  }
}

// ================================================================ NVFP4
// E4M3 block scale from an unnormalised 16-block maximum, as the fp64 formula:
// r = fp32(fp64(smax / sqrt(b)) / (6 t)), s_b = E4M3(r).
__device__ __forceinline__ uint32_t nvfp4_scale_code(double smax, double sqrt_b, float t) {
  if (!(t > 0.0f)) return 0u;
  const double y = smax / sqrt_b;
  const float r = __double2float_rn(y / (6.0 * (double)t));
  return e4m3_encode_rne_sat(r);
}

// tensor scale from the exact global max |S|
__device__ __forceinline__ float nvfp4_tensor_scale(double gmax_abs_s, double sqrt_b) {
  return __double2float_rn((gmax_abs_s / sqrt_b) / 2688.0);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
k_nvfp4(const T* __restrict__ x, const int8_t* __restrict__ signs,
        uint8_t* __restrict__ codes, uint8_t* __restrict__ bscales,
        float* __restrict__ tensor_scale, const NvWorkspace* __restrict__ ws,
        int64_t tokens, Geometry g) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  const int nb = g.n / 16;
  float* bmax = buf + g.n;
  uint8_t* bsc = reinterpret_cast<uint8_t*>(bmax + nb);
  uint8_t* bflag = bsc + nb;
  double* red = reinterpret_cast<double*>(
      (reinterpret_cast<uintptr_t>(bflag + nb) + 15) & ~uintptr_t(15));

  float t;
  if (ws) {
    t = nvfp4_tensor_scale(__longlong_as_double((long long)ws->gmax_bits), g.sqrt_b);
    if (blockIdx.x == 0 && threadIdx.x == 0) *tensor_scale = t;
  } else {
    t = *tensor_scale;
  }

  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const T* xr = x + row * g.n;
    transform_row(xr, signs, buf, g, false);
    const float mh = row_absmax(buf, g.n, red);
    const double E = error_bound(g, mh);
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
      float m = 0.0f;
#pragma unroll
      for (int e = 0; e < 16; ++e) m = fmaxf(m, fabsf(buf[16 * k + e]));
      bmax[k] = m;
      const uint32_t c_lo = nvfp4_scale_code(fmax((double)m - E, 0.0), g.sqrt_b, t);
      const uint32_t c_hi = nvfp4_scale_code((double)m + E, g.sqrt_b, t);
      bsc[k] = (uint8_t)c_lo;
      bflag[k] = c_lo != c_hi;
    }
    __syncthreads();
    for (int k = 0; k < nb; ++k) {
      if (!bflag[k]) continue;                 // uniform: shared flag
      const double smax = exact_max_abs(xr, signs, g, buf, 16 * k, 16 * k + 16,
                                        thr_down((double)bmax[k] - 2.0 * E), red);
      if (threadIdx.x == 0) bsc[k] = (uint8_t)nvfp4_scale_code(smax, g.sqrt_b, t);
    }
    __syncthreads();
    uint2* crow = reinterpret_cast<uint2*>(codes + row * (g.n / 2));
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
      const uint32_t sc = bsc[k];
      const double den = (double)e4m3_decode(sc) * (double)t;
      float v[16];
      if (den > 0.0) {
        const float c = __double2float_rn(1.0 / (g.sqrt_b * den));
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const float a = buf[16 * k + e] * c;
          v[e] = (a == 0.0f) ? 0.0f : a;        // -0 carries no sign bit
        }
        crow[k] = make_uint2(e2m1x8_hw(v), e2m1x8_hw(v + 8));
      } else {
        uint32_t w0 = 0, w1 = 0;
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          w0 |= (buf[16 * k + e] < 0.0f ? 8u : 0u) << (4 * e);
          w1 |= (buf[16 * k + 8 + e] < 0.0f ? 8u : 0u) << (4 * e);
        }
        crow[k] = make_uint2(w0, w1);
      }
      bscales[sf_offset(row, k, nb, g.sf_kc4)] = (uint8_t)sc;
    }
    __syncthreads();
  }
}

// ================================================================ MXFP4
// Shared exponent of a 32-block from the largest |S| of the block: e =
// floor(log2(smax / sqrt(b))) - 2, clamped to [-127, 127] (OCP MX: the
// largest E2M1 exponent is 2); an all-zero block gets -127.  Monotone in
// smax, so equal exponents at both ends of an interval decide it.
__device__ __forceinline__ int mx_exponent(double smax, double sqrt_b) {
  const double y = smax / sqrt_b;
  if (!(y > 0.0)) return -127;
  const int e = ilogb(y) - 2;
  return e < -127 ? -127 : (e > 127 ? 127 : e);
}

template <typename T>
__global__ void __launch_bounds__(kThreads)
k_mxfp4(const T* __restrict__ x, const int8_t* __restrict__ signs,
        uint8_t* __restrict__ codes, uint8_t* __restrict__ scales, int64_t tokens, Geometry g) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  const int nb = g.n / 32;
  float* bmax = buf + g.n;
  uint8_t* bsc = reinterpret_cast<uint8_t*>(bmax + nb);
  uint8_t* bflag = bsc + nb;
  double* red = reinterpret_cast<double*>(
      (reinterpret_cast<uintptr_t>(bflag + nb) + 15) & ~uintptr_t(15));
  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const T* xr = x + row * g.n;
    transform_row(xr, signs, buf, g, false);
    const float mh = row_absmax(buf, g.n, red);
    const double E = error_bound(g, mh);
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
      float m = 0.0f;
#pragma unroll
      for (int e = 0; e < 32; ++e) m = fmaxf(m, fabsf(buf[32 * k + e]));
      bmax[k] = m;
      const int lo = mx_exponent(fmax((double)m - E, 0.0), g.sqrt_b);
      const int hi = mx_exponent((double)m + E, g.sqrt_b);
      bsc[k] = (uint8_t)(lo + 127);
      bflag[k] = lo != hi;
    }
    __syncthreads();
    for (int k = 0; k < nb; ++k) {
      if (!bflag[k]) continue;                 // uniform: shared flag
      const double smax = exact_max_abs(xr, signs, g, buf, 32 * k, 32 * k + 32,
                                        thr_down((double)bmax[k] - 2.0 * E), red);
      if (threadIdx.x == 0) bsc[k] = (uint8_t)(mx_exponent(smax, g.sqrt_b) + 127);
    }
    __syncthreads();
    uint4* crow = reinterpret_cast<uint4*>(codes + row * (g.n / 2));
    for (int k = threadIdx.x; k < nb; k += blockDim.x) {
      const int e = (int)bsc[k] - 127;
      const float c = (float)ldexp(1.0 / g.sqrt_b, -e);   // 1 / (sqrt(b) 2^e)
      float v[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float a = buf[32 * k + i] * c;
        v[i] = (a == 0.0f) ? 0.0f : a;          // -0 carries no sign bit
      }
      crow[k] = make_uint4(e2m1x8_hw(v), e2m1x8_hw(v + 8), e2m1x8_hw(v + 16), e2m1x8_hw(v + 24));
      scales[row * nb + k] = bsc[k];
    }
    __syncthreads();
  }
}

__global__ void k_dequant_mxfp4(const uint8_t* __restrict__ codes,
                                const uint8_t* __restrict__ scales, float* __restrict__ out,
                                int64_t tokens, int n) {
  const int64_t words = tokens * (int64_t)(n / 8);
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < words;
       q += (int64_t)gridDim.x * blockDim.x) {
    const float sx = ldexpf(1.0f, (int)scales[q >> 2] - 127);   // exact power of two
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes)[q];
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = e2m1_decode((w >> (4 * k)) & 15u) * sx;
    float4* o = reinterpret_cast<float4*>(out + 8 * q);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// Dynamic tensor scale, step 1: per-row computed max and error bound, and a
// global lower bound on max|S| (atomicMax on non-negative float bits).
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_nvfp4_rowstats(const T* __restrict__ x, const int8_t* __restrict__ signs,
                 NvWorkspace* __restrict__ ws, int64_t tokens, Geometry g) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  double* red = reinterpret_cast<double*>(buf + g.n);
  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    transform_row(x + row * g.n, signs, buf, g, false);
    const float mh = row_absmax(buf, g.n, red);
    const double E = error_bound(g, mh);
    if (threadIdx.x == 0) {
      ws->rows[row] = make_float2(mh, __double2float_ru(E));
      atomicMax(&ws->lower_bits, __float_as_uint(thr_down((double)mh - E)));
    }
    __syncthreads();
  }
}

// Inputs j0 .. j0 + 7 with the signs applied, exact in fp64.
__device__ __forceinline__ void load8_f64(const uint16_t* __restrict__ xr,
                                          const int8_t* __restrict__ signs, int j0,
                                          double (&v)[8]) {
  const uint4 w = __ldg(reinterpret_cast<const uint4*>(xr + j0));
  const uint2 sv = signs ? __ldg(reinterpret_cast<const uint2*>(signs + j0)) : make_uint2(0, 0);
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint32_t sw = k < 2 ? sv.x : sv.y;
    const uint32_t sb0 = (sw >> (16 * (k & 1) + 7)) & 1u;
    const uint32_t sb1 = (sw >> (16 * (k & 1) + 15)) & 1u;
    v[2 * k] = (double)__uint_as_float((ww[k] << 16) ^ (sb0 << 31));
    v[2 * k + 1] = (double)__uint_as_float((ww[k] & 0xffff0000u) ^ (sb1 << 31));
  }
}
__device__ __forceinline__ void load8_f64(const float* __restrict__ xr,
                                          const int8_t* __restrict__ signs, int j0,
                                          double (&v)[8]) {
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const float4 f = __ldg(reinterpret_cast<const float4*>(xr + j0) + h);
    const uint32_t sw = signs ? __ldg(reinterpret_cast<const uint32_t*>(signs + j0) + h) : 0u;
    const float e[4] = {f.x, f.y, f.z, f.w};
#pragma unroll
    for (int k = 0; k < 4; ++k)
      v[4 * h + k] = (double)__uint_as_float(__float_as_uint(e[k]) ^ (((sw >> (8 * k + 7)) & 1u) << 31));
  }
}

// Row j = 0 .. n-1 with the signs applied, in fp64, with the butterflies of
// strides 1, 2 and 4 already done (each thread holds whole groups of eight).
template <typename T>
__device__ __forceinline__ void load_row_f64_h8(const T* __restrict__ xr,
                                                const int8_t* __restrict__ signs, double* buf,
                                                int n) {
#pragma unroll 2
  for (int gi = threadIdx.x; gi < n / 8; gi += blockDim.x) {
    double v[8];
    load8_f64(xr, signs, 8 * gi, v);
#pragma unroll
    for (int st = 1; st < 8; st <<= 1)
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (!(k & st)) {
          const double a = v[k], b = v[k | st];
          v[k] = a + b;
          v[k | st] = a - b;
        }
#pragma unroll
    for (int k = 0; k < 8; ++k) buf[8 * gi + k] = v[k];
  }
}

// Block-wide max of doubles; `red` is shared scratch of >= 32 doubles.
__device__ __forceinline__ double block_max_d(double v, double* red) {
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5, nw = blockDim.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmax(v, __shfl_xor_sync(0xffffffffu, v, o));
  __syncthreads();
  if (lane == 0) red[wid] = v;
  __syncthreads();
  double t = red[0];
  for (int i = 1; i < nw; ++i) t = fmax(t, red[i]);
  return t;
}

// Dynamic tensor scale, step 2: max|S| over the rows that can hold the
// global maximum, in fp64.  Each CTA screens a contiguous range of rows with
// all its threads at once (one row's statistics per thread); a candidate row
// is transformed whole in fp64 (exact inputs, fp64 butterflies and Paley
// sums: the same precision as an fp64 dot product per output), so no
// per-output candidate search is needed.
template <typename T>
__global__ void __launch_bounds__(kThreads)
k_nvfp4_global(const T* __restrict__ x, const int8_t* __restrict__ signs,
               NvWorkspace* __restrict__ ws, int64_t tokens, Geometry g) {
  extern __shared__ __align__(16) float smem[];
  double* dbuf = reinterpret_cast<double*>(smem);   // g.n values
  double* red = dbuf + g.n;
  __shared__ int64_t cand[kThreads];
  __shared__ int ncand;
  const float L = __uint_as_float(ws->lower_bits);
  const int64_t per = (tokens + gridDim.x - 1) / gridDim.x;
  const int64_t r0 = (int64_t)blockIdx.x * per;
  const int64_t r1 = r0 + per < tokens ? r0 + per : tokens;
  for (int64_t base = r0; base < r1; base += blockDim.x) {
    if (threadIdx.x == 0) ncand = 0;
    __syncthreads();
    const int64_t row = base + threadIdx.x;
    if (row < r1) {
      const float2 st = ws->rows[row];
      if ((double)st.x + (double)st.y >= (double)L) cand[atomicAdd(&ncand, 1)] = row;
    }
    __syncthreads();
    const int nc = ncand;
    for (int c = 0; c < nc; ++c) {
      load_row_f64_h8(x + cand[c] * g.n, signs, dbuf, g.n);
      __syncthreads();
      fwht_smem(dbuf, g.n, g.m, 8);
      if (g.paley) paley_smem<false>(dbuf, g.m);
      double m = 0.0;
      for (int i = threadIdx.x; i < g.n; i += blockDim.x) m = fmax(m, fabs(dbuf[i]));
      m = block_max_d(m, red);
      if (threadIdx.x == 0)
        atomicMax(&ws->gmax_bits, (unsigned long long)__double_as_longlong(m));
      __syncthreads();
    }
    __syncthreads();   // every thread has read ncand before the next reset
  }
}

// ============================================================= dequant
__global__ void k_dequant_int4_sym(const uint8_t* __restrict__ codes,
                                   const float* __restrict__ scales,
                                   float* __restrict__ out, int64_t tokens, int n) {
  const int64_t words = tokens * (int64_t)(n / 8);
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < words;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = q / (n / 8);
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes)[q];
    const float s = scales[row];
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      int c = (w >> (4 * k)) & 15;
      c = c >= 8 ? c - 16 : c;
      v[k] = (float)c * s;
    }
    float4* o = reinterpret_cast<float4*>(out + 8 * q);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

__global__ void k_dequant_int4_asym(const uint8_t* __restrict__ codes,
                                    const uint16_t* __restrict__ scales,
                                    const uint16_t* __restrict__ zeros,
                                    float* __restrict__ out, int64_t tokens, int n,
                                    int group) {
  const int64_t words = tokens * (int64_t)(n / 8);
  const int gpr = n / group;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < words;
       q += (int64_t)gridDim.x * blockDim.x) {
    const int64_t row = q / (n / 8);
    const int col = (int)(q - row * (n / 8)) * 8;
    const int64_t gi = row * gpr + col / group;
    const float s = f16_bits_to_f32(scales[gi]);
    const float z = f16_bits_to_f32(zeros[gi]);
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes)[q];
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = s * ((float)((w >> (4 * k)) & 15) - z);
    float4* o = reinterpret_cast<float4*>(out + 8 * q);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

__global__ void k_dequant_nvfp4(const uint8_t* __restrict__ codes,
                                const uint8_t* __restrict__ bscales,
                                const float* __restrict__ tensor_scale,
                                float* __restrict__ out, int64_t tokens, int n) {
  const int64_t words = tokens * (int64_t)(n / 8);
  const float t = *tensor_scale;
  for (int64_t q = blockIdx.x * (int64_t)blockDim.x + threadIdx.x; q < words;
       q += (int64_t)gridDim.x * blockDim.x) {
    const float sb = e4m3_decode(bscales[q >> 1]);
    const uint32_t w = reinterpret_cast<const uint32_t*>(codes)[q];
    float v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = (e2m1_decode((w >> (4 * k)) & 15u) * sb) * t;
    float4* o = reinterpret_cast<float4*>(out + 8 * q);
    o[0] = make_float4(v[0], v[1], v[2], v[3]);
    o[1] = make_float4(v[4], v[5], v[6], v[7]);
  }
}

// ================================================ dequant + inverse rotation
// One row per CTA (grid-stride): the row's codes are dequantized into shared
// memory exactly as kq_dequant writes them (each value the product of code
// and scale(s), rounded once to fp32), then rotated back as kq_rht with
// KQ_INVERSE does: FWHT, the transposed Paley factor, 1/sqrt(b), signs.
template <bool kBf16Out>
__global__ void __launch_bounds__(kThreads)
k_dequant_rht_inv(int fmt, const uint8_t* __restrict__ codes, const void* __restrict__ scales,
                  const uint16_t* __restrict__ zeros, const float* __restrict__ tensor_scale,
                  const int8_t* __restrict__ signs, void* __restrict__ out, int64_t tokens,
                  Geometry g, int group) {
  extern __shared__ __align__(16) float smem[];
  float* buf = smem;
  const int words = g.n / 8;
  const float t = fmt == 2 ? *tensor_scale : 0.0f;
  for (int64_t row = blockIdx.x; row < tokens; row += gridDim.x) {
    const uint32_t* cw = reinterpret_cast<const uint32_t*>(codes + row * (g.n / 2));
    for (int c = threadIdx.x; c < words; c += blockDim.x) {
      const uint32_t w = cw[c];
      float v[8];
      if (fmt == 0) {
        const float s = static_cast<const float*>(scales)[row];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          int q = (w >> (4 * k)) & 15;
          q = q >= 8 ? q - 16 : q;
          v[k] = (float)q * s;
        }
      } else if (fmt == 1) {
        const int64_t gi = row * (g.n / group) + (8 * c) / group;
        const float s = f16_bits_to_f32(static_cast<const uint16_t*>(scales)[gi]);
        const float z = f16_bits_to_f32(zeros[gi]);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = s * ((float)((w >> (4 * k)) & 15) - z);
      } else if (fmt == 3) {
        const float sx =
            ldexpf(1.0f, (int)static_cast<const uint8_t*>(scales)[row * (g.n / 32) + (c >> 2)] - 127);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = e2m1_decode((w >> (4 * k)) & 15u) * sx;
      } else {
        const float sb =
            e4m3_decode(static_cast<const uint8_t*>(scales)[row * (g.n / 16) + (c >> 1)]);
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = (e2m1_decode((w >> (4 * k)) & 15u) * sb) * t;
      }
      float4* b4 = reinterpret_cast<float4*>(buf + 8 * c);
      b4[0] = make_float4(v[0], v[1], v[2], v[3]);
      b4[1] = make_float4(v[4], v[5], v[6], v[7]);
    }
    __syncthreads();
    fwht_smem(buf, g.n, g.m);
    if (g.paley) paley_smem<true>(buf, g.m);
    for (int c = threadIdx.x; c < g.n / 4; c += blockDim.x) {
      float4 v = reinterpret_cast<const float4*>(buf)[c];
      v.x *= g.inv_sqrt_b;
      v.y *= g.inv_sqrt_b;
      v.z *= g.inv_sqrt_b;
      v.w *= g.inv_sqrt_b;
      if (signs) {
        const uint32_t sw = __ldg(reinterpret_cast<const uint32_t*>(signs) + c);
        v.x = __uint_as_float(__float_as_uint(v.x) ^ (((sw >> 7) & 1u) << 31));
        v.y = __uint_as_float(__float_as_uint(v.y) ^ (((sw >> 15) & 1u) << 31));
        v.z = __uint_as_float(__float_as_uint(v.z) ^ (((sw >> 23) & 1u) << 31));
        v.w = __uint_as_float(__float_as_uint(v.w) ^ (((sw >> 31) & 1u) << 31));
      }
      if (kBf16Out) {
        uint32_t lo, hi;
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(lo) : "f"(v.y), "f"(v.x));
        asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(hi) : "f"(v.w), "f"(v.z));
        reinterpret_cast<uint2*>(static_cast<uint16_t*>(out) + row * g.n)[c] = make_uint2(lo, hi);
      } else {
        reinterpret_cast<float4*>(static_cast<float*>(out) + row * g.n)[c] = v;
      }
    }
    __syncthreads();
  }
}

// ============================================================= launchers
namespace {

int grid_for(const void* kernel, size_t smem, int64_t tokens) {
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (smem > 48 * 1024)
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t g = (int64_t)sms * per_sm;
  return (int)(tokens < g ? tokens : g);
}

}  // namespace

cudaError_t launch_rht(const void* x, int dtype, int64_t tokens, const Geometry& g,
                       const int8_t* signs, float* out, int inverse, cudaStream_t s) {
  const size_t smem = (size_t)g.n * sizeof(float);
  if (dtype == 1) {
    auto k = k_rht<uint16_t>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const uint16_t*>(x), signs, out, tokens, g, inverse);
  } else {
    auto k = k_rht<float>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const float*>(x), signs, out, tokens, g, inverse);
  }
  return cudaGetLastError();
}

cudaError_t launch_int4_sym(const void* x, int dtype, int64_t tokens, const Geometry& g,
                            const int8_t* signs, uint8_t* codes, float* scales,
                            cudaStream_t s) {
  const size_t smem = 2 * (size_t)g.n * sizeof(float) + 64 * sizeof(double);
  if (dtype == 1) {
    auto k = k_int4_sym<uint16_t>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const uint16_t*>(x), signs, codes, scales, tokens, g);
  } else {
    auto k = k_int4_sym<float>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const float*>(x), signs, codes, scales, tokens, g);
  }
  return cudaGetLastError();
}

cudaError_t launch_int4_asym(const void* x, int dtype, int64_t tokens, const Geometry& g,
                             const int8_t* signs, int group, uint8_t* codes,
                             uint16_t* scales, uint16_t* zeros, cudaStream_t s) {
  const int ng = g.n / group;
  const size_t smem = (size_t)g.n * 4 + (size_t)ng * (4 + 4 + 2 + 2 + 4) + 64 + 64 * 8;
  if (dtype == 1) {
    auto k = k_int4_asym<uint16_t>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const uint16_t*>(x), signs, codes, scales, zeros, tokens, g, group);
  } else {
    auto k = k_int4_asym<float>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const float*>(x), signs, codes, scales, zeros, tokens, g, group);
  }
  return cudaGetLastError();
}

cudaError_t launch_nvfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                         const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                         float* tensor_scale, NvWorkspace* ws, cudaStream_t s) {
  const int nb = g.n / 16;
  const size_t smem = (size_t)g.n * 4 + (size_t)nb * (4 + 1 + 1) + 16 + 64 * 8;
  const size_t smem_stats = (size_t)g.n * 4 + 64 * 8;
  const size_t smem_glob = (size_t)g.n * 8 + 64 * 8;
  cudaError_t err;
  if (ws) {
    const int ph = g.dyn ? g.dyn : 7;
    if (ph & 1) {
      err = cudaMemsetAsync(ws, 0, sizeof(NvWorkspace), s);
      if (err != cudaSuccess) return err;
      if (dtype == 1) {
        auto k1 = k_nvfp4_rowstats<uint16_t>;
        k1<<<grid_for((const void*)k1, smem_stats, tokens), kThreads, smem_stats, s>>>(
            static_cast<const uint16_t*>(x), signs, ws, tokens, g);
      } else {
        auto k1 = k_nvfp4_rowstats<float>;
        k1<<<grid_for((const void*)k1, smem_stats, tokens), kThreads, smem_stats, s>>>(
            static_cast<const float*>(x), signs, ws, tokens, g);
      }
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
    }
    if (ph & 2) {
      if (dtype == 1) {
        auto k2 = k_nvfp4_global<uint16_t>;
        k2<<<grid_for((const void*)k2, smem_glob, tokens), kThreads, smem_glob, s>>>(
            static_cast<const uint16_t*>(x), signs, ws, tokens, g);
      } else {
        auto k2 = k_nvfp4_global<float>;
        k2<<<grid_for((const void*)k2, smem_glob, tokens), kThreads, smem_glob, s>>>(
            static_cast<const float*>(x), signs, ws, tokens, g);
      }
      err = cudaGetLastError();
      if (err != cudaSuccess) return err;
    }
    if (!(ph & 4)) return cudaSuccess;
  }
  if (dtype == 1) {
    auto k = k_nvfp4<uint16_t>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const uint16_t*>(x), signs, codes, bscales, tensor_scale, ws, tokens, g);
  } else {
    auto k = k_nvfp4<float>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const float*>(x), signs, codes, bscales, tensor_scale, ws, tokens, g);
  }
  return cudaGetLastError();
}

cudaError_t launch_nvfp4_global(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                const int8_t* signs, NvWorkspace* ws, cudaStream_t s) {
  const size_t smem_glob = (size_t)g.n * 8 + 64 * 8;
  if (dtype == 1) {
    auto k2 = k_nvfp4_global<uint16_t>;
    k2<<<grid_for((const void*)k2, smem_glob, tokens), kThreads, smem_glob, s>>>(
        static_cast<const uint16_t*>(x), signs, ws, tokens, g);
  } else {
    auto k2 = k_nvfp4_global<float>;
    k2<<<grid_for((const void*)k2, smem_glob, tokens), kThreads, smem_glob, s>>>(
        static_cast<const float*>(x), signs, ws, tokens, g);
  }
  return cudaGetLastError();
}

cudaError_t launch_dequant(int fmt, const uint8_t* codes, const void* scales,
                           const void* zeros, const float* tensor_scale, int64_t tokens,
                           int n, int group, float* out, cudaStream_t s) {
  int dev = 0, sms = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t words = tokens * (int64_t)(n / 8);
  int64_t blocks = (words + 255) / 256;
  const int64_t cap = (int64_t)sms * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (fmt == 0)
    k_dequant_int4_sym<<<(int)blocks, 256, 0, s>>>(
        codes, static_cast<const float*>(scales), out, tokens, n);
  else if (fmt == 1)
    k_dequant_int4_asym<<<(int)blocks, 256, 0, s>>>(
        codes, static_cast<const uint16_t*>(scales), static_cast<const uint16_t*>(zeros),
        out, tokens, n, group);
  else if (fmt == 3)
    k_dequant_mxfp4<<<(int)blocks, 256, 0, s>>>(
        codes, static_cast<const uint8_t*>(scales), out, tokens, n);
  else
    k_dequant_nvfp4<<<(int)blocks, 256, 0, s>>>(
        codes, static_cast<const uint8_t*>(scales), tensor_scale, out, tokens, n);
  return cudaGetLastError();
}

cudaError_t launch_dequant_rht_inv(int fmt, const uint8_t* codes, const void* scales,
                                  const void* zeros, const float* tensor_scale,
                                  int64_t tokens, const Geometry& g, int group,
                                  const int8_t* signs, void* out, int out_bf16, cudaStream_t s) {
  const size_t smem = (size_t)g.n * sizeof(float);
  auto k = out_bf16 ? k_dequant_rht_inv<true> : k_dequant_rht_inv<false>;
  k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
      fmt, codes, scales, static_cast<const uint16_t*>(zeros), tensor_scale, signs, out,
      tokens, g, group);
  return cudaGetLastError();
}

cudaError_t launch_mxfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                         const int8_t* signs, uint8_t* codes, uint8_t* scales,
                         cudaStream_t s) {
  const int nb = g.n / 32;
  const size_t smem = (size_t)g.n * 4 + (size_t)nb * 6 + 16 + 64 * 8;
  if (dtype == 1) {
    auto k = k_mxfp4<uint16_t>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const uint16_t*>(x), signs, codes, scales, tokens, g);
  } else {
    auto k = k_mxfp4<float>;
    k<<<grid_for((const void*)k, smem, tokens), kThreads, smem, s>>>(
        static_cast<const float*>(x), signs, codes, scales, tokens, g);
  }
  return cudaGetLastError();
}

}  // namespace kq
