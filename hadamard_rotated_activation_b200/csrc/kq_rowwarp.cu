// Warp-per-row kernels for a Hadamard transform over the whole row, rows of
// N = 2048 or 4096 (the hidden size 4096 of "Bug: Qwen3-8B integration
// issue", Model Details; full-row RHT of the QuaRot reviews).
//
// One warp owns one row; lane l keeps N/32 values in registers.  Rows stream
// into a per-warp double buffer in shared memory by asynchronous copies, one
// row ahead of the computation.
//   phase 1: lane l reads the bf16 pairs (h*64 + 2l, +1), h = 0..N/64-1, so
//            element bits {0, 6..log2 N - 1} are in-lane: stage 0 in scalar
//            fp32 while converting, the rest on packed f32x2 pairs.
//   transposition through shared memory (fp32, XOR-swizzled 16-byte chunks:
//            the 8-byte writes and 16-byte reads are conflict-free).
//   phase 2: lane l holds elements l*N/32 .. l*N/32 + N/32 - 1, so bits 1..5
//            are in-lane (f32x2) and every NVFP4 16-block and INT4 nibble pair
//            is local to one lane.
// The sign vector is applied as an XOR of the bf16 sign bits with a per-CTA
// table of masks built once from the int8 signs.
//
// Exact scales: the fp32 transform is within E = gamma_L * sum|x| of the exact
// sums (L = log2 N roundings per path), sum|x| accumulated while loading.
// Undecided scales are recomputed by the warp as exact fp64 dot products.
#include <cfloat>
#include <climits>
#include <cstdint>

#include "kq_device.cuh"
#include "kq_internal.h"

namespace kq {
namespace rw {

constexpr int kWarps = 2;
constexpr int kThreads = 32 * kWarps;

enum { kInt4 = 0, kNvfp4 = 1, kNvStats = 2 };

struct Params {
  const void* x;                // [T, N] bf16 bits or fp32
  const int8_t* signs;          // [N] or null
  uint8_t* codes;               // [T, N/2]
  float* scales32;              // INT4: fp32 [T]
  uint8_t* scales8;             // NVFP4: E4M3 [T, N/16]
  float* tensor_scale;          // NVFP4: read if static, written if dynamic
  NvWorkspace* ws;              // NVFP4 dynamic
  int64_t tokens;
  float gamma;                  // gamma_L with a safety factor (rounded up)
  int sf_kc4;                   // NVFP4 scale layout (Geometry::sf_kc4)
};

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

__device__ __forceinline__ float e4m3_recip(uint32_t c) {
  const uint32_t e = (c >> 3) & 15u, m = c & 7u;
  if (e == 0) return 512.0f / (float)m;
  const float r = 1.0f / (1.0f + 0.125f * (float)m);
  return ldexpf(r, 7 - (int)e);
}

// smem word address of element i in a row buffer of N floats whose rows of
// R = N/32 words have their 16-byte chunks XOR-swizzled by the row index.
template <int N>
__device__ __forceinline__ int swz(int i) {
  constexpr int R = N / 32, C = R / 4;
  const int r = i / R, w = i % R;
  const int c = (w >> 2) ^ (r % C);
  return r * R + (c << 2) + (w & 3);
}

// Starts copying row `row` (N bf16, contiguous) into `raw` with coalesced
// 16-byte asynchronous copies, as one commit group.
template <int N>
__device__ __forceinline__ void prefetch_row(const uint16_t* __restrict__ x, int64_t row,
                                             uint16_t* raw) {
  const int lane = threadIdx.x & 31;
  const uint4* src = reinterpret_cast<const uint4*>(x + row * N);
  const uint32_t base = (uint32_t)__cvta_generic_to_shared(raw);
#pragma unroll
  for (int j = 0; j < N / 256; ++j) {
    const int idx = lane + 32 * j;
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" :: "r"(base + 16u * idx),
                 "l"(src + idx) : "memory");
  }
  asm volatile("cp.async.commit_group;" ::: "memory");
}

// Exact S_i of the staged row (Sylvester, natural order), warp-cooperative
// fp64: lane l sums the pairs l + 32 q.  Every lane gets the result.
template <int N>
__device__ __noinline__ double warp_exact_S(const uint16_t* raw, const uint32_t* smask, int i) {
  const int lane = threadIdx.x & 31;
  const uint32_t* rw32 = reinterpret_cast<const uint32_t*>(raw);
  double acc = 0.0;
#pragma unroll 8
  for (int q = 0; q < N / 64; ++q) {
    const int pr = lane + 32 * q;
    const uint32_t w = rw32[pr] ^ smask[pr];
    const int j = 2 * pr;
    const double a = (double)__uint_as_float(w << 16);
    const double b = (double)__uint_as_float(w & 0xffff0000u);
    acc += (__popc(i & j) & 1) ? -a : a;
    acc += (__popc(i & (j + 1)) & 1) ? -b : b;
  }
  return warp_sum_d(acc);
}

// Transform the staged row; v[p] = {S[l*R + 2p], S[l*R + 2p + 1]} (R = N/32).
// Returns this lane's part of sum|x|.
template <int N>
__device__ __forceinline__ float row_transform(const uint16_t* raw, const uint32_t* smask,
                                               float* tbuf, float2 (&v)[N / 64]) {
  constexpr int H = N / 64;    // pairs per lane in phase 1
  constexpr int R = N / 32;
  const int lane = threadIdx.x & 31;
  const uint32_t* rw32 = reinterpret_cast<const uint32_t*>(raw);
  float abs_sum = 0.0f;
  float2 a[H];
#pragma unroll
  for (int h = 0; h < H; ++h) {
    const uint32_t w = rw32[h * 32 + lane] ^ smask[h * 32 + lane];
    const float lo = __uint_as_float(w << 16), hi = __uint_as_float(w & 0xffff0000u);
    abs_sum += fabsf(lo);
    abs_sum += fabsf(hi);
    a[h] = make_float2(lo + hi, lo - hi);          // element bit 0
  }
#pragma unroll
  for (int s = 1; s < H; s <<= 1)                  // element bits 6..
#pragma unroll
    for (int h = 0; h < H; ++h)
      if (!(h & s)) bfly2(a[h], a[h | s]);
  // transposition through tbuf (N floats)
  __syncwarp();
#pragma unroll
  for (int h = 0; h < H; ++h)
    *reinterpret_cast<float2*>(tbuf + swz<N>(h * 64 + 2 * lane)) = a[h];
  __syncwarp();
#pragma unroll
  for (int q = 0; q < R / 4; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(tbuf + swz<N>(lane * R + 4 * q));
    v[2 * q] = make_float2(f.x, f.y);
    v[2 * q + 1] = make_float2(f.z, f.w);
  }
#pragma unroll
  for (int s = 1; s < 32; s <<= 1)                 // element bits 1..5
#pragma unroll
    for (int p = 0; p < R / 2; ++p)
      if (!(p & s)) bfly2(v[p], v[p | s]);
  return abs_sum;
}

// Stores the lane's R/2 code bytes of one row with coalesced 16-byte stores,
// staged through `tbuf` (free after the transform).
template <int N>
__device__ __forceinline__ void store_row_codes(float* tbuf, const uint4* cw, uint8_t* crow) {
  constexpr int K = N / 32 / 32;   // 16-byte chunks per lane (R/2 bytes)
  const int lane = threadIdx.x & 31;
  uint4* st = reinterpret_cast<uint4*>(tbuf);
  __syncwarp();
#pragma unroll
  for (int k = 0; k < K; ++k) st[lane * K + (k ^ (lane % K))] = cw[k];
  __syncwarp();
  uint4* dst = reinterpret_cast<uint4*>(crow);
#pragma unroll
  for (int j = 0; j < K; ++j) {
    const int idx = lane + 32 * j;
    const int t = idx / K, k = idx % K;
    dst[idx] = st[t * K + (k ^ (t % K))];
  }
}

template <int N, int kMode>
__global__ void __launch_bounds__(kThreads)
k_rowwarp(Params P) {
  constexpr int R = N / 32;      // values per lane
  constexpr int K = R / 32;      // 16-byte code chunks per lane
  extern __shared__ __align__(16) uint32_t sm[];
  const int lane = threadIdx.x & 31, wid = threadIdx.x >> 5;
  uint32_t* smask = sm;                                               // N/2 pair masks
  uint16_t* raws = reinterpret_cast<uint16_t*>(sm + N / 2) + wid * 2 * N;   // 2 rows
  float* tbuf = reinterpret_cast<float*>(sm + N / 2 + kWarps * N) + wid * N;

  // per-pair sign masks (bit 15: even element, bit 31: odd element)
  for (int pidx = threadIdx.x; pidx < N / 2; pidx += blockDim.x) {
    uint32_t m = 0;
    if (P.signs) {
      const uint32_t two =
          (uint32_t)__ldg(reinterpret_cast<const uint16_t*>(P.signs) + pidx);
      m = __byte_perm(two, 0, 0x1404) & 0x80008000u;
    }
    smask[pidx] = m;
  }
  __syncthreads();

  float t = 0.0f, c6 = 0.0f, inv_bt = 0.0f;
  constexpr double kSqrtN = (N == 4096) ? 64.0 : 45.254833995939045;
  if (kMode == kNvfp4) {
    if (P.ws) {
      const double g = __longlong_as_double((long long)P.ws->gmax_bits);
      t = __double2float_rn((g / kSqrtN) / 2688.0);
      if (blockIdx.x == 0 && threadIdx.x == 0) *P.tensor_scale = t;
    } else {
      t = *P.tensor_scale;
    }
    c6 = (t > 0.0f) ? (float)(1.0 / (kSqrtN * 6.0 * (double)t)) : 0.0f;
    inv_bt = (t > 0.0f) ? (float)(1.0 / (kSqrtN * (double)t)) : 0.0f;
  }

  const uint16_t* x = static_cast<const uint16_t*>(P.x);
  const int64_t gw = (int64_t)blockIdx.x * kWarps + wid;
  const int64_t nw = (int64_t)gridDim.x * kWarps;
  if (gw < P.tokens) prefetch_row<N>(x, gw, raws);
  int it = 0;
  for (int64_t row = gw; row < P.tokens; row += nw, ++it) {
    const uint16_t* raw = raws + (it & 1) * N;
    __syncwarp();
    const bool more = row + nw < P.tokens;
    if (more) prefetch_row<N>(x, row + nw, raws + ((it + 1) & 1) * N);
    if (more)
      asm volatile("cp.async.wait_group 1;" ::: "memory");
    else
      asm volatile("cp.async.wait_group 0;" ::: "memory");
    __syncwarp();

    float2 v[R / 2];
    const float part = row_transform<N>(raw, smask, tbuf, v);
    float sum_abs = part;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) sum_abs += __shfl_xor_sync(0xffffffffu, sum_abs, o);
    // |S_hat - S| <= gamma_L * sum|x| for every output of the row
    const float E = __fmul_ru(P.gamma, sum_abs);

    if (kMode == kNvStats) {
      float m = 0.0f;
#pragma unroll
      for (int p = 0; p < R / 2; ++p) m = fmax3(m, fabsf(v[p].x), fabsf(v[p].y));
      m = warp_max(m);
      if (lane == 0) {
        P.ws->rows[row] = make_float2(m, E);
        atomicMax(&P.ws->lower_bits, __float_as_uint(fmaxf(__fsub_rd(m, E), 0.0f)));
      }
      continue;
    }

    uint4 cw[K];
    if (kMode == kInt4) {
      float m = 0.0f;
#pragma unroll
      for (int p = 0; p < R / 2; ++p) m = fmax3(m, fabsf(v[p].x), fabsf(v[p].y));
      const float mh = warp_max(m);
      const float lo_s = __double2float_rn((fmax((double)mh - E, 0.0) / kSqrtN) / 7.0);
      const float hi_s = __double2float_rn((((double)mh + E) / kSqrtN) / 7.0);
      float scale = lo_s;
      if (lo_s != hi_s) {
        // candidates: |S_hat| >= mh - 2E, as a per-lane bitmask over R values
        const float thr = __fsub_rd(mh, 2.0f * E);
        uint32_t cm[K];
#pragma unroll
        for (int w = 0; w < K; ++w) cm[w] = 0;
#pragma unroll
        for (int p = 0; p < R / 2; ++p) {
          if (fabsf(v[p].x) >= thr) cm[(2 * p) >> 5] |= 1u << ((2 * p) & 31);
          if (fabsf(v[p].y) >= thr) cm[(2 * p + 1) >> 5] |= 1u << ((2 * p + 1) & 31);
        }
        uint32_t any = 0;
#pragma unroll
        for (int w = 0; w < K; ++w) any |= cm[w];
        double best = 0.0;
        unsigned todo = __ballot_sync(0xffffffffu, any != 0);
        while (todo) {
          const int src = __ffs(todo) - 1;
          todo &= todo - 1;
#pragma unroll
          for (int w = 0; w < K; ++w) {
            uint32_t b = __shfl_sync(0xffffffffu, cm[w], src);
            while (b) {
              const int e = __ffs(b) - 1;
              b &= b - 1;
              best = fmax(best, fabs(warp_exact_S<N>(raw, smask, src * R + 32 * w + e)));
            }
          }
        }
        scale = __double2float_rn((best / kSqrtN) / 7.0);
      }
      if (lane == 0) P.scales32[row] = scale;
      const float c = scale > 0.0f ? __double2float_rn(1.0 / (kSqrtN * (double)scale)) : 0.0f;
#pragma unroll
      for (int k = 0; k < K; ++k) {
        uint32_t words[4];
#pragma unroll
        for (int w = 0; w < 4; ++w) {
          uint32_t word = 0;
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float2 a = v[16 * k + 4 * w + e];
            int qx = __float2int_rn(a.x * c), qy = __float2int_rn(a.y * c);
            qx = max(-8, min(7, qx));
            qy = max(-8, min(7, qy));
            word |= ((uint32_t)(qx & 15) << (8 * e)) | ((uint32_t)(qy & 15) << (8 * e + 4));
          }
          words[w] = word;
        }
        cw[k] = make_uint4(words[0], words[1], words[2], words[3]);
      }
      store_row_codes<N>(tbuf, cw, P.codes + row * (N / 2));
      continue;
    }

    // ---- NVFP4: lane holds NB blocks of 16
    constexpr int NB = R / 16;
    float bm[NB];
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      float m = 0.0f;
#pragma unroll
      for (int p = 8 * j; p < 8 * j + 8; ++p) m = fmax3(m, fabsf(v[p].x), fabsf(v[p].y));
      bm[j] = m;
    }
    uint32_t sc[NB / 4];
#pragma unroll
    for (int w = 0; w < NB / 4; ++w) sc[w] = 0;
    uint32_t undecided = 0;
#pragma unroll
    for (int j = 0; j < NB; ++j) {
      const float lo = fmaxf(bm[j] - E, 0.0f) * c6 * (1.0f - 0x1p-20f);
      const float hi = (bm[j] + E) * c6 * (1.0f + 0x1p-20f);
      const uint32_t cc = e4m3_pair(lo, hi);
      sc[j >> 2] |= (cc & 0xffu) << (8 * (j & 3));
      if ((cc & 0xffu) != (cc >> 8)) undecided |= 1u << j;
    }
    if (t <= 0.0f) undecided = 0;
    unsigned todo = __ballot_sync(0xffffffffu, undecided != 0);
    while (todo) {
      const int src = __ffs(todo) - 1;
      todo &= todo - 1;
      const uint32_t und = __shfl_sync(0xffffffffu, undecided, src);
      for (int j = 0; j < NB; ++j) {
        if (!((und >> j) & 1u)) continue;
        uint32_t cand = 0;
        if (lane == src) {
          float bmj = 0.0f;
#pragma unroll
          for (int q = 0; q < NB; ++q)
            if (q == j) bmj = bm[q];
          const float thr = bmj - 2.0f * E;
#pragma unroll
          for (int q = 0; q < NB; ++q) {
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
        double best = 0.0;
        while (cand) {
          const int e = __ffs(cand) - 1;
          cand &= cand - 1;
          best = fmax(best, fabs(warp_exact_S<N>(raw, smask, src * R + 16 * j + e)));
        }
        const float r = __double2float_rn((best / kSqrtN) / (6.0 * (double)t));
        const uint32_t code = e4m3_pair(r, r) & 0xffu;
        if (lane == src) {
          const int w = j >> 2, sh = 8 * (j & 3);
#pragma unroll
          for (int q = 0; q < NB / 4; ++q)
            if (q == w) sc[q] = (sc[q] & ~(0xffu << sh)) | (code << sh);
        }
      }
    }
    const float2 zero2 = make_float2(0.0f, 0.0f);
#pragma unroll
    for (int k = 0; k < NB / 2; ++k) {
      uint32_t words[4];
#pragma unroll
      for (int jj = 0; jj < 2; ++jj) {
        const int j = 2 * k + jj;
        const uint32_t code = (sc[j >> 2] >> (8 * (j & 3))) & 0xffu;
        if (code != 0 && t > 0.0f) {
          const float c = inv_bt * e4m3_recip(code);
          const float2 c2 = make_float2(c, c);
          float q[16];
#pragma unroll
          for (int p = 0; p < 8; ++p) {
            const float2 a = fma2(v[8 * j + p], c2, zero2);   // + 0 turns -0 into +0
            q[2 * p] = a.x;
            q[2 * p + 1] = a.y;
          }
          words[2 * jj] = e2m1x8_hw(q);
          words[2 * jj + 1] = e2m1x8_hw(q + 8);
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
      cw[k] = make_uint4(words[0], words[1], words[2], words[3]);
    }
    store_row_codes<N>(tbuf, cw, P.codes + row * (N / 2));
    if (P.sf_kc4 != 0) {
      // one or two words of the tensor-core layout
#pragma unroll
      for (int j = 0; j < NB / 4; ++j)
        *reinterpret_cast<uint32_t*>(P.scales8 + sf_offset(row, lane * NB + 4 * j, N / 16,
                                                           P.sf_kc4)) = sc[j];
    } else if (NB == 8) {
      *reinterpret_cast<uint2*>(P.scales8 + row * (N / 16) + lane * NB) = make_uint2(sc[0], sc[1]);
    } else {
      *reinterpret_cast<uint32_t*>(P.scales8 + row * (N / 16) + lane * NB) = sc[0];
    }
  }
}

}  // namespace rw

// ------------------------------------------------------------- launchers
namespace {

template <int N, int kMode>
cudaError_t launch_rw(rw::Params& P, cudaStream_t s) {
  auto k = rw::k_rowwarp<N, kMode>;
  // sign masks + per warp: two staged rows (bf16) + one row of fp32
  const size_t smem = (size_t)N / 2 * 4 + (size_t)rw::kWarps * (2 * N * 2 + N * 4);
  cudaFuncSetAttribute((const void*)k, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  int dev = 0, sms = 0, per_sm = 0;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, (const void*)k, rw::kThreads, smem);
  if (per_sm < 1) per_sm = 1;
  const int64_t need = (P.tokens + rw::kWarps - 1) / rw::kWarps;
  const int64_t cap = (int64_t)sms * per_sm;
  k<<<(int)(need < cap ? need : cap), rw::kThreads, smem, s>>>(P);
  return cudaGetLastError();
}

float gamma_for(int log2n) {
  const double u = 0x1p-24, L = log2n;
  return (float)((L * u / (1.0 - L * u)) * 1.01);
}

template <int kMode>
cudaError_t dispatch(int n, rw::Params& P, cudaStream_t s) {
  if (n == 4096) return launch_rw<4096, kMode>(P, s);
  return launch_rw<2048, kMode>(P, s);
}

}  // namespace

bool rowwarp_supported(const Geometry& g, int dtype) {
  return dtype == 1 && !g.paley && g.b == g.n && (g.n == 4096 || g.n == 2048);
}

cudaError_t launch_rowwarp_int4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                const int8_t* signs, uint8_t* codes, float* scales,
                                cudaStream_t s) {
  rw::Params P{};
  P.x = x;
  P.signs = signs;
  P.codes = codes;
  P.scales32 = scales;
  P.tokens = tokens;
  P.gamma = gamma_for(g.n == 4096 ? 12 : 11);
  return dispatch<rw::kInt4>(g.n, P, s);
}

cudaError_t launch_rowwarp_nvfp4(const void* x, int dtype, int64_t tokens, const Geometry& g,
                                 const int8_t* signs, uint8_t* codes, uint8_t* bscales,
                                 float* tensor_scale, NvWorkspace* ws, cudaStream_t s) {
  rw::Params P{};
  P.x = x;
  P.signs = signs;
  P.codes = codes;
  P.scales8 = bscales;
  P.tensor_scale = tensor_scale;
  P.ws = ws;
  P.tokens = tokens;
  P.sf_kc4 = g.sf_kc4;
  P.gamma = gamma_for(g.n == 4096 ? 12 : 11);
  if (ws) {
    const int ph = g.dyn ? g.dyn : 7;
    if (ph & 1) {
      cudaError_t e = cudaMemsetAsync(ws, 0, kNvWorkspaceHeader, s);
      if (e != cudaSuccess) return e;
      e = dispatch<rw::kNvStats>(g.n, P, s);
      if (e != cudaSuccess) return e;
    }
    if (ph & 2) {
      cudaError_t e = launch_nvfp4_global(x, dtype, tokens, g, signs, ws, s);
      if (e != cudaSuccess) return e;
    }
    if (!(ph & 4)) return cudaSuccess;
  }
  return dispatch<rw::kNvfp4>(g.n, P, s);
}

}  // namespace kq
