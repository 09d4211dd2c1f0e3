/*
 * kq.h -- C ABI of the fused randomized Hadamard rotation + 4-bit
 * quantization library for NVIDIA B200 (sm_100a).
 *
 * What the library computes
 * -------------------------
 * The randomized Hadamard transform (RHT) of activation rows followed by a
 * 4-bit quantizer, as discussed on these pages:
 *   - "QuaRot: Outlier-Free 4-Bit Inference in Rotated LLMs" (OpenReview
 *     reviews): review 1 Summary (online Hadamard run with the fast
 *     Walsh-Hadamard algorithm), review 2 Summary (the RHT is invertible up to
 *     machine epsilon; activations are then rounded to nearest INT4),
 *     review 3 Questions (the Hadamard block computes Y = X H^T), final
 *     comments (RHT per batch of tokens = data parallel; RHT for the KV cache).
 *   - "Bug: Qwen3-8B integration issue" (KronQ issue #2), Model Details table:
 *     12288 = 12 x 1024 is Hadamard-compatible.
 *   - "Methodology checks for NVFP4 W4A4 on Qwen3-8B" (forum thread):
 *     block-Hadamard-128 (discrete_descent's note) and NVFP4 at 4.50 bits per
 *     element (krylov_schur section 3 table).
 *
 * Rotation.  For a row x of `dim` values, a +-1 sign vector s (the diagonal D)
 * and Hadamard blocks of width b (b = dim when block == 0):
 *     y_i = (1/sqrt(b)) * sum_j H_b[i][j] * s_j * x_j      (inside each block)
 * H_b is the Sylvester-Hadamard matrix in natural order,
 * H[i][j] = (-1)^popcount(i & j), when b is a power of two, and
 * Paley-12 (construction I, q = 11) kron Sylvester(b/12) when b = 12 * 2^k
 * (full-row mode only).  The inverse is x_j = s_j * sum_i H_b[i][j] y_i / sqrt(b).
 *
 * Quantizers (readings of points the pages leave open are noted):
 *   INT4 symmetric per token: scale = fp32(amax_row / 7), q = clamp(rint(y /
 *     scale), -8, 7), ties to even.  A zero row has scale 0 and codes 0.
 *   INT4 asymmetric per group of `group` elements: scale = fp16((max - min) /
 *     15), z = rint(-min / scale) stored as fp16, u = clamp(rint(y / scale) + z,
 *     0, 15).
 *   NVFP4: tensor scale t = fp32(amax_tensor / 2688) (2688 = 6 * 448) when
 *     dynamic, else supplied; per 16 elements r = fp32(amax_16 / (6 t)),
 *     block scale s_b = E4M3(r) (nearest even, saturating at 448), codes =
 *     E2M1(y / (value(s_b) * t)) (nearest even, saturating at 6), sign bit set
 *     when y < 0.
 *   Scales are computed from the exact rotated values (the library recomputes
 *   the deciding elements in fp64 when its fp32 transform cannot decide the
 *   rounding), so they equal an fp64 evaluation of the formulas bit for bit.
 *
 * Layouts (all row-major, no padding between rows):
 *   x            [tokens, dim] of fp32 or bf16 (kq_dtype).
 *   out          [tokens, dim] fp32.
 *   codes        [tokens, dim/2] bytes; element 2k in bits 0-3, 2k+1 in
 *                bits 4-7.  INT4 symmetric: two's complement nibble.
 *                INT4 asymmetric: 0..15.  NVFP4: E2M1 (bit 3 = sign).
 *   INT4 sym scales   fp32 [tokens].
 *   INT4 asym scales  fp16 [tokens, dim/group], zeros fp16 [tokens, dim/group].
 *   NVFP4 block_scales E4M3 bytes [tokens, dim/16]; tensor_scale one fp32.
 *   signs        int8 [dim] of +1/-1, or NULL (no D).
 *
 * Ownership and execution: every pointer is a device pointer owned by the
 * caller.  The library never allocates, frees, synchronizes, or keeps a pointer
 * after a call returns.  Work is enqueued on `stream` (NULL = the legacy
 * default stream) and runs asynchronously.  Calls are safe from several host
 * threads on different streams; outputs of calls that overlap on the GPU must
 * not alias.
 *
 * Errors: arguments are validated on the host before anything is launched.  A
 * bad argument returns KQ_ERR_INVALID_ARG / KQ_ERR_UNSUPPORTED /
 * KQ_ERR_MISALIGNED and enqueues nothing.  KQ_ERR_CUDA means a launch failed
 * (the CUDA error is reported by kq_last_cuda_error()).  No call traps on the
 * device.  Inputs must be finite; NaN or Inf inputs give unspecified outputs.
 * tokens == 0 is a valid no-op: shapes and flags are still checked, but
 * data pointers may then be NULL.
 *
 * Supported shapes:
 *   dim = 2^k with 32 <= dim <= 16384, or dim = 12 * 2^k with
 *   384 <= dim <= 12288 (the 12 * 2^k form only with block == 0).
 *   block = 0 (Hadamard over the whole row) or a power of two with
 *   16 <= block <= dim that divides dim.
 * Alignment: x, out and codes 16-byte aligned; scales/zeros/block_scales at
 * their element size.
 */
#ifndef KQ_H
#define KQ_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define KQ_API __attribute__((visibility("default")))
#else
#define KQ_API
#endif

struct CUstream_st;
/* Same type as cudaStream_t. */
typedef struct CUstream_st* kq_stream_t;

typedef enum {
  KQ_OK = 0,
  KQ_ERR_INVALID_ARG = -1,  /* null pointer, negative size, bad flag combination */
  KQ_ERR_UNSUPPORTED = -2,  /* shape, block, group or dtype outside the list above */
  KQ_ERR_MISALIGNED = -3,   /* a pointer breaks the alignment rule */
  KQ_ERR_CUDA = -4          /* a kernel launch or memset failed */
} kq_status;

typedef enum { KQ_F32 = 0, KQ_BF16 = 1 } kq_dtype;

/* flags */
enum {
  KQ_INVERSE = 1,        /* kq_rht: inverse transform x = D H^T y / sqrt(b) */
  KQ_SCALE_STATIC = 2,   /* kq_rht_quant_nvfp4: *tensor_scale is an input */
  KQ_SCALE_DYNAMIC = 4,  /* kq_rht_quant_nvfp4: *tensor_scale is computed and written */
  KQ_SCALES_MMA = 8,     /* kq_rht_quant_nvfp4: block scales in the tensor-core layout */
  KQ_DYN_STATS = 16,     /* KQ_SCALE_DYNAMIC: run the statistics phase (see below) */
  KQ_DYN_EXACT = 32,     /* KQ_SCALE_DYNAMIC: run the exact-maximum phase */
  KQ_DYN_QUANT = 64      /* KQ_SCALE_DYNAMIC: run the quantization phase */
};

/* formats for kq_dequant */
enum { KQ_FMT_INT4_SYM = 0, KQ_FMT_INT4_ASYM = 1, KQ_FMT_NVFP4 = 2, KQ_FMT_MXFP4 = 3 };

/*
 * kq_rht -- rotation only, fp32 output.
 * Forward (flags = 0): out = y as defined above (QuaRot reviews, review 2
 * Summary and review 3 Questions: Y = X H^T).  Inverse (flags = KQ_INVERSE):
 * out = x_j = s_j sum_i H[i][j] y_i / sqrt(b), the exact inverse of the forward
 * map ("fully invertible up to machine epsilon", review 2 Summary).
 * x: [tokens, dim] fp32 or bf16; signs: int8[dim] or NULL; out: fp32
 * [tokens, dim] (may not alias x).
 */
KQ_API kq_status kq_rht(const void* x, int dtype, int64_t tokens, int dim,
                        int block, const int8_t* signs, float* out, int flags,
                        kq_stream_t stream);

/*
 * kq_rht_quant_int4 -- rotation fused with INT4 quantization into packed
 * nibbles (QuaRot reviews, review 2 Summary/Weaknesses: RTN INT4 on rotated
 * activations; final comments: KV cache at 4 bits; NVFP4 thread,
 * discrete_descent's INT4-g128 note).
 * asym == 0: symmetric per token; group must be 0; scales = fp32 [tokens];
 *            zeros must be NULL.
 * asym == 1: asymmetric per group; group must be 128 and divide dim;
 *            scales and zeros = fp16 [tokens, dim/group].
 * codes: [tokens, dim/2] bytes.
 */
KQ_API kq_status kq_rht_quant_int4(const void* x, int dtype, int64_t tokens,
                                   int dim, int block, const int8_t* signs,
                                   int group, int asym, uint8_t* codes,
                                   void* scales, void* zeros,
                                   kq_stream_t stream);

/*
 * kq_rht_quant_int4_kv -- kq_rht_quant_int4 with asym = 1 that writes each
 * token straight into a KV cache (QuaRot reviews, final comments: the KV
 * cache at 4 bits with a per-head 128-point Hadamard): token t's codes,
 * scales and zero points go to cache row slot_mapping[t] instead of row t.
 * A negative slot skips the token (padding); slots at or above num_slots
 * are skipped too (nothing is written).  Two tokens with the same slot:
 * either one's row ends up there.
 * x: bf16 [tokens, dim]; block = 128 and group = 128 (one Hadamard block per
 * head); signs: int8[dim] or NULL, 16-byte aligned.  slot_mapping: int64
 * [tokens] in device memory, 8-byte aligned.  codes_cache: [num_slots, dim/2]
 * (16-byte aligned); scales_cache, zeros_cache: fp16 [num_slots, dim/128].
 * Rows not named by the mapping are left as they are.  Errors: as
 * kq_rht_quant_int4, KQ_ERR_UNSUPPORTED for another dtype, block or group.
 */
KQ_API kq_status kq_rht_quant_int4_kv(const void* x, int dtype, int64_t tokens,
                                      int dim, int block, const int8_t* signs,
                                      int group, const int64_t* slot_mapping,
                                      int64_t num_slots, uint8_t* codes_cache,
                                      uint16_t* scales_cache, uint16_t* zeros_cache,
                                      kq_stream_t stream);

/*
 * kq_rht_quant_nvfp4 -- rotation fused with NVFP4 quantization (NVFP4 thread,
 * krylov_schur section 3 table: E2M1 codes + one E4M3 scale per 16 elements,
 * 4.50 bits per element; per-tensor fp32 scale).
 * flags must hold exactly one of KQ_SCALE_STATIC (tensor_scale is read) or
 * KQ_SCALE_DYNAMIC (tensor_scale = fp32(amax/2688) of this call's rotated
 * tensor is computed and written).  For the same tensor scale both modes give
 * identical codes and block scales.
 * Dynamic mode needs `workspace`, a device buffer of at least
 * kq_workspace_size(tokens, dim, block) bytes, 16-byte aligned; its contents on
 * entry do not matter and are clobbered.  Static mode ignores it.
 * codes: [tokens, dim/2]; block_scales: E4M3 [tokens, dim/16]; tensor_scale:
 * one fp32 in device memory.
 * Dynamic mode runs three phases on the stream: (1) statistics -- the
 * workspace is cleared, each row's computed max |S| and error bound are
 * written, and bytes 0-3 of the workspace receive a lower bound on max |S|
 * over the rows (an fp32); (2) exact maximum -- rows whose upper bound
 * reaches that lower bound are transformed exactly and bytes 8-15 receive
 * max |S| over them (an fp64, unnormalized); (3) quantization with
 * t = fp32(max|S| / sqrt(b) / 2688), written to *tensor_scale.  Flags
 * KQ_DYN_STATS, KQ_DYN_EXACT and KQ_DYN_QUANT select a subset (none: all
 * three).  When all three run on bf16 rows with block = 128 and at most 8192
 * rows, phases 2 and 3 share one kernel launch (each CTA finds the exact
 * maximum before quantizing); the workspace then holds the same quantities.  A tensor split over ranks (QuaRot reviews, final comments: RHT
 * per batch of data is data parallelism) gets the tensor scale of the whole
 * tensor by running phase 1 on every rank, an all-reduce(max) of bytes 0-3
 * of every rank's workspace (as int32: a non-negative fp32 orders like its
 * bits), phase 2, an all-reduce(max) of bytes 8-15 (as int64), then phase 3:
 * the rank holding the largest row finds it among its candidates, so every
 * rank gets the single-tensor result.  A rank with no rows sets both words
 * to zero itself (tokens == 0 launches nothing).
 * KQ_SCALES_MMA (optional, needs dim % 64 == 0 and 16-byte aligned
 * block_scales) writes the block scales instead in the scale-factor layout of
 * the tcgen05 block-scaled MMA, which kq_gemm_nvfp4 reads: 512-byte atoms of
 * 128 rows x 4 blocks; the scale of row r, block c sits at byte
 * ((r / 128) * (dim / 64) + c / 4) * 512 + (r % 32) * 16 + ((r / 32) % 4) * 4 + c % 4.
 * The buffer then holds ceil(tokens / 128) * 128 * dim / 16 bytes; the bytes of
 * the padding rows are not written.  Codes and scale values are the same as
 * without the flag.  kq_dequant and kq_dequant_rht_inverse read the row-major
 * layout only.
 */
KQ_API kq_status kq_rht_quant_nvfp4(const void* x, int dtype, int64_t tokens,
                                    int dim, int block, const int8_t* signs,
                                    uint8_t* codes, uint8_t* block_scales,
                                    float* tensor_scale, void* workspace,
                                    size_t ws_bytes, int flags,
                                    kq_stream_t stream);

/*
 * kq_rht_quant_mxfp4 -- rotation fused with MXFP4 quantization (named in the
 * NVFP4 thread, discrete_descent's comparison of rotations under NVFP4, MXFP4
 * and INT4-g128; the bit-level layout is the OCP Microscaling (MX) v1.0
 * format): E2M1 codes, one E8M0 power-of-two scale per 32 consecutive
 * elements, no tensor scale.  A block's scale is X = 2^e with
 * e = floor(log2(max |y|)) - 2 over the block, clamped to [-127, 127] and
 * stored as the byte e + 127 (an all-zero block stores 0); code = E2M1(y / X),
 * nearest even, saturating at 6.  The scale byte is exact: blocks whose
 * exponent the fp32 transform leaves undecided are recomputed in fp64.
 * codes: [tokens, dim/2] (16-byte aligned); scales: E8M0 bytes
 * [tokens, dim/32].  dim, block, signs and errors as for kq_rht.
 */
KQ_API kq_status kq_rht_quant_mxfp4(const void* x, int dtype, int64_t tokens,
                                    int dim, int block, const int8_t* signs,
                                    uint8_t* codes, uint8_t* scales,
                                    kq_stream_t stream);

/*
 * kq_dequant -- codes and scales back to fp32: each output is the exact
 * product of the code value and its scale(s), rounded once to fp32.
 * fmt = KQ_FMT_INT4_SYM: scales fp32 [tokens]; zeros and tensor_scale unused.
 * fmt = KQ_FMT_INT4_ASYM: scales, zeros fp16 [tokens, dim/group]; group = 128.
 * fmt = KQ_FMT_NVFP4: scales = E4M3 bytes [tokens, dim/16]; tensor_scale =
 *   device fp32.
 * fmt = KQ_FMT_MXFP4: scales = E8M0 bytes [tokens, dim/32]; tensor_scale and
 *   zeros unused.
 * out: fp32 [tokens, dim].
 */
KQ_API kq_status kq_dequant(int fmt, const uint8_t* codes, const void* scales,
                            const void* zeros, const float* tensor_scale,
                            int64_t tokens, int dim, int group, float* out,
                            kq_stream_t stream);

/*
 * kq_dequant_rht_inverse -- the receiving end of the round trip in one call:
 * out = the inverse rotation (as kq_rht with KQ_INVERSE) of the values that
 * kq_dequant would write, x_j = s_j sum_i H[i][j] yq_i / sqrt(b) (QuaRot
 * reviews, review 2 Summary: the rotation is undone exactly by its transpose,
 * H^T = H for the Sylvester factor).  No intermediate tensor is written.
 * fmt, codes, scales, zeros, tensor_scale, group: as for kq_dequant.
 * dim, block, signs: the geometry and signs the codes were produced with (as
 * for kq_rht).  out: [tokens, dim], fp32 (out_dtype = KQ_F32) or bf16
 * (KQ_BF16: the fp32 result rounded to nearest even), 16-byte aligned; may
 * not alias the inputs.  Errors: as kq_dequant and kq_rht (KQ_ERR_UNSUPPORTED
 * for a geometry kq_rht rejects or another out_dtype, KQ_ERR_MISALIGNED,
 * KQ_ERR_INVALID_ARG); nothing is launched on an error.  Results agree with
 * kq_dequant followed by kq_rht(KQ_INVERSE) to fp32 rounding (the order of
 * the sums may differ).
 */
KQ_API kq_status kq_dequant_rht_inverse(int fmt, const uint8_t* codes,
                                        const void* scales, const void* zeros,
                                        const float* tensor_scale, int64_t tokens,
                                        int dim, int block, int group,
                                        const int8_t* signs, void* out,
                                        int out_dtype, kq_stream_t stream);

/*
 * kq_gemm_nvfp4 -- the 4-bit GEMM that consumes rotated, NVFP4-quantized
 * activations (QuaRot reviews, review 2 and review 4 Strengths: the speedup of
 * the rotated 4-bit path is the 4-bit GEMM; review 3 Questions: with Y = X H^T
 * applied to activations and weights alike, X W^T is unchanged), run on the
 * block-scaled tensor cores:
 *   C[m][n] = ta * tb * sum_k (E2M1(a[m][k]) E4M3(sa[m][k/16]))
 *                             (E2M1(b[n][k]) E4M3(sb[n][k/16])),
 * accumulated in fp32, scaled by ta * tb (fp32) and stored as fp32 or bf16.
 *   a_codes  [m, k/2] packed E2M1 codes (element 2i in the low nibble), as
 *            kq_rht_quant_nvfp4 writes them;  b_codes [n, k/2] likewise.
 *   a_scales, b_scales  E4M3 block scales in the KQ_SCALES_MMA layout, buffers
 *            of ceil(rows / 128) * 128 * k / 16 bytes (padding rows are read;
 *            their products reach only output rows that are not stored).
 *   a_tensor_scale, b_tensor_scale  one fp32 each, device memory.
 *   c        [m, n] row-major, c_dtype KQ_F32 or KQ_BF16 (round to nearest even).
 * Device pointers owned by the caller, 16-byte aligned (tensor scales 4);
 * C must not alias the inputs.  Supported: m >= 0 (m == 0 is a no-op),
 * n % 128 == 0, k % 256 == 0.  Errors: KQ_ERR_INVALID_ARG (null pointer,
 * non-positive n or k), KQ_ERR_UNSUPPORTED (shape or c_dtype),
 * KQ_ERR_MISALIGNED, KQ_ERR_CUDA; nothing is launched on an error.
 */
KQ_API kq_status kq_gemm_nvfp4(const uint8_t* a_codes, const uint8_t* a_scales,
                               const float* a_tensor_scale, const uint8_t* b_codes,
                               const uint8_t* b_scales, const float* b_tensor_scale,
                               int64_t m, int64_t n, int64_t k, void* c, int c_dtype,
                               kq_stream_t stream);

/*
 * kq_device_errors -- failure reports of the tensor-core kernels.  Every
 * wait of those kernels is bounded (about two seconds); when one runs out the
 * kernel records it in its family's error word and returns without writing
 * the affected outputs, instead of hanging.  flags: host array of 6 words,
 * filled and then cleared on the device: [0] the 4096-wide kernels (bit 0: a
 * wait ran out; bit 1: the fix-up queue stayed full, a block kept its
 * provisional scale; bit 2: a fix-up warp waited too long), [1] the
 * 12288-wide kernel, [2] the block-128 GEMM kernel, [3] the fused dequant +
 * inverse kernel, [4] kq_diag_wait_timeout (bit 0), [5] the NVFP4 GEMM
 * (since ABI version 1.1; 1.0 had 5 words).  All zero: no failure
 * since the last call.  The read synchronizes the device.  The pages have no
 * counterpart to this entry point.
 */
KQ_API kq_status kq_device_errors(unsigned int* flags);

/*
 * kq_diag_wait_timeout -- diagnostic, no page counterpart: one CTA waits on
 * a barrier that nothing arrives at, with a limit of limit_cycles clock
 * cycles (1 .. 4e9), then sets bit 0 of word [4] of kq_device_errors and
 * exits.  It exercises the bounded-wait failure path without any fault.
 */
KQ_API kq_status kq_diag_wait_timeout(long long limit_cycles, kq_stream_t stream);

/*
 * kq_rht_quant_nvfp4_dynamic_noalloc -- kq_rht_quant_nvfp4 with
 * KQ_SCALE_DYNAMIC, for callers that cannot allocate device memory.  The
 * pages have no counterpart to this entry point; it exists for integration.
 *
 * Who needs it: code that may not call cudaMalloc or any allocator -- a plugin
 * whose host framework owns all device memory and passes it no workspace, or a
 * serving loop that reserves HBM up front and cannot afford cudaMalloc (which
 * may synchronize the device) on its hot path.  The caller still passes the
 * input and all outputs, exactly as for kq_rht_quant_nvfp4.
 *
 * The dynamic tensor scale's workspace lives instead in a fixed array of
 * KQ_NOALLOC_SCRATCH_BYTES (1 MiB) of the library's own device memory, which
 * every GPU that loads the library holds until the process exits.  tokens
 * above KQ_NOALLOC_MAX_TOKENS returns KQ_ERR_UNSUPPORTED and launches nothing.
 * The call allocates nothing and calls no allocating routine.
 *
 * The first call on each device looks up the array's device address (with
 * that device current) and caches it together with the current CUDA context;
 * a call in another context (another context made current, or the primary
 * context recreated after cudaDeviceReset) looks it up again.  Make the first
 * call in each context before any stream capture.  All calls share the one array and it keeps the last call's
 * contents (each call clears what must start at zero), so calls that overlap
 * on the GPU -- on different streams or from different threads -- race and
 * must be serialized by the caller.
 */
#define KQ_NOALLOC_SCRATCH_BYTES (1u << 20)
#define KQ_NOALLOC_MAX_TOKENS ((KQ_NOALLOC_SCRATCH_BYTES - 16u) / 8u)
KQ_API kq_status kq_rht_quant_nvfp4_dynamic_noalloc(
    const void* x, int dtype, int64_t tokens, int dim, int block, const int8_t* signs,
    uint8_t* codes, uint8_t* block_scales, float* tensor_scale, kq_stream_t stream);

/* Bytes of workspace the dynamic NVFP4 path needs (0 on bad arguments). */
KQ_API size_t kq_workspace_size(int64_t tokens, int dim, int block);

/* Human-readable name of a status code (static string). */
KQ_API const char* kq_status_str(int status);

/* The CUDA error code behind the calling thread's last KQ_ERR_CUDA (0 if none). */
KQ_API int kq_last_cuda_error(void);

/*
 * Diagnostic (the pages have no counterpart): arms a simulated launch failure
 * for the calling thread.  The next call of an entry point that passes its
 * argument checks and would enqueue work enqueues nothing, returns
 * KQ_ERR_CUDA and sets kq_last_cuda_error() to cuda_error; that disarms it.
 * Calls rejected by their checks, and calls with tokens == 0, leave it armed.
 * 0 disarms.  It lets the error path of every entry point be tested on a
 * machine without a GPU, and without making a GPU fail.
 */
KQ_API void kq_diag_fail_next_launch(int cuda_error);

/* ABI version: (major << 16) | minor. */
KQ_API int kq_version(void);

/*
 * Diagnostic: two accumulation steps of the tensor-core contraction the
 * 4096-wide bf16 paths are built on, on caller data.  The pages have no
 * counterpart; the test suite uses it to check the accumulation model the
 * kernels' error bound rests on (each tcgen05.mma step truncates its terms
 * toward zero to a multiple of 2^(emax - 25) and its sum to fp32).
 *   a   bf16 bits [128][32], row-major (M x K).
 *   b   bf16 bits [32][128], row-major (K x N).
 *   d1  fp32 [128][128]: A[:, 0:16] B[0:16, :] (accumulation from zero).
 *   d2  fp32 [128][128]: d1 + A[:, 16:32] B[16:32, :] (accumulated in place).
 *   status  one uint32: 0, or 1 if a wait timed out (then d1, d2 are undefined).
 * Device pointers owned by the caller; one CTA is enqueued on `stream`.
 */
KQ_API kq_status kq_diag_tc_steps(const uint16_t* a, const uint16_t* b, float* d1, float* d2,
                                  unsigned int* status, kq_stream_t stream);

/*
 * Diagnostic: the same two steps with fp16 operands (a and b hold fp16 bits),
 * the operand type of the fused dequant + inverse kernel.  Arguments, layout
 * and errors as kq_diag_tc_steps.  The pages have no counterpart.
 */
KQ_API kq_status kq_diag_tc_steps_f16(const uint16_t* a, const uint16_t* b, float* d1,
                                      float* d2, unsigned int* status, kq_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* KQ_H */
