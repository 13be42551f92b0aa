/*
 * fp4mx.h — C ABI of libfp4mx.so: block-scaled 4-bit (E2M1) microscaling on NVIDIA B200 (sm_100a).
 *
 * Every entry point takes plain pointers and sizes.  Pointers documented as "device" must point to
 * memory the caller allocated on the current CUDA device; the library never allocates, frees or
 * synchronises.  All work is enqueued on the caller's `stream` (a cudaStream_t passed as void*;
 * NULL = the legacy default stream) and returns as soon as it is enqueued.
 *
 * Error behaviour (all entry points):
 *   - argument errors (bad sizes, unsupported combinations, NULL required pointers, misaligned
 *     buffers) return FP4_EINVAL or FP4_EUNSUPPORTED synchronously, before anything is launched;
 *     a format is never silently replaced by another one;
 *   - a failed launch returns FP4_ECUDA; fp4_last_error() then describes it;
 *   - data problems are never trapped on the device: non-finite inputs are counted in
 *     fp4_counts.nonfinite and the outputs of the affected blocks are unspecified.
 *
 * Sources the operations follow (cited by page title and section):
 *   [E]  "Sub-4-Bit Microscaling (NVFP4, MXFP4 & Walsh-Hadamard Rotation)" (Eluvix docs),
 *        §1 E2M1, §2 MXFP4 vs NVFP4, §3 Walsh-Hadamard rotation.
 *   [A]  "MXFP4 Quantization: Audit the 4.25-Bit Blocks", sections "Read the FP4 E2M1 value
 *        lattice", "Read the shared E8M0 scale", "Encode one MXFP4 block step by step",
 *        "Publish the MXFP4 audit receipt".
 *   [X]  metrale `hardware::exec` module docs: the activation format picks the MMA kind; NVFP4
 *        runs on the block-scaled FP4 MMA.
 *   [P]  podcast "Adaptive Block-Scaled Data Types for FP4 Training" (segments on block scaling,
 *        the Hadamard transform and stochastic rounding, and Four Over Six).
 */
#ifndef FP4MX_H
#define FP4MX_H

#include <stddef.h>

#if defined(__GNUC__)
#define FP4_API __attribute__((visibility("default")))
#else
#define FP4_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum fp4_status {
  FP4_OK = 0,
  FP4_EINVAL = 1,        /* bad argument: size, NULL pointer, alignment, layout precondition */
  FP4_EUNSUPPORTED = 2,  /* well-formed request for a combination this library does not run */
  FP4_ECUDA = 3          /* a CUDA call or kernel launch failed */
} fp4_status;

typedef enum fp4_dtype { FP4_F32 = 0, FP4_BF16 = 1 } fp4_dtype;

/* MXFP4: 32 E2M1 elements share one E8M0 byte (value 2^(byte-127), 0xFF = NaN, never produced).
 * NVFP4: 16 E2M1 elements share one E4M3 byte (positive, OCP E4M3FN: bias 7, max 448) under one
 *        FP32 per-tensor global scale s_g.   [E] §2, [P] block-scaling segment.
 * IF4:   NVFP4 whose blocks may instead hold INT4: a scale byte with bit 7 set (the sign bit NVFP4
 *        never uses) marks a block of sign-magnitude integers k in -7..7 (bit 3 the sign, bits 0-2
 *        |k|) with value k * d * s7, d the E4M3 value of the low 7 bits, s7 = fl(s_g * fl(6/7)).
 *        Written by nvfp4_quantize with FP4_NV_IF4; read by fp4_dequantize.  [P] IF4 segment. */
typedef enum fp4_format { FP4_MXFP4 = 0, FP4_NVFP4 = 1, FP4_IF4 = 2 } fp4_format;

/* NVFP4 block mode (the `mode` argument of the NVFP4 quantisers).
 * PLAIN   : every block scales its maximum to 6.
 * FOUR_SIX: each block also tries a maximum of 4 and keeps the lower-error one ([P] Four Over
 *           Six segment); the global scale uses M = 256.
 * IF4     : each block also tries INT4 on the step 6/7 of the E2M1 unit and keeps the lower-error
 *           one, flagged in scale bit 7 (format FP4_IF4; [P] IF4 segment); M = 448, round to
 *           nearest only. */
typedef enum fp4_nv_mode { FP4_NV_PLAIN = 0, FP4_NV_FOUR_SIX = 1, FP4_NV_IF4 = 2 } fp4_nv_mode;

/* RNE: round to nearest on the E2M1 lattice {0,.5,1,1.5,2,3,4,6}, an exact tie takes the code with
 * the even mantissa bit ([A] "Read the FP4 E2M1 value lattice").
 * STOCHASTIC: round up to the next lattice point with probability (a-lo)/(hi-lo), decided by one
 * 32-bit Philox4x32-10 word per element ([P] stochastic-rounding segment).  The word for flat
 * row-major element index i is output word (i & 3) of Philox4x32-10 with key (seed low 32 bits,
 * seed high 32 bits) and counter (i>>2 low 32, i>>2 high 32, 0, 0); the element rounds up iff
 * word < ceil(p * 2^32).  Block scales are always chosen with RNE. */
typedef enum fp4_round { FP4_RNE = 0, FP4_STOCHASTIC = 1 } fp4_round;

/* MXFP4 shared-exponent rule.
 * OCP_FLOOR : e = floor(log2 amax) - 2 clamped to [-127,127]; the block top may exceed 6 and
 *             saturate ([A] "Read the shared E8M0 scale", worked example with max 13).
 * NOSAT_CEIL: the smallest e with amax <= 6 * 2^e, clamped; never saturates but can leave the top
 *             lattice steps 4 and 6 unused ([E] §2 "sawtooth cliff").
 * An all-zero block uses e = 0 (byte 127) under both rules. */
typedef enum fp4_mx_policy { FP4_MX_OCP_FLOOR = 0, FP4_MX_NOSAT_CEIL = 1 } fp4_mx_policy;

/* Scale-byte layout.
 * ROWMAJOR : scales[r * (cols/B) + j] is the scale of block j of row r.
 * MMA_TILED: the layout the sm_100 block-scaled MMA reads from tensor memory.  Rows are grouped in
 *            tiles of 128 and block columns in groups of 4; each (128 x 4) tile is 512 contiguous
 *            bytes, tiles ordered block-column-group fastest:
 *              off(r, j) = ((r/128) * (cols/B/4) + j/4) * 512 + (r%32)*16 + ((r%128)/32)*4 + j%4
 *            Requires rows % 128 == 0 and (cols/B) % 4 == 0.  fp4_block_gemm requires it. */
typedef enum fp4_scale_layout { FP4_SCALES_ROWMAJOR = 0, FP4_SCALES_MMA_TILED = 1 } fp4_scale_layout;

/* Encoding counters, tensor totals.  Lives in DEVICE memory; every quantize call zeroes it on its
 * stream before counting.  underflow: nonzero source whose code is +-0.  saturation: normalised
 * magnitude strictly above 6 (clamped to +-6), an infinite one included.  nonfinite: Inf/NaN source elements.
 * blocks_four: blocks that took the alternative candidate: the max->4 scaling under FOUR_SIX,
 * INT4 under IF4 (whose saturation bound is 7 integer steps).  Counts come from the chosen
 * encoding only.  [A] "Read the FP4 E2M1 value lattice", "Expose outlier and dead-zone damage". */
typedef struct fp4_counts {
  unsigned long long underflow;
  unsigned long long saturation;
  unsigned long long nonfinite;
  unsigned long long blocks_four;
} fp4_counts;

/* Operation ids for fp4_workspace_size.  FP4_OP_NVFP4_QUANTIZE is nvfp4_quantize's need (8 KiB: one
 * 32-bit partial maximum per CTA of the amax pass, which the quantise pass reduces, so nothing is
 * zeroed between calls).  FP4_OP_FWHT_QUANTIZE is the minimum for fwht_quantize and
 * swiglu_fwht_quantize (the amax word); FP4_OP_FWHT_QUANTIZE_STORED the size that also holds the
 * fp32 rotation of a [rows, cols] tensor, which lets the two-pass NVFP4 call rotate once. */
typedef enum fp4_op { FP4_OP_MX_QUANTIZE = 0, FP4_OP_NVFP4_QUANTIZE = 1, FP4_OP_FWHT_QUANTIZE = 2,
                      FP4_OP_DEQUANTIZE = 3, FP4_OP_BLOCK_GEMM = 4, FP4_OP_FWHT_QUANTIZE_STORED = 5,
                      FP4_OP_BLOCK_GEMM_IF4 = 6 } fp4_op;

/* ---------------------------------------------------------------------------------------------
 * mx_quantize — MXFP4 quantisation of a row-major [rows, cols] tensor, blocks of 32 along rows.
 * Follows [A] "Encode one MXFP4 block step by step": per block amax, shared exponent e (policy),
 * y = x * 2^-e (exact), E2M1 encode (RNE or stochastic), saturate at 6, nibble pack.
 *   x      : device, [rows, cols] of `dtype`, 32-byte aligned (the same for every quantiser).
 *   block  : must be 32 (no block-size inference; anything else is FP4_EINVAL).
 *   q      : device, [rows, cols/2] bytes, 8-byte aligned; element 2j in the low nibble of byte j, 2j+1 high
 *            ([A] "Encode one MXFP4 block": values 0 and 1 share the first byte, low half first).
 *   scales : device, rows*cols/32 E8M0 bytes in `layout`.
 *   counts : device fp4_counts or NULL (no counting).
 * Preconditions: rows >= 0, cols % 32 == 0 (an incomplete block is rejected), cols > 0 if rows > 0.
 * Empty tensors (rows == 0) are accepted and launch nothing except zeroing `counts`. */
FP4_API fp4_status mx_quantize(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                       fp4_mx_policy policy, fp4_round round, unsigned long long seed,
                       fp4_scale_layout layout, unsigned char* q, unsigned char* scales,
                       fp4_counts* counts, void* stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_quantize — NVFP4 two-level quantisation, blocks of 16 along rows.  [E] §2, [P] Four Over
 * Six and IF4 segments.  Global scale s_g = fl(amax_t / (6*M)) with M = 448 (M = 256 under
 * FP4_NV_FOUR_SIX, the reduced global range that keeps the max->4 candidate finite); s_g = 1 when
 * amax_t == 0.  For target T (6, and also 4 under FOUR_SIX): inv_T = fl(1/fl(T*s_g)); block code =
 * E4M3_RNE_satfinite(fl(amax_b * inv_T)) with decoded value d; elements y = fl(x * fl(1/fl(d*s_g)))
 * are E2M1-encoded; a code of 0 encodes the whole block as signed zeros.  Under FOUR_SIX each block
 * keeps the candidate whose fp32 sum of squared dequantisation errors is strictly lower (ties
 * keep 6).  Under FP4_NV_IF4 the T = 6 block also gets an INT4 candidate: D7 = fl(d * s7),
 * s7 = fl(s_g * fl(6/7)), R7 = fl(1/D7); |k| = nearest integer (ties to even) to
 * min(|fl(x * R7)|, 7), the sign that of fl(x * R7); reconstruction fl(fl(k*d) * s7).  It is kept,
 * with scale bit 7 set, iff R7 is a finite nonzero number and its fp32 sequential error sum is
 * strictly below the E2M1 one (ties and NaN keep E2M1).  IF4 assumes s_g > 0: a caller-supplied
 * negative global scale gives in-bounds but unspecified bytes.
 *   mode       : fp4_nv_mode (0, 1 or 2; other values are FP4_EINVAL); FP4_NV_IF4 with
 *                FP4_STOCHASTIC is FP4_EUNSUPPORTED.
 *   global_in  : device float or NULL.  NULL: a first pass reduces amax_t over the tensor (two
 *                passes over x).  Non-NULL: the caller fixes s_g = *global_in (one pass).
 *   global_out : device float or NULL; receives the s_g used.
 *   q, scales, counts : as in mx_quantize (E4M3 scale bytes).
 *   workspace  : device, >= fp4_workspace_size(FP4_OP_NVFP4_QUANTIZE, rows, cols) bytes, 16-byte
 *                aligned; required when global_in == NULL.  Clobbered; needs no initialisation (the
 *                amax pass writes every word the quantise pass reads).
 * Preconditions: block == 16, cols % 16 == 0. */
FP4_API fp4_status nvfp4_quantize(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                          fp4_round round, int mode, unsigned long long seed,
                          fp4_scale_layout layout, const float* global_in, float* global_out,
                          unsigned char* q, unsigned char* scales, fp4_counts* counts,
                          void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * fwht_quantize — normalised Walsh-Hadamard rotation of every row (length d), fused ahead of the
 * quantiser.  [E] §3 "Orthogonal Walsh-Hadamard Outlier Rotation": H_d has entries +-1/sqrt(d)
 * (Sylvester order, H[i][j] = (-1)^popcount(i&j)/sqrt(d)) and is applied by O(d log2 d) butterflies.
 * The rotation is computed in fp32 in a fixed order: unnormalised radix-2 stages h = 1,2,4,...,d/2,
 * each mapping (a,b) -> (a+b, a-b) for index pairs (i, i+h) with (i & h) == 0, then one multiply by
 * c = fl(1/sqrt(d)).  The rotated fp32 values are then quantised exactly as nvfp4_quantize
 * (format FP4_NVFP4, block 16; the global amax is taken over the rotated tensor) or as
 * mx_quantize with FP4_MX_OCP_FLOOR (format FP4_MXFP4, block 32).  Stochastic rounding indexes
 * Philox by the flat element index of the rotated [rows, d] tensor.
 * With `signs` the rotation is randomised ([P], random Hadamard transform): Q = c * H * D, where
 * D = diag(+-1) negates channel i (before the butterflies) when bit i % 32 of signs[i / 32] is set.
 * Q is orthogonal, so rotating both GEMM operands along K with the same signs leaves A * B^T
 * unchanged up to quantisation.
 *   d           : power of two, 1024 <= d <= 16384.
 *   signs       : device uint32 [d / 32], 4-byte aligned, or NULL (plain rotation); caller-owned.
 *   rotated_out : device float [rows, d] or NULL; receives the rotated values.
 *   workspace   : device, 16-byte aligned; >= fp4_workspace_size(FP4_OP_FWHT_QUANTIZE) bytes when
 *                 NVFP4 runs without global_in (two passes).  Clobbered.
 *   other arguments as in nvfp4_quantize; four_six is the NVFP4 block mode (fp4_nv_mode:
 *   FP4_NV_PLAIN, FP4_NV_FOUR_SIX, or FP4_NV_IF4 with FP4_RNE only) and, with global_in/out,
 *   applies to FP4_NVFP4 only.
 * The two-pass NVFP4 call (global_in NULL) takes one of two routes with the same results: when
 * rotated_out is 32-byte aligned, or the workspace holds fp4_workspace_size(
 * FP4_OP_FWHT_QUANTIZE_STORED, rows, d) bytes, the first pass rotates once and stores the fp32
 * rotation there, and the second quantises the stored values; otherwise each pass rotates (no
 * extra memory, more arithmetic). */
FP4_API fp4_status fwht_quantize(const void* x, fp4_dtype dtype, long rows, long d,
                         const unsigned int* signs, fp4_format format,
                         int block, fp4_round round, int four_six, unsigned long long seed,
                         fp4_scale_layout layout, const float* global_in, float* global_out,
                         float* rotated_out, unsigned char* q, unsigned char* scales,
                         fp4_counts* counts, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * swiglu_fwht_quantize — the SwiGLU activation fused ahead of the (optionally randomised) rotation and
 * the quantiser.  [E] §3 places the rotation in the SwiGLU epilogue; here the activation
 * a = fl(SiLU(g) * u) is formed in fp32 from the two bf16 inputs and rotated without being stored, so
 * it is never rounded to bf16.  SiLU(g) = g * fl(1 / fl(1 + e^-g)); the exponential follows Cody and
 * Waite's argument reduction (x = n ln2 + r, n = rint(x log2 e), ln2 = 0x1.62ep-1 + 0x1.0bfbe8p-15)
 * with the degree-6 Taylor polynomial of e^r in Horner form and an exact scaling by 2^n; e^x = +Inf
 * above 88.5 and +0 below -103.  Every step is one fp32 rounding, so the activation is reproducible
 * bit for bit.  Everything after the activation is fwht_quantize.
 *   g, u  : device bf16 [rows, d] each, row-major, 32-byte aligned (dtype must be FP4_BF16, else
 *           FP4_EUNSUPPORTED).
 *   other arguments as in fwht_quantize. */
FP4_API fp4_status swiglu_fwht_quantize(const void* g, const void* u, fp4_dtype dtype, long rows, long d,
                                const unsigned int* signs, fp4_format format, int block, fp4_round round,
                                int four_six, unsigned long long seed, fp4_scale_layout layout,
                                const float* global_in, float* global_out, float* rotated_out,
                                unsigned char* q, unsigned char* scales, fp4_counts* counts,
                                void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * fp4_dequantize — x_hat = fl((v * d) * s_g) per element, v the E2M1 value of the nibble and d the
 * decoded block scale (v*d is exact); MXFP4 has no s_g (x_hat = v * 2^e, exact).  FP4_IF4 (block
 * 16): a block whose scale byte has bit 7 set is INT4, x_hat = fl((k * d) * s7) with d the E4M3
 * value of the low 7 bits and s7 = fl(s_g * fl(6/7)); other blocks follow NVFP4.  bf16 output is
 * the round-to-nearest-even of that fp32 value.  [A] "Encode one MXFP4 block step by step"
 * (reconstruction = lattice value times scale), [X] block scales applied in FP32, [P] IF4 segment.
 *   q, scales : device, as written by the quantisers (`layout` names the scale layout).
 *   global    : device float, NVFP4 and IF4 only (NULL for MXFP4).
 *   out       : device [rows, cols] of out_dtype, 16-byte aligned. */
FP4_API fp4_status fp4_dequantize(const unsigned char* q, const unsigned char* scales, fp4_format format,
                          int block, fp4_scale_layout layout, const float* global, long rows,
                          long cols, fp4_dtype out_dtype, void* out, void* stream);

/* ---------------------------------------------------------------------------------------------
 * fp4_block_gemm — W4A4 block-scaled GEMM C = alpha * A * B^T on the sm_100 tensor cores
 * (tcgen05.mma kind::mxf4nvf4 with block scales, FP32 accumulation in tensor memory).
 * [E] §2 (NVFP4 on the 5th-generation tensor core), [X] (NVFP4 activations take the block-scaled
 * FP4 MMA).  C[m][n] = alpha * sum_kb dA[m][kb] * dB[n][kb] * sum_{k in kb} vA[m][k] * vB[n][k],
 * alpha = (*Ag) * (*Bg) for NVFP4 and 1 for MXFP4; C is stored as bf16 (RNE), row-major with
 * leading dimension ldc (elements).
 *   Aq : device [M, K/2] packed E2M1, K-major (as written by the quantisers for a [M, K] tensor).
 *   As : device scales of A in FP4_SCALES_MMA_TILED layout (E4M3 for NVFP4, E8M0 for MXFP4).
 *   Bq, Bs : the same for B [N, K].
 *   Ag, Bg : device floats (NVFP4 global scales); ignored (may be NULL) for MXFP4.
 *   workspace : device, >= fp4_workspace_size(FP4_OP_BLOCK_GEMM, M, N) bytes, 16-byte aligned; the
 *               kernel's status word (0 = ok, nonzero = a bounded pipeline wait gave up) is its
 *               first 4 bytes; see fp4_gemm_status_word.
 * FP4_IF4 ([P] IF4 segment): blocks whose scale byte has bit 7 set hold INT4 integers k whose step
 * is six sevenths of the E2M1 unit, so a mixed FP4 x INT4 block pair carries the factor 6/7 and an
 * INT4 x INT4 pair 36/49.  No block-scaled MMA kind carries those factors (E4M3 and UE8M0 block
 * scales cannot hold d * 6/7), so both operands are first expanded into the workspace as fp16
 * without the per-tensor scale: v * d for an E2M1 block (exact) and the RNE fp16 of
 * fl(fl(k * d) * fl(6/7)) for an INT4 block (relative error below 2^-11).  Then tcgen05.mma
 * kind::f16 computes C = (*Ag) * (*Bg) * A16 * B16^T with FP32 accumulation.  An NVFP4 operand is
 * an IF4 operand without INT4 blocks.  Ag and Bg are required; the workspace must hold
 * fp4_workspace_size(FP4_OP_BLOCK_GEMM_IF4, M + N, K) bytes (the status word first).
 * Preconditions: M % 128 == 0, N % 256 == 0, K % 256 == 0, ldc >= N, ldc % 8 == 0, all pointers
 * 16-byte aligned.  Other shapes return FP4_EUNSUPPORTED. */
FP4_API fp4_status fp4_block_gemm(fp4_format format, int M, int N, int K,
                          const unsigned char* Aq, const unsigned char* As, const float* Ag,
                          const unsigned char* Bq, const unsigned char* Bs, const float* Bg,
                          void* C, long ldc, void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * fp4_to_e4m3 — E2M1 nibbles to E4M3 bytes through the exact identity of [X] (metrale
 * `hardware::exec`): with a nibble in bits 7..4 of a byte b, (b & 0x80) | ((b & 0x70) >> 2) is the
 * E4M3 encoding of the nibble's value times 2^-6 (-0 gives 0x80).  It lets the FP8 tensor-core
 * MMA take FP4 operands exactly (fp4_block_gemm_e4m3).
 *   q   : device [rows, cols/2] packed E2M1 as the quantisers write (element 2j low nibble), 16-byte aligned.
 *   out : device [rows, cols] bytes, element k of a row at byte k, 16-byte aligned.  Caller-owned.
 * Preconditions: rows >= 0, cols > 0, cols % 32 == 0; rows == 0 launches nothing. */
FP4_API fp4_status fp4_to_e4m3(const unsigned char* q, long rows, long cols, unsigned char* out, void* stream);

/* ---------------------------------------------------------------------------------------------
 * fp4_block_gemm_e4m3 — the MXFP4 block-scaled GEMM on the FP8 tensor-core path: C = A * B^T with
 * the operands given as their E4M3 expansions (fp4_to_e4m3 of MXFP4 nibbles) and the MXFP4 E8M0
 * scales unchanged, run as tcgen05.mma kind::mxf8f6f4 block_scale scale_vec::1X (one scale per 32
 * values) with FP32 accumulation; the epilogue multiplies by 2^12, undoing the 2^-6 of each
 * operand, so C equals fp4_block_gemm(FP4_MXFP4, ...) up to the order of the FP32 accumulation.
 * [X] (FP4 operands run exactly on the FP8 MMA after that conversion) — an independent second tensor-
 * core GEMM for cross-checking the FP4 one.  MXFP4 only: the FP8 kind takes UE8M0 scales per 32,
 * which cannot carry NVFP4's E4M3 scales per 16.
 *   A8 : device [M, K] E4M3 bytes; B8 : device [N, K] E4M3 bytes (K-major).
 *   As, Bs : device MXFP4 scales in FP4_SCALES_MMA_TILED layout (as written by mx_quantize).
 *   C, ldc, workspace, ws_bytes : as in fp4_block_gemm (workspace of FP4_OP_BLOCK_GEMM size).
 * Preconditions: M % 128 == 0, N % 256 == 0, K % 128 == 0 (else FP4_EUNSUPPORTED), ldc >= N,
 * ldc % 8 == 0, all pointers 16-byte aligned.  Runs on the 1-SM kernel (128 x 256 tiles). */
FP4_API fp4_status fp4_block_gemm_e4m3(int M, int N, int K, const unsigned char* A8, const unsigned char* As,
                                       const unsigned char* B8, const unsigned char* Bs, void* C, long ldc,
                                       void* workspace, size_t ws_bytes, void* stream);

/* ---------------------------------------------------------------------------------------------
 * nvfp4_quantize_noalloc — nvfp4_quantize without a caller-supplied workspace, for callers that
 * cannot allocate device memory: for example a plugin inside another runtime that receives only
 * its input and output buffers, or a latency-critical loop that must not call cudaMalloc (which
 * can synchronise the device).  The source pages have no counterpart; this is a library
 * convenience.
 *   Arguments, results and errors are those of nvfp4_quantize, minus `workspace`/`ws_bytes`.
 *   Scratch: a fixed 8 KiB array in this library's device memory (per GPU, kept until the process
 *   exits).  A shape whose workspace need (fp4_workspace_size) exceeds it is rejected with
 *   FP4_EUNSUPPORTED; today every shape needs the same 8 KiB and fits.
 *   Allocation: none (no cudaMalloc, no cudaFree, no allocating library call).
 *   First call on a device: looks up the array's device address with cudaGetSymbolAddress, with
 *   that device current; make that first call before any stream capture.  The address is kept for
 *   the life of the process: after a cudaDeviceReset (or anything else that tears down and
 *   re-creates the device's primary context) it is stale, so such a process must not call this
 *   entry point again.
 *   Sharing: all calls on a device share the one array and it keeps the last call's contents; each
 *   call's amax pass overwrites every word its quantise pass reads.  Calls that overlap on the GPU
 *   (in flight at the same time on different streams) race on it: serialise them. */
FP4_API fp4_status nvfp4_quantize_noalloc(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                                          fp4_round round, int mode, unsigned long long seed,
                                          fp4_scale_layout layout, const float* global_in, float* global_out,
                                          unsigned char* q, unsigned char* scales, fp4_counts* counts,
                                          void* stream);

/* Bytes of device workspace `op` needs for the given sizes (rows/cols; M/N for the GEMM). */
FP4_API size_t fp4_workspace_size(fp4_op op, long rows, long cols);

/* Byte offset, inside fp4_block_gemm's workspace, of its 32-bit device status word.  Bit i set
 * means the pipeline wait at site i gave up: 0 a stage slot to refill, 1 the accumulator to be
 * released, 2 a stage to land, 3 the accumulator to be ready, 4 the last stage releases, 5 the last
 * accumulator release, 6-9 the scale-copy stages of the 2-SM kernel.  The kernel then stops every
 * role, waits (bounded) for the copies and MMAs it issued, frees tensor memory and returns; its
 * output is incomplete.  A failure of this kind is reported, never trapped ([H]: refuse, never
 * substitute). */
FP4_API size_t fp4_gemm_status_word(void);

/* Limit, in nanoseconds, of each pipeline wait inside the GEMM kernels launched after this call
 * (fp4_block_gemm, fp4_block_gemm_e4m3); returns the previous limit.  The default is 2000000000
 * (2 s), far above any wait of a working pipeline.  A small limit makes the kernel give up early,
 * which is how the fault path is exercised without faulting: 0 gives up at the first wait that has
 * not completed already.  Process-wide; launches already enqueued keep their limit. */
FP4_API unsigned long long fp4_set_gemm_wait_limit(unsigned long long ns);

/* Static description of a status code. */
FP4_API const char* fp4_status_str(fp4_status s);

/* Human-readable detail of the last non-OK status returned on the calling thread. */
FP4_API const char* fp4_last_error(void);

#ifdef __cplusplus
}
#endif

#endif /* FP4MX_H */
