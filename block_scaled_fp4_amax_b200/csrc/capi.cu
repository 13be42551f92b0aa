// capi.cu — the extern "C" boundary of libfp4mx.so (declared in include/fp4mx.h).
//
// Each entry point validates its arguments on the host and returns an error before anything is
// enqueued; a format or block size is never inferred or silently replaced (the "refuse, never
// substitute" rule of the heterogeneous-microscaling evaluation page, and the reject rules of the
// MXFP4 audit page's "Publish the MXFP4 audit receipt" section).  Valid calls enqueue work on the
// caller's stream and return without synchronising.
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include "../../include/fp4mx.h"
#include "launch.h"

namespace {

thread_local char g_err[512] = "";

fp4_status fail(fp4_status s, const char* fmt, ...) __attribute__((format(printf, 2, 3)));
fp4_status fail(fp4_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

fp4_status cuda_fail(cudaError_t e, const char* what) {
  return fail(FP4_ECUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

bool aligned(const void* p, size_t a) { return (reinterpret_cast<uintptr_t>(p) % a) == 0; }

constexpr long long kMaxElems = 1LL << 40;
constexpr size_t kAmaxWorkspace = 256;  // the rotations' 32-bit amax word, padded
// nvfp4_quantize's amax pass: one 32-bit partial maximum per CTA of that pass
constexpr size_t kAmaxSlotsWorkspace = fp4k::kAmaxSlots * sizeof(uint32_t);
constexpr size_t kGemmWorkspace = 256;  // one 32-bit status word, padded

fp4_status check_quant_common(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                              int want_block, fp4_round round, fp4_scale_layout layout,
                              unsigned char* q, unsigned char* scales) {
  if (dtype != FP4_F32 && dtype != FP4_BF16) return fail(FP4_EINVAL, "dtype %d is not FP4_F32/FP4_BF16", (int)dtype);
  if (block != want_block)
    return fail(FP4_EINVAL, "block %d does not match the format's block size %d", block, want_block);
  if (rows < 0 || cols <= 0) return fail(FP4_EINVAL, "bad shape [%ld, %ld]", rows, cols);
  if (cols % want_block) return fail(FP4_EINVAL, "cols %ld is not a multiple of the block size %d (incomplete block)", cols, want_block);
  if ((long long)rows * cols > kMaxElems) return fail(FP4_EUNSUPPORTED, "tensor larger than 2^40 elements");
  if (round != FP4_RNE && round != FP4_STOCHASTIC) return fail(FP4_EINVAL, "round %d unknown", (int)round);
  if (layout != FP4_SCALES_ROWMAJOR && layout != FP4_SCALES_MMA_TILED) return fail(FP4_EINVAL, "layout %d unknown", (int)layout);
  if (layout == FP4_SCALES_MMA_TILED && (rows % 128 || (cols / want_block) % 4))
    return fail(FP4_EINVAL, "MMA-tiled scales need rows %% 128 == 0 and (cols/block) %% 4 == 0");
  if (rows > 0 && (!x || !q || !scales)) return fail(FP4_EINVAL, "NULL x, q or scales");
  if (x && !aligned(x, 32)) return fail(FP4_EINVAL, "x must be 32-byte aligned");
  if (q && !aligned(q, 8)) return fail(FP4_EINVAL, "q must be 8-byte aligned");
  return FP4_OK;
}

fp4_status zero_counts(fp4_counts* counts, cudaStream_t s) {
  if (!counts) return FP4_OK;
  if (!aligned(counts, 8)) return fail(FP4_EINVAL, "counts must be 8-byte aligned");
  cudaError_t e = cudaMemsetAsync(counts, 0, sizeof(fp4_counts), s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "zeroing counts");
}

}  // namespace

namespace fp4k {
void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

int num_sms() {
  static int cache[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || n <= 0) n = 148;
    cache[dev] = n;
  }
  return cache[dev];
}
}  // namespace fp4k

extern "C" {

const char* fp4_status_str(fp4_status s) {
  switch (s) {
    case FP4_OK: return "FP4_OK";
    case FP4_EINVAL: return "FP4_EINVAL: invalid argument";
    case FP4_EUNSUPPORTED: return "FP4_EUNSUPPORTED: unsupported combination";
    case FP4_ECUDA: return "FP4_ECUDA: CUDA error";
  }
  return "unknown fp4_status";
}

const char* fp4_last_error(void) { return g_err; }

size_t fp4_workspace_size(fp4_op op, long rows, long cols) {
  (void)rows;
  (void)cols;
  switch (op) {
    case FP4_OP_NVFP4_QUANTIZE: return kAmaxSlotsWorkspace;
    case FP4_OP_FWHT_QUANTIZE: return kAmaxWorkspace;
    case FP4_OP_FWHT_QUANTIZE_STORED:
      // the amax word, padding to a 256-byte boundary, and the fp32 rotation
      return rows > 0 && cols > 0 ? 2 * kAmaxWorkspace + (size_t)rows * (size_t)cols * sizeof(float) : kAmaxWorkspace;
    case FP4_OP_BLOCK_GEMM: return kGemmWorkspace;
    case FP4_OP_BLOCK_GEMM_IF4:
      // rows = M + N, cols = K: the status word, padding, and both fp16 operands
      return rows > 0 && cols > 0 ? 2 * kGemmWorkspace + 2 * (size_t)rows * (size_t)cols : kGemmWorkspace;
    default: return 0;
  }
}

size_t fp4_gemm_status_word(void) { return 0; }

unsigned long long fp4_set_gemm_wait_limit(unsigned long long ns) { return fp4k::set_gemm_wait_limit(ns); }

fp4_status mx_quantize(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                       fp4_mx_policy policy, fp4_round round, unsigned long long seed,
                       fp4_scale_layout layout, unsigned char* q, unsigned char* scales,
                       fp4_counts* counts, void* stream) {
  fp4_status st = check_quant_common(x, dtype, rows, cols, block, 32, round, layout, q, scales);
  if (st != FP4_OK) return st;
  if (policy != FP4_MX_OCP_FLOOR && policy != FP4_MX_NOSAT_CEIL) return fail(FP4_EINVAL, "policy %d unknown", (int)policy);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if ((st = zero_counts(counts, s)) != FP4_OK) return st;
  fp4k::QuantLaunch L{};
  L.x = x; L.bf16 = dtype == FP4_BF16; L.rows = rows; L.cols = cols; L.nv = false;
  L.policy = policy; L.sr = round == FP4_STOCHASTIC; L.mode = 0; L.seed = seed;
  L.tiled = layout == FP4_SCALES_MMA_TILED; L.reverse = 0;
  L.q = q; L.scales = scales; L.counts = reinterpret_cast<unsigned long long*>(counts);
  cudaError_t e = fp4k::launch_quantize(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "mx_quantize launch");
}

fp4_status nvfp4_quantize(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                          fp4_round round, int mode, unsigned long long seed,
                          fp4_scale_layout layout, const float* global_in, float* global_out,
                          unsigned char* q, unsigned char* scales, fp4_counts* counts,
                          void* workspace, size_t ws_bytes, void* stream) {
  fp4_status st = check_quant_common(x, dtype, rows, cols, block, 16, round, layout, q, scales);
  if (st != FP4_OK) return st;
  if (mode != FP4_NV_PLAIN && mode != FP4_NV_FOUR_SIX && mode != FP4_NV_IF4)
    return fail(FP4_EINVAL, "NVFP4 block mode %d unknown", mode);
  if (mode == FP4_NV_IF4 && round != FP4_RNE) return fail(FP4_EUNSUPPORTED, "IF4 is defined with round to nearest only");
  if (!global_in && (!workspace || ws_bytes < kAmaxSlotsWorkspace || !aligned(workspace, 16)))
    return fail(FP4_EINVAL, "a 16-byte aligned workspace of %zu bytes is required when global_in is NULL",
                kAmaxSlotsWorkspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (counts && !aligned(counts, 8)) return fail(FP4_EINVAL, "counts must be 8-byte aligned");
  // with an amax pass (and a non-empty tensor) that pass zeroes the counters; otherwise a memset does
  const bool amax_pass = !global_in && (long long)rows * cols > 0;
  if (!amax_pass && (st = zero_counts(counts, s)) != FP4_OK) return st;
  // the amax pass writes one partial maximum per CTA into the workspace (no zeroing needed); the
  // quantise pass reduces them
  uint32_t* amax = static_cast<uint32_t*>(workspace);
  cudaError_t e;
  if (amax_pass) {
    if ((e = fp4k::launch_amax(x, dtype == FP4_BF16, (long long)rows * cols, amax,
                               reinterpret_cast<unsigned long long*>(counts), s)) != cudaSuccess)
      return cuda_fail(e, "nvfp4 amax launch");
  }
  fp4k::QuantLaunch L{};
  L.x = x; L.bf16 = dtype == FP4_BF16; L.rows = rows; L.cols = cols; L.nv = true;
  L.policy = 0; L.sr = round == FP4_STOCHASTIC; L.mode = mode; L.seed = seed;
  L.tiled = layout == FP4_SCALES_MMA_TILED; L.reverse = global_in ? 0 : 1;
  L.global_in = global_in; L.amax_bits = amax; L.global_out = global_out;
  L.amax_slots = amax_pass ? fp4k::amax_grid((long long)rows * cols, dtype == FP4_BF16) : 0;
  L.q = q; L.scales = scales; L.counts = reinterpret_cast<unsigned long long*>(counts);
  L.pdl = amax_pass;
  e = fp4k::launch_quantize(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "nvfp4_quantize launch");
}

static fp4_status fwht_quantize_impl(const void* x, const void* u, fp4_dtype dtype, long rows, long d,
                                     const unsigned int* signs, fp4_format format,
                         int block, fp4_round round, int four_six, unsigned long long seed,
                         fp4_scale_layout layout, const float* global_in, float* global_out,
                         float* rotated_out, unsigned char* q, unsigned char* scales,
                         fp4_counts* counts, void* workspace, size_t ws_bytes, void* stream) {
  if (format != FP4_MXFP4 && format != FP4_NVFP4) return fail(FP4_EINVAL, "format %d unknown", (int)format);
  const bool nv = format == FP4_NVFP4;
  if (d < 1024 || d > 16384 || (d & (d - 1))) return fail(FP4_EINVAL, "d = %ld must be a power of two in [1024, 16384]", d);
  fp4_status st = check_quant_common(x, dtype, rows, d, block, nv ? 16 : 32, round, layout, q, scales);
  if (st != FP4_OK) return st;
  if (four_six != FP4_NV_PLAIN && four_six != FP4_NV_FOUR_SIX && four_six != FP4_NV_IF4)
    return fail(FP4_EINVAL, "NVFP4 block mode %d unknown", four_six);
  if (!nv && four_six) return fail(FP4_EUNSUPPORTED, "four-over-six and IF4 are defined for NVFP4 only");
  if (four_six == FP4_NV_IF4 && round != FP4_RNE) return fail(FP4_EUNSUPPORTED, "IF4 is defined with round to nearest only");
  if (nv && !global_in && (!workspace || ws_bytes < kAmaxWorkspace || !aligned(workspace, 16)))
    return fail(FP4_EINVAL, "a 16-byte aligned workspace of %zu bytes is required when global_in is NULL", kAmaxWorkspace);
  if (rotated_out && !aligned(rotated_out, 16)) return fail(FP4_EINVAL, "rotated_out must be 16-byte aligned");
  if (signs && !aligned(signs, 4)) return fail(FP4_EINVAL, "signs must be 4-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (counts && !aligned(counts, 8)) return fail(FP4_EINVAL, "counts must be 8-byte aligned");
  // with an amax pass (and a non-empty tensor) that pass zeroes the counters; otherwise a memset does
  const bool amax_pass = nv && !global_in && rows > 0;
  if (!amax_pass && (st = zero_counts(counts, s)) != FP4_OK) return st;
  fp4k::FwhtLaunch L{};
  L.x = x; L.bf16 = dtype == FP4_BF16; L.rows = rows; L.d = (int)d; L.nv = nv;
  L.sr = round == FP4_STOCHASTIC; L.mode = nv ? four_six : 0; L.seed = seed;
  L.tiled = layout == FP4_SCALES_MMA_TILED;
  L.global_in = nv ? global_in : nullptr;
  L.amax_bits = static_cast<uint32_t*>(workspace);
  L.global_out = nv ? global_out : nullptr;
  L.rotated_out = rotated_out;
  L.signs = signs;
  L.u = u;
  L.pdl = amax_pass;
  L.q = q; L.scales = scales; L.counts = reinterpret_cast<unsigned long long*>(counts);
  cudaError_t e;
  // Stored-rotation route for the two-pass call: the first pass keeps the fp32 rotation (in
  // rotated_out, or in the workspace past the amax word) and the second pass quantises it, so the
  // butterflies run once.  Both routes give the same bytes.
  float* rot = nullptr;
  if (amax_pass) {
    const size_t rot_bytes = (size_t)rows * (size_t)d * sizeof(float);
    if (rotated_out && aligned(rotated_out, 32)) {
      rot = rotated_out;
    } else if (!rotated_out && ws_bytes >= 2 * kAmaxWorkspace + rot_bytes) {
      // the first 256-byte boundary past the amax word's 256 bytes
      const uintptr_t w = reinterpret_cast<uintptr_t>(workspace);
      rot = reinterpret_cast<float*>((w + 2 * kAmaxWorkspace) & ~(uintptr_t)(kAmaxWorkspace - 1));
    }
  }
  if (amax_pass) {
    if ((e = cudaMemsetAsync(L.amax_bits, 0, sizeof(uint32_t), s)) != cudaSuccess) return cuda_fail(e, "zeroing amax");
    if (rot) {
      L.rotated_out = rot;
      if ((e = fp4k::launch_fwht_store(L, s)) != cudaSuccess) return cuda_fail(e, "fwht store launch");
      fp4k::QuantLaunch Q{};
      Q.x = rot; Q.bf16 = false; Q.rows = rows; Q.cols = d; Q.nv = true;
      Q.policy = 0; Q.sr = L.sr; Q.mode = L.mode; Q.seed = seed;
      Q.tiled = L.tiled; Q.reverse = 1;  // start on the rows the first pass left in L2
      Q.global_in = nullptr; Q.amax_bits = L.amax_bits; Q.amax_slots = 1; Q.global_out = L.global_out;
      Q.q = q; Q.scales = scales; Q.counts = L.counts; Q.pdl = true;
      e = fp4k::launch_quantize(Q, s);
      return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fwht_quantize stored-rotation launch");
    }
    if ((e = fp4k::launch_fwht_amax(L, s)) != cudaSuccess) return cuda_fail(e, "fwht amax launch");
  }
  e = fp4k::launch_fwht_quantize(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fwht_quantize launch");
}

fp4_status fwht_quantize(const void* x, fp4_dtype dtype, long rows, long d, const unsigned int* signs,
                         fp4_format format, int block, fp4_round round, int four_six, unsigned long long seed,
                         fp4_scale_layout layout, const float* global_in, float* global_out,
                         float* rotated_out, unsigned char* q, unsigned char* scales,
                         fp4_counts* counts, void* workspace, size_t ws_bytes, void* stream) {
  return fwht_quantize_impl(x, nullptr, dtype, rows, d, signs, format, block, round, four_six, seed, layout,
                            global_in, global_out, rotated_out, q, scales, counts, workspace, ws_bytes, stream);
}

fp4_status swiglu_fwht_quantize(const void* g, const void* u, fp4_dtype dtype, long rows, long d,
                                const unsigned int* signs, fp4_format format, int block, fp4_round round, int four_six, unsigned long long seed,
                                fp4_scale_layout layout, const float* global_in, float* global_out,
                                float* rotated_out, unsigned char* q, unsigned char* scales,
                                fp4_counts* counts, void* workspace, size_t ws_bytes, void* stream) {
  if (dtype != FP4_BF16) return fail(FP4_EUNSUPPORTED, "swiglu_fwht_quantize takes bf16 g and u");
  if (rows > 0 && !u) return fail(FP4_EINVAL, "NULL u");
  if (u && !aligned(u, 32)) return fail(FP4_EINVAL, "u must be 32-byte aligned");
  return fwht_quantize_impl(g, u, dtype, rows, d, signs, format, block, round, four_six, seed, layout, global_in,
                            global_out, rotated_out, q, scales, counts, workspace, ws_bytes, stream);
}

fp4_status fp4_dequantize(const unsigned char* q, const unsigned char* scales, fp4_format format,
                          int block, fp4_scale_layout layout, const float* global, long rows,
                          long cols, fp4_dtype out_dtype, void* out, void* stream) {
  if (format != FP4_MXFP4 && format != FP4_NVFP4 && format != FP4_IF4)
    return fail(FP4_EINVAL, "format %d unknown", (int)format);
  const bool nv = format != FP4_MXFP4;
  const int B = nv ? 16 : 32;
  if (block != B) return fail(FP4_EINVAL, "block %d does not match the format's block size %d", block, B);
  if (out_dtype != FP4_F32 && out_dtype != FP4_BF16) return fail(FP4_EINVAL, "out dtype %d unknown", (int)out_dtype);
  if (rows < 0 || cols <= 0 || cols % B) return fail(FP4_EINVAL, "bad shape [%ld, %ld] for block %d", rows, cols, B);
  if ((long long)rows * cols > kMaxElems) return fail(FP4_EUNSUPPORTED, "tensor larger than 2^40 elements");
  if (layout != FP4_SCALES_ROWMAJOR && layout != FP4_SCALES_MMA_TILED) return fail(FP4_EINVAL, "layout %d unknown", (int)layout);
  if (layout == FP4_SCALES_MMA_TILED && (rows % 128 || (cols / B) % 4))
    return fail(FP4_EINVAL, "MMA-tiled scales need rows %% 128 == 0 and (cols/block) %% 4 == 0");
  if (rows == 0) return FP4_OK;
  if (!q || !scales || !out) return fail(FP4_EINVAL, "NULL q, scales or out");
  if (nv && !global) return fail(FP4_EINVAL, "NVFP4 and IF4 dequantisation need the global scale");
  if (!aligned(q, 8) || !aligned(out, 16)) return fail(FP4_EINVAL, "q must be 8-byte and out 16-byte aligned");
  fp4k::DequantLaunch L{q, scales, (int)format, layout == FP4_SCALES_MMA_TILED, nv ? global : nullptr,
                        rows, cols, out_dtype == FP4_BF16, out};
  cudaError_t e = fp4k::launch_dequant(L, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fp4_dequantize launch");
}

// IF4 GEMM: both operands expanded to fp16 in the workspace (E2M1 blocks exact, INT4 blocks with
// their six-sevenths step), then the kind::f16 tensor-core GEMM with alpha = (*Ag) * (*Bg).
static fp4_status if4_block_gemm(int M, int N, int K, const unsigned char* Aq, const unsigned char* As,
                                 const float* Ag, const unsigned char* Bq, const unsigned char* Bs, const float* Bg,
                                 void* C, long ldc, void* workspace, size_t ws_bytes, cudaStream_t s) {
  if (M % 128 || N % 256 || K % 64)
    return fail(FP4_EUNSUPPORTED, "IF4 GEMM shape %d x %d x %d: needs M %% 128, N %% 256, K %% 64 == 0", M, N, K);
  if (!Ag || !Bg) return fail(FP4_EINVAL, "IF4 GEMM needs both global scales");
  const size_t need = fp4_workspace_size(FP4_OP_BLOCK_GEMM_IF4, (long)M + N, K);
  if (!workspace || ws_bytes < need || !aligned(workspace, 16))
    return fail(FP4_EINVAL, "the IF4 GEMM needs a 16-byte aligned workspace of %zu bytes "
                "(fp4_workspace_size(FP4_OP_BLOCK_GEMM_IF4, M + N, K))", need);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  const uintptr_t w = reinterpret_cast<uintptr_t>(workspace);
  uint8_t* a16 = reinterpret_cast<uint8_t*>((w + 2 * kGemmWorkspace) & ~(uintptr_t)(kGemmWorkspace - 1));
  uint8_t* b16 = a16 + 2 * (size_t)M * (size_t)K;
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "zeroing gemm status");
  if ((e = fp4k::launch_if4_to_f16(Aq, As, M, K, a16, s)) != cudaSuccess) return cuda_fail(e, "IF4 operand A expansion");
  if ((e = fp4k::launch_if4_to_f16(Bq, Bs, N, K, b16, s)) != cudaSuccess) return cuda_fail(e, "IF4 operand B expansion");
  fp4k::GemmLaunch L{true, false, true, M, N, K, a16, nullptr, b16, nullptr, Ag, Bg, C, ldc, status};
  e = fp4k::launch_gemm(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "IF4 fp16 GEMM launch");
}

fp4_status fp4_block_gemm(fp4_format format, int M, int N, int K, const unsigned char* Aq,
                          const unsigned char* As, const float* Ag, const unsigned char* Bq,
                          const unsigned char* Bs, const float* Bg, void* C, long ldc,
                          void* workspace, size_t ws_bytes, void* stream) {
  if (format != FP4_MXFP4 && format != FP4_NVFP4 && format != FP4_IF4)
    return fail(FP4_EINVAL, "format %d unknown", (int)format);
  const bool nv = format == FP4_NVFP4;
  if (M <= 0 || N <= 0 || K <= 0) return fail(FP4_EINVAL, "bad GEMM shape %d x %d x %d", M, N, K);
  if (M % 128 || N % 256 || K % 256)
    return fail(FP4_EUNSUPPORTED, "GEMM shape %d x %d x %d: needs M %% 128, N %% 256, K %% 256 == 0", M, N, K);
  if (!Aq || !As || !Bq || !Bs || !C) return fail(FP4_EINVAL, "NULL operand pointer");
  if (nv && (!Ag || !Bg)) return fail(FP4_EINVAL, "NVFP4 GEMM needs both global scales");
  if (ldc < N || ldc % 8) return fail(FP4_EINVAL, "ldc %ld must be >= N and a multiple of 8", ldc);
  if (!aligned(Aq, 16) || !aligned(Bq, 16) || !aligned(As, 16) || !aligned(Bs, 16) || !aligned(C, 16))
    return fail(FP4_EINVAL, "GEMM operands must be 16-byte aligned");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (format == FP4_IF4) return if4_block_gemm(M, N, K, Aq, As, Ag, Bq, Bs, Bg, C, ldc, workspace, ws_bytes, s);
  if (!workspace || ws_bytes < kGemmWorkspace || !aligned(workspace, 16))
    return fail(FP4_EINVAL, "a 16-byte aligned workspace of %zu bytes is required", kGemmWorkspace);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "zeroing gemm status");
  fp4k::GemmLaunch L{nv, false, false, M, N, K, Aq, As, Bq, Bs, nv ? Ag : nullptr, nv ? Bg : nullptr, C, ldc, status};
  e = fp4k::launch_gemm(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fp4_block_gemm launch");
}

fp4_status fp4_to_e4m3(const unsigned char* q, long rows, long cols, unsigned char* out, void* stream) {
  if (rows < 0 || cols <= 0 || cols % 32)
    return fail(FP4_EINVAL, "bad shape [%ld, %ld]: cols must be a positive multiple of 32", rows, cols);
  if ((long long)rows * cols > kMaxElems) return fail(FP4_EUNSUPPORTED, "tensor larger than 2^40 elements");
  if (rows == 0) return FP4_OK;
  if (!q || !out) return fail(FP4_EINVAL, "NULL q or out");
  if (!aligned(q, 16) || !aligned(out, 16)) return fail(FP4_EINVAL, "q and out must be 16-byte aligned");
  cudaError_t e = fp4k::launch_e2m1_to_e4m3(q, (long long)rows * cols / 2, out, static_cast<cudaStream_t>(stream));
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fp4_to_e4m3 launch");
}

fp4_status fp4_block_gemm_e4m3(int M, int N, int K, const unsigned char* A8, const unsigned char* As,
                               const unsigned char* B8, const unsigned char* Bs, void* C, long ldc,
                               void* workspace, size_t ws_bytes, void* stream) {
  if (M <= 0 || N <= 0 || K <= 0) return fail(FP4_EINVAL, "bad GEMM shape %d x %d x %d", M, N, K);
  if (M % 128 || N % 256 || K % 128)
    return fail(FP4_EUNSUPPORTED, "GEMM shape %d x %d x %d: needs M %% 128, N %% 256, K %% 128 == 0", M, N, K);
  if (!A8 || !As || !B8 || !Bs || !C) return fail(FP4_EINVAL, "NULL operand pointer");
  if (ldc < N || ldc % 8) return fail(FP4_EINVAL, "ldc %ld must be >= N and a multiple of 8", ldc);
  if (!aligned(A8, 16) || !aligned(B8, 16) || !aligned(As, 16) || !aligned(Bs, 16) || !aligned(C, 16))
    return fail(FP4_EINVAL, "GEMM operands must be 16-byte aligned");
  if (!workspace || ws_bytes < kGemmWorkspace || !aligned(workspace, 16))
    return fail(FP4_EINVAL, "a 16-byte aligned workspace of %zu bytes is required", kGemmWorkspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  cudaError_t e = cudaMemsetAsync(status, 0, sizeof(uint32_t), s);
  if (e != cudaSuccess) return cuda_fail(e, "zeroing gemm status");
  fp4k::GemmLaunch L{false, true, false, M, N, K, A8, As, B8, Bs, nullptr, nullptr, C, ldc, status};
  e = fp4k::launch_gemm(L, s);
  return e == cudaSuccess ? FP4_OK : cuda_fail(e, "fp4_block_gemm_e4m3 launch");
}

}  // extern "C"
