// launch.h — internal interface between the C ABI (capi.cu) and the kernel translation units.
// Arguments arrive here already validated; launchers only configure grids and enqueue.
#pragma once

#include <cuda_runtime.h>
#include <utility>
#include <stdint.h>

namespace fp4k {

// Launch `kernel` with an optional programmatic-dependent-launch attribute (see grid_dep_wait).
template <typename... KArgs, typename... Args>
inline cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s, bool pdl,
                              Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

int num_sms();  // SM count of the current device (cached per device)

// Records the message fp4_last_error() returns on the calling thread.
void set_last_error(const char* msg);

struct QuantLaunch {
  const void* x;
  bool bf16;
  long long rows, cols;
  bool nv;        // NVFP4 (block 16, E4M3) vs MXFP4 (block 32, E8M0)
  int policy;     // MXFP4 exponent rule
  bool sr;        // stochastic rounding
  int mode;       // NVFP4 block mode: 0 plain, 1 four-over-six, 2 IF4
  unsigned long long seed;
  int tiled;      // scale layout
  int reverse;    // walk tiles last-to-first
  const float* global_in;    // NVFP4: caller-fixed s_g, or NULL to derive from the amax words
  const uint32_t* amax_bits;  // amax_slots words whose maximum is the tensor amax (magnitude bits)
  int amax_slots;             // 1 (a single word reduced by atomicMax) or the amax pass's grid
  float* global_out;
  uint8_t* q;
  uint8_t* scales;
  unsigned long long* counts;  // 4 counters or NULL
  bool pdl;       // launched right after the amax pass: programmatic dependent launch
};

struct DequantLaunch {
  const uint8_t* q;
  const uint8_t* scales;
  int format;     // 0 MXFP4, 1 NVFP4, 2 IF4
  int tiled;
  const float* global;
  long long rows, cols;
  bool out_bf16;
  void* out;
};

struct FwhtLaunch {
  const void* x;
  bool bf16;
  long long rows;
  int d;
  bool nv;
  bool sr;
  int mode;       // NVFP4 block mode: 0 plain, 1 four-over-six, 2 IF4
  unsigned long long seed;
  int tiled;
  const float* global_in;
  uint32_t* amax_bits;   // workspace word (pass 1 output / pass 2 input)
  float* global_out;
  float* rotated_out;
  const uint32_t* signs;  // randomised rotation: bit i negates channel i (nullptr: plain rotation)
  const void* u;          // SwiGLU path (bf16): x is g, u the up projection; nullptr otherwise
  bool pdl;               // quantise pass right after the amax pass: programmatic dependent launch
  uint8_t* q;
  uint8_t* scales;
  unsigned long long* counts;
};

struct GemmLaunch {
  bool nv;
  bool e4m3;  // MXFP4 through the FP8 MMA: Aq/Bq are E4M3 expansions [rows, K] (kind::mxf8f6f4)
  bool f16;   // fp16 operands [rows, K] (kind::f16, no block scales; alpha = (*Ag) * (*Bg))
  int M, N, K;
  const uint8_t *Aq, *As, *Bq, *Bs;
  const float *Ag, *Bg;
  void* C;
  long long ldc;
  uint32_t* status;  // device status word
};

cudaError_t launch_quantize(const QuantLaunch& L, cudaStream_t s);
// Upper bound of the tensor-amax pass's grid: the number of 32-bit slots its output needs.
constexpr int kAmaxSlots = 2048;
// CTAs of the tensor-amax pass over n_elems values (at most kAmaxSlots; 0 for an empty tensor).
int amax_grid(long long n_elems, bool bf16);
// Tensor amax as per-CTA partial maxima: CTA i writes the magnitude bits of its maximum to
// slots[i], i < amax_grid(n_elems, bf16), so nothing needs zeroing first.  Also zeroes `counts`
// (4 words) if non-null.  Lets the following quantise pass, launched with QuantLaunch::pdl and
// amax_slots = amax_grid(...), be scheduled as it retires.
cudaError_t launch_amax(const void* x, bool bf16, long long n_elems, uint32_t* slots,
                        unsigned long long* counts, cudaStream_t s);
cudaError_t launch_dequant(const DequantLaunch& L, cudaStream_t s);
// IF4 operand [rows, cols] (packed nibbles, MMA-tiled scales) -> fp16 [rows, cols] without the
// per-tensor scale: v * d for E2M1 blocks, RNE fp16 of fl(fl(k * d) * fl(6/7)) for INT4 blocks.  `out`
// must be 32-byte aligned (256-bit stores), else cudaErrorInvalidValue.
cudaError_t launch_if4_to_f16(const uint8_t* q, const uint8_t* scales, long long rows, long long cols, void* out,
                              cudaStream_t s);
// E2M1 nibbles -> E4M3 bytes; n_bytes (packed input bytes) a multiple of 16, both 16-byte aligned.
cudaError_t launch_e2m1_to_e4m3(const uint8_t* q, long long n_bytes, uint8_t* out, cudaStream_t s);
cudaError_t launch_fwht_amax(const FwhtLaunch& L, cudaStream_t s);
// Rotate once, store the normalised fp32 rotation to L.rotated_out ([rows, d]) and reduce the
// tensor amax into *L.amax_bits; zeroes L.counts.  The quantise pass is then launch_quantize on
// the stored values.
cudaError_t launch_fwht_store(const FwhtLaunch& L, cudaStream_t s);
cudaError_t launch_fwht_quantize(const FwhtLaunch& L, cudaStream_t s);
cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t s);
// Limit (ns) of each pipeline wait in GEMM launches made after the call; returns the previous one.
unsigned long long set_gemm_wait_limit(unsigned long long ns);

}  // namespace fp4k
