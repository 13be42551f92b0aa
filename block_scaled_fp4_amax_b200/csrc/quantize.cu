// quantize.cu — MXFP4 / NVFP4 block quantisers, the tensor-amax reduction and the dequantiser.
//
// All three are HBM-bound streaming kernels.  The row-major tensor is viewed as a flat array of
// 32-byte chunks (16 bf16 or 8 fp32 values); a warp reads 32 consecutive chunks (1 KiB, one
// 256-bit load per lane) per step, kUnroll steps in flight per lane.  A quantisation block of B
// values is G = B / E adjacent lanes: for the bf16 NVFP4 case G = 1, so a lane owns a whole block
// (amax, scale, both 4/6 candidates and their error sums without any cross-lane traffic).  Blocks
// never straddle rows because cols % B == 0.
//
// Per-element work is kept to the encode itself: the block amax is an integer max over the
// magnitude bits (which also exposes Inf/NaN: a block with a non-finite value has amax bits
// >= 0x7F800000, is rejected from the audit counters and only then counts its non-finite values
// per element); saturation is counted per element only when
// the block's normalised maximum exceeds 6; underflow = zero codes minus zero inputs, both from
// popcounts over the packed bits.
//
// Sources: "MXFP4 Quantization: Audit the 4.25-Bit Blocks" ("Read the shared E8M0 scale",
// "Encode one MXFP4 block step by step"); "Sub-4-Bit Microscaling" §1-§2 (E2M1, NVFP4 two-level
// scaling); podcast "Adaptive Block-Scaled Data Types" (stochastic rounding, Four Over Six).
#include "fp4_device.cuh"
#include "launch.h"

namespace fp4k {

constexpr int kThreads = 256;
constexpr int kUnroll = 4;      // 32-byte chunks in flight per lane
constexpr int kUnroll46 = 2;    // four-over-six and IF4: compute-bound, so a smaller body is worth more

// NVFP4 block modes: plain, four-over-six, IF4 (E2M1 or INT4 per block)
constexpr int kPlain = 0, kFourSix = 1, kIF4 = 2;

// ---------------------------------------------------------------------------------------------
// MXFP4 shared exponent from the amax bit pattern (exact): OCP floor(log2 amax) - 2, or the
// smallest e with amax <= 6 * 2^e; clamped to [-127, 127]; an all-zero block takes e = 0.  A
// non-finite maximum (Inf or NaN: exponent field 255) counts as 2^128, e = 126 under both rules.
__device__ __forceinline__ int mx_exponent(uint32_t bits, int policy) {
  const int ef = (int)((bits >> 23) & 0xFFu);
  if (bits == 0u) return 0;
  if (ef == 0) return -127;  // subnormal maximum: below 2^-126, clamps
  if (ef == 255) return 126;
  const int E = ef - 127;
  const int e = (policy == 0) ? E - 2 : (((bits & 0x7FFFFFu) <= 0x400000u) ? E - 2 : E - 1);
  return e < -127 ? -127 : e;
}

struct NvScale {
  float s_g, inv6, inv4;
};

// The tensor amax from `n` <= kAmaxSlots words of magnitude bits (the amax pass's per-CTA maxima,
// or one word): an integer maximum, which orders non-negative floats (NaN patterns above +Inf).
// Every thread of the CTA (kThreads of them) calls it and gets the result.  The loads have a fixed
// trip count, so they are all in flight together: one L2 round trip.
__device__ __forceinline__ uint32_t cta_amax_bits(const uint32_t* slots, int n) {
  __shared__ uint32_t red;
  if (threadIdx.x == 0) red = 0u;
  __syncthreads();
  uint32_t m = 0u;
#pragma unroll
  for (int k = 0; k < kAmaxSlots / kThreads; ++k) {
    const int i = (int)threadIdx.x + k * kThreads;
    if (i < n) m = max(m, __ldcg(slots + i));
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  if ((threadIdx.x & 31) == 0 && m) atomicMax(&red, m);
  __syncthreads();
  return red;
}

__device__ __forceinline__ NvScale nv_scales(const float* global_in, const uint32_t* amax_bits, int amax_slots,
                                             float six_m) {
  NvScale s;
  if (global_in) {
    s.s_g = *global_in;
  } else {
    const float amax = __uint_as_float(cta_amax_bits(amax_bits, amax_slots));
    s.s_g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, six_m);
  }
  s.inv6 = __frcp_rn(__fmul_rn(6.0f, s.s_g));
  s.inv4 = __frcp_rn(__fmul_rn(4.0f, s.s_g));
  return s;
}

struct QuantParams {
  const void* x;
  long long n_chunks;  // rows * cols / E
  DivU32 nb;           // blocks per row (with its division multiplier)
  int policy;          // MXFP4 exponent rule
  int tiled;           // scale layout
  int reverse;         // walk the tiles last-to-first (re-use the tail a previous pass left in L2)
  PhiloxKeys keys;     // stochastic-rounding round keys (from the seed)
  uint32_t zero;       // 0, read at run time: makes in-register nibble decodes opaque
  const float* global_in;
  const uint32_t* amax_bits;
  int amax_slots;
  float* global_out;
  float six_m;
  uint8_t* q;
  uint8_t* scales;
  unsigned long long* counts;
};

// Reload one chunk's values for an exact decision (an L2 hit: the kernel read them moments ago).
template <typename T>
__device__ __forceinline__ void reload_chunk(const char* xb, long long c, bool valid, float* v) {
  U8 raw;
  if (valid) {  // plain 16-byte loads: ptxas 12.9 crashed on the 256-bit load asm in these functions
    const uint4 lo = __ldg(reinterpret_cast<const uint4*>(xb + c * 32));
    const uint4 hi = __ldg(reinterpret_cast<const uint4*>(xb + c * 32 + 16));
    raw.w[0] = lo.x; raw.w[1] = lo.y; raw.w[2] = lo.z; raw.w[3] = lo.w;
    raw.w[4] = hi.x; raw.w[5] = hi.y; raw.w[6] = hi.z; raw.w[7] = hi.w;
  } else {
#pragma unroll
    for (int i = 0; i < 8; ++i) raw.w[i] = 0u;
  }
  Vec32<T>::unpack(raw, v);
}

// Exact four-over-six choice for one chunk (the rare case the estimates cannot decide): compares
// the two fp32 sequential error sums.  Out of line so the unrolled main loop keeps a single copy
// of it; called by the whole warp (the block sums shuffle when G > 1).
template <typename T, int G>
__device__ __noinline__ uint32_t four_six_exact(const char* xb, long long c, bool valid, uint32_t w6a, uint32_t w6b,
                                                uint32_t w4a, uint32_t w4b, uint32_t sc6, uint32_t sc4, float s_g,
                                                uint32_t zero) {
  constexpr int E = Vec32<T>::E;
  float v[E], sq[E];
  reload_chunk<T>(xb, c, valid, v);
  const int lane = threadIdx.x & 31;
  const uint32_t w6[2] = {w6a, w6b}, w4[2] = {w4a, w4b};
  sq_errors_n<E>(v, w6, sc6, s_g, zero, sq);
  const float sse6 = block_sse_n<E, G>(sq, lane);
  sq_errors_n<E>(v, w4, sc4, s_g, zero, sq);
  const float sse4 = block_sse_n<E, G>(sq, lane);
  return sse4 < sse6 ? 1u : 0u;
}

// Exact IF4 choice for one chunk, as four_six_exact: the E2M1 error sum against the INT4 one
// (the INT4 candidate is rebuilt from the values; `wa`/`wb` are the E2M1 words, whose sign bits
// it takes).  Returns 1 when INT4 is strictly lower.
template <typename T, int G>
__device__ __noinline__ uint32_t if4_exact(const char* xb, long long c, bool valid, uint32_t wa, uint32_t wb,
                                           uint32_t sc, float s_g, float R7, float s7, uint32_t zero) {
  constexpr int E = Vec32<T>::E;
  float v[E], sq[E];
  reload_chunk<T>(xb, c, valid, v);
  const int lane = threadIdx.x & 31;
  const uint32_t w[2] = {wa, wb};
  uint32_t w7[2];
  sq_errors_n<E>(v, w, sc, s_g, zero, sq);
  const float sse6 = block_sse_n<E, G>(sq, lane);
  int4_candidate_n<E>(v, R7, e4m3_value(sc), s7, w, w7, sq);
  const float sse7 = block_sse_n<E, G>(sq, lane);
  return sse7 < sse6 ? 1u : 0u;
}

template <typename T, bool NV, bool SR, int MODE>
__global__ void __launch_bounds__(kThreads) quantize_kernel(QuantParams p) {
  constexpr bool FOUR_SIX = MODE == kFourSix;
  constexpr bool IF4 = MODE == kIF4;
  constexpr int E = Vec32<T>::E;  // 16 (bf16) or 8 (fp32)
  constexpr int B = NV ? 16 : 32;
  constexpr int G = B / E;
  constexpr int W = E / 8;        // packed words per chunk
  constexpr int U = MODE != kPlain ? kUnroll46 : kUnroll;
  constexpr bool kBF = E == 16;   // bf16 input: saturations counted with bf16x2 compares
  const int lane = threadIdx.x & 31;
  const long long warp = ((long long)blockIdx.x * kThreads + threadIdx.x) >> 5;
  const long long nwarps = ((long long)gridDim.x * kThreads) >> 5;
  const long long per_tile = 32LL * U;
  const long long ntiles = (p.n_chunks + per_tile - 1) / per_tile;
  grid_dep_wait();  // after the amax pass (programmatic launch): its results are visible from here

  NvScale ns{1.0f, 1.0f, 1.0f};
  __shared__ float2 tab[NV ? kScaleTab : 1];
  __shared__ float2 tab7[IF4 ? kScaleTab : 1];
  float s7 = 0.0f;
  if (NV) {
    ns = nv_scales(p.global_in, p.amax_bits, p.amax_slots, p.six_m);
    if (p.global_out && blockIdx.x == 0 && threadIdx.x == 0) *p.global_out = ns.s_g;
    fill_scale_tab(tab, ns.s_g);
    if (IF4) {
      s7 = __fmul_rn(ns.s_g, kSixSevenths);
      fill_int4_tab(tab7, s7);
    }
    __syncthreads();
  }
  uint32_t cnt[4] = {0u, 0u, 0u, 0u};  // underflow, saturation, nonfinite, blocks_four
  const char* xb = reinterpret_cast<const char*>(p.x);

  for (long long t = warp; t < ntiles; t += nwarps) {
    const long long tile = p.reverse ? (ntiles - 1 - t) : t;
    const long long c0 = tile * per_tile + lane;
    U8 raw[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long c = c0 + 32LL * u;
      if (c < p.n_chunks) {
        raw[u] = ld32<true>(xb + c * 32);
      } else {
#pragma unroll
        for (int i = 0; i < 8; ++i) raw[u].w[i] = 0u;
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const long long c = c0 + 32LL * u;
      const bool valid = c < p.n_chunks;
      float v[E];
      Vec32<T>::unpack(raw[u], v);
      bool any_zero;
      uint32_t am = Vec32<T>::max_mag(raw[u], any_zero);
#pragma unroll
      for (int o = 1; o < G; o <<= 1) am = max(am, __shfl_xor_sync(0xFFFFFFFFu, am, o));
      if (am >= 0x7F800000u && valid) {
#pragma unroll
        for (int i = 0; i < E; ++i) cnt[2] += !isfinite(v[i]);
      }
      const float amax = __uint_as_float(am);
      const unsigned long long idx0 = (unsigned long long)c * E;
      uint32_t rnd[E];
      if (SR) sr_words<E>(idx0, p.keys, rnd);
      uint32_t w[W], sc, sat = 0, four = 0;
      if (!NV) {
        const int e = mx_exponent(am, p.policy);
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
        const float top = __fmul_rn(amax, inv);
        encode_n<E, SR, !kBF>(v, inv, top, rnd, w, sat);
        if constexpr (kBF) {
          // 6 * 2^e is a normal bf16 for e in [-127, 126]; a non-finite block (e = 126 or 127 from
          // an Inf/NaN maximum) keeps the general count, as does e = 127
          if (e <= 125 && am < 0x7F800000u) {
            const uint32_t n = mx_sat_count_bf16x16(raw[u].w, e);
            sat = top > 6.0f ? n : 0u;
          } else {
            // a NaN top (a NaN in the block, e = 126) still counts the block's infinities
            const float D = __uint_as_float(e > -127 ? (uint32_t)(e + 127) << 23 : 0x00400000u);
            const uint32_t n = sat_count_bf16x16(raw[u].w, D, inv);
            sat = !(top <= 6.0f) ? n : 0u;
          }
        }
        sc = (uint32_t)(e + 127);
      } else if (IF4) {
        // E2M1 and INT4 candidates with their scaled-domain residual estimates; the exact fp32
        // error sums only where the estimates are too close to call (INT4 kept iff strictly lower)
        float D, A, R;
        sc = nv_candidate_resid_n<E, false, !kBF>(v, amax, ns.inv6, tab, rnd, p.zero, w, sat, D, A, &R);
        if constexpr (kBF) {
          const uint32_t n = sat_count_bf16x16(raw[u].w, D, R);
          sat = __fmul_rn(amax, R) > 6.0f ? n : 0u;
        }
        const float2 DR7 = tab7[sc];
        uint32_t w7[W];
        float A7 = int4_encode_resid_n<E>(v, DR7.y, w, w7);
#pragma unroll
        for (int o = 1; o < G; o <<= 1) {
          A += __shfl_xor_sync(0xFFFFFFFFu, A, o);
          A7 += __shfl_xor_sync(0xFFFFFFFFu, A7, o);
        }
        const bool eligible = DR7.y != 0.0f;
        bool pick;
        bool undecided = if4_undecided(am, amax, D, DR7.x, A, A7, eligible, pick);
        if (__any_sync(0xFFFFFFFFu, undecided)) {  // rare: warp-uniform, so the common path is unchanged
          if constexpr (G == 1) {
            if (undecided && eligible && ns.s_g > 0.0f && s7 > 0.0f && am < 0x7F800000u &&
                if4_single_term(w, w7, amax, sc, ns.s_g, s7)) {
              undecided = false;
              pick = false;
            }
          }
          if (__any_sync(0xFFFFFFFFu, undecided)) {  // the exact sums shuffle: the whole warp calls
            const uint32_t lower = if4_exact<T, G>(xb, c, valid, w[0], w[W - 1], sc, ns.s_g, DR7.y, s7, p.zero);
            pick = eligible && lower != 0u;
          }
        }
        if (pick) {
          sc |= 0x80u;
          four = 1;
          sat = 0;
          if (__fmul_rn(amax, DR7.y) > 7.0f) {
            if constexpr (kBF) {
              sat = sat_count_bf16x16(raw[u].w, DR7.x, DR7.y, 7.0f);
            } else {
#pragma unroll
              for (int i = 0; i < E; ++i) sat += fabsf(__fmul_rn(v[i], DR7.y)) > 7.0f;
            }
          }
#pragma unroll
          for (int k = 0; k < W; ++k) w[k] = w7[k];
        }
      } else if (!FOUR_SIX) {
        float2 DR;
        sc = nv_candidate_n<E, SR, !kBF>(v, amax, ns.inv6, tab, rnd, w, sat, &DR);
        if constexpr (kBF) {
          const uint32_t n = sat_count_bf16x16(raw[u].w, DR.x, DR.y);
          sat = __fmul_rn(amax, DR.y) > 6.0f ? n : 0u;
        }
      } else {
        float D6, D4, A6, A4, R6, R4;
        uint32_t w4[W], sat4;
        const uint32_t sc6 =
            nv_candidate_resid_n<E, SR, !kBF>(v, amax, ns.inv6, tab, rnd, p.zero, w, sat, D6, A6, &R6);
        const uint32_t sc4 =
            nv_candidate_resid_n<E, SR, !kBF>(v, amax, ns.inv4, tab, rnd, p.zero, w4, sat4, D4, A4, &R4);
        if constexpr (kBF) {
          // target 6: about half the blocks saturate their maximum, so count without a branch;
          // target 4 normalises the maximum to about 4 and saturates only with a clamped scale
          const uint32_t n = sat_count_bf16x16(raw[u].w, D6, R6);
          sat = __fmul_rn(amax, R6) > 6.0f ? n : 0u;
          if (__fmul_rn(amax, R4) > 6.0f) sat4 = sat_count_bf16x16(raw[u].w, D4, R4);
        }
#pragma unroll
        for (int o = 1; o < G; o <<= 1) {  // butterfly: every lane of the block gets the same sums
          A6 += __shfl_xor_sync(0xFFFFFFFFu, A6, o);
          A4 += __shfl_xor_sync(0xFFFFFFFFu, A4, o);
        }
        bool pick4;
        bool undecided = four_six_undecided(am, amax, D6, D4, A6, A4, sc6, sc4, pick4);
        if (__any_sync(0xFFFFFFFFu, undecided)) {  // rare: warp-uniform, so the common path is unchanged
          if constexpr (G == 1) {
            // the outlier-block shape: one nonzero code per candidate, decided from one term
            if (undecided && ns.s_g > 0.0f && am < 0x7F800000u && four_six_single_term(w, w4, amax, sc6, sc4, ns.s_g)) {
              undecided = false;
              pick4 = false;
            }
          }
          if (__any_sync(0xFFFFFFFFu, undecided))  // the exact sums shuffle: the whole warp calls
            pick4 = four_six_exact<T, G>(xb, c, valid, w[0], w[W - 1], w4[0], w4[W - 1], sc6, sc4, ns.s_g, p.zero) != 0u;
        }
        sc = sc6;
        if (pick4) {
          sc = sc4;
          sat = sat4;
          four = 1;
#pragma unroll
          for (int k = 0; k < W; ++k) w[k] = w4[k];
        }
      }
      if (valid) {
        // a block holding Inf or NaN is rejected: it adds only to the non-finite count, and its
        // codes and scale byte are unspecified
        const bool audit = am < 0x7F800000u;
        const int zc = zero_codes_n<E>(w);
        // a +-0 input always gives a zero code, so inputs are counted only when both occur
        cnt[0] += audit ? (uint32_t)(zc - ((zc > 0 && any_zero) ? Vec32<T>::zeros(raw[u]) : 0)) : 0u;
        cnt[1] += audit ? sat : 0u;
        if (W == 2) {
          reinterpret_cast<uint2*>(p.q)[c] = make_uint2(w[0], w[W - 1]);
        } else {
          reinterpret_cast<uint32_t*>(p.q)[c] = w[0];
        }
        if ((lane & (G - 1)) == 0) {
          const unsigned long long blk = (unsigned long long)c / G;
          p.scales[scale_offset(blk, p.nb, p.tiled)] = (uint8_t)sc;
          cnt[3] += audit ? four : 0u;
        }
      }
    }
  }
  if (p.counts) flush_counts<4>(cnt, p.counts);
}

// ---------------------------------------------------------------------------------------------
// Tensor amax (NVFP4 global scale, first pass): max |x| over the whole tensor as an integer max
// of the magnitude bits (monotone for non-negative floats).  Each CTA stores its maximum in its own
// slot, so nothing needs zeroing before the pass (a memset on the stream costs about as much as 7%
// of this kernel); the quantise pass reduces the slots.  Loads keep their L2 lines so the
// second pass, walking the tiles in reverse, starts on resident data.
template <typename T>
__global__ void __launch_bounds__(kThreads) amax_kernel(const void* x, long long n_chunks,
                                                        uint32_t* slots, unsigned long long* counts) {
  grid_dep_trigger();  // the quantise pass may take SMs as this grid's CTAs retire
  // the counters the following quantise pass accumulates into start at zero (stream order)
  if (counts && blockIdx.x == 0 && threadIdx.x < 4) counts[threadIdx.x] = 0ull;
  constexpr int E = Vec32<T>::E;
  const char* xb = reinterpret_cast<const char*>(x);
  const long long tid = (long long)blockIdx.x * kThreads + threadIdx.x;
  const long long stride = (long long)gridDim.x * kThreads;
  uint32_t m = 0u;
  long long c = tid;
  for (; c + 3 * stride < n_chunks; c += 4 * stride) {
    U8 r[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) r[u] = ld32<false>(xb + (c + u * stride) * 32);
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      float v[E];
      Vec32<T>::unpack(r[u], v);
#pragma unroll
      for (int i = 0; i < E; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
    }
  }
  for (; c < n_chunks; c += stride) {
    float v[E];
    Vec32<T>::unpack(ld32<false>(xb + c * 32), v);
#pragma unroll
    for (int i = 0; i < E; ++i) m = max(m, __float_as_uint(v[i]) & 0x7FFFFFFFu);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t wm[kThreads / 32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0u;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) b = max(b, wm[w]);
    slots[blockIdx.x] = b;
  }
}

// ---------------------------------------------------------------------------------------------
// Dequantiser: each lane expands 8 packed bytes (16 values).  x_hat = fl(fl(v*d)*s_g) (NVFP4) or
// v * 2^(byte-127) (MXFP4, exact); IF4 blocks whose scale byte has bit 7 set hold INT4 nibbles,
// x_hat = fl(fl(k*d)*s7) with d from the low 7 bits and s7 = fl(s_g * fl(6/7)).  bf16 output is
// the RNE cast of the fp32 value.
template <int FMT, bool OUT_BF16, bool V8>  // FMT: 0 MXFP4, 1 NVFP4, 2 IF4; V8: 256-bit stores
__global__ void __launch_bounds__(kThreads) dequant_kernel(const uint8_t* q, const uint8_t* scales,
                                                           const float* global, long long n_groups,
                                                           DivU32 nb, int tiled, void* out) {
  constexpr bool NV = FMT != 0;
  constexpr int B = NV ? 16 : 32;
  const float s_g = NV ? *global : 1.0f;
  const float s7 = FMT == 2 ? __fmul_rn(s_g, kSixSevenths) : 0.0f;
  const long long stride = (long long)gridDim.x * kThreads;
  for (long long g = (long long)blockIdx.x * kThreads + threadIdx.x; g < n_groups; g += stride) {
    const uint2 w = *reinterpret_cast<const uint2*>(q + g * 8);
    const unsigned long long blk = (unsigned long long)(g * 16) / B;
    const uint8_t sb = scales[scale_offset(blk, nb, tiled)];
    const bool int4 = FMT == 2 && (sb & 0x80u);
    float d;
    if (NV) d = e4m3_value(FMT == 2 ? (sb & 0x7Fu) : sb);
    else d = __uint_as_float((uint32_t)sb << 23);  // 2^(sb-127); sb = 0 -> 0 (handled below)
    float v[16];
    if (int4) {
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        const uint32_t c = ((i < 8 ? w.x : w.y) >> (4 * (i & 7))) & 15u;
        const float m = (float)(c & 7u);
        v[i] = (c & 8u) ? -m : m;
      }
    } else {
      e2m1_unpack<8>(w.x, v);
      e2m1_unpack<8>(w.y, v + 8);
    }
    const float sf = int4 ? s7 : s_g;
    float o[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      if (NV) {
        o[i] = __fmul_rn(__fmul_rn(v[i], d), sf);
      } else if (sb != 0) {
        o[i] = __fmul_rn(v[i], d);
      } else {
        o[i] = __fmul_rn(__fmul_rn(v[i], 0x1p-64f), 0x1p-63f);  // v * 2^-127, exact (subnormal)
      }
    }
    if (OUT_BF16) {
      uint32_t pw[8];
#pragma unroll
      for (int i = 0; i < 8; ++i) pw[i] = bf16x2_pack(o[2 * i], o[2 * i + 1]);
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(out) + g * 16;
      if (V8) {
        st32(dst, pw);
      } else {
        reinterpret_cast<uint4*>(dst)[0] = make_uint4(pw[0], pw[1], pw[2], pw[3]);
        reinterpret_cast<uint4*>(dst)[1] = make_uint4(pw[4], pw[5], pw[6], pw[7]);
      }
    } else {
      float* dst = reinterpret_cast<float*>(out) + g * 16;
      if (V8) {
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          uint32_t w8[8];
#pragma unroll
          for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(o[8 * h + i]);
          st32(dst + 8 * h, w8);
        }
      } else {
#pragma unroll
        for (int i = 0; i < 4; ++i)
          reinterpret_cast<float4*>(dst)[i] = make_float4(o[4 * i], o[4 * i + 1], o[4 * i + 2], o[4 * i + 3]);
      }
    }
  }
}

// ---------------------------------------------------------------------------------------------
// E2M1 -> E4M3 expansion (metrale `hardware::exec`: the exact conversion that lets the FP8 MMA take
// FP4 operands).  With a nibble in bits 7..4 of a byte b, (b & 0x80) | ((b & 0x70) >> 2) is the E4M3
// encoding of its value times 2^-6.  Each thread turns 16 packed bytes (32 nibbles) into 32 bytes.
template <bool V8>
__global__ void __launch_bounds__(kThreads) e2m1_to_e4m3_kernel(const uint4* q, uint4* out, long long n16) {
  const long long stride = (long long)gridDim.x * kThreads;
  for (long long i = (long long)blockIdx.x * kThreads + threadIdx.x; i < n16; i += stride) {
    const uint4 w = q[i];
    const uint32_t in[4] = {w.x, w.y, w.z, w.w};
    uint32_t o[8];
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const uint32_t even = (in[k] << 4) & 0xF0F0F0F0u;  // elements 0, 2, 4, 6 of the word, one per byte
      const uint32_t odd = in[k] & 0xF0F0F0F0u;          // elements 1, 3, 5, 7
      const uint32_t e = (even & 0x80808080u) | ((even & 0x70707070u) >> 2);
      const uint32_t d = (odd & 0x80808080u) | ((odd & 0x70707070u) >> 2);
      o[2 * k] = __byte_perm(e, d, 0x5140);      // elements 0 1 2 3
      o[2 * k + 1] = __byte_perm(e, d, 0x7362);  // elements 4 5 6 7
    }
    if (V8) {
      st32(out + 2 * i, o);
    } else {
      out[2 * i] = make_uint4(o[0], o[1], o[2], o[3]);
      out[2 * i + 1] = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

// ---------------------------------------------------------------------------------------------
// IF4 -> fp16 GEMM operand (the IF4 GEMM: "Adaptive Block-Scaled Data Types" podcast, IF4 segment).
// An E2M1 block gives v * d, exact in fp16 (at most 6 significant bits, magnitudes 2^-10 .. 2688);
// an INT4 block (scale bit 7) gives the RNE fp16 of fl(fl(k * d) * fl(6/7)): its integer step is six
// sevenths of the E2M1 unit, so a mixed block pair carries 6/7 and an INT4 pair 36/49 into the
// product.  The per-tensor scale stays out of the element (fp16 range); the GEMM epilogue applies
// both.  Scales are read in the MMA tile layout; each thread expands one 16-block (8 packed bytes)
// into one 256-bit store.
__global__ void __launch_bounds__(kThreads) if4_to_f16_kernel(const uint8_t* q, const uint8_t* scales,
                                                              long long n_groups, DivU32 nb, uint4* out) {
  const long long stride = (long long)gridDim.x * kThreads;
  for (long long g = (long long)blockIdx.x * kThreads + threadIdx.x; g < n_groups; g += stride) {
    const uint2 w = *reinterpret_cast<const uint2*>(q + g * 8);
    const uint8_t sb = scales[scale_offset((unsigned long long)g, nb, true)];
    const uint32_t code = sb & 0x7Fu;
    uint32_t h[8];
    if (sb & 0x80u) {
      const float d = e4m3_value(code);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float f[2];
#pragma unroll
        for (int j = 0; j < 2; ++j) {
          const int e = 2 * i + j;
          const uint32_t c = ((e < 8 ? w.x : w.y) >> (4 * (e & 7))) & 15u;
          const float k = (c & 8u) ? -(float)(c & 7u) : (float)(c & 7u);
          f[j] = __fmul_rn(__fmul_rn(k, d), kSixSevenths);  // k * d exact, then one rounding
        }
        asm("cvt.rn.f16x2.f32 %0, %1, %2;" : "=r"(h[i]) : "f"(f[1]), "f"(f[0]));
      }
    } else {
      uint32_t dh2;
      asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(dh2) : "h"((uint16_t)(code | (code << 8))));
      uint32_t v[8];
      e2m1x8_to_f16x2(w.x, v);
      e2m1x8_to_f16x2(w.y, v + 4);
#pragma unroll
      for (int i = 0; i < 8; ++i) asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(h[i]) : "r"(v[i]), "r"(dh2));
    }
    st32(out + 2 * g, h);
  }
}

// ---------------------------------------------------------------------------------------------
// Launchers

// The 256-bit store variants need 32-byte aligned output (the API promises 16).
static bool aligned32(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 31u) == 0; }

static int grid_for(long long work_items, int per_cta) {
  const long long want = (work_items + per_cta - 1) / per_cta;
  const long long cap = (long long)num_sms() * (2048 / kThreads);
  return (int)(want < 1 ? 1 : (want > cap ? cap : want));
}

// One wave of resident CTAs (the kernel loops over tiles), so no CTA waits in a tail wave.
template <typename T, bool NV, bool SR, int MODE>
static cudaError_t launch_q(const QuantParams& p, bool pdl, cudaStream_t s) {
  static int per_sm = 0;  // resident CTAs per SM for this instantiation (same on every sm_100 device)
  if (per_sm == 0) {
    int n = 0;
    if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, quantize_kernel<T, NV, SR, MODE>, kThreads, 0) != cudaSuccess ||
        n < 1)
      n = 1;
    per_sm = n;
  }
  constexpr int U = MODE != kPlain ? kUnroll46 : kUnroll;
  const long long tiles = (p.n_chunks + 32LL * U - 1) / (32LL * U);
  const long long want = (tiles * 32 + kThreads - 1) / kThreads;
  const long long cap = (long long)num_sms() * per_sm;
  const int grid = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  return launch_pdl(quantize_kernel<T, NV, SR, MODE>, dim3(grid), dim3(kThreads), 0, s, pdl, p);
}

template <typename T>
static cudaError_t dispatch_q(const QuantParams& p, bool nv, bool sr, int mode, bool pdl, cudaStream_t s) {
  if (!nv) return sr ? launch_q<T, false, true, kPlain>(p, pdl, s) : launch_q<T, false, false, kPlain>(p, pdl, s);
  if (mode == kIF4) return launch_q<T, true, false, kIF4>(p, pdl, s);  // round to nearest only
  if (mode == kFourSix)
    return sr ? launch_q<T, true, true, kFourSix>(p, pdl, s) : launch_q<T, true, false, kFourSix>(p, pdl, s);
  return sr ? launch_q<T, true, true, kPlain>(p, pdl, s) : launch_q<T, true, false, kPlain>(p, pdl, s);
}

cudaError_t launch_quantize(const QuantLaunch& L, cudaStream_t s) {
  QuantParams p;
  const int E = L.bf16 ? 16 : 8;
  p.x = L.x;
  p.n_chunks = (long long)(L.rows * L.cols / E);
  p.nb = make_divu32((uint32_t)(L.cols / (L.nv ? 16 : 32)));
  p.policy = L.policy;
  p.tiled = L.tiled;
  p.reverse = L.reverse;
  p.keys = philox_keys(L.seed);
  p.zero = 0u;
  p.global_in = L.global_in;
  p.amax_bits = L.amax_bits;
  p.amax_slots = L.amax_slots;
  p.global_out = L.global_out;
  p.six_m = L.mode == kFourSix ? 1536.0f : 2688.0f;
  p.q = L.q;
  p.scales = L.scales;
  p.counts = L.counts;
  if (p.n_chunks == 0) return cudaSuccess;
  return L.bf16 ? dispatch_q<__nv_bfloat16>(p, L.nv, L.sr, L.mode, L.pdl, s)
                : dispatch_q<float>(p, L.nv, L.sr, L.mode, L.pdl, s);
}

int amax_grid(long long n_elems, bool bf16) {
  const long long chunks = n_elems / (bf16 ? 16 : 8);
  if (chunks == 0) return 0;
  const int grid = grid_for(chunks / 4 + 1, kThreads);
  return grid < kAmaxSlots ? grid : kAmaxSlots;
}

cudaError_t launch_amax(const void* x, bool bf16, long long n_elems, uint32_t* slots,
                        unsigned long long* counts, cudaStream_t s) {
  const long long chunks = n_elems / (bf16 ? 16 : 8);
  const int grid = amax_grid(n_elems, bf16);
  if (grid == 0) return cudaSuccess;
  if (bf16) amax_kernel<__nv_bfloat16><<<grid, kThreads, 0, s>>>(x, chunks, slots, counts);
  else amax_kernel<float><<<grid, kThreads, 0, s>>>(x, chunks, slots, counts);
  return cudaGetLastError();
}

cudaError_t launch_e2m1_to_e4m3(const uint8_t* q, long long n_bytes, uint8_t* out, cudaStream_t s) {
  const long long n16 = n_bytes / 16;
  if (n16 == 0) return cudaSuccess;
  const int grid = grid_for(n16, kThreads);
  const uint4* in = reinterpret_cast<const uint4*>(q);
  uint4* o = reinterpret_cast<uint4*>(out);
  if (aligned32(out)) e2m1_to_e4m3_kernel<true><<<grid, kThreads, 0, s>>>(in, o, n16);
  else e2m1_to_e4m3_kernel<false><<<grid, kThreads, 0, s>>>(in, o, n16);
  return cudaGetLastError();
}

cudaError_t launch_if4_to_f16(const uint8_t* q, const uint8_t* scales, long long rows, long long cols, void* out,
                              cudaStream_t s) {
  const long long groups = rows * cols / 16;
  if (groups == 0) return cudaSuccess;
  const int grid = grid_for(groups, kThreads);
  const DivU32 nb = make_divu32((uint32_t)(cols / 16));
  if (!aligned32(out)) return cudaErrorInvalidValue;  // the GEMM workspace places it 256-byte aligned
  if4_to_f16_kernel<<<grid, kThreads, 0, s>>>(q, scales, groups, nb, reinterpret_cast<uint4*>(out));
  return cudaGetLastError();
}

cudaError_t launch_dequant(const DequantLaunch& L, cudaStream_t s) {
  const long long groups = L.rows * L.cols / 16;
  if (groups == 0) return cudaSuccess;
  const DivU32 nb = make_divu32((uint32_t)(L.cols / (L.format != 0 ? 16 : 32)));
  const int grid = grid_for(groups, kThreads);
  const float* gl = L.format != 0 ? L.global : nullptr;
  auto go = [&](auto kernel) { kernel<<<grid, kThreads, 0, s>>>(L.q, L.scales, gl, groups, nb, L.tiled, L.out); };
  auto pick = [&](auto fmt) {
    constexpr int F = decltype(fmt)::value;
    if (aligned32(L.out)) {
      if (L.out_bf16) go(dequant_kernel<F, true, true>); else go(dequant_kernel<F, false, true>);
    } else {
      if (L.out_bf16) go(dequant_kernel<F, true, false>); else go(dequant_kernel<F, false, false>);
    }
  };
  if (L.format == 2) pick(std::integral_constant<int, 2>{});
  else if (L.format == 1) pick(std::integral_constant<int, 1>{});
  else pick(std::integral_constant<int, 0>{});
  return cudaGetLastError();
}

}  // namespace fp4k
