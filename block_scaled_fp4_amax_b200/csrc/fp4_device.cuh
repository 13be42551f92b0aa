// fp4_device.cuh — device-side building blocks shared by the quantise / rotate / dequantise
// kernels of libfp4mx: 256-bit lane loads, the sm_100 FP4/FP8 conversion instructions,
// Philox4x32-10, the E2M1 rounding rules and the block encoders.
//
// Every floating-point step that decides a code is an explicitly rounded fp32 intrinsic
// (__fmul_rn, __fadd_rn, __fsub_rn, __frcp_rn, __fdiv_rn) so the compiler cannot contract or
// reorder it.
#pragma once

#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>

namespace fp4k {

// ---------------------------------------------------------------------------------------------
// Programmatic dependent launch (sm_90 and later).  A kernel launched with programmatic stream
// serialisation may be scheduled while its predecessor on the stream still runs.  grid_dep_wait()
// blocks until that predecessor has completed and its memory is visible (a no-op after an
// ordinary launch); grid_dep_trigger() lets the dependent grid be scheduled once every CTA of this
// grid has started, so its CTAs take SMs as this grid's CTAs retire instead of after a launch gap.
__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_trigger() { asm volatile("griddepcontrol.launch_dependents;" ::: "memory"); }

// ---------------------------------------------------------------------------------------------
// Loads.
// 32 bytes per lane (sm_100 256-bit load): a warp reads 1 KiB of contiguous memory per
// instruction.  `Stream` marks the lines evict-first in L2 (last use); otherwise they are kept
// for a following pass.
struct U8 {
  uint32_t w[8];
};
template <bool Stream>
__device__ __forceinline__ U8 ld32(const void* p) {
  U8 r;
  if (Stream) {
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_first.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]),
                   "=r"(r.w[6]), "=r"(r.w[7])
                 : "l"(p));
  } else {
    asm volatile("ld.global.nc.L1::no_allocate.L2::evict_last.v8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r.w[0]), "=r"(r.w[1]), "=r"(r.w[2]), "=r"(r.w[3]), "=r"(r.w[4]), "=r"(r.w[5]),
                   "=r"(r.w[6]), "=r"(r.w[7])
                 : "l"(p));
  }
  return r;
}

// Stores.
// 32 bytes per lane (sm_100 256-bit store, `p` 32-byte aligned): each lane fills whole 32-byte
// sectors, where two 16-byte stores from lanes 32 bytes apart would half-fill twice as many.
__device__ __forceinline__ void st32(void* p, const uint32_t (&w)[8]) {
  asm volatile("st.global.v8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};" ::"l"(p), "r"(w[0]), "r"(w[1]), "r"(w[2]),
               "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
               : "memory");
}

// Element traits for a 32-byte chunk: E values, unpacked to fp32 (exact), and the number of
// values that are +-0 (from the bit patterns: the magnitude bits of a nonzero value, plus all
// ones, carry into the top bit of its field).
template <typename T> struct Vec32;
template <> struct Vec32<float> {
  static constexpr int E = 8;
  __device__ __forceinline__ static void unpack(const U8& r, float* v) {
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r.w[i]);
  }
  __device__ __forceinline__ static int zeros(const U8& r) {
    int nz = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) nz += (r.w[i] & 0x7FFFFFFFu) != 0u;
    return 8 - nz;
  }
  // Largest magnitude bit pattern of the chunk; `any_zero` is set if some value is +-0.
  __device__ __forceinline__ static uint32_t max_mag(const U8& r, bool& any_zero) {
    uint32_t m = 0u, mn = 0xFFFFFFFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a = r.w[i] & 0x7FFFFFFFu;
      m = max(m, a);
      mn = min(mn, a);
    }
    any_zero = mn == 0u;
    return m;
  }
};
template <> struct Vec32<__nv_bfloat16> {
  static constexpr int E = 16;
  // bf16 -> fp32 as the exact mixed-precision sum x + (-0): it runs on the FMA pipe, where two
  // shifts/masks per pair would load the integer pipe, the busiest one in the quantisers.
  __device__ __forceinline__ static void unpack(const U8& r, float* v) {
#pragma unroll
    for (int i = 0; i < 8; ++i)
      asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tadd.rn.f32.bf16 %0, l, 0f80000000;\n\t"
          "add.rn.f32.bf16 %1, u, 0f80000000;\n\t}" : "=f"(v[2 * i]), "=f"(v[2 * i + 1]) : "r"(r.w[i]));
  }
  __device__ __forceinline__ static int zeros(const U8& r) {
    int nz = 0;
#pragma unroll
    for (int i = 0; i < 8; ++i) nz += __popc(((r.w[i] & 0x7FFF7FFFu) + 0x7FFF7FFFu) & 0x80008000u);
    return 16 - nz;
  }
  // Largest magnitude as an fp32 bit pattern (lane-wise bf16x2 max of the sign-cleared values, on
  // the half-precision pipe; a NaN makes the result the canonical NaN 0x7FFF, above +Inf, so the
  // block still reads as non-finite); `any_zero` is set if some value is +-0 (lane-wise minimum
  // magnitude 0; the bf16 minimum ignores NaN operands).
  __device__ __forceinline__ static uint32_t max_mag(const U8& r, bool& any_zero) {
    uint32_t m = 0u, mn = 0x7FFF7FFFu;
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const uint32_t a = r.w[i] & 0x7FFF7FFFu;
      asm("max.NaN.bf16x2 %0, %0, %1;" : "+r"(m) : "r"(a));
      asm("min.bf16x2 %0, %0, %1;" : "+r"(mn) : "r"(a));
    }
    any_zero = ((mn & 0xFFFFu) == 0u) | ((mn >> 16) == 0u);
    return max(m & 0xFFFFu, m >> 16) << 16;
  }
};

// Number of +-0 codes among the 8 nibbles of a packed word.
__device__ __forceinline__ int zero_nibbles(uint32_t p) {
  return 8 - __popc(((p & 0x77777777u) + 0x77777777u) & 0x88888888u);
}

// ---------------------------------------------------------------------------------------------
// E2M1 encode of pairs with the sm_100 conversion (round to nearest even, saturating to +-6).
// Packs 8 values into one 32-bit word: value i in bits [4i, 4i+4) — element 2j in the low
// nibble of byte j.
__device__ __forceinline__ uint32_t e2m1x8(const float* y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b2, %6, %5;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b3, %8, %7;\n\t"
      "mov.b32 %0, {b0, b1, b2, b3};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]), "f"(y[4]), "f"(y[5]), "f"(y[6]), "f"(y[7]));
  return out;
}
__device__ __forceinline__ uint32_t e2m1x4(const float* y) {
  uint32_t out;
  asm("{\n\t.reg .b8 b0, b1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b0, %2, %1;\n\t"
      "cvt.rn.satfinite.e2m1x2.f32 b1, %4, %3;\n\t"
      "mov.b32 %0, {b0, b1, 0, 0};\n\t}"
      : "=r"(out)
      : "f"(y[0]), "f"(y[1]), "f"(y[2]), "f"(y[3]));
  return out;
}

// Two f16 halves of a 32-bit word to fp32 (exact), without type punning.
__device__ __forceinline__ void f16x2_to_f32(uint32_t h, float& lo, float& hi) {
  asm("{\n\t.reg .b16 l, u;\n\tmov.b32 {l, u}, %2;\n\tcvt.f32.f16 %0, l;\n\tcvt.f32.f16 %1, u;\n\t}"
      : "=f"(lo), "=f"(hi) : "r"(h));
}

// Round two fp32 values to bf16 (RNE) and pack them: `lo` in bits 0-15, `hi` in bits 16-31.
__device__ __forceinline__ uint32_t bf16x2_pack(float lo, float hi) {
  uint32_t r;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(r) : "f"(hi), "f"(lo));
  return r;
}

// The 8 nibbles of `codes` as four f16x2 words (byte b -> h[b], low nibble in the low half).
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t codes, uint32_t* h) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(h[0]), "=r"(h[1]), "=r"(h[2]), "=r"(h[3]) : "r"(codes));
}

// Decode the low E nibbles of `codes` back to fp32 (exact) through f16x2.
template <int E>
__device__ __forceinline__ void e2m1_unpack(uint32_t codes, float* v) {
  uint32_t h[4];
  e2m1x8_to_f16x2(codes, h);
#pragma unroll
  for (int i = 0; i < E / 2; ++i) f16x2_to_f32(h[i], v[2 * i], v[2 * i + 1]);
}

// Two fp32 values in one 64-bit register (first value in the low half) and the sm_100 packed
// fp32 arithmetic on such pairs: each half is an IEEE fp32 operation rounded to nearest even.
typedef unsigned long long f32x2;
__device__ __forceinline__ f32x2 f2_pack(float lo, float hi) {
  f32x2 r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "r"(__float_as_uint(lo)), "r"(__float_as_uint(hi)));
  return r;
}
__device__ __forceinline__ void f2_unpack(f32x2 v, float& lo, float& hi) {
  uint32_t a, b;
  asm("mov.b64 {%0, %1}, %2;" : "=r"(a), "=r"(b) : "l"(v));
  lo = __uint_as_float(a);
  hi = __uint_as_float(b);
}
__device__ __forceinline__ f32x2 f2_mul(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_sub(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("sub.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}
__device__ __forceinline__ f32x2 f2_add(f32x2 a, f32x2 b) {
  f32x2 d;
  asm("add.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// E4M3 (E4M3FN) round to nearest even, saturating at 448; u >= 0.  Returns the code byte.
__device__ __forceinline__ uint32_t e4m3_code(float u) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(0.0f), "f"(u));
  return r & 0xFFu;
}
// Exact fp32 value of an E4M3 code byte.
__device__ __forceinline__ float e4m3_value(uint32_t code) {
  uint32_t h;
  const uint16_t c = (uint16_t)code;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(h) : "h"(c));
  float lo, hi;
  f16x2_to_f32(h, lo, hi);
  return lo;
}

// ---------------------------------------------------------------------------------------------
// Philox4x32-10 (Salmon et al., SC'11): ten rounds of two 32x32->64 multiplies with the round
// keys advanced by the Weyl increments.  Counter (blk lo, blk hi, 0, 0), key (seed lo, seed hi).
// The round keys depend only on the seed (key + r * Weyl increment), so the host computes them once
// and the kernels read them from their parameter block: a round is then two 32x32->64 multiplies
// and two three-input XORs.
struct PhiloxKeys {
  uint32_t k0[10], k1[10];
};
inline PhiloxKeys philox_keys(unsigned long long seed) {
  PhiloxKeys K;
  for (int r = 0; r < 10; ++r) {
    K.k0[r] = (uint32_t)seed + (uint32_t)r * 0x9E3779B9u;
    K.k1[r] = (uint32_t)(seed >> 32) + (uint32_t)r * 0xBB67AE85u;
  }
  return K;
}

struct Philox4 { uint32_t w[4]; };
__device__ __forceinline__ Philox4 philox4x32_10(uint64_t blk, const PhiloxKeys& K) {
  uint32_t c0 = (uint32_t)blk, c1 = (uint32_t)(blk >> 32), c2 = 0u, c3 = 0u;
#pragma unroll
  for (int r = 0; r < 10; ++r) {
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ K.k0[r];
    const uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ K.k1[r];
    c0 = n0; c1 = (uint32_t)p1; c2 = n2; c3 = (uint32_t)p0;
  }
  Philox4 o;
  o.w[0] = c0; o.w[1] = c1; o.w[2] = c2; o.w[3] = c3;
  return o;
}

// Random words for E consecutive elements starting at flat index idx0 (idx0 % 4 == 0).
template <int E>
__device__ __forceinline__ void sr_words(uint64_t idx0, const PhiloxKeys& K, uint32_t* r) {
#pragma unroll
  for (int k = 0; k < E / 4; ++k) {
    Philox4 p = philox4x32_10((idx0 >> 2) + k, K);
#pragma unroll
    for (int i = 0; i < 4; ++i) r[4 * k + i] = p.w[i];
  }
}

__device__ __forceinline__ uint32_t f2u_ceil(float x) {  // x in [0, 2^32): ceil, exact
  uint32_t u;
  asm("cvt.rpi.u32.f32 %0, %1;" : "=r"(u) : "f"(x));
  return u;
}

// Stochastic rounding of y onto the E2M1 lattice, returned directly as its 4-bit code (sign in
// bit 3).  For a = |y| <= 6 with lo the largest lattice point <= a and p = (a - lo)/step, the value
// rounds up iff r < ceil(p * 2^32); a > 6 (and Inf/NaN) gives 6.  The lattice is consecutive in
// code order, so the result is code(lo) + up, capped at 7:
//   a in [1, 8): the points of [2^e, 2^(e+1)) are 2^e * {1, 1.5}, so code(lo) = 2 + 2e + (top
//     mantissa bit) = (bits >> 22) - 252, and p * 2^32 is the remaining 22-bit mantissa field
//     shifted left by 10 (an exact integer);
//   a < 1: points 0, 0.5, 1 (codes 0, 1, 2); T = a * 2^33 is exact, code(lo) = [T >= 2^32] and
//     p * 2^32 = T - [T >= 2^32] * 2^32 (exact), whose ceiling is the threshold.
__device__ __forceinline__ uint32_t sr_code(float y, uint32_t r) {
  const uint32_t bits = __float_as_uint(y);
  const uint32_t ab = bits & 0x7FFFFFFFu;
  const float T = __fmul_rn(__uint_as_float(ab), 8589934592.0f);  // 2^33
  const bool half = T >= 4294967296.0f;                           // a >= 0.5
  const uint32_t th_small = f2u_ceil(half ? __fsub_rn(T, 4294967296.0f) : T);
  const bool ge1 = ab >= 0x3F800000u;
  const uint32_t th = ge1 ? (ab & 0x003FFFFFu) << 10 : th_small;
  const uint32_t lo = ge1 ? (ab >> 22) - 252u : (half ? 1u : 0u);
  const uint32_t code = min(lo + (r < th ? 1u : 0u), 7u);
  return code | ((bits >> 28) & 8u);
}

// N stochastically rounded codes packed 8 per word, value 0 in the lowest nibble.
template <int N>
__device__ __forceinline__ void sr_pack_n(const float* y, const uint32_t* rnd, uint32_t* w) {
#pragma unroll
  for (int k = 0; k < (N + 7) / 8; ++k) {
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 7; i >= 0; --i) {
      const int j = 8 * k + i;
      acc = (acc << 4) | (j < N ? sr_code(y[j], rnd[j]) : 0u);
    }
    w[k] = acc;
  }
}

// ---------------------------------------------------------------------------------------------
// Block encoding helpers shared by the quantiser and the fused rotation (N = values per lane,
// 1..16; packed words hold 8 nibbles each, value 0 in the lowest nibble).

template <int N>
__device__ __forceinline__ void e2m1_pack_n(const float* y, uint32_t* w) {
  if constexpr (N >= 8) {
#pragma unroll
    for (int k = 0; k < N / 8; ++k) w[k] = e2m1x8(y + 8 * k);
  } else {
    float t[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) t[i] = (i < N) ? y[i] : 0.0f;
    w[0] = e2m1x4(t);
  }
}

template <int N>
__device__ __forceinline__ void e2m1_unpack_n(const uint32_t* w, float* q) {
  if constexpr (N >= 8) {
#pragma unroll
    for (int k = 0; k < N / 8; ++k) e2m1_unpack<8>(w[k], q + 8 * k);
  } else {
    float o[4];
    e2m1_unpack<4>(w[0], o);
#pragma unroll
    for (int i = 0; i < N; ++i) q[i] = o[i];
  }
}

template <int N>
__device__ __forceinline__ int zero_codes_n(const uint32_t* w) {
  if constexpr (N >= 8) {
    int z = 0;
#pragma unroll
    for (int k = 0; k < N / 8; ++k) z += zero_nibbles(w[k]);
    return z;
  } else {
    return zero_nibbles(w[0]) - (8 - N);  // the 8 - N padding nibbles encode 0.0
  }
}

// N values scaled by R and E2M1-encoded (RNE or stochastic); with CNT, saturations are counted per
// value only when the block maximum normalises above 6 (`top` = fl(amax * R), monotone in |x|);
// without it the caller counts them (sat_count_bf16x16).  `y` receives the scaled values
// fl(v * R) (before any stochastic rounding).
template <int N, bool SR, bool CNT = true>
__device__ __forceinline__ void encode_y_n(const float* v, float R, float top, const uint32_t* rnd,
                                           float* y, uint32_t* w, uint32_t& sat) {
  if constexpr (N % 2 == 0) {
    const f32x2 R2 = f2_pack(R, R);
#pragma unroll
    for (int j = 0; j < N; j += 2) f2_unpack(f2_mul(f2_pack(v[j], v[j + 1]), R2), y[j], y[j + 1]);
  } else {
#pragma unroll
    for (int i = 0; i < N; ++i) y[i] = __fmul_rn(v[i], R);
  }
  if (CNT && !(top <= 6.0f)) {  // a NaN top (a NaN in the block) still counts its infinities
#pragma unroll
    for (int i = 0; i < N; ++i) sat += fabsf(y[i]) > 6.0f;
  }
  if (SR) {
    sr_pack_n<N>(y, rnd, w);
  } else {
    e2m1_pack_n<N>(y, w);
  }
}

template <int N, bool SR, bool CNT = true>
__device__ __forceinline__ void encode_n(const float* v, float R, float top, const uint32_t* rnd,
                                         uint32_t* w, uint32_t& sat) {
  float y[N];
  encode_y_n<N, SR, CNT>(v, R, top, rnd, y, w, sat);
}

// Count of the 16 bf16 values (8 packed words) whose magnitude is at least the bf16 magnitude
// pattern t (both halves of t2), by bf16x2 compares accumulated in bf16x2 (exact small integers).
__device__ __forceinline__ uint32_t count_ge_bf16x16(const uint32_t* w, uint32_t t2) {
  uint32_t acc;
  asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(acc) : "r"(w[0] & 0x7FFF7FFFu), "r"(t2));
#pragma unroll
  for (int i = 1; i < 8; ++i) {
    uint32_t s;
    asm("set.ge.bf16x2.bf16x2 %0, %1, %2;" : "=r"(s) : "r"(w[i] & 0x7FFF7FFFu), "r"(t2));
    asm("add.rn.bf16x2 %0, %0, %1;" : "+r"(acc) : "r"(s));
  }
  return (uint32_t)(__uint_as_float(acc << 16) + __uint_as_float(acc & 0xFFFF0000u));
}

// MXFP4 saturation count of 16 bf16 values under the shared exponent e (scale 2^e, normal 6 * 2^e):
// scaling by 2^-e is exact, so |v| * 2^-e > 6 iff |v| > 6 * 2^e, i.e. |v| is at least the bf16
// value one step above 6 * 2^e = 1.5 * 2^(e+2) (bf16 pattern ((e + 129) << 7) | 0x40).
__device__ __forceinline__ uint32_t mx_sat_count_bf16x16(const uint32_t* w, int e) {
  const uint32_t t = (((uint32_t)(e + 129)) << 7 | 0x40u) + 1u;
  return count_ge_bf16x16(w, t | (t << 16));
}

// Saturation count of 16 bf16 values (8 packed words) under the scale pair (D, R = fl(1/D)):
// the number of values with fl(|v| * R) > lim (6 for E2M1, 7 for IF4's INT4).  The predicate is
// monotone in |v|, so it holds exactly for |v| >= t, t the smallest bf16 magnitude that satisfies
// it.  lim * D and the real threshold (lim + 2^-22) / R differ by about 2^-22 relative while one
// bf16 step is at least 2^-8, so t is one of the three bf16 values from b0 = bf16_rd(fl(lim * D))
// up, and two predicate tests pick it.  The count is then 8 bf16x2 compares accumulated in bf16x2
// (exact small integers).  Only meaningful when the block maximum saturates (fl(amax * R) > lim,
// so D is positive and finite).
__device__ __forceinline__ uint32_t sat_count_bf16x16(const uint32_t* w, float D, float R, float lim = 6.0f) {
  const uint32_t xb = __float_as_uint(__fmul_rn(lim, D)) & 0xFFFF0000u;
  const uint32_t tb = (__fmul_rn(__uint_as_float(xb), R) > lim)             ? xb
                      : (__fmul_rn(__uint_as_float(xb + 0x10000u), R) > lim) ? xb + 0x10000u
                                                                             : xb + 0x20000u;
  return count_ge_bf16x16(w, (tb >> 16) | (tb & 0xFFFF0000u));
}

// NVFP4 per-code scale table: for every E4M3 code byte c, D = fl(value(c) * s_g) and
// R = fl(1 / D) (all 256 bytes, so a caller-supplied negative or non-finite global scale indexes
// inside it and behaves as the direct computation would).  Filled once per CTA into shared memory,
// it replaces the per-block decode, multiply and reciprocal.  Entry 0 holds R = 0: a block whose
// scale code is 0 has only finite values (a non-finite amax gives code 0x7E or 0x7F), so v * 0 is
// the signed zero that block encodes to, and no branch is needed for it.
constexpr int kScaleTab = 256;
__device__ __forceinline__ void fill_scale_tab(float2* tab, float s_g) {
  for (int c = threadIdx.x; c < kScaleTab; c += blockDim.x) {
    const float D = __fmul_rn(e4m3_value((uint32_t)c), s_g);
    tab[c] = make_float2(D, c == 0 ? 0.0f : __frcp_rn(D));
  }
}

// One NVFP4 candidate (target T through inv_t = fl(1/fl(T*s_g))): returns the E4M3 code and
// writes the packed nibbles and the saturation count.
template <int N, bool SR, bool CNT = true>
__device__ __forceinline__ uint32_t nv_candidate_n(const float* v, float amax, float inv_t, const float2* tab,
                                                   const uint32_t* rnd, uint32_t* w, uint32_t& sat,
                                                   float2* DR_out = nullptr) {
  const uint32_t sc = e4m3_code(__fmul_rn(amax, inv_t));
  sat = 0;
  const float2 DR = tab[sc];  // R = 0 for code 0: every value encodes to its signed zero
  encode_n<N, SR, CNT>(v, DR.y, __fmul_rn(amax, DR.y), rnd, w, sat);
  if (DR_out) *DR_out = DR;
  return sc;
}

// Squared dequantisation errors fl((x - fl(fl(q*d)*s_g))^2), d the value of E4M3 `code`.
//
// The packed words are decoded as `w ^ opaque0`, opaque0 a zero the kernel reads from its
// parameters.  With CUDA 12.9 on sm_100a, `cvt.rn.f16x2.e2m1x2` applied to bytes 2 and 3 of a word
// that was just assembled in registers from `cvt.rn.satfinite.e2m1x2.f32` results returned zeros in
// some kernels (observed by comparing the decoded values with the stored nibbles).  A decode of a
// word the compiler cannot trace back to those byte registers (one loaded from memory, or XORed
// with a value only known at run time) is correct, so every in-register decode goes through it.
// For pairs, v*d is formed in f16x2 straight from the nibble conversion: |v| <= 6 has two
// significant bits and d four, so the product (at least 2^-10, at most 2688) is exact in f16.
template <int N>
__device__ __forceinline__ void sq_errors_n(const float* v, const uint32_t* w, uint32_t code, float s_g,
                                            uint32_t opaque0, float* sq) {
  if constexpr (N % 2 == 0) {
    uint32_t dh2;
    asm("cvt.rn.f16x2.e4m3x2 %0, %1;" : "=r"(dh2) : "h"((uint16_t)(code | (code << 8))));
#pragma unroll
    for (int k = 0; k < (N + 7) / 8; ++k) {
      uint32_t h[4];
      e2m1x8_to_f16x2(w[k] ^ opaque0, h);
#pragma unroll
      for (int b = 0; b < 4; ++b) {
        const int j = 8 * k + 2 * b;
        if (j < N) {
          uint32_t qd;
          asm("mul.rn.f16x2 %0, %1, %2;" : "=r"(qd) : "r"(h[b]), "r"(dh2));
          float lo, hi;
          f16x2_to_f32(qd, lo, hi);
          // scalar __fmul_rn/__fsub_rn: never contracted into an FMA (packed f32x2 mul + sub
          // pairs can be, which would round the error differently)
          const float el = __fsub_rn(v[j], __fmul_rn(lo, s_g));
          const float eh = __fsub_rn(v[j + 1], __fmul_rn(hi, s_g));
          sq[j] = __fmul_rn(el, el);
          sq[j + 1] = __fmul_rn(eh, eh);
        }
      }
    }
    return;
  }
  const float d = e4m3_value(code);
  uint32_t wo[(N + 7) / 8];
#pragma unroll
  for (int k = 0; k < (N + 7) / 8; ++k) wo[k] = w[k] ^ opaque0;
  float q[N];
  e2m1_unpack_n<N>(wo, q);
#pragma unroll
  for (int i = 0; i < N; ++i) {
    const float xhat = __fmul_rn(__fmul_rn(q[i], d), s_g);
    const float e = __fsub_rn(v[i], xhat);
    sq[i] = __fmul_rn(e, e);
  }
}

// fp32 sum of a block's squared errors in element order.  G = 1: the lane owns the block; G > 1:
// every lane of the block adds the broadcast values of lanes 0..G-1 (each holding N values).
template <int N, int G>
__device__ __forceinline__ float block_sse_n(const float* sq, int lane) {
  float acc = 0.0f;
  if constexpr (G == 1) {
#pragma unroll
    for (int i = 0; i < N; ++i) acc = __fadd_rn(acc, sq[i]);
  } else {
    const int base = lane & ~(G - 1);
#pragma unroll
    for (int g = 0; g < G; ++g) {
#pragma unroll
      for (int i = 0; i < N; ++i) acc = __fadd_rn(acc, __shfl_sync(0xFFFFFFFFu, sq[i], base + g));
    }
  }
  return acc;
}

// ---------------------------------------------------------------------------------------------
// IF4 ("Adaptive Block-Scaled Data Types" podcast, IF4 segment): every 16-block is encoded as
// plain NVFP4 E2M1 and as sign-magnitude INT4 on the step D7 = fl(d * s7), s7 = fl(s_g * fl(6/7))
// (the block maximum lands on 7 instead of 6).  INT4 is kept iff its fp32 sequential error sum is
// strictly lower, and the choice is bit 7 of the E4M3 scale byte.
constexpr float kSixSevenths = 0x1.b6db6ep-1f;  // fl(6/7)

// Per-code INT4 step table: for every E4M3 byte c, D7 = fl(value(c) * s7) and R7 = fl(1 / D7)
// when that is a finite nonzero number, else 0 (code 0 included).  A block whose R7 is 0 keeps
// E2M1: its INT4 candidate has no usable step.
__device__ __forceinline__ void fill_int4_tab(float2* tab, float s7) {
  for (int c = threadIdx.x; c < kScaleTab; c += blockDim.x) {
    const float D7 = __fmul_rn(e4m3_value((uint32_t)c), s7);
    const float R7 = __frcp_rn(D7);
    tab[c] = make_float2(D7, (fabsf(R7) < INFINITY && R7 != 0.0f) ? R7 : 0.0f);
  }
}

// Sum over the 8 nibble positions i of (bits of 2^23) << 4i, modulo 2^32: what packing the raw
// bit patterns of fl(a + 2^23) adds on top of the integers a.
__host__ __device__ constexpr uint32_t int4_pack_fold() {
  uint32_t f = 0u;
  for (int i = 0; i < 8; ++i) f += 0x4B000000u << (4 * i);
  return f;
}

// INT4 candidate of N values (N % 8 == 0) with step reciprocal R7, E4M3 scale value d and
// s7: the packed sign-magnitude nibbles and the squared errors fl((x - fl(fl(k*d)*s7))^2).
//   |k| = nearest integer to min(|fl(x * R7)|, 7), ties to even: adding 2^23 rounds a value in
//   [0, 7] to an integer in the low mantissa bits (one ulp is 1 there), so the bit patterns pack
//   with one shift-add per value and a constant correction (int4_pack_fold).
//   The sign bits are those of the E2M1 candidate's nibbles (`w_e2m1`): both are the sign of
//   fl(x * R), and R, R7 have the sign of s_g.
//   x_hat has the sign of x (or is zero), so |x - x_hat| = |x| - |x_hat| exactly; |k| * d is exact
//   (at most 7 significant bits).
template <int N>
__device__ __forceinline__ void int4_candidate_n(const float* v, float R7, float d, float s7,
                                                 const uint32_t* w_e2m1, uint32_t* w7, float* sq) {
  static_assert(N % 8 == 0, "whole packed words");
  const f32x2 R2 = f2_pack(R7, R7), M2 = f2_pack(0x1p23f, 0x1p23f), d2 = f2_pack(d, d);
#pragma unroll
  for (int k = 0; k < N / 8; ++k) {
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int j = 8 * k + i;
      float y0, y1;
      f2_unpack(f2_mul(f2_pack(v[j], v[j + 1]), R2), y0, y1);
      const f32x2 t = f2_add(f2_pack(fminf(fabsf(y0), 7.0f), fminf(fabsf(y1), 7.0f)), M2);
      float t0, t1;
      f2_unpack(t, t0, t1);
      acc += __float_as_uint(t0) << (4 * i);
      acc += __float_as_uint(t1) << (4 * i + 4);
      float kd0, kd1;
      f2_unpack(f2_mul(f2_sub(t, M2), d2), kd0, kd1);
      const float e0 = __fsub_rn(fabsf(v[j]), __fmul_rn(kd0, s7));
      const float e1 = __fsub_rn(fabsf(v[j + 1]), __fmul_rn(kd1, s7));
      sq[j] = __fmul_rn(e0, e0);
      sq[j + 1] = __fmul_rn(e1, e1);
    }
    w7[k] = (acc - int4_pack_fold()) | (w_e2m1[k] & 0x88888888u);
  }
}

// The INT4 candidate for the estimate path: the packed nibbles of int4_candidate_n and the
// residual sum sum (k - y)^2 = sum (|y| - |k|)^2 (k has the sign of y), formed with FMAs into
// two partial sums (an estimate; if4_undecided allows for its rounding).
template <int N>
__device__ __forceinline__ float int4_encode_resid_n(const float* v, float R7, const uint32_t* w_e2m1, uint32_t* w7) {
  static_assert(N % 8 == 0, "whole packed words");
  const f32x2 R2 = f2_pack(R7, R7), M2 = f2_pack(0x1p23f, 0x1p23f);
  f32x2 acc2 = 0ull;  // even and odd values in the two halves: one packed FMA per pair
#pragma unroll
  for (int k = 0; k < N / 8; ++k) {
    uint32_t acc = 0u;
#pragma unroll
    for (int i = 0; i < 8; i += 2) {
      const int j = 8 * k + i;
      float y0, y1;
      f2_unpack(f2_mul(f2_pack(v[j], v[j + 1]), R2), y0, y1);
      const float a0 = fabsf(y0), a1 = fabsf(y1);
      const f32x2 t = f2_add(f2_pack(fminf(a0, 7.0f), fminf(a1, 7.0f)), M2);
      float t0, t1;
      f2_unpack(t, t0, t1);
      acc += __float_as_uint(t0) << (4 * i);
      acc += __float_as_uint(t1) << (4 * i + 4);
      // residual |y| - |k|, the clamp's excess above 7 included
      const f32x2 r = f2_sub(f2_pack(a0, a1), f2_sub(t, M2));
      asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc2) : "l"(r));
    }
    w7[k] = (acc - int4_pack_fold()) | (w_e2m1[k] & 0x88888888u);
  }
  float a0, a1;
  f2_unpack(acc2, a0, a1);
  return a0 + a1;
}

// ---------------------------------------------------------------------------------------------
// Four-over-six selection without the exact error sums in the common case.
//
// The selection rule compares S_T = fp32 sequential sum of fl(fl(v - fl(fl(q*d)*s_g))^2) for the
// two candidates T = 6, 4.  A cheaper estimate of the same quantity is the scaled-domain residual
//   A_T = fl(D^2) * sum (q_i - y_i)^2,   y_i = fl(v_i * R), R = fl(1/D), D = fl(d * s_g),
// since (q_i - y_i) * D = -(e_i + theta_i v_i) with e_i = v_i - q_i d s_g and |theta_i| <= 3u
// (u = 2^-24).  With Q = sum e_i^2 and P = sum |e_i||v_i| <= 4 amax sqrt(Q), first-order rounding
// analysis gives |A_T - Q| <= 6uP + 22uQ and |S_T - Q| <= 2uP + 20uQ (16 terms, every operation
// one rounding, no overflow, normal D), so |A_T - S_T| <= 32u amax sqrt(Q) + 42uQ.
// The margin below is four times that (2^-17 = 128u on each term, sqrt(Q) <= 1.0001 sqrt(A_T) +
// 2^-19 amax), plus 2^-35 amax^2 for the second-order terms and 2^-139 for subnormal squares;
// amax sqrt(A) <= (amax^2 + A) / 2 then gives the square-root-free form used below.
// When |A_4 - A_6| exceeds it, sign(A_4 - A_6) = sign(S_4 - S_6) and the estimate decides; the
// caller computes S_T exactly otherwise.


// sum over N values of (q_i - y_i)^2: q_i decoded from the packed nibbles (exact in f16), the
// difference formed in fp32 from the f16 operand directly, the squares accumulated by packed FMAs
// into two partial sums (the estimate's bound allows any rounding order).  `opaque0` is a kernel-parameter zero
// (see sq_errors_n).
template <int N>
__device__ __forceinline__ float resid_sq_n(const uint32_t* w, const float* y, uint32_t opaque0) {
  static_assert(N % 2 == 0, "pairs");
  f32x2 acc = 0ull;  // even and odd values in the two halves: one packed FMA per pair
#pragma unroll
  for (int k = 0; k < (N + 7) / 8; ++k) {
    uint32_t h[4];
    e2m1x8_to_f16x2(w[k] ^ opaque0, h);
#pragma unroll
    for (int b = 0; b < 4; ++b) {
      const int j = 8 * k + 2 * b;
      if (j < N) {
        f32x2 r;
        asm("{\n\t.reg .b16 l, u;\n\t.reg .f32 rl, rh;\n\tmov.b32 {l, u}, %1;\n\t"
            "sub.rn.f32.f16 rl, l, %2;\n\tsub.rn.f32.f16 rh, u, %3;\n\tmov.b64 %0, {rl, rh};\n\t}"
            : "=l"(r) : "r"(h[b]), "f"(y[j]), "f"(y[j + 1]));
        asm("fma.rn.f32x2 %0, %1, %1, %0;" : "+l"(acc) : "l"(r));
      }
    }
  }
  float a0, a1;
  f2_unpack(acc, a0, a1);
  return a0 + a1;
}

// One NVFP4 candidate as nv_candidate_n, plus D = fl(d * s_g) and the residual sum A (both 0
// when the scale code is 0).
template <int N, bool SR, bool CNT = true>
__device__ __forceinline__ uint32_t nv_candidate_resid_n(const float* v, float amax, float inv_t, const float2* tab,
                                                         const uint32_t* rnd, uint32_t opaque0, uint32_t* w,
                                                         uint32_t& sat, float& D, float& A, float* R_out = nullptr) {
  const uint32_t sc = e4m3_code(__fmul_rn(amax, inv_t));
  sat = 0;
  const float2 DR = tab[sc];  // code 0: D = 0, R = 0, so y = +-0, the codes are zeros and A = 0
  D = DR.x;
  if (R_out) *R_out = DR.y;
  float y[N];
  encode_y_n<N, SR, CNT>(v, DR.y, __fmul_rn(amax, DR.y), rnd, y, w, sat);
  A = resid_sq_n<N>(w, y, opaque0);
  return sc;
}

// Decide four-over-six from the estimates when the margin allows.  `am` is the block amax bit
// pattern and A6/A4 the residual sums of the whole block.  Returns true when the exact sums are
// needed; otherwise `four` holds the decision.
__device__ __forceinline__ bool four_six_undecided(uint32_t am, float amax, float D6, float D4, float A6,
                                                   float A4, uint32_t sc6, uint32_t sc4, bool& four) {
  // equal scale codes make the two candidates identical (same scale, codes and errors): an exact
  // tie, which keeps 6 (a clamped scale, for example, under a small caller-supplied global scale)
  if (sc6 == sc4) {
    four = false;
    return false;
  }
  const float a6 = __fmul_rn(__fmul_rn(D6, D6), A6);
  const float a4 = __fmul_rn(__fmul_rn(D4, D4), A4);
  const float sa = a6 + a4;
  // amax (sqrt a6 + sqrt a4) <= amax^2 + (a6 + a4) / 2, so this is at least the margin above
  const float m = 7.62939453e-06f * (1.02f * amax * amax + 2.0f * sa) + __uint_as_float(0x00000400u);  // 2^-17, 2^-139
  const float diff = a4 - a6;
  // amax in [2^-50, 2^60); D4 >= D6 (monotone rounding of amax/(T s_g)) and D6 >= 2^-60 (so both
  // codes are nonzero and D is normal); finite estimates (a NaN fails `<`)
  const bool in_range = (am >= 0x26800000u) & (am < 0x5D800000u) & (D6 >= __uint_as_float(0x21800000u)) &
                        (sa < INFINITY);
  four = (am != 0u) & (diff < 0.0f);
  // an all-zero block has equal (zero) sums and keeps 6 without the exact path
  return (am != 0u) & !(in_range & (fabsf(diff) > m));
}

// ---------------------------------------------------------------------------------------------
// Exact decisions for one common shape of undecided block.
//
// On tensors with outlier channels the blocks holding an outlier often fall inside the estimate's
// margin: their small values encode to zero under both candidates, so the two sums differ only in
// the outlier's term and the estimates differ by rounding noise.  Such a block has, in each
// candidate, exactly one nonzero code, at the same position.  That element is the block maximum
// (codes are monotone in |x|), so |x| = amax there, and every other element has x_hat = +-0 in both
// candidates and the same error term fl(x_i^2).  The fp32 sequential error sums then differ in one
// term t = fl(fl(amax - xh)^2), xh = fl(fl(|q| d) s), and such a sum is monotone in each term: if the
// alternative's term is not below the incumbent's, its sum is not below either, and the incumbent
// stays (ties included).  Only the other outcome still needs the exact sums.  Valid for positive
// finite scales (s > 0, d > 0), a finite amax and a lane holding the whole block (two words).

// Bit 3 of every nibble whose 3-bit magnitude is nonzero.
__device__ __forceinline__ uint32_t nonzero_nibbles(uint32_t w) {
  return ((w & 0x77777777u) + 0x77777777u) & 0x88888888u;
}

// If the blocks wa and wb (two words each) both hold exactly one nonzero code, at the same position,
// their 3-bit magnitudes through ca, cb; false otherwise.
__device__ __forceinline__ bool single_nonzero_code(const uint32_t* wa, const uint32_t* wb, uint32_t& ca,
                                                    uint32_t& cb) {
  const uint32_t m0 = nonzero_nibbles(wa[0]), m1 = nonzero_nibbles(wa[1]);
  if (m0 != nonzero_nibbles(wb[0]) || m1 != nonzero_nibbles(wb[1]) || __popc(m0) + __popc(m1) != 1) return false;
  // the words' other nibbles have magnitude 0, so or-folding leaves the one nonzero magnitude
  uint32_t a = (wa[0] | wa[1]) & 0x77777777u, b = (wb[0] | wb[1]) & 0x77777777u;
  a |= a >> 16; b |= b >> 16;
  a |= a >> 8; b |= b >> 8;
  a |= a >> 4; b |= b >> 4;
  ca = a & 7u;
  cb = b & 7u;
  return true;
}

// E2M1 magnitude of a 3-bit code: 0, 0.5, 1, 1.5, 2, 3, 4, 6.
__device__ __forceinline__ float e2m1_magnitude(uint32_t c) {
  return c < 4u ? 0.5f * (float)c : (c == 7u ? 6.0f : (float)(c - 2u));
}

// fl(fl(amax - fl(fl(q d) s))^2): the squared error of the block maximum, as the exact sums form it.
__device__ __forceinline__ float max_term(float amax, float q, float d, float s) {
  const float e = __fsub_rn(amax, __fmul_rn(__fmul_rn(q, d), s));
  return __fmul_rn(e, e);
}

// Four-over-six: true when the single-term shape settles the choice, which is then 6 (kept).
__device__ __forceinline__ bool four_six_single_term(const uint32_t* w6, const uint32_t* w4, float amax,
                                                     uint32_t sc6, uint32_t sc4, float s_g) {
  uint32_t c6, c4;
  if (!single_nonzero_code(w6, w4, c6, c4)) return false;
  const float t6 = max_term(amax, e2m1_magnitude(c6), e4m3_value(sc6), s_g);
  const float t4 = max_term(amax, e2m1_magnitude(c4), e4m3_value(sc4), s_g);
  return t4 >= t6;
}

// IF4: the same for the E2M1 candidate (words w, scale code sc) against the INT4 one (words w7, the
// same scale, integer magnitudes, factor s7 = fl(s_g * fl(6/7))): true when E2M1 is kept.
__device__ __forceinline__ bool if4_single_term(const uint32_t* w, const uint32_t* w7, float amax, uint32_t sc,
                                                float s_g, float s7) {
  uint32_t c, k;
  if (!single_nonzero_code(w, w7, c, k)) return false;
  const float d = e4m3_value(sc);
  const float te = max_term(amax, e2m1_magnitude(c), d, s_g);
  const float ti = max_term(amax, (float)k, d, s7);
  return ti >= te;
}

// IF4: the same test for the E2M1 candidate (D, A) against the INT4 one (D7, A7).  The INT4
// reconstruction fl(fl(k*d)*s7), its step D7 = fl(d*s7) and y = fl(v*fl(1/D7)) take the rounded
// steps of the E2M1 ones (k*d exact, then one product with a per-tensor factor), so the bound
// holds as derived; D7 <= D, so the range test is on D7.  `eligible` is false when the INT4 step
// has no finite nonzero reciprocal: such a block keeps E2M1 without the exact path.  Returns true
// when the exact sums are needed; otherwise `int4` holds the decision.
__device__ __forceinline__ bool if4_undecided(uint32_t am, float amax, float D, float D7, float A, float A7,
                                              bool eligible, bool& int4) {
  const float a6 = __fmul_rn(__fmul_rn(D, D), A);
  const float a7 = __fmul_rn(__fmul_rn(D7, D7), A7);
  const float sa = a6 + a7;
  const float m = 7.62939453e-06f * (1.02f * amax * amax + 2.0f * sa) + __uint_as_float(0x00000400u);  // 2^-17, 2^-139
  const float diff = a7 - a6;
  const bool in_range = (am >= 0x26800000u) & (am < 0x5D800000u) & (D7 >= __uint_as_float(0x21800000u)) &
                        (sa < INFINITY);
  const bool live = eligible & (am != 0u);
  int4 = live & (diff < 0.0f);
  return live & !(in_range & (fabsf(diff) > m));
}

// ---------------------------------------------------------------------------------------------
// Scale-byte placement.  Row-major: the flat block index.  MMA tile layout: 128 x 4 tiles of
// 512 bytes, block-column groups fastest (the layout tcgen05.cp 32x128b.warpx4 expects).
__device__ __forceinline__ uint64_t scale_offset_rj(uint64_t r, uint32_t j, uint32_t nb) {
  return ((r >> 7) * (nb >> 2) + (j >> 2)) * 512u + (r & 31u) * 16u + ((r >> 5) & 3u) * 4u + (j & 3u);
}
// For a blocks-per-row count known at compile time (the compiler divides by a constant).
__device__ __forceinline__ uint64_t scale_offset(uint64_t blk, uint32_t nb, bool tiled) {
  if (!tiled) return blk;
  const uint64_t r = blk / nb;
  return scale_offset_rj(r, (uint32_t)(blk - r * nb), nb);
}

// Unsigned 32-bit division by an invariant divisor through a precomputed multiplier (Granlund and
// Montgomery, "Division by Invariant Integers using Multiplication", PLDI 1994, section 4): with
// l = ceil(log2 d) and m = floor(2^32 (2^l - d) / d) + 1, every n < 2^32 has
// n / d = (t + ((n - t) >> min(l, 1))) >> max(l - 1, 0), t the high word of m * n.
struct DivU32 {
  uint32_t d, m, s1, s2;
};
inline DivU32 make_divu32(uint32_t d) {
  uint32_t l = 0;
  while (l < 32 && (1ull << l) < d) ++l;
  DivU32 v;
  v.d = d;
  v.m = (uint32_t)(((1ull << 32) * ((1ull << l) - d)) / d + 1);
  v.s1 = l < 1 ? l : 1;
  v.s2 = l > 1 ? l - 1 : 0;
  return v;
}
__device__ __forceinline__ uint32_t div_u32(uint32_t n, const DivU32& v) {
  const uint32_t t = __umulhi(v.m, n);
  return (t + ((n - t) >> v.s1)) >> v.s2;
}
// For a run-time blocks-per-row count: the 32-bit path by multiplier, 64-bit division beyond it.
__device__ __forceinline__ uint64_t scale_offset(uint64_t blk, const DivU32& nb, bool tiled) {
  if (!tiled) return blk;
  if (blk < (1ull << 32)) {
    const uint32_t r = div_u32((uint32_t)blk, nb);
    return scale_offset_rj(r, (uint32_t)blk - r * nb.d, nb.d);
  }
  const uint64_t r = blk / nb.d;
  return scale_offset_rj(r, (uint32_t)(blk - r * nb.d), nb.d);
}

// ---------------------------------------------------------------------------------------------
// Counter reduction: per-thread partial counts -> one atomicAdd per CTA and counter.
template <int NC>
__device__ __forceinline__ void flush_counts(uint32_t (&c)[NC], unsigned long long* dst) {
  __shared__ unsigned long long red[NC];
  if (threadIdx.x < NC) red[threadIdx.x] = 0ull;
  __syncthreads();
#pragma unroll
  for (int i = 0; i < NC; ++i) {
    uint32_t v = c[i];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
    if ((threadIdx.x & 31) == 0 && v) atomicAdd(&red[i], (unsigned long long)v);
  }
  __syncthreads();
  if (threadIdx.x < NC && red[threadIdx.x]) atomicAdd(dst + threadIdx.x, red[threadIdx.x]);
}

}  // namespace fp4k
