/*
 * fp4_oracle.c — plain, slow CPU definition of block-scaled 4-bit microscaling.
 *
 * TEST INFRASTRUCTURE.  Only the tests, the smoke check and the bench's CPU-baseline leg may call
 * this code.  It shares nothing with the CUDA library: no headers, tables or helpers.  Every
 * encoder here works by enumerating its lattice (the audit page advises enumerating the lattice
 * rather than re-deriving a bit trick), and every floating-point step is a single IEEE fp32 (or
 * exact fp64) operation written out in the order the definition gives.  Build with
 * -O2 -ffp-contract=off and without fast-math so that no operation is fused or reassociated.
 *
 * Sources (page title and section):
 *   [E] "Sub-4-Bit Microscaling (NVFP4, MXFP4 & Walsh-Hadamard Rotation)", §1-§3.
 *   [A] "MXFP4 Quantization: Audit the 4.25-Bit Blocks".
 *   [X] metrale `hardware::exec` docs (E2M1 -> E4M3 conversion).
 *   [P] "Adaptive Block-Scaled Data Types for FP4 Training" podcast (block scaling, stochastic
 *       rounding, Hadamard transform, Four Over Six).
 *   Philox4x32-10: Salmon, Moraes, Dror, Shaw, "Parallel Random Numbers: As Easy as 1, 2, 3",
 *       SC'11, §4 (the Philox round function and key schedule).
 *
 * Readings where the pages are silent are listed beside each function.
 */
#include <math.h>
#include <stdint.h>
#include <string.h>

typedef struct {
  uint64_t underflow, saturation, nonfinite, blocks_four;
} ora_counts;

/* ------------------------------------------------------------------------------------------ */
/* E2M1 element.  [E] §1: 1 sign, 2 exponent, 1 mantissa bit, exponent bias 1, no Inf/NaN.
 * [A] "Read the FP4 E2M1 value lattice": exponent field 0 is subnormal (0 and 0.5).           */

double ora_e2m1_value(int code) {
  int s = (code >> 3) & 1, e = (code >> 1) & 3, m = code & 1;
  double mag = (e == 0) ? 0.5 * m : ldexp(1.0 + 0.5 * m, e - 1);
  return s ? -mag : mag;
}

/* Nearest lattice magnitude code (0..7) for a >= 0, a <= 6.  Exact ties take the code whose
 * mantissa bit is even ([A] "Read the FP4 E2M1 value lattice": ties-to-even on the lattice). */
static int e2m1_nearest_mag(double a) {
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c < 8; ++c) {
    double d = fabs(a - ora_e2m1_value(c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* RNE encode of a normalised value y.  Magnitudes strictly above 6, infinities included, clamp to
 * 6 ([A]: "the lab clamps them to signed 6").  The sign bit always follows signbit(y), so a
 * negative value that rounds to zero encodes -0 (0x8).  Returns the 4-bit code.
 * Domain: y is not NaN.  E2M1 has no NaN ([E] §1) and [A]'s receipt rejects non-finite input, so
 * the quantisers never encode a block that holds one (see ora_block_rejected); a NaN here gets
 * the placeholder -1, which no caller stores. */
int ora_e2m1_encode_rne(float y) {
  if (isnan(y)) return -1;
  double a = fabs((double)y);
  int mag = (a > 6.0) ? 7 : e2m1_nearest_mag(a);
  return (signbit(y) ? 8 : 0) | mag;
}

/* ------------------------------------------------------------------------------------------ */
/* Philox4x32-10 (Salmon et al. SC'11).  Round: with multipliers M0, M1, the pair products
 * (hi,lo) = M0*c0 and M1*c2 give (c0,c1,c2,c3) <- (hi(M1*c2)^c1^k0, lo(M1*c2), hi(M0*c0)^c3^k1,
 * lo(M0*c0)); between rounds the key is bumped by the Weyl constants.                         */

void ora_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2], uint32_t out[4]) {
  const uint32_t M0 = 0xD2511F53u, M1 = 0xCD9E8D57u;
  const uint32_t W0 = 0x9E3779B9u, W1 = 0xBB67AE85u;
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    uint64_t p0 = (uint64_t)M0 * c0;
    uint64_t p1 = (uint64_t)M1 * c2;
    uint32_t n0 = (uint32_t)(p1 >> 32) ^ c1 ^ k0;
    uint32_t n1 = (uint32_t)p1;
    uint32_t n2 = (uint32_t)(p0 >> 32) ^ c3 ^ k1;
    uint32_t n3 = (uint32_t)p0;
    c0 = n0; c1 = n1; c2 = n2; c3 = n3;
    k0 += W0;
    k1 += W1;
  }
  out[0] = c0; out[1] = c1; out[2] = c2; out[3] = c3;
}

/* The 32-bit random word of flat element index idx: key = (seed lo, seed hi), counter =
 * (idx/4 lo, idx/4 hi, 0, 0), word idx%4.  (Reading: the pages fix no mapping; this one keys
 * Philox on (seed, element index) as the problem statement asks, one call per 4 elements.)   */
uint32_t ora_sr_word(uint64_t seed, uint64_t idx) {
  uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  uint64_t blk = idx >> 2;
  uint32_t ctr[4] = {(uint32_t)blk, (uint32_t)(blk >> 32), 0u, 0u};
  uint32_t out[4];
  ora_philox4x32_10(ctr, key, out);
  return out[idx & 3];
}

/* Stochastic rounding of y onto the E2M1 lattice ([P]: round up or down with probability given by
 * the distance, so the expectation is y).  For a = |y| <= 6 let lo <= a < hi be consecutive
 * lattice magnitudes (lo = a when a is a lattice point); p = (a-lo)/(hi-lo) is exact; the value
 * rounds up iff r < ceil(p * 2^32).  a > 6 clamps to 6 (saturation, as for RNE).             */
int ora_e2m1_encode_sr(float y, uint32_t r) {
  if (isnan(y)) return -1; /* outside the domain, as for RNE */
  double a = fabs((double)y);
  int sign = signbit(y) ? 8 : 0;
  if (a > 6.0) return sign | 7;
  int lo = 0;
  for (int c = 0; c < 8; ++c)
    if (ora_e2m1_value(c) <= a) lo = c;
  if (lo == 7) return sign | 7; /* a == 6 exactly */
  double vlo = ora_e2m1_value(lo), vhi = ora_e2m1_value(lo + 1);
  double p = (a - vlo) / (vhi - vlo);
  double thresh = ceil(ldexp(p, 32));
  int up = (double)r < thresh;
  return sign | (up ? lo + 1 : lo);
}

/* ------------------------------------------------------------------------------------------ */
/* FP8 E4M3 (OCP E4M3FN): 1 sign, 4 exponent (bias 7), 3 mantissa bits; exponent field 0 is
 * subnormal; 0x7F/0xFF are NaN, so the largest finite magnitude is 448 (0x7E).  The NVFP4 block
 * scale is a positive E4M3 value ([E] §2, [P] block-scaling segment).                          */

double ora_e4m3_value(int code) {
  int s = (code >> 7) & 1, e = (code >> 3) & 15, m = code & 7;
  if (e == 15 && m == 7) return NAN;
  double mag = (e == 0) ? ldexp(m / 8.0, -6) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -mag : mag;
}

/* Round-to-nearest-even onto the positive E4M3 lattice, saturating to 448 (the "satfinite"
 * reading: a magnitude above 448, Inf included, becomes 448).  Ties take the even code.
 * Domain: u >= 0 and not NaN (a block maximum of a finite block times a per-tensor factor); a
 * NaN gets the placeholder -1, which no caller stores.                                       */
int ora_e4m3_encode_rne_satfinite(float u) {
  if (isnan(u)) return -1;
  double a = (double)u;
  if (!(a <= 448.0)) return 0x7E;
  int best = 0;
  double bestd = INFINITY;
  for (int c = 0; c <= 0x7E; ++c) {
    double d = fabs(a - ora_e4m3_value(c));
    if (d < bestd || (d == bestd && (c & 1) == 0 && (best & 1) == 1)) {
      best = c;
      bestd = d;
    }
  }
  return best;
}

/* ------------------------------------------------------------------------------------------ */
/* bf16 output rounding: round-to-nearest-even of an fp32 value to its top 16 bits.             */
uint16_t ora_f32_to_bf16_rne(float f) {
  uint32_t u;
  memcpy(&u, &f, 4);
  if ((u & 0x7F800000u) == 0x7F800000u && (u & 0x007FFFFFu)) return (uint16_t)((u >> 16) | 0x40);
  uint32_t low = u & 0xFFFFu, hi = u >> 16;
  if (low > 0x8000u || (low == 0x8000u && (hi & 1u))) hi += 1;
  return (uint16_t)hi;
}

/* ------------------------------------------------------------------------------------------ */
/* MXFP4.  [A] "Read the shared E8M0 scale": block exponent from the block maximum, clamped to
 * [-127, 127], byte = e + 127 (byte 0 for -127, 254 for 127, 0xFF never produced); all-zero block
 * uses e = 0.  policy 0 (OCP floor): e = floor(log2(amax/4)) = floor(log2 amax) - 2, taken
 * exactly from the binary exponent.  policy 1 (no saturation, [E] §2 sawtooth): the smallest e
 * with amax <= 6 * 2^e.                                                                       */

static int floor_log2(double a) { /* a > 0 finite: exact via frexp (a = f * 2^x, f in [.5,1)) */
  int x;
  frexp(a, &x);
  return x - 1;
}

/* Domain: amax finite (a block holding Inf or NaN is rejected before its exponent is taken); a
 * non-finite amax gets the placeholder 0.                                                      */
int ora_mx_exponent(float amax, int policy) {
  if (amax == 0.0f || !isfinite(amax)) return 0;
  double a = (double)amax;
  int e;
  if (policy == 0) {
    e = floor_log2(a) - 2;
  } else {
    e = floor_log2(a) - 3; /* 8 * 2^(E-3) > a, so this is below the answer: step up */
    while (!(a <= ldexp(6.0, e))) e += 1;
  }
  if (e < -127) e = -127;
  if (e > 127) e = 127;
  return e;
}

/* ------------------------------------------------------------------------------------------ */
/* Rejected blocks.  [A] "Publish the MXFP4 audit receipt" lists non-finite input among the inputs
 * to reject, and E2M1 has no Inf or NaN ([E] §1).  Reading: a block holding an Inf or a NaN is
 * rejected.  Its non-finite values are counted in `nonfinite`; its codes and scale byte are left
 * unspecified (the oracle writes zeros there as placeholders, not as a definition) and it adds
 * nothing to the underflow, saturation and blocks_four counters, which audit encoded values.
 * Returns the number of non-finite values among the n (0: the block is encoded).              */
int ora_block_nonfinite(const float* x, int n) {
  int k = 0;
  for (int i = 0; i < n; ++i)
    if (!isfinite(x[i])) k += 1;
  return k;
}

/* Encode one block with a given shared exponent e (the manual path of the audit page, and the
 * inner step of ora_mx_quantize): y = x * 2^-e in fp32 (exact unless it underflows), then RNE
 * or stochastic E2M1.  idx0 is the flat index of x[0] (for the random word).  Codes land in
 * codes[0..n-1] (one per byte, unpacked). */
void ora_mx_encode_block(const float* x, int n, int e, int round, uint64_t seed, uint64_t idx0,
                         uint8_t* codes, ora_counts* cnt) {
  int bad = ora_block_nonfinite(x, n);
  if (bad) { /* rejected: placeholder codes, only the non-finite count */
    cnt->nonfinite += (uint64_t)bad;
    memset(codes, 0, (size_t)n);
    return;
  }
  float inv_scale = ldexpf(1.0f, -e);
  for (int i = 0; i < n; ++i) {
    float y = x[i] * inv_scale;
    int c = (round == 0) ? ora_e2m1_encode_rne(y) : ora_e2m1_encode_sr(y, ora_sr_word(seed, idx0 + i));
    if (fabsf(y) > 6.0f) cnt->saturation += 1;
    if (x[i] != 0.0f && (c & 7) == 0) cnt->underflow += 1;
    codes[i] = (uint8_t)c;
  }
}

/* Largest magnitude of n values; a NaN anywhere makes it NaN (the IEEE maximum that propagates
 * NaN, as torch.amax does).  Only the tensor maximum of the two-pass NVFP4 scale depends on the
 * NaN rule: a rejected block's own maximum is never used.                                       */
static float block_amax(const float* x, int n) {
  float m = 0.0f;
  for (int i = 0; i < n; ++i) {
    float a = fabsf(x[i]);
    if (isnan(a) || a > m) m = a;
    if (isnan(m)) break;
  }
  return m;
}

/* Pack element 2j into the low nibble and 2j+1 into the high nibble of byte j
 * ([A] "Encode one MXFP4 block step by step": the first byte holds element 0 in its low half and
 * element 1 in its high half). */
static void pack_pairs(const uint8_t* codes, int n, uint8_t* out) {
  for (int j = 0; j < n / 2; ++j) out[j] = (uint8_t)((codes[2 * j] & 15) | ((codes[2 * j + 1] & 15) << 4));
}

/* x: [rows, cols] fp32 row-major; q: [rows, cols/2]; scales: [rows, cols/32] row-major bytes. */
/* idx_base: flat element index of x[0] in the tensor the rows belong to (the random words of
 * stochastic rounding are indexed by it; 0 for a whole tensor).  spec (nullable): one byte per
 * block, 1 where the block's outputs are defined (every value finite), 0 for a rejected block.
 * With a finite block the normalised values x * 2^-e are finite, so nothing else is left open. */
void ora_mx_quantize_at(const float* x, long rows, long cols, int policy, int round, uint64_t seed,
                        uint64_t idx_base, uint8_t* q, uint8_t* scales, ora_counts* cnt, uint8_t* spec) {
  const int B = 32;
  long nb = cols / B;
  uint8_t codes[32];
  for (long r = 0; r < rows; ++r) {
    for (long j = 0; j < nb; ++j) {
      const float* xb = x + r * cols + j * B;
      int bad = ora_block_nonfinite(xb, B);
      int e = bad ? 0 : ora_mx_exponent(block_amax(xb, B), policy);
      scales[r * nb + j] = bad ? 0 : (uint8_t)(e + 127); /* rejected block: placeholder byte */
      if (spec) spec[r * nb + j] = bad ? 0 : 1;
      ora_mx_encode_block(xb, B, e, round, seed, idx_base + (uint64_t)(r * cols + j * B), codes, cnt);
      pack_pairs(codes, B, q + r * (cols / 2) + j * (B / 2));
    }
  }
}

void ora_mx_quantize(const float* x, long rows, long cols, int policy, int round, uint64_t seed,
                     uint8_t* q, uint8_t* scales, ora_counts* cnt) {
  ora_mx_quantize_at(x, rows, cols, policy, round, seed, 0, q, scales, cnt, 0);
}

/* ------------------------------------------------------------------------------------------ */
/* NVFP4 two-level scaling.  [E] §2: an E4M3 scale per 16 elements under an FP32 per-tensor
 * scale.  Reading (the pages fix the formats, not the rounding steps): s_g = fl(amax_t / (6*M))
 * with M = 448 (M = 256 under four-over-six, see below), s_g = 1 for an all-zero tensor; for
 * target T: inv_T = fl(1/fl(T*s_g)), block code = E4M3_RNE_satfinite(fl(amax_b * inv_T)), d its
 * value; a zero code encodes the block as signed zeros; otherwise R = fl(1/fl(d*s_g)) and
 * y_i = fl(x_i * R).
 * Four over six ([P] Four Over Six segment): each block is encoded with T = 6 and with T = 4 and
 * keeps T = 4 iff its fp32 sum of squared errors is strictly lower; the global scale uses M = 256
 * (the segment's smaller per-tensor scale that avoids overflow and costs about 43% of the dynamic
 * range: 1 - 256/448 = 42.9%), which keeps the T = 4 code of the largest block (384) inside
 * E4M3's range.                                                                                */

float ora_nvfp4_global_scale(float amax_t, int four_six) {
  if (amax_t == 0.0f) return 1.0f;
  float six_m = four_six ? 1536.0f : 2688.0f;
  return amax_t / six_m;
}

/* One candidate encoding of a 16-block of finite values: returns the sum of squared
 * dequantisation errors.  *defined is cleared when one of the reading's fp32 steps gives a NaN
 * (the scale argument u, or a normalised value y): E4M3 and E2M1 encodings of a NaN are not
 * fixed by the pages.  That needs a per-tensor scale outside its domain (fl(T*s_g) rounding to
 * zero or overflowing, or a reciprocal of fl(d*s_g) that overflows), never a normal one.      */
static float nv_candidate(const float* x, int n, float amax_b, float s_g, float T, int round,
                          uint64_t seed, uint64_t idx0, uint8_t* codes, int* scale_code,
                          ora_counts* c, int* defined) {
  float ts = T * s_g;
  float inv_t = 1.0f / ts;
  float u = amax_b * inv_t;
  memset(c, 0, sizeof(*c));
  memset(codes, 0, (size_t)n);
  *scale_code = 0;
  if (isnan(u)) {
    *defined = 0;
    return NAN;
  }
  int sc = ora_e4m3_encode_rne_satfinite(u);
  float d = (float)ora_e4m3_value(sc);
  *scale_code = sc;
  if (sc == 0) {
    for (int i = 0; i < n; ++i) {
      codes[i] = (uint8_t)(signbit(x[i]) ? 8 : 0);
      if (x[i] != 0.0f) c->underflow += 1;
    }
  } else {
    float ds = d * s_g;
    float R = 1.0f / ds;
    for (int i = 0; i < n; ++i) {
      float y = x[i] * R;
      if (isnan(y)) {
        *defined = 0;
        return NAN;
      }
      int code = (round == 0) ? ora_e2m1_encode_rne(y) : ora_e2m1_encode_sr(y, ora_sr_word(seed, idx0 + i));
      if (fabsf(y) > 6.0f) c->saturation += 1; /* an overflowed (infinite) y included */
      if (x[i] != 0.0f && (code & 7) == 0) c->underflow += 1;
      codes[i] = (uint8_t)code;
    }
  }
  float sse = 0.0f;
  for (int i = 0; i < n; ++i) {
    float vd = (float)(ora_e2m1_value(codes[i]) * (double)d); /* exact: <= 6 significant bits */
    float xhat = vd * s_g;
    float err = x[i] - xhat;
    float sq = err * err;
    sse = sse + sq;
  }
  return sse;
}

/* ------------------------------------------------------------------------------------------ */
/* IF4 ([P] IF4 segment): each 16-block takes the NVFP4 block scale (block amax over 6, cast to
 * E4M3), is encoded twice, as E2M1 and as a signed integer scaled by 7/6 (the block maximum lands
 * on 7 instead of 6, so an integer step is 6/7 of the E2M1 unit), and keeps the encoding with the
 * lower squared error.  The choice goes into the scale byte's sign bit, which NVFP4 never uses
 * (0 = E2M1, 1 = INT4).  Readings where the segment is silent:
 *   - the INT4 nibble is sign-magnitude like E2M1: bit 3 is the sign of y, bits 0-2 hold |k| <= 7,
 *     so the integer lattice is -7..7 and -0 is encodable;
 *   - the step is formed in fp32 as s7 = fl(s_g * fl(6/7)) per tensor, D7 = fl(d * s7),
 *     R7 = fl(1 / D7); y = fl(x * R7); k = nearest integer to y, ties to even, |k| clamped to 7;
 *     the reconstruction is fl(fl(k * d) * s7) (k * d is exact), the INT4 analogue of
 *     fl(fl(v * d) * s_g);
 *   - INT4 is kept iff its fp32 sequential error sum is strictly lower (a tie or a NaN keeps E2M1),
 *     and only when R7 is a finite nonzero number: a block whose scale code is 0 (both
 *     reconstructions are zero) or whose INT4 step has no usable reciprocal keeps E2M1;
 *   - the global scale is plain NVFP4's (M = 448); round to nearest only;
 *   - counters of an INT4 block: saturation |y| > 7, underflow x != 0 with k = 0.               */

double ora_int4_value(int code) {
  int mag = code & 7;
  return (code & 8) ? -(double)mag : (double)mag;
}

/* Nearest of the integers 0..7 to |y| (ties to the even one), by enumerating the lattice; a
 * magnitude above 7, Inf included, clamps to 7.  The sign bit follows signbit(y).  Domain as
 * for E2M1: y is not NaN (placeholder -1 otherwise).                                           */
int ora_int4_encode_rne(float y) {
  if (isnan(y)) return -1;
  double a = fabs((double)y);
  int best = 7;
  if (!(a > 7.0)) {
    double bestd = INFINITY;
    best = 0;
    for (int k = 0; k < 8; ++k) {
      double d = fabs(a - (double)k);
      if (d < bestd || (d == bestd && (k & 1) == 0 && (best & 1) == 1)) {
        best = k;
        bestd = d;
      }
    }
  }
  return (signbit(y) ? 8 : 0) | best;
}

/* The INT4 candidate of one block with E4M3 scale code sc (nonzero): codes, counters and the
 * fp32 sequential sum of squared errors.  Returns NaN (the candidate is not taken) when R7 is not
 * a finite nonzero number.                                                                     */
static float if4_int_candidate(const float* x, int n, int sc, float s_g, uint8_t* codes, ora_counts* c) {
  float six_sevenths = 6.0f / 7.0f;
  float s7 = s_g * six_sevenths;
  float d = (float)ora_e4m3_value(sc);
  float D7 = d * s7;
  float R7 = 1.0f / D7;
  memset(c, 0, sizeof(*c));
  if (!isfinite(R7) || R7 == 0.0f) return NAN;
  for (int i = 0; i < n; ++i) {
    float y = x[i] * R7;
    int code = ora_int4_encode_rne(y);
    if (fabsf(y) > 7.0f) c->saturation += 1; /* an overflowed (infinite) y included */
    if (x[i] != 0.0f && (code & 7) == 0) c->underflow += 1;
    codes[i] = (uint8_t)code;
  }
  float sse = 0.0f;
  for (int i = 0; i < n; ++i) {
    float kd = (float)(ora_int4_value(codes[i]) * (double)d); /* exact: <= 7 significant bits */
    float xhat = kd * s7;
    float err = x[i] - xhat;
    float sq = err * err;
    sse = sse + sq;
  }
  return sse;
}

/* x: [rows, cols] fp32; q: [rows, cols/2]; scales: [rows, cols/16] row-major E4M3 bytes.
 * mode: 0 plain NVFP4, 1 four over six, 2 IF4.
 * global_in: NULL -> s_g from the tensor amax; else s_g = *global_in.
 * spec (nullable): one byte per block, 1 where the block's outputs are defined.  A block is left
 * unspecified (placeholder zeros; only its non-finite values counted) when it is rejected (holds
 * Inf or NaN), when the per-tensor scale is not finite (the tensor maximum of a tensor holding a
 * NaN or an Inf), or when a step of a candidate it compares gives a NaN (nv_candidate).  A finite
 * s_g >= 2^-118 rules the last case out: every nonzero block scale fl(d*s_g) is then at least
 * 2^-127 and has a finite reciprocal.                                                          */
void ora_nvfp4_quantize_spec(const float* x, long rows, long cols, int round, int mode, uint64_t seed,
                             const float* global_in, float* global_out, uint8_t* q, uint8_t* scales,
                             ora_counts* cnt, uint8_t* spec) {
  const int B = 16;
  long nb = cols / B;
  float s_g;
  if (global_in) {
    s_g = *global_in;
  } else {
    float amax_t = 0.0f; /* NaN-propagating maximum, as block_amax */
    for (long i = 0; i < rows * cols; ++i) {
      float a = fabsf(x[i]);
      if (isnan(a) || a > amax_t) amax_t = a;
      if (isnan(amax_t)) break;
    }
    s_g = ora_nvfp4_global_scale(amax_t, mode == 1);
  }
  if (global_out) *global_out = s_g;
  uint8_t c6[16], c4[16];
  for (long r = 0; r < rows; ++r) {
    for (long j = 0; j < nb; ++j) {
      const float* xb = x + r * cols + j * B;
      uint64_t idx0 = (uint64_t)(r * cols + j * B);
      int bad = ora_block_nonfinite(xb, B);
      cnt->nonfinite += (uint64_t)bad;
      int defined = !bad && isfinite(s_g);
      float amax_b = 0.0f, sse6 = 0.0f, sse4 = 0.0f;
      ora_counts k6, k4;
      int sc6 = 0, sc4 = 0;
      if (defined) {
        amax_b = block_amax(xb, B);
        sse6 = nv_candidate(xb, B, amax_b, s_g, 6.0f, round, seed, idx0, c6, &sc6, &k6, &defined);
        if (mode == 1) sse4 = nv_candidate(xb, B, amax_b, s_g, 4.0f, round, seed, idx0, c4, &sc4, &k4, &defined);
      }
      if (spec) spec[r * nb + j] = (uint8_t)defined;
      if (!defined) { /* placeholders: the outputs of this block are not fixed */
        scales[r * nb + j] = 0;
        memset(q + r * (cols / 2) + j * (B / 2), 0, B / 2);
        continue;
      }
      const uint8_t* pick = c6;
      int sc = sc6;
      ora_counts k = k6;
      if (mode == 1) {
        if (sse4 < sse6) {
          pick = c4;
          sc = sc4;
          k = k4;
          cnt->blocks_four += 1;
        }
      } else if (mode == 2 && sc6 != 0) {
        float sse7 = if4_int_candidate(xb, B, sc6, s_g, c4, &k4);
        if (sse7 < sse6) {
          pick = c4;
          sc = sc6 | 0x80;
          k = k4;
          cnt->blocks_four += 1;
        }
      }
      cnt->underflow += k.underflow;
      cnt->saturation += k.saturation;
      scales[r * nb + j] = (uint8_t)sc;
      pack_pairs(pick, B, q + r * (cols / 2) + j * (B / 2));
    }
  }
}

void ora_nvfp4_quantize(const float* x, long rows, long cols, int round, int mode, uint64_t seed,
                        const float* global_in, float* global_out, uint8_t* q, uint8_t* scales,
                        ora_counts* cnt) {
  ora_nvfp4_quantize_spec(x, rows, cols, round, mode, seed, global_in, global_out, q, scales, cnt, 0);
}

/* ------------------------------------------------------------------------------------------ */
/* Dequantisation ([A] "Encode one MXFP4 block step by step": reconstruction = lattice value times
 * the block scale; [X]: block scales applied in FP32).  x_hat = fl(fl(v*d) * s_g) for NVFP4, where
 * v*d is exact, and x_hat = v * 2^(byte-127) for MXFP4 (exact).  format 2 is IF4: a scale byte
 * with bit 7 set holds an INT4 block, x_hat = fl(fl(k*d) * s7) with d from the low 7 bits and
 * s7 = fl(s_g * fl(6/7)); otherwise the NVFP4 rule.  Row-major scales.                         */
void ora_dequantize(const uint8_t* q, const uint8_t* scales, int format, long rows, long cols,
                    float s_g, float* out) {
  int B = (format == 0) ? 32 : 16;
  long nb = cols / B;
  float six_sevenths = 6.0f / 7.0f;
  float s7 = s_g * six_sevenths;
  for (long r = 0; r < rows; ++r) {
    for (long k = 0; k < cols; ++k) {
      uint8_t byte = q[r * (cols / 2) + k / 2];
      int code = (k & 1) ? (byte >> 4) : (byte & 15);
      uint8_t sb = scales[r * nb + k / B];
      double v = ora_e2m1_value(code);
      if (format == 0) {
        out[r * cols + k] = (float)ldexp(v, (int)sb - 127);
      } else if (format == 2 && (sb & 0x80)) {
        float kd = (float)(ora_int4_value(code) * ora_e4m3_value(sb & 0x7F));
        out[r * cols + k] = kd * s7;
      } else {
        float vd = (float)(v * ora_e4m3_value(sb));
        out[r * cols + k] = vd * s_g;
      }
    }
  }
}

/* E2M1 nibbles to E4M3 bytes ([X]: devices without the FP4 MMA run the operands on the FP8 MMA
 * after an exact conversion, the factor 2^6 being absorbed by the scale).  Definition: the E4M3 encoding of
 * value(n) * 2^-6 (exact: at most 2 significant bits, magnitude in [2^-7, 6 * 2^-6]), with the
 * nibble's sign bit, so -0 maps to 0x80.  q: [rows, cols/2] packed as the quantisers write;
 * out: [rows, cols], one byte per element.                                                      */
void ora_e2m1_to_e4m3(const uint8_t* q, long rows, long cols, uint8_t* out) {
  for (long r = 0; r < rows; ++r) {
    for (long k = 0; k < cols; ++k) {
      uint8_t byte = q[r * (cols / 2) + k / 2];
      int code = (k & 1) ? (byte >> 4) : (byte & 15);
      double mag = fabs(ora_e2m1_value(code));
      int e = ora_e4m3_encode_rne_satfinite((float)ldexp(mag, -6));
      out[r * cols + k] = (uint8_t)((code & 8 ? 0x80 : 0) | e);
    }
  }
}

/* Exact fp64 dequantisation (for the GEMM reference), with no rounding: v * 2^(byte-127) (MXFP4),
 * v * d * s_g (NVFP4, and IF4 blocks whose scale byte has bit 7 clear), k * d * s_g * 6/7 (IF4
 * INT4 blocks, d from the low 7 bits).  [P] IF4 segment: an INT4 block's integer step is 6/7 of the
 * E2M1 unit (its maximum lands on 7), so in a product of two blocks a mixed FP4 x INT4 pair carries
 * the factor 6/7 and an INT4 x INT4 pair 36/49, applied once in full precision before the sum; here
 * the factor is the exact ratio 6/7 (the fp32 quantiser's s7 = fl(s_g * fl(6/7)) is a rounding of
 * it).  The product of two reconstructions carries exactly those factors.                       */
void ora_dequantize_f64(const uint8_t* q, const uint8_t* scales, int format, long rows, long cols,
                        float s_g, double* out) {
  int B = (format == 0) ? 32 : 16;
  long nb = cols / B;
  for (long r = 0; r < rows; ++r) {
    for (long k = 0; k < cols; ++k) {
      uint8_t byte = q[r * (cols / 2) + k / 2];
      int code = (k & 1) ? (byte >> 4) : (byte & 15);
      uint8_t sb = scales[r * nb + k / B];
      double v = ora_e2m1_value(code);
      if (format == 0) {
        out[r * cols + k] = ldexp(v, (int)sb - 127);
      } else if (format == 2 && (sb & 0x80)) {
        out[r * cols + k] = ora_int4_value(code) * ora_e4m3_value(sb & 0x7F) * (double)s_g * 6.0 / 7.0;
      } else {
        out[r * cols + k] = v * ora_e4m3_value(sb) * (double)s_g;
      }
    }
  }
}

/* ------------------------------------------------------------------------------------------ */
/* SwiGLU activation a = SiLU(g) * u in fp32, for the fused SiLU -> rotation -> quantiser path
 * ([E] §3 places the rotation in the SwiGLU epilogue).  The exponential is written out so that a
 * second implementation can reproduce it bit for bit: Cody and Waite's argument reduction (W. J.
 * Cody and W. Waite, "Software Manual for the Elementary Functions", 1980) x = n ln2 + r with
 * n = rint(x log2(e)) and ln2 split into an 11-bit head and a tail, then the degree-6 Taylor
 * polynomial of e^r in Horner form (|r| <= 0.35: truncation below 2^-24 relative), then an exact
 * scaling by 2^n.  Every operation is one fp32 rounding, in the order written.
 *   exp: x > 88.5 -> +Inf, x < -103 -> +0; otherwise the steps above.
 *   SiLU(g) = g * fl(1 / fl(1 + exp(-g)))  (one correctly rounded reciprocal)
 *   a = fl(SiLU(g) * u)                                                                          */
static float ora_pow2(int k) { /* 2^k for k in [-126, 127], exact */
  uint32_t b = (uint32_t)(k + 127) << 23;
  float f;
  memcpy(&f, &b, 4);
  return f;
}

/* p * 2^n, p in [0.7, 1.42], n in [-149, 128]: one rounding at most (only a subnormal result rounds) */
static float ora_scale_pow2(float p, int n) {
  if (n > 127) return (p * ora_pow2(127)) * ora_pow2(n - 127);
  if (n >= -126) return p * ora_pow2(n);
  return (p * ora_pow2(n + 64)) * ora_pow2(-64);
}

/* ln2 head: 12 significant bits, so n * head is exact for |n| <= 4096; tail = fl(ln2 - head) */
float ora_exp_cw(float x) {
  if (x != x) return x;
  if (x > 88.5f) return INFINITY;
  if (x < -103.0f) return 0.0f;
  const float log2e = 0x1.715476p+0f, ln2_hi = 0x1.62ep-1f, ln2_lo = 0x1.0bfbe8p-15f;
  float t = x * log2e;
  float n = rintf(t);
  float r = x - n * ln2_hi;
  r = r - n * ln2_lo;
  float p = 0x1.6c16c2p-10f;   /* fl(1/720) */
  p = p * r + 0x1.111112p-7f;  /* fl(1/120) */
  p = p * r + 0x1.555556p-5f;  /* fl(1/24) */
  p = p * r + 0x1.555556p-3f;  /* fl(1/6) */
  p = p * r + 0.5f;
  p = p * r + 1.0f;
  p = p * r + 1.0f;
  return ora_scale_pow2(p, (int)n);
}

float ora_silu_mul(float g, float u) {
  float e = ora_exp_cw(-g);
  float s = g * (1.0f / (1.0f + e));
  return s * u;
}

void ora_silu_mul_rows(const float* g, const float* u, long n, float* a) {
  for (long i = 0; i < n; ++i) a[i] = ora_silu_mul(g[i], u[i]);
}

/* ------------------------------------------------------------------------------------------ */
/* Normalised Walsh-Hadamard rotation of each row ([E] §3: H_d with entries +-1/sqrt(d), applied by
 * O(d log2 d) add/subtract butterflies).  Reading: natural (Sylvester) order; fp32; the
 * unnormalised stages run in the fixed order h = 1, 2, 4, ..., d/2, each mapping
 * (x[i], x[i+h]) -> (x[i]+x[i+h], x[i]-x[i+h]) for (i & h) == 0; then each value is multiplied by
 * c = fl(1/sqrt(d)).                                                                           */

float ora_fwht_norm_const(long d) { return (float)(1.0L / sqrtl((long double)d)); }

/* Randomised rotation ([P], the random Hadamard transform segment: a Hadamard transform with random
 * signs).  Reading: Q = c * H * D, D = diag(s) with s_i = -1 where bit i of the caller's sign vector
 * is set (bit i % 32 of word i / 32) and +1 otherwise; the signs multiply the input before the
 * butterflies (negation is exact), so with no bits set this is the plain rotation.  Q is
 * orthogonal (H * H = d * I), and its inverse is c * D * H.                                     */
void ora_rht_rows(const float* x, long rows, long d, const uint32_t* signs, float* y) {
  float c = ora_fwht_norm_const(d);
  for (long r = 0; r < rows; ++r) {
    float* v = y + r * d;
    for (long i = 0; i < d; ++i) {
      const int neg = signs ? (int)((signs[i / 32] >> (i % 32)) & 1u) : 0;
      v[i] = neg ? -x[r * d + i] : x[r * d + i];
    }
    for (long h = 1; h < d; h *= 2) {
      for (long i = 0; i < d; ++i) {
        if (i & h) continue;
        float a = v[i], b = v[i + h];
        v[i] = a + b;
        v[i + h] = a - b;
      }
    }
    for (long i = 0; i < d; ++i) v[i] = v[i] * c;
  }
}

void ora_fwht_rows(const float* x, long rows, long d, float* y) { ora_rht_rows(x, rows, d, 0, y); }
