// fwht.cu — online normalised Walsh-Hadamard rotation fused ahead of the FP4 quantisers.
//
// "Sub-4-Bit Microscaling" §3: activations are multiplied by H_d (entries +-1/sqrt(d)) with an
// O(d log2 d) add/subtract butterfly before quantisation, which spreads an outlier channel over
// all d channels.  The rotation is computed in fp32 in a fixed order — unnormalised radix-2
// stages h = 1, 2, 4, ..., d/2, each (a, b) -> (a + b, a - b) on pairs (i, i + h) with i & h == 0,
// then one multiply by c = fl(1/sqrt(d)) — so the rotated values, and therefore every code, are
// reproducible bit for bit.
//
// Data movement (d = 2^LOG_D, 32 values per thread, T = d/32 threads per row):
//   round A : the thread loads its 32 consecutive values (index bits 0-4) straight from global
//             memory and runs stages h = 1..16 in registers; writes fp32 to shared memory;
//   round B : the thread gathers the 32 values that differ in index bits 5-9, stages h=32..512;
//   last    : the thread gathers the values that differ in the remaining high bits together with
//             2^L consecutive values (index bits 0..L-1, L = 5 - #high bits) and runs the last
//             stages;
//   quantise: the values go back through the row buffer so that each thread holds 32 consecutive
//             rotated values (two NVFP4 blocks or one MXFP4 block), multiplies by c and quantises
//             whole blocks from registers.
// Shared memory holds one fp32 row per row slot; 16-byte chunks are XOR-swizzled by the low
// three bits of their 32-value row so that every round's accesses are bank-conflict free.
//
// Two optional inputs change what is rotated, not how:
//   signs : the randomised rotation c * H * D ([P], random Hadamard transform): bit j of a
//           thread's sign word negates its round-A value j before the butterflies;
//   u     : the SwiGLU path (bf16): x holds g, and the rotated input is fl(SiLU(g) * u).
#include "fp4_device.cuh"
#include "launch.h"

namespace fp4k {

template <int LOG_D>
struct Geom {
  static constexpr int D = 1 << LOG_D;
  static constexpr int T = D / 32;                 // threads per row
  static constexpr int CTA = T < 256 ? 256 : T;    // threads per CTA
  static constexpr int ROWS = CTA / T;             // row slots per CTA
  static constexpr int NR = (LOG_D + 4) / 5;       // rounds
  static constexpr int HI = 5 * (NR - 1);          // first index bit of the last round
  static constexpr int NH = LOG_D - HI;            // high bits in the last round
  static constexpr int L = 5 - NH;                 // consecutive low bits held in the last round
  static_assert(LOG_D >= 10 && LOG_D <= 14, "d must be in [1024, 16384]");
};

__device__ __forceinline__ int swz(int i) {  // word offset of element i inside its row slot
  const int row = i >> 5;
  return (row << 5) | ((((i >> 2) & 7) ^ (row & 7)) << 2) | (i & 3);
}

// One butterfly stage on local bit BIT: (v[p], v[p+h]) -> (v[p]+v[p+h], v[p]-v[p+h]).  For
// BIT >= 1 the pairs (p, p+1) and (p+h, p+h+1) are processed together with the sm_100 packed
// fp32 add/sub (each half an IEEE fp32 operation, so the result is identical to two scalar ones).
template <int BIT>
__device__ __forceinline__ void stage(float (&v)[32]) {
  if constexpr (BIT == 0) {
#pragma unroll
    for (int p = 0; p < 32; p += 2) {
      const float a = v[p], b = v[p + 1];
      v[p] = __fadd_rn(a, b);
      v[p + 1] = __fsub_rn(a, b);
    }
  } else {
    constexpr int H = 1 << BIT;
#pragma unroll
    for (int p = 0; p < 32; p += 2) {
      if (!(p & H)) {
        const f32x2 a = f2_pack(v[p], v[p + 1]), b = f2_pack(v[p + H], v[p + H + 1]);
        f2_unpack(f2_add(a, b), v[p], v[p + 1]);
        f2_unpack(f2_sub(a, b), v[p + H], v[p + H + 1]);
      }
    }
  }
}
template <int LO, int HI_>
__device__ __forceinline__ void stages(float (&v)[32]) {  // local bits LO..HI_-1 in order
  if constexpr (LO < HI_) {
    stage<LO>(v);
    stages<LO + 1, HI_>(v);
  }
}

// SwiGLU activation fl(SiLU(g) * u) with a written-out exponential, every step one explicitly rounded
// fp32 operation: Cody and Waite's argument reduction ("Software Manual for the Elementary
// Functions", 1980) x = n ln2 + r, n = rint(x log2 e), ln2 split into a 12-significant-bit head
// (n * head exact) and a tail; the degree-6 Taylor polynomial of e^r in Horner form; an exact scaling
// by 2^n.  SiLU(g) = g * fl(1 / fl(1 + e^-g)) with a correctly rounded reciprocal.
__device__ __forceinline__ float pow2_exact(int k) { return __uint_as_float((uint32_t)(k + 127) << 23); }
__device__ __forceinline__ float exp_cw(float x) {
  if (x != x) return x;
  if (x > 88.5f) return __int_as_float(0x7F800000);
  if (x < -103.0f) return 0.0f;
  const float n = rintf(__fmul_rn(x, 0x1.715476p+0f));
  float r = __fsub_rn(x, __fmul_rn(n, 0x1.62ep-1f));
  r = __fsub_rn(r, __fmul_rn(n, 0x1.0bfbe8p-15f));
  float q = 0x1.6c16c2p-10f;
  q = __fadd_rn(__fmul_rn(q, r), 0x1.111112p-7f);
  q = __fadd_rn(__fmul_rn(q, r), 0x1.555556p-5f);
  q = __fadd_rn(__fmul_rn(q, r), 0x1.555556p-3f);
  q = __fadd_rn(__fmul_rn(q, r), 0.5f);
  q = __fadd_rn(__fmul_rn(q, r), 1.0f);
  q = __fadd_rn(__fmul_rn(q, r), 1.0f);
  const int k = (int)n;
  if (k > 127) return __fmul_rn(__fmul_rn(q, pow2_exact(127)), pow2_exact(k - 127));
  if (k >= -126) return __fmul_rn(q, pow2_exact(k));
  return __fmul_rn(__fmul_rn(q, pow2_exact(k + 64)), pow2_exact(-64));
}
__device__ __forceinline__ float silu_mul(float g, float u) {
  const float e = exp_cw(-g);
  return __fmul_rn(__fmul_rn(g, __frcp_rn(__fadd_rn(1.0f, e))), u);
}

template <typename T>
struct RowLoad {
  static constexpr int NV = 32 * (int)sizeof(T) / 32;  // 32-byte chunks per thread
};

// Round A + B + last-round rotation of one row into v[32] (last-round order: j = low | h << L).
// `raw` holds this thread's round-A chunks, elements [32 t, 32 t + 32); bit j of `sgn` negates
// element 32 t + j first (randomised rotation; 0 = plain).  Leaves the values unnormalised.
template <typename T, int LOG_D, bool GATED = false>
__device__ __forceinline__ void rotate_row(const U8 (&raw)[RowLoad<T>::NV], const U8* rawu, float* srow, int t,
                                           uint32_t sgn, float (&v)[32]) {
  using G = Geom<LOG_D>;
  // round A: index bits 0-4 local
#pragma unroll
  for (int c = 0; c < RowLoad<T>::NV; ++c) Vec32<T>::unpack(raw[c], v + c * Vec32<T>::E);
  if constexpr (GATED) {  // raw holds g, rawu holds u: the rotated input is fl(SiLU(g) * u)
#pragma unroll
    for (int c = 0; c < RowLoad<T>::NV; ++c) {
      float w[Vec32<T>::E];
      Vec32<T>::unpack(rawu[c], w);
#pragma unroll
      for (int i = 0; i < Vec32<T>::E; ++i) v[c * Vec32<T>::E + i] = silu_mul(v[c * Vec32<T>::E + i], w[i]);
    }
  }
  if (sgn) {
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __uint_as_float(__float_as_uint(v[j]) ^ ((sgn << (31 - j)) & 0x80000000u));
  }
  stages<0, 5>(v);
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const int i = (t << 5) | (q << 2);
    *reinterpret_cast<float4*>(srow + swz(i)) = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
  }
  __syncthreads();
  if constexpr (G::NR == 3) {
    // round B: index bits 5-9 local; lane = bits 0-4, rest = bits 10..
    const int lo5 = t & 31, hi = t >> 5;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = srow[swz(lo5 | (j << 5) | (hi << 10))];
    stages<0, 5>(v);
#pragma unroll
    for (int j = 0; j < 32; ++j) srow[swz(lo5 | (j << 5) | (hi << 10))] = v[j];
    __syncthreads();
  }
  // last round: high bits HI.. plus low bits 0..L-1
  constexpr int L = G::L, NH = G::NH, HI = G::HI;
#pragma unroll
  for (int h = 0; h < (1 << NH); ++h) {
    const int i0 = (t << L) | (h << HI);
    if constexpr (L >= 2) {
#pragma unroll
      for (int q = 0; q < (1 << L) / 4; ++q) {
        const float4 f = *reinterpret_cast<const float4*>(srow + swz(i0 + 4 * q));
        v[(h << L) + 4 * q] = f.x; v[(h << L) + 4 * q + 1] = f.y;
        v[(h << L) + 4 * q + 2] = f.z; v[(h << L) + 4 * q + 3] = f.w;
      }
    } else if constexpr (L == 1) {
      const float2 f = *reinterpret_cast<const float2*>(srow + swz(i0));
      v[h << 1] = f.x; v[(h << 1) + 1] = f.y;
    } else {
      v[h] = srow[swz(i0)];
    }
  }
  stages<L, 5>(v);
  __syncthreads();  // shared row free for the next row
}

template <typename T, int LOG_D>
__device__ __forceinline__ void load_row(const T* x, long long row, long long rows, int t,
                                         U8 (&raw)[RowLoad<T>::NV]) {
  constexpr int D = 1 << LOG_D;
  if (row < rows) {
    const char* p = reinterpret_cast<const char*>(x + row * D + (long long)t * 32);
#pragma unroll
    for (int c = 0; c < RowLoad<T>::NV; ++c) raw[c] = ld32<false>(p + 32 * c);
  } else {
#pragma unroll
    for (int c = 0; c < RowLoad<T>::NV; ++c) for (int i = 0; i < 8; ++i) raw[c].w[i] = 0u;
  }
}

struct FwhtParams {
  const void* x;
  long long rows;
  float c;            // fl(1/sqrt(d))
  int tiled;
  int reverse;
  PhiloxKeys keys;
  uint32_t zero;      // 0, read at run time: makes in-register nibble decodes opaque
  const float* global_in;
  uint32_t* amax_bits;
  float* global_out;
  float six_m;
  float* rotated_out;
  const uint32_t* signs;
  const void* u;      // SwiGLU path: x holds g, u holds the up projection (same layout)
  uint8_t* q;
  uint8_t* scales;
  unsigned long long* counts;
};

// Pass 1 (NVFP4 without a caller scale): amax of the rotated tensor.
template <typename T, int LOG_D, bool GATED>
__global__ void __launch_bounds__(Geom<LOG_D>::CTA) fwht_amax_kernel(FwhtParams p) {
  using G = Geom<LOG_D>;
  grid_dep_trigger();  // the quantise pass may take SMs as this grid's CTAs retire
  // the counters the following quantise pass accumulates into start at zero (stream order)
  if (p.counts && blockIdx.x == 0 && threadIdx.x < 4) p.counts[threadIdx.x] = 0ull;
  extern __shared__ __align__(16) float smem[];
  const int slot = threadIdx.x / G::T, t = threadIdx.x % G::T;
  float* srow = smem + slot * G::D;
  const T* x = reinterpret_cast<const T*>(p.x);
  const uint32_t sgn = p.signs ? p.signs[t] : 0u;
  const long long step = (long long)gridDim.x * G::ROWS;
  float m = 0.0f;
  U8 raw[RowLoad<T>::NV], nxt[RowLoad<T>::NV], rawu[GATED ? RowLoad<T>::NV : 1];
  long long row = (long long)blockIdx.x * G::ROWS + slot;
  if (!GATED) load_row<T, LOG_D>(x, row, p.rows, t, raw);
  for (long long base = (long long)blockIdx.x * G::ROWS; base < p.rows; base += step) {
    if constexpr (GATED) {  // two inputs per row: loaded for the current row, no prefetch
      load_row<T, LOG_D>(x, row, p.rows, t, raw);
      load_row<T, LOG_D>(reinterpret_cast<const T*>(p.u), row, p.rows, t, rawu);
    } else {
      load_row<T, LOG_D>(x, row + step, p.rows, t, nxt);
    }
    float v[32];
    rotate_row<T, LOG_D, GATED>(raw, rawu, srow, t, sgn, v);
    if (row < p.rows) {
#pragma unroll
      for (int j = 0; j < 32; ++j) m = fmaxf(m, fabsf(v[j]));
    }
    if (!GATED) {
#pragma unroll
      for (int c = 0; c < RowLoad<T>::NV; ++c) raw[c] = nxt[c];
    }
    row += step;
  }
  // |fl(c*u)| is monotone in |u|: scale the maximum once.
  m = __fmul_rn(m, p.c);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ float wm[32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    float b = 0.0f;
    for (int w = 0; w < G::CTA / 32; ++w) b = fmaxf(b, wm[w]);
    atomicMax(p.amax_bits, __float_as_uint(b));
  }
}

// Last-round order -> natural order in the (free) row buffer: the thread writes its 2^NH groups of
// 2^L consecutive values (consecutive 16-byte chunks across a warp, conflict-free), then syncs.
template <int LOG_D>
__device__ __forceinline__ void to_row_buffer(float* srow, int t, const float (&v)[32]) {
  using G = Geom<LOG_D>;
  constexpr int L = G::L, NH = G::NH, HI = G::HI;
#pragma unroll
  for (int h = 0; h < (1 << NH); ++h) {
    const int i0 = (t << L) | (h << HI);
    if constexpr (L >= 2) {
#pragma unroll
      for (int q = 0; q < (1 << L) / 4; ++q) {
        const float* f = v + (h << L) + 4 * q;
        *reinterpret_cast<float4*>(srow + swz(i0 + 4 * q)) = make_float4(f[0], f[1], f[2], f[3]);
      }
    } else if constexpr (L == 1) {
      *reinterpret_cast<float2*>(srow + swz(i0)) = make_float2(v[h << 1], v[(h << 1) + 1]);
    } else {
      srow[swz(i0)] = v[h];
    }
  }
  __syncthreads();
}

// Last-round order -> 32 consecutive values per thread, through the (free) row buffer: the thread
// writes its 2^NH groups of 2^L consecutive values and reads back elements [32 t, 32 t + 32), so
// that every quantisation block lies inside one thread.  Both the writes (consecutive 16-byte
// chunks across a warp) and the reads (one swizzled 128-byte row per thread) are conflict-free.
template <int LOG_D>
__device__ __forceinline__ void to_consecutive(float* srow, int t, float (&v)[32]) {
  using G = Geom<LOG_D>;
  constexpr int L = G::L, NH = G::NH, HI = G::HI;
#pragma unroll
  for (int h = 0; h < (1 << NH); ++h) {
    const int i0 = (t << L) | (h << HI);
    if constexpr (L >= 2) {
#pragma unroll
      for (int q = 0; q < (1 << L) / 4; ++q) {
        const float* f = v + (h << L) + 4 * q;
        *reinterpret_cast<float4*>(srow + swz(i0 + 4 * q)) = make_float4(f[0], f[1], f[2], f[3]);
      }
    } else if constexpr (L == 1) {
      *reinterpret_cast<float2*>(srow + swz(i0)) = make_float2(v[h << 1], v[(h << 1) + 1]);
    } else {
      srow[swz(i0)] = v[h];
    }
  }
  __syncthreads();
#pragma unroll
  for (int q = 0; q < 8; ++q) {
    const float4 f = *reinterpret_cast<const float4*>(srow + swz((t << 5) + 4 * q));
    v[4 * q] = f.x; v[4 * q + 1] = f.y; v[4 * q + 2] = f.z; v[4 * q + 3] = f.w;
  }
  __syncthreads();  // row buffer free for the next row
}

// Pass 1 of the stored-rotation path (NVFP4 without a caller scale, given room for the rotated
// tensor): rotate once, normalise, store the fp32 rotation row-major to p.rotated_out and reduce
// the tensor amax.  The quantise pass then reads the stored values (quantize_kernel on fp32 input),
// so the butterflies run once instead of twice, for 4 more bytes per element of traffic each way.
// The maximum is an integer max over the magnitude bits, which keeps a NaN (its bits lie above
// every finite value's and Inf's), as the tensor maximum does in the two-rotation path's reading.
template <typename T, int LOG_D, bool GATED>
__global__ void __launch_bounds__(Geom<LOG_D>::CTA) fwht_store_kernel(FwhtParams p) {
  using G = Geom<LOG_D>;
  constexpr int D = G::D;
  grid_dep_trigger();
  if (p.counts && blockIdx.x == 0 && threadIdx.x < 4) p.counts[threadIdx.x] = 0ull;
  extern __shared__ __align__(16) float smem[];
  const int slot = threadIdx.x / G::T, t = threadIdx.x % G::T;
  float* srow = smem + slot * D;
  const T* x = reinterpret_cast<const T*>(p.x);
  const uint32_t sgn = p.signs ? p.signs[t] : 0u;
  const long long step = (long long)gridDim.x * G::ROWS;
  uint32_t m = 0u;
  U8 raw[RowLoad<T>::NV], nxt[RowLoad<T>::NV], rawu[GATED ? RowLoad<T>::NV : 1];
  long long row = (long long)blockIdx.x * G::ROWS + slot;
  if (!GATED) load_row<T, LOG_D>(x, row, p.rows, t, raw);
  for (long long base = (long long)blockIdx.x * G::ROWS; base < p.rows; base += step) {
    if constexpr (GATED) {
      load_row<T, LOG_D>(x, row, p.rows, t, raw);
      load_row<T, LOG_D>(reinterpret_cast<const T*>(p.u), row, p.rows, t, rawu);
    } else {
      load_row<T, LOG_D>(x, row + step, p.rows, t, nxt);
    }
    float v[32];
    rotate_row<T, LOG_D, GATED>(raw, rawu, srow, t, sgn, v);
    // through the row buffer in natural order, then out in 512-byte warp-contiguous pieces: thread
    // t stores the 16-byte groups t, t + T, t + 2T, ... of the row
    to_row_buffer<LOG_D>(srow, t, v);
    if (row < p.rows) {
      float4* dst = reinterpret_cast<float4*>(p.rotated_out + row * D);
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        const int grp = t + q * G::T;
        float4 f = *reinterpret_cast<const float4*>(srow + swz(4 * grp));
        f.x = __fmul_rn(f.x, p.c); f.y = __fmul_rn(f.y, p.c);
        f.z = __fmul_rn(f.z, p.c); f.w = __fmul_rn(f.w, p.c);
        m = max(m, max(max(__float_as_uint(f.x) & 0x7FFFFFFFu, __float_as_uint(f.y) & 0x7FFFFFFFu),
                       max(__float_as_uint(f.z) & 0x7FFFFFFFu, __float_as_uint(f.w) & 0x7FFFFFFFu)));
        dst[grp] = f;
      }
    }
    __syncthreads();  // row buffer free for the next row
    if (!GATED) {
#pragma unroll
      for (int c = 0; c < RowLoad<T>::NV; ++c) raw[c] = nxt[c];
    }
    row += step;
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) m = max(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
  __shared__ uint32_t wm[32];
  if ((threadIdx.x & 31) == 0) wm[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x == 0) {
    uint32_t b = 0u;
    for (int w = 0; w < G::CTA / 32; ++w) b = max(b, wm[w]);
    atomicMax(p.amax_bits, b);
  }
}

// Pass 2: rotate again, normalise, quantise from registers (whole blocks per thread).
// MODE: 0 plain, 1 four-over-six, 2 IF4 (NVFP4 only).
template <typename T, int LOG_D, bool NV, bool SR, int MODE, bool GATED>
__global__ void __launch_bounds__(Geom<LOG_D>::CTA, Geom<LOG_D>::CTA <= 256 ? 2 : 1) fwht_quant_kernel(FwhtParams p) {
  constexpr bool FOUR_SIX = MODE == 1, IF4 = MODE == 2;
  using G = Geom<LOG_D>;
  constexpr int D = G::D;
  constexpr int B = NV ? 16 : 32;
  constexpr int W = B / 8;  // packed nibble words per block
  extern __shared__ __align__(16) float smem[];
  const int slot = threadIdx.x / G::T, t = threadIdx.x % G::T;
  float* srow = smem + slot * D;
  const T* x = reinterpret_cast<const T*>(p.x);
  const uint32_t sgn = p.signs ? p.signs[t] : 0u;
  const long long step = (long long)gridDim.x * G::ROWS;
  const uint32_t nb = D / B;
  grid_dep_wait();  // after the amax pass (programmatic launch): its results are visible from here

  float s_g = 1.0f, inv6 = 1.0f, inv4 = 1.0f;
  if (NV) {
    if (p.global_in) {
      s_g = *p.global_in;
    } else {
      const float amax = __uint_as_float(*p.amax_bits);
      s_g = (amax == 0.0f) ? 1.0f : __fdiv_rn(amax, p.six_m);
    }
    inv6 = __frcp_rn(__fmul_rn(6.0f, s_g));
    inv4 = __frcp_rn(__fmul_rn(4.0f, s_g));
    if (p.global_out && blockIdx.x == 0 && threadIdx.x == 0) *p.global_out = s_g;
  }
  __shared__ float2 tab[NV ? kScaleTab : 1];
  __shared__ float2 tab7[IF4 ? kScaleTab : 1];
  const float s7 = IF4 ? __fmul_rn(s_g, kSixSevenths) : 0.0f;
  if (NV) fill_scale_tab(tab, s_g);  // first read after the rotation's __syncthreads
  if (IF4) fill_int4_tab(tab7, s7);
  uint32_t cnt[4] = {0u, 0u, 0u, 0u};
  U8 raw[RowLoad<T>::NV], nxt[RowLoad<T>::NV], rawu[GATED ? RowLoad<T>::NV : 1];
  auto phys = [&](long long r) { return p.reverse ? (p.rows - 1 - r) : r; };
  long long row = (long long)blockIdx.x * G::ROWS + slot;
  if (!GATED) load_row<T, LOG_D>(x, row < p.rows ? phys(row) : row, p.rows, t, raw);
  for (long long base = (long long)blockIdx.x * G::ROWS; base < p.rows; base += step) {
    if constexpr (GATED) {  // two inputs per row: loaded for the current row, no prefetch
      const long long pr = row < p.rows ? phys(row) : row;
      load_row<T, LOG_D>(x, pr, p.rows, t, raw);
      load_row<T, LOG_D>(reinterpret_cast<const T*>(p.u), pr, p.rows, t, rawu);
    } else {
      const long long rn = row + step;
      load_row<T, LOG_D>(x, rn < p.rows ? phys(rn) : rn, p.rows, t, nxt);
    }
    float v[32];
    rotate_row<T, LOG_D, GATED>(raw, rawu, srow, t, sgn, v);
    to_consecutive<LOG_D>(srow, t, v);
    const bool valid = row < p.rows;  // uniform over the row's warps
    const long long prow = valid ? phys(row) : 0;
#pragma unroll
    for (int j = 0; j < 32; ++j) v[j] = __fmul_rn(v[j], p.c);
    if (valid && p.rotated_out) {
      float4* dst = reinterpret_cast<float4*>(p.rotated_out + prow * D + (t << 5));
#pragma unroll
      for (int q = 0; q < 8; ++q) dst[q] = make_float4(v[4 * q], v[4 * q + 1], v[4 * q + 2], v[4 * q + 3]);
    }
#pragma unroll
    for (int b = 0; b < 32 / B; ++b) {
      const float* g = v + b * B;
      const int i0 = (t << 5) + b * B;  // index in row of g[0]
      const unsigned long long idx0 = (unsigned long long)prow * D + i0;
      uint32_t am = 0u, mn = 0xFFFFFFFFu;
#pragma unroll
      for (int i = 0; i < B; ++i) {
        const uint32_t a = __float_as_uint(g[i]) & 0x7FFFFFFFu;
        am = max(am, a);
        mn = min(mn, a);
      }
      const float amax = __uint_as_float(am);
      uint32_t w[W], sc, sat = 0, four = 0;
      if (!NV) {
        // MXFP4 OCP rule: e = floor(log2 amax) - 2, clamped to [-127, 127], all-zero -> 0
        const int ef = (int)((am >> 23) & 0xFFu);
        int e = (am == 0u) ? 0 : (ef == 0 ? -127 : ef - 129);
        e = e < -127 ? -127 : e;
        const float inv = __uint_as_float((uint32_t)(127 - e) << 23);
        const float top = __fmul_rn(amax, inv);
#pragma unroll
        for (int hf = 0; hf < B / 16; ++hf) {  // two 16-value halves under the block's one scale
          uint32_t rnd[16];
          if (SR) sr_words<16>(idx0 + 16 * hf, p.keys, rnd);
          encode_n<16, SR>(g + 16 * hf, inv, top, rnd, w + 2 * hf, sat);
        }
        sc = (uint32_t)(e + 127);
      } else if constexpr (FOUR_SIX) {
        uint32_t rnd[B];
        if (SR) sr_words<B>(idx0, p.keys, rnd);
        uint32_t w4[W], sat4;
        float D6, D4, A6, A4;
        sc = nv_candidate_resid_n<B, SR>(g, amax, inv6, tab, rnd, p.zero, w, sat, D6, A6);
        const uint32_t sc4 = nv_candidate_resid_n<B, SR>(g, amax, inv4, tab, rnd, p.zero, w4, sat4, D4, A4);
        bool pick4;
        const bool undecided = four_six_undecided(am, amax, D6, D4, A6, A4, sc, sc4, pick4);
        if (__any_sync(0xFFFFFFFFu, undecided)) {  // warp-uniform branch
          float sq[B];
          sq_errors_n<B>(g, w, sc, s_g, p.zero, sq);
          const float sse6 = block_sse_n<B, 1>(sq, 0);
          sq_errors_n<B>(g, w4, sc4, s_g, p.zero, sq);
          const float sse4 = block_sse_n<B, 1>(sq, 0);
          pick4 = sse4 < sse6;
        }
        if (pick4) {
          sc = sc4;
          sat = sat4;
          four = 1;
#pragma unroll
          for (int k = 0; k < W; ++k) w[k] = w4[k];
        }
      } else if constexpr (IF4) {
        // E2M1 or INT4 (round to nearest): residual estimates, exact sums inside the margin
        uint32_t rnd[B];  // unused without stochastic rounding
        float D6, A6, R6;
        sc = nv_candidate_resid_n<B, false>(g, amax, inv6, tab, rnd, p.zero, w, sat, D6, A6, &R6);
        const float2 DR7 = tab7[sc];
        uint32_t w7[W];
        const float A7 = int4_encode_resid_n<B>(g, DR7.y, w, w7);
        const bool eligible = DR7.y != 0.0f;
        bool pick;
        const bool undecided = if4_undecided(am, amax, D6, DR7.x, A6, A7, eligible, pick);
        if (__any_sync(0xFFFFFFFFu, undecided)) {  // warp-uniform branch
          float sq[B];
          sq_errors_n<B>(g, w, sc, s_g, p.zero, sq);
          const float sse6 = block_sse_n<B, 1>(sq, 0);
          uint32_t wx[W];
          int4_candidate_n<B>(g, DR7.y, e4m3_value(sc), s7, w, wx, sq);
          const float sse7 = block_sse_n<B, 1>(sq, 0);
          pick = eligible && sse7 < sse6;
        }
        if (pick) {
          sc |= 0x80u;
          four = 1;
          sat = 0;
          if (__fmul_rn(amax, DR7.y) > 7.0f) {
#pragma unroll
            for (int i = 0; i < B; ++i) sat += fabsf(__fmul_rn(g[i], DR7.y)) > 7.0f;
          }
#pragma unroll
          for (int k = 0; k < W; ++k) w[k] = w7[k];
        }
      } else {
        uint32_t rnd[B];
        if (SR) sr_words<B>(idx0, p.keys, rnd);
        sc = nv_candidate_n<B, SR>(g, amax, inv6, tab, rnd, w, sat);
      }
      if (valid) {
        if (am >= 0x7F800000u) {
#pragma unroll
          for (int i = 0; i < B; ++i) cnt[2] += !isfinite(g[i]);
        }
        // a block holding Inf or NaN is rejected: only its non-finite values are counted
        const bool audit = am < 0x7F800000u;
        const int zc = zero_codes_n<B>(w);
        int zx = 0;  // a +-0 input always gives a zero code: count inputs only when both occur
        if (zc > 0 && mn == 0u) {
#pragma unroll
          for (int i = 0; i < B; ++i) zx += g[i] == 0.0f;
        }
        cnt[0] += audit ? (uint32_t)(zc - zx) : 0u;
        cnt[1] += audit ? sat : 0u;
        uint2* q2 = reinterpret_cast<uint2*>(p.q + prow * (D / 2) + i0 / 2);
#pragma unroll
        for (int k = 0; k < W; k += 2) q2[k / 2] = make_uint2(w[k], w[k + 1]);
        const unsigned long long blk = (unsigned long long)prow * nb + (unsigned)(i0 / B);
        p.scales[scale_offset(blk, nb, p.tiled)] = (uint8_t)sc;
        cnt[3] += audit ? four : 0u;
      }
    }
    if (!GATED) {
#pragma unroll
      for (int c = 0; c < RowLoad<T>::NV; ++c) raw[c] = nxt[c];
    }
    row += step;
  }
  if (p.counts) flush_counts<4>(cnt, p.counts);
}

// ---------------------------------------------------------------------------------------------
// CTAs to launch: the resident count of the amax pass (the lighter kernel), also for the quantise
// pass, whose CTAs then run as about one and a half waves over rows of equal cost; that measured
// slightly faster than one wave of the quantise pass's own resident count (uneven row tails).
template <int LOG_D, typename K>
static int fwht_grid(K kernel, long long rows) {
  using G = Geom<LOG_D>;
  const int smem = G::ROWS * G::D * 4;
  int per_sm = 0;
  cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kernel, G::CTA, smem);
  if (per_sm < 1) per_sm = 1;
  const long long want = (rows + G::ROWS - 1) / G::ROWS;
  const long long cap = (long long)num_sms() * per_sm;
  return (int)(want < 1 ? 1 : (want < cap ? want : cap));
}

static FwhtParams make_params(const FwhtLaunch& L) {
  FwhtParams p;
  p.x = L.x; p.rows = L.rows;
  p.c = (float)(1.0 / sqrt((double)L.d));
  p.tiled = L.tiled; p.reverse = 0; p.keys = philox_keys(L.seed); p.zero = 0u;
  p.global_in = L.global_in; p.amax_bits = L.amax_bits; p.global_out = L.global_out;
  p.six_m = L.mode == 1 ? 1536.0f : 2688.0f;
  p.rotated_out = L.rotated_out; p.signs = L.signs; p.u = L.u; p.q = L.q; p.scales = L.scales; p.counts = L.counts;
  return p;
}

template <typename T, int LOG_D, bool GATED>
static cudaError_t amax_d(const FwhtParams& p, cudaStream_t s) {
  using G = Geom<LOG_D>;
  const int smem = G::ROWS * G::D * 4;
  auto k = fwht_amax_kernel<T, LOG_D, GATED>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  k<<<fwht_grid<LOG_D>(k, p.rows), G::CTA, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, int LOG_D, bool NV, bool SR, int FS, bool GATED>
static cudaError_t quant_d(const FwhtParams& p, bool pdl, cudaStream_t s) {
  using G = Geom<LOG_D>;
  const int smem = G::ROWS * G::D * 4;
  auto k = fwht_quant_kernel<T, LOG_D, NV, SR, FS, GATED>;
  cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  cudaFuncSetAttribute(fwht_amax_kernel<T, LOG_D, GATED>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  return launch_pdl(k, dim3(fwht_grid<LOG_D>(fwht_amax_kernel<T, LOG_D, GATED>, p.rows)), dim3(G::CTA), smem, s,
                    pdl, p);
}

template <typename T, int LOG_D, bool GATED>
static cudaError_t quant_sel(const FwhtParams& p, const FwhtLaunch& L, cudaStream_t s) {
  const bool d = L.pdl;
  if (!L.nv)
    return L.sr ? quant_d<T, LOG_D, false, true, 0, GATED>(p, d, s) : quant_d<T, LOG_D, false, false, 0, GATED>(p, d, s);
  if (L.mode == 2) return quant_d<T, LOG_D, true, false, 2, GATED>(p, d, s);  // IF4: round to nearest only
  if (L.mode == 1)
    return L.sr ? quant_d<T, LOG_D, true, true, 1, GATED>(p, d, s) : quant_d<T, LOG_D, true, false, 1, GATED>(p, d, s);
  return L.sr ? quant_d<T, LOG_D, true, true, 0, GATED>(p, d, s) : quant_d<T, LOG_D, true, false, 0, GATED>(p, d, s);
}

template <typename T, int LOG_D, bool GATED>
static cudaError_t store_d(const FwhtParams& p, cudaStream_t s) {
  using G = Geom<LOG_D>;
  const int smem = G::ROWS * G::D * 4;
  auto k = fwht_store_kernel<T, LOG_D, GATED>;
  cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
  if (e != cudaSuccess) return e;
  k<<<fwht_grid<LOG_D>(k, p.rows), G::CTA, smem, s>>>(p);
  return cudaGetLastError();
}

template <typename T, bool GATED>
static cudaError_t dispatch_store(const FwhtParams& p, int d, cudaStream_t s) {
  switch (d) {
    case 1024: return store_d<T, 10, GATED>(p, s);
    case 2048: return store_d<T, 11, GATED>(p, s);
    case 4096: return store_d<T, 12, GATED>(p, s);
    case 8192: return store_d<T, 13, GATED>(p, s);
    case 16384: return store_d<T, 14, GATED>(p, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T, bool GATED>
static cudaError_t dispatch_amax(const FwhtParams& p, int d, cudaStream_t s) {
  switch (d) {
    case 1024: return amax_d<T, 10, GATED>(p, s);
    case 2048: return amax_d<T, 11, GATED>(p, s);
    case 4096: return amax_d<T, 12, GATED>(p, s);
    case 8192: return amax_d<T, 13, GATED>(p, s);
    case 16384: return amax_d<T, 14, GATED>(p, s);
  }
  return cudaErrorInvalidValue;
}

template <typename T, bool GATED>
static cudaError_t dispatch_quant(const FwhtParams& p, const FwhtLaunch& L, cudaStream_t s) {
  switch (L.d) {
    case 1024: return quant_sel<T, 10, GATED>(p, L, s);
    case 2048: return quant_sel<T, 11, GATED>(p, L, s);
    case 4096: return quant_sel<T, 12, GATED>(p, L, s);
    case 8192: return quant_sel<T, 13, GATED>(p, L, s);
    case 16384: return quant_sel<T, 14, GATED>(p, L, s);
  }
  return cudaErrorInvalidValue;
}

// The SwiGLU (gated) path is built for bf16 inputs only.
cudaError_t launch_fwht_amax(const FwhtLaunch& L, cudaStream_t s) {
  if (L.rows == 0) return cudaSuccess;
  FwhtParams p = make_params(L);
  if (L.u) return L.bf16 ? dispatch_amax<__nv_bfloat16, true>(p, L.d, s) : cudaErrorInvalidValue;
  return L.bf16 ? dispatch_amax<__nv_bfloat16, false>(p, L.d, s) : dispatch_amax<float, false>(p, L.d, s);
}

cudaError_t launch_fwht_store(const FwhtLaunch& L, cudaStream_t s) {
  if (L.rows == 0) return cudaSuccess;
  FwhtParams p = make_params(L);
  if (L.u) return L.bf16 ? dispatch_store<__nv_bfloat16, true>(p, L.d, s) : cudaErrorInvalidValue;
  return L.bf16 ? dispatch_store<__nv_bfloat16, false>(p, L.d, s) : dispatch_store<float, false>(p, L.d, s);
}

cudaError_t launch_fwht_quantize(const FwhtLaunch& L, cudaStream_t s) {
  if (L.rows == 0) return cudaSuccess;
  FwhtParams p = make_params(L);
  p.reverse = (L.nv && !L.global_in) ? 1 : 0;
  if (L.u) return L.bf16 ? dispatch_quant<__nv_bfloat16, true>(p, L, s) : cudaErrorInvalidValue;
  return L.bf16 ? dispatch_quant<__nv_bfloat16, false>(p, L, s) : dispatch_quant<float, false>(p, L, s);
}

}  // namespace fp4k
