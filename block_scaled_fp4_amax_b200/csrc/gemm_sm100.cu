// gemm_sm100.cu — W4A4 block-scaled GEMM on the sm_100 tensor cores.
//
// C[m][n] = alpha * sum_k dA[m][k/B] dB[n][k/B] vA[m][k] vB[n][k], FP32 accumulation in tensor
// memory, bf16 output.  NVFP4 operands (E4M3 scale per 16, alpha = product of the global scales)
// run tcgen05.mma kind::mxf4nvf4 with scale_vec::4X; MXFP4 operands (E8M0 scale per 32) the same
// kind with scale_vec::2X.  ("Sub-4-Bit Microscaling" §2: NVFP4 on the 5th-generation tensor
// core; metrale `hardware::exec`: NVFP4 activations take the block-scaled FP4 MMA.)
//
// Two kernels share the PTX helpers below.
//
// gemm_pair_kernel (M % 256 == 0): clusters of two CTAs on neighbouring SMs, each pair computing a
// 256 x 256 tile with tcgen05 cta_group::2 (each SM holds half of A and half of B per stage), K
// consumed 256 values per stage in a 5-6 stage ring.  Twelve warps per CTA:
//   warp 0     TMA producer (both CTAs): operand tiles by 2-D tensor maps with 128-byte swizzle,
//              scale tiles by 3-D tensor maps; all loads complete on the leader's barrier;
//   warps 2-3  (leader) copy each stage's scales smem -> TMEM (tcgen05.cp) into one of three
//              TMEM scale buffers, half of the scale atoms each — issued from their own warps so
//              the copies queue separately from the MMAs and overlap them;
//   warp 1     (leader) issues tcgen05.mma kind::mxf4nvf4 and the commits that free smem stages,
//              scale buffers and, per tile, hand the accumulator to the epilogue;
//   warps 4-11 epilogue (both CTAs): each tcgen05.lds a 32-row x 128-column part of the FP32
//              accumulator, releases it, then scales by alpha, rounds to bf16 and stores.
// gemm_kernel (M % 256 == 128): the same pipeline on one SM with 128 x 256 tiles.
// Every mbarrier wait is bounded in time; on expiry the kernel records the site in the caller's
// status word, tells the other roles to stop, drains what it issued and frees tensor memory.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>

#include <atomic>
#include <cstdint>

#include "launch.h"

namespace fp4k {
namespace gemm {

constexpr int BM = 128, BN = 256, BKB = 128;  // tile rows, tile cols, K bytes per stage (256 values)
constexpr int STAGES = 4;
constexpr int NUM_THREADS = 192;
constexpr int A_BYTES = BM * BKB, B_BYTES = BN * BKB;
constexpr int TMEM_COLS = 512;
constexpr int ACC_COL = 0, SFA_COL = 256, SFB_COL = 288;
constexpr unsigned long long kTimeoutNs = 2000000000ull;  // 2 s: default pipeline wait limit, and every drain wait

struct Params {
  int M, N, K;
  int nv;           // 1: NVFP4 (16-blocks, E4M3), 0: MXFP4 (32-blocks, E8M0)
  int atoms;        // 512-byte scale atoms per 128 rows per stage (4 NVFP4, 2 MXFP4)
  int atoms_row;    // scale atoms per 128-row group over the whole K
  const uint8_t* As;
  const uint8_t* Bs;
  const float* Ag;
  const float* Bg;
  __nv_bfloat16_raw* C;
  long long ldc;
  uint32_t* status;
  unsigned long long wait_ns;  // limit of each pipeline wait (kTimeoutNs unless set otherwise)
  int group_m;                 // M tiles walked together before the walk moves along N
};

// Output tile of linear index `tile`: bands of group_m M tiles, M fastest inside a band, the bands
// one after another, so that the A rows of one band stay in L2 while all of B streams past them.
__device__ __forceinline__ void tile_coords(int tile, int tiles_m, int tiles_n, int group_m, int& tm, int& tn) {
  const int per_group = group_m * tiles_n;
  const int g = tile / per_group, r = tile - g * per_group;
  tm = g * group_m + r % group_m;
  tn = r / group_m;
}

// ---------------------------------------------------------------------------------------------
// PTX wrappers
__device__ __forceinline__ uint32_t smem_u32(const void* p) { return (uint32_t)__cvta_generic_to_shared(p); }

__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count));
}
__device__ __forceinline__ void mbar_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes) : "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ bool mbar_try(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile("{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
               "selp.u32 %0, 1, 0, p;\n\t}"
               : "=r"(ok) : "r"(bar), "r"(parity) : "memory");
  return ok != 0;
}
__device__ __forceinline__ unsigned long long now_ns() {
  unsigned long long t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

// Bounded wait: true when the phase completed; false when this or another role gave up.  A wait
// longer than `limit` ns records its site in the status word and tells the other roles to stop.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag,
                                          uint32_t* status, uint32_t site, unsigned long long limit) {
  if (mbar_try(bar, parity)) return true;
  const unsigned long long t0 = now_ns();
  while (true) {
    if (mbar_try(bar, parity)) return true;
    if (*abort_flag) return false;
    if (now_ns() - t0 > limit) {
      atomicOr(status, 1u << site);
      *abort_flag = 1;
      return false;
    }
  }
}

// mbar_wait for code that every lane of a warp runs up to a warp-collective instruction (the
// epilogue's tcgen05.ld.sync.aligned): the lanes vote, so all of them see the same outcome (one lane
// giving up while another passes would leave the warp diverged at that instruction).  The MMA and
// scale-copy warps run their loops on every lane, lane 0 alone issuing, with no warp-collective
// instruction inside the loop: a lane that gives up simply leaves the loop early, and the lanes
// meet again at the __syncwarp after it.  (Running the loop on lane 0 alone, inside a divergent
// branch, measured 3-4% slower.)
__device__ __forceinline__ bool warp_wait(uint32_t bar, uint32_t parity, volatile int* abort_flag, uint32_t* status,
                                          uint32_t site, unsigned long long limit) {
  return __all_sync(0xFFFFFFFFu, mbar_wait(bar, parity, abort_flag, status, site, limit));
}

// Drain wait (exit paths): until the phase completes or kTimeoutNs passes, whatever the flags say.
__device__ __forceinline__ void mbar_drain(uint32_t bar, uint32_t parity) {
  const unsigned long long t0 = now_ns();
  while (!mbar_try(bar, parity) && now_ns() - t0 < kTimeoutNs) {
  }
}

// After `issued` fills of a ring of `stages` full barriers (fill g on stage g % stages, phase
// parity (g / stages) & 1), wait (bounded) until the last fill of every stage has landed.
__device__ __forceinline__ void drain_fills(uint32_t full0, uint32_t issued, uint32_t stages) {
  for (uint32_t s = 0; s < stages && s < issued; ++s) {
    const uint32_t last = s + stages * ((issued - 1 - s) / stages);
    mbar_drain(full0 + 8 * s, (last / stages) & 1);
  }
}

__device__ __forceinline__ void tma_load_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];"
      ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void bulk_load(uint32_t dst, const void* src, uint32_t bytes, uint32_t bar) {
  asm volatile("cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
               ::"r"(dst), "l"(src), "r"(bytes), "r"(bar) : "memory");
}

__device__ __forceinline__ void tc_fence_before() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void tc_fence_after() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
// scales: 32 rows x 16 bytes from shared memory, replicated into the four 32-lane quarters
__device__ __forceinline__ void tc_cp_sf(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
template <bool NV>
__device__ __forceinline__ void tc_mma(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                       uint32_t sfb, uint32_t accumulate) {
  if constexpr (NV) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate) : "memory");
  } else {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::1.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate) : "memory");
  }
}

// fp16 operands without block scales (the IF4 GEMM's expanded operands): kind::f16, K = 16 per
// instruction, FP32 accumulation.
__device__ __forceinline__ void tc_mma_f16(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
               ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate) : "memory");
}

// The FP8 route for MXFP4 operands expanded to E4M3: kind::mxf8f6f4, one UE8M0 scale per 32 values
// (scale_vec::1X), K = 32 per instruction.
__device__ __forceinline__ void tc_mma_f8(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                          uint32_t sfb, uint32_t accumulate) {
  asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
               "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale.scale_vec::1X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
               ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate) : "memory");
}

// Two fp32 accumulator words scaled by alpha and rounded to bf16 (RNE), the first in the low half.
__device__ __forceinline__ uint32_t bf16x2_scaled(uint32_t lo, uint32_t hi, float alpha) {
  uint32_t b;
  asm("cvt.rn.bf16x2.f32 %0, %1, %2;"
      : "=r"(b)
      : "f"(__fmul_rn(__uint_as_float(hi), alpha)), "f"(__fmul_rn(__uint_as_float(lo), alpha)));
  return b;
}

#define TC_LD32(taddr, r)                                                                                   \
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15," \
               "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"                       \
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]), \
                 "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),        \
                 "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),      \
                 "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),      \
                 "=r"(r[29]), "=r"(r[30]), "=r"(r[31])                                                           \
               : "r"(taddr))

// Shared-memory matrix descriptor (sm_100 format, version 1).
//   K-major operand tile, 128-byte swizzle: 8-row groups 1024 bytes apart (SBO), no LBO.
//   Scale tile (no swizzle): 8 rows of 16 bytes per core matrix, core matrices 128 bytes apart.
__device__ __forceinline__ uint64_t desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(1024 >> 4) << 32) | (1ull << 46) | (2ull << 61);
}
__device__ __forceinline__ uint64_t desc_sf(uint32_t saddr) {
  return (uint64_t)((saddr >> 4) & 0x3FFF) | ((uint64_t)(128 >> 4) << 32) | (1ull << 46);
}

// Instruction descriptor, kind::mxf4nvf4: E2M1 x E2M1, K-major A and B, M = 128, N = 256,
// scale type bit 23 (0 = UE4M3, 1 = UE8M0), scale-factor byte ids for A (29-30) and B (4-5).
__host__ __device__ constexpr uint32_t idesc(bool nv, uint32_t sfa_id, uint32_t sfb_id) {
  return (sfb_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(BN >> 3) << 17) | ((nv ? 0u : 1u) << 23) |
         ((uint32_t)(BM >> 4) << 24) | (sfa_id << 29);
}

// Instruction descriptor, kind::mxf8f6f4: E4M3 x E4M3 (format code 0 in bits 7-9 and 10-12),
// K-major A and B, M = 128, N = 256, UE8M0 scales (bit 23), scale byte ids as above.
__host__ __device__ constexpr uint32_t idesc_f8(uint32_t sfa_id, uint32_t sfb_id) {
  return (sfb_id << 4) | ((uint32_t)(BN >> 3) << 17) | (1u << 23) | ((uint32_t)(BM >> 4) << 24) | (sfa_id << 29);
}

// Instruction descriptor, kind::f16: F32 accumulator (bits 4-5 = 1), F16 x F16 (format 0 in bits
// 7-9 and 10-12), K-major A and B, M = 128, N = 256.
__host__ __device__ constexpr uint32_t idesc_f16() {
  return (1u << 4) | ((uint32_t)(BN >> 3) << 17) | ((uint32_t)(BM >> 4) << 24);
}

// Operand kinds of the 1-SM kernel.
constexpr int kMxFp4 = 0, kNvFp4 = 1, kMxE4m3 = 2, kF16 = 3;

// ---------------------------------------------------------------------------------------------
// KIND kMxFp4 / kNvFp4: packed E2M1 operands, 256 values (128 bytes) per row per stage, four K=64
// MMAs.  kMxE4m3: the E4M3 expansions of MXFP4 operands, 128 values (128 bytes) per stage, four
// K=32 MMAs of kind::mxf8f6f4, each taking one of the stage's four UE8M0 scales per row (scale
// byte id 0-3 of the atom's 32-bit tensor-memory column).  kF16: fp16 operands, 64 values (128
// bytes) per stage, four K=16 MMAs of kind::f16, no scales.
template <int KIND>
__global__ void __launch_bounds__(NUM_THREADS, 1)
gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, Params p) {
  constexpr bool NV = KIND == kNvFp4, F8 = KIND == kMxE4m3, F16 = KIND == kF16;
  constexpr int ATOMS = F16 ? 0 : (NV ? 4 : (F8 ? 1 : 2));  // scale atoms per 128 rows per stage
  constexpr int SFA_BYTES = ATOMS * 512;
  constexpr int SFB_BYTES = 2 * ATOMS * 512;  // two 128-row groups
  constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  constexpr uint32_t TX_BYTES = STAGE_BYTES;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;                                  // STAGES x A_BYTES
  uint8_t* sB = sA + STAGES * A_BYTES;                 // STAGES x B_BYTES
  uint8_t* sSFA = sB + STAGES * B_BYTES;               // STAGES x SFA_BYTES
  uint8_t* sSFB = sSFA + STAGES * SFA_BYTES;           // STAGES x SFB_BYTES
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + STAGES * SFB_BYTES);
  // bars: full[STAGES], empty[STAGES], tmem_full, tmem_empty, drain
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * STAGES + 3);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + STAGES);
  const uint32_t tmem_full = smem_u32(bars + 2 * STAGES), tmem_empty = smem_u32(bars + 2 * STAGES + 1);
  const uint32_t drain = smem_u32(bars + 2 * STAGES + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;");
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int tiles_m = p.M / BM, tiles_n = p.N / BN;
  const int num_tiles = tiles_m * tiles_n;
  const int kt_count = p.K / (F16 ? 64 : (F8 ? 128 : 256));

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
      uint32_t g = 0;  // global k-iteration counter
      uint32_t issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x) {
        int tm, tn;
        tile_coords(tile, tiles_m, tiles_n, p.group_m, tm, tn);
        for (int kt = 0; kt < kt_count; ++kt, ++g) {
          const int s = g % STAGES;
          const uint32_t ph = (g / STAGES) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, abort_flag, p.status, 0, p.wait_ns)) { ok = false; break; }
          const uint32_t fb = full0 + 8 * s;
          mbar_expect_tx(fb, TX_BYTES);
          issued = g + 1;
          tma_load_2d(smem_u32(sA + s * A_BYTES), &tmA, kt * BKB, tm * BM, fb);
          tma_load_2d(smem_u32(sB + s * B_BYTES), &tmB, kt * BKB, tn * BN, fb);
          if constexpr (!F16) {
            const uint8_t* sfa = p.As + ((size_t)tm * p.atoms_row + (size_t)kt * ATOMS) * 512;
            bulk_load(smem_u32(sSFA + s * SFA_BYTES), sfa, SFA_BYTES, fb);
#pragma unroll
            for (int rg = 0; rg < 2; ++rg) {
              const uint8_t* sfb = p.Bs + ((size_t)(2 * tn + rg) * p.atoms_row + (size_t)kt * ATOMS) * 512;
              bulk_load(smem_u32(sSFB + s * SFB_BYTES + rg * ATOMS * 512), sfb, ATOMS * 512, fb);
            }
          }
        }
      }
      if (ok) {
        // wait for the MMA side to release the last STAGES fills, so that no tcgen05.commit
        // arrival is still in flight towards this CTA's barriers when it exits
        for (int i = 0; i < STAGES; ++i, ++g) {
          const int s = g % STAGES;
          if (!mbar_wait(empty0 + 8 * s, ((g / STAGES) & 1) ^ 1, abort_flag, p.status, 4, p.wait_ns)) {
            ok = false;
            break;
          }
        }
      }
      // a wait gave up: every fill issued must still land before the CTA's shared memory goes away
      if (!ok) drain_fills(full0, issued, STAGES);
    }
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (lane 0 issues)
    {
    uint32_t g = 0, j = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < num_tiles && ok; tile += gridDim.x, ++j) {
      if (!mbar_wait(tmem_empty, (j & 1) ^ 1, abort_flag, p.status, 1, p.wait_ns)) { ok = false; break; }
      tc_fence_after();
      for (int kt = 0; kt < kt_count; ++kt, ++g) {
        const int s = g % STAGES;
        const uint32_t ph = (g / STAGES) & 1;
        if (!mbar_wait(full0 + 8 * s, ph, abort_flag, p.status, 2, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + s * A_BYTES), b0 = smem_u32(sB + s * B_BYTES);
          const uint32_t fa = smem_u32(sSFA + s * SFA_BYTES), fbs = smem_u32(sSFB + s * SFB_BYTES);
#pragma unroll
          for (int a = 0; a < ATOMS; ++a) {
            tc_cp_sf(tmem + SFA_COL + 4 * a, desc_sf(fa + a * 512));
            tc_cp_sf(tmem + SFB_COL + 8 * a, desc_sf(fbs + a * 512));
            tc_cp_sf(tmem + SFB_COL + 8 * a + 4, desc_sf(fbs + (ATOMS + a) * 512));
          }
#pragma unroll
          for (int t = 0; t < 4; ++t) {  // four MMAs of 32 bytes of K per stage
            const uint32_t acc = (kt > 0 || t > 0) ? 1u : 0u;
            if constexpr (F16) {
              tc_mma_f16(tmem + ACC_COL, desc_sw128(a0 + 32 * t), desc_sw128(b0 + 32 * t), idesc_f16(), acc);
            } else if constexpr (F8) {
              tc_mma_f8(tmem + ACC_COL, desc_sw128(a0 + 32 * t), desc_sw128(b0 + 32 * t), idesc_f8(t, t),
                        tmem + SFA_COL, tmem + SFB_COL, acc);
            } else {
              const int atom = NV ? t : (t >> 1);
              const uint32_t sf_id = NV ? 0u : (uint32_t)((t & 1) * 2);
              tc_mma<NV>(tmem + ACC_COL, desc_sw128(a0 + 32 * t), desc_sw128(b0 + 32 * t), idesc(NV, sf_id, sf_id),
                         tmem + SFA_COL + 4 * atom, tmem + SFB_COL + 8 * atom, acc);
            }
          }
          tc_commit(empty0 + 8 * s);  // stage free once these MMAs have read it
        }
      }
      if (!ok) break;
      if (lane == 0) tc_commit(tmem_full);
    }
    if (lane == 0) {
      // on every path: the barrier arrives once every MMA and scale copy this thread issued has
      // completed, so none is still running when tensor memory is freed (the epilogue may have
      // given up on a tile whose MMAs are in flight)
      tc_commit(drain);
      mbar_drain(drain, 0);
    }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    // E4M3 operands hold value * 2^-6 each, so their products carry 2^-12
    const float alpha = F8 ? 4096.0f : (p.nv ? __fmul_rn(*p.Ag, *p.Bg) : 1.0f);
    uint32_t j = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++j) {
      int tm, tn;
      tile_coords(tile, tiles_m, tiles_n, p.group_m, tm, tn);
      if (!warp_wait(tmem_full, j & 1, abort_flag, p.status, 3, p.wait_ns)) break;
      tc_fence_after();
      const int row = tm * BM + q * 32 + lane;
      uint4* crow = reinterpret_cast<uint4*>(p.C + (size_t)row * p.ldc + (size_t)tn * BN);
#pragma unroll 1
      for (int c = 0; c < BN / 32; ++c) {
        uint32_t r[32];
        TC_LD32(tmem + ACC_COL + ((uint32_t)(q * 32) << 16) + c * 32, r);
        asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
        uint32_t packed[16];
#pragma unroll
        for (int i = 0; i < 16; ++i) {
          const float lo = __fmul_rn(__uint_as_float(r[2 * i]), alpha);
          const float hi = __fmul_rn(__uint_as_float(r[2 * i + 1]), alpha);
          uint32_t b;
          asm("cvt.rn.bf16x2.f32 %0, %1, %2;" : "=r"(b) : "f"(hi), "f"(lo));
          packed[i] = b;
        }
#pragma unroll
        for (int v = 0; v < 4; ++v)
          crow[c * 4 + v] = make_uint4(packed[4 * v], packed[4 * v + 1], packed[4 * v + 2], packed[4 * v + 3]);
      }
      tc_fence_before();
      mbar_arrive(tmem_empty);  // accumulator read out: the next tile may start
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

template <int KIND>
constexpr int smem_bytes() {
  constexpr int atoms = KIND == kF16 ? 0 : (KIND == kNvFp4 ? 4 : (KIND == kMxE4m3 ? 1 : 2));
  return 1024 + STAGES * (A_BYTES + B_BYTES + atoms * 512 * 3) + 256;
}

// ---------------------------------------------------------------------------------------------
// 2-SM variant: a cluster of two CTAs on neighbouring SMs computes a 256 x 256 output tile with
// tcgen05 cta_group::2.  CTA r of the pair holds rows [128r, 128r+128) of the A tile and of the B
// tile (the MMA splits M across the pair for A and D, N across the pair for B) plus the scales
// for its A rows and for all 256 B rows.  Both CTAs' tensor-map loads complete on the leader's
// (rank 0) barrier, which the leader arms for the pair's bytes; the leader alone issues
// tcgen05.cp and tcgen05.mma, and its commits arrive on the barriers of both CTAs.  Each SM then
// reads 32 KB of operands per 256-value K stage instead of 48 KB, and 5-6 stages fit.

__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_rank(uint32_t saddr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(saddr), "r"(rank));
  return r;
}
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr) : "memory");
}
__device__ __forceinline__ void tma_pair_2d(uint32_t dst, const CUtensorMap* map, int x, int y, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3}], [%4];" ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(bar) : "memory");
}
__device__ __forceinline__ void tma_pair_3d(uint32_t dst, const CUtensorMap* map, int x, int y, int z, uint32_t bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%2, %3, %4}], [%5];" ::"r"(dst), "l"(map), "r"(x), "r"(y), "r"(z), "r"(bar) : "memory");
}
__device__ __forceinline__ void tc_commit_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;"
               ::"r"(bar), "h"((uint16_t)3) : "memory");
}
__device__ __forceinline__ void tc_commit_local_pair(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(bar) : "memory");
}
__device__ __forceinline__ void tc_cp_sf_pair(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::2.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc) : "memory");
}
template <bool NV>
__device__ __forceinline__ void tc_mma_pair(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                                            uint32_t sfb, uint32_t accumulate) {
  if constexpr (NV) {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::4X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate) : "memory");
  } else {
    asm volatile("{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %6, 0;\n\t"
                 "tcgen05.mma.cta_group::2.kind::mxf4nvf4.block_scale.scale_vec::2X [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
                 ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate) : "memory");
  }
}

// M = 256 (the pair), N = 256
__host__ __device__ constexpr uint32_t idesc_pair(bool nv, uint32_t sfa_id, uint32_t sfb_id) {
  return (sfb_id << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(256 >> 3) << 17) | ((nv ? 0u : 1u) << 23) |
         ((uint32_t)(256 >> 4) << 24) | (sfa_id << 29);
}

template <bool NV> struct PairCfg {
  static constexpr int ATOMS = NV ? 4 : 2;
  static constexpr int S = NV ? 5 : 6;
  static constexpr int NB = 3;  // scale buffers in tensor memory
  static constexpr int A_HALF = 128 * BKB, B_HALF = 128 * BKB;
  static constexpr int SFA_BYTES = ATOMS * 512, SFB_BYTES = 2 * ATOMS * 512;
  static constexpr int STAGE = A_HALF + B_HALF + SFA_BYTES + SFB_BYTES;
  static constexpr int SMEM = 1024 + S * STAGE + 512;
  static constexpr uint32_t SF_BUF = 12u * ATOMS;  // TMEM columns per scale buffer: SFA 4*ATOMS + SFB 8*ATOMS
};
// warp 0 TMA, 1 MMA, 2-3 scale copies, 4-11 epilogue (two warps per tensor-memory lane quadrant,
// one per 128-column half of the accumulator)
constexpr int PAIR_THREADS = 384;
constexpr int PAIR_CP_WARPS = 2;

template <bool NV>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const __grid_constant__ CUtensorMap tmSA, const __grid_constant__ CUtensorMap tmSB, Params p) {
  using C = PairCfg<NV>;
  constexpr int S = C::S, ATOMS = C::ATOMS, NB = C::NB;
  static_assert(SFA_COL + NB * (int)C::SF_BUF <= TMEM_COLS, "scale buffers exceed the tensor-memory allocation");
  constexpr uint32_t TX_PAIR = 2u * C::STAGE;

  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + S * C::A_HALF;
  uint8_t* sSFA = sB + S * C::B_HALF;
  uint8_t* sSFB = sSFA + S * C::SFA_BYTES;
  uint64_t* bars = reinterpret_cast<uint64_t*>(sSFB + S * C::SFB_BYTES);
  // bars: full[S] (leader), empty[S], sf_full[NB], sf_empty[NB], tmem_full, tmem_empty (leader),
  // drain[1 + PAIR_CP_WARPS] (MMA warp, each scale-copy warp)
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(bars + 2 * S + 2 * NB + 3 + PAIR_CP_WARPS);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const uint32_t full0 = smem_u32(bars), empty0 = smem_u32(bars + S);
  const uint32_t sf_full0 = smem_u32(bars + 2 * S), sf_empty0 = smem_u32(bars + 2 * S + NB);
  const uint32_t tmem_full = smem_u32(bars + 2 * S + 2 * NB), tmem_empty = smem_u32(bars + 2 * S + 2 * NB + 1);
  const uint32_t drain0 = smem_u32(bars + 2 * S + 2 * NB + 2);

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int b = 0; b < NB; ++b) {
      mbar_init(sf_full0 + 8 * b, PAIR_CP_WARPS);  // one commit per scale-copy warp
      mbar_init(sf_empty0 + 8 * b, 1);
    }
    mbar_init(tmem_full, 1);
    mbar_init(tmem_empty, 16);  // 8 epilogue warps in each CTA of the pair
    for (int i = 0; i <= PAIR_CP_WARPS; ++i) mbar_init(drain0 + 8 * i, 1);
    *abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(tmem_slot)),
                 "r"(TMEM_COLS));
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;");
  }
  tc_fence_before();
  cluster_sync();  // barriers initialised and tensor memory allocated in both CTAs
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  const int tiles_m = p.M / 256, tiles_n = p.N / 256;
  const int num_tiles = tiles_m * tiles_n;
  const int kt_count = p.K / 256;
  const int cid = blockIdx.x >> 1, ncl = gridDim.x >> 1;
  const uint32_t my_tiles = (uint32_t)((num_tiles - cid + ncl - 1) / ncl);
  const uint32_t total = my_tiles * (uint32_t)kt_count;

  if (warp == 0) {
    // ------------------------------------------------------------------ TMA producer (both CTAs)
    if (lane == 0) {
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmA) : "memory");
      asm volatile("prefetch.tensormap [%0];" ::"l"(&tmB) : "memory");
      uint32_t g = 0;
      bool ok = true, issued = false;
      uint32_t issued_n = 0;
      for (int tile = cid; tile < num_tiles && ok; tile += ncl) {
        int tm, tn;
        tile_coords(tile, tiles_m, tiles_n, p.group_m, tm, tn);
        for (int kt = 0; kt < kt_count; ++kt, ++g) {
          const int s = g % S;
          const uint32_t ph = (g / S) & 1;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1, abort_flag, p.status, 0, p.wait_ns)) { ok = false; break; }
          const uint32_t fb = map_rank(full0 + 8 * s, 0);  // the leader's barrier
          if (leader) mbar_expect_tx(full0 + 8 * s, TX_PAIR);
          tma_pair_2d(smem_u32(sA + s * C::A_HALF), &tmA, kt * BKB, tm * 256 + (int)rank * 128, fb);
          tma_pair_2d(smem_u32(sB + s * C::B_HALF), &tmB, kt * BKB, tn * 256 + (int)rank * 128, fb);
          tma_pair_3d(smem_u32(sSFA + s * C::SFA_BYTES), &tmSA, 0, kt * ATOMS, tm * 2 + (int)rank, fb);
          tma_pair_3d(smem_u32(sSFB + s * C::SFB_BYTES), &tmSB, 0, kt * ATOMS, tn * 2, fb);
          issued = true;
          issued_n = g + 1;
        }
      }
      if (ok) {
        // the last S releases: no tcgen05.commit arrival is still on its way to this CTA
        for (int i = 0; i < S; ++i, ++g) {
          const int s = g % S;
          if (!mbar_wait(empty0 + 8 * s, ((g / S) & 1) ^ 1, abort_flag, p.status, 4, p.wait_ns)) {
            ok = false;
            break;
          }
        }
      }
      if (!ok && issued) {
        if (leader) {
          // both CTAs' fills complete on the leader's barriers: wait (bounded) for the last phase
          // of every stage issued, so that they have landed before the final cluster barrier
          drain_fills(full0, issued_n, S);
        } else {
          // this CTA cannot observe its fills (they complete on the leader's barrier): give them a
          // fixed, bounded time to land before shared memory is released
          const unsigned long long t0 = now_ns();
          while (now_ns() - t0 < 2000000ull) {
          }
        }
      }
    }
  } else if (warp == 2 || warp == 3) {
    // ------------------------------------------------------------------ scale copies (leader)
    // Issued from their own warps so that they queue separately from the MMAs, and split over two
    // warps (each a contiguous half of the stage's scale atoms, all three copies of an atom):
    // tcgen05.cp issue from one thread was the limit with NVFP4's 12 copies per stage.  Iteration
    // g's scales go to TMEM buffer g % NB once its stage has landed and the MMAs that last read
    // the buffer have completed; each warp's commit then counts towards the buffer being ready.
    const int ci = warp - 2;
    constexpr int PER = ATOMS / PAIR_CP_WARPS;
    static_assert(ATOMS % PAIR_CP_WARPS == 0, "whole atoms per copy warp");
    if (leader) {
      bool ok = true;
      uint32_t g = 0;
      for (; g < total && ok; ++g) {
        const int s = g % S, b = g % NB;
        if (!mbar_wait(full0 + 8 * s, (g / S) & 1, abort_flag, p.status, 6, p.wait_ns)) { ok = false; break; }
        if (!mbar_wait(sf_empty0 + 8 * b, ((g / NB) & 1) ^ 1, abort_flag, p.status, 7, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t fa = smem_u32(sSFA + s * C::SFA_BYTES), fbs = smem_u32(sSFB + s * C::SFB_BYTES);
          const uint32_t sfa = tmem + SFA_COL + b * C::SF_BUF, sfb = sfa + 4 * ATOMS;
#pragma unroll
          for (int i = 0; i < PER; ++i) {
            const int a = ci * PER + i;
            tc_cp_sf_pair(sfa + 4 * a, desc_sf(fa + a * 512));
            tc_cp_sf_pair(sfb + 8 * a, desc_sf(fbs + a * 512));
            tc_cp_sf_pair(sfb + 8 * a + 4, desc_sf(fbs + (ATOMS + a) * 512));
          }
          tc_commit_local_pair(sf_full0 + 8 * b);
        }
      }
      if (ok) {
        // the MMA warp's last releases of the scale buffers have landed
        for (int i = 0; i < NB; ++i, ++g) {
          const int b = g % NB;
          if (!mbar_wait(sf_empty0 + 8 * b, ((g / NB) & 1) ^ 1, abort_flag, p.status, 8, p.wait_ns)) break;
        }
      }
      if (lane == 0) {
        // on every path: arrives once this warp's scale copies have completed
        const uint32_t dr = drain0 + 8 * (1 + ci);
        tc_commit_local_pair(dr);
        mbar_drain(dr, 0);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------------ MMA issuer (leader, lane 0)
    if (leader) {
      bool ok = true;
      uint32_t j = 0;
      for (uint32_t g = 0; g < total && ok; ++g) {
        const uint32_t kt = g % (uint32_t)kt_count;
        const int s = g % S, b = g % NB;
        j = g / (uint32_t)kt_count;
        if (kt == 0) {
          if (!mbar_wait(tmem_empty, (j & 1) ^ 1, abort_flag, p.status, 1, p.wait_ns)) { ok = false; break; }
        }
        if (!mbar_wait(full0 + 8 * s, (g / S) & 1, abort_flag, p.status, 2, p.wait_ns)) { ok = false; break; }
        if (!mbar_wait(sf_full0 + 8 * b, (g / NB) & 1, abort_flag, p.status, 9, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        if (lane == 0) {
          const uint32_t a0 = smem_u32(sA + s * C::A_HALF), b0 = smem_u32(sB + s * C::B_HALF);
          const uint32_t sfa = tmem + SFA_COL + b * C::SF_BUF, sfb = sfa + 4 * ATOMS;
#pragma unroll
          for (int t = 0; t < 4; ++t) {
            const int atom = NV ? t : (t >> 1);
            const uint32_t sf_id = NV ? 0u : (uint32_t)((t & 1) * 2);
            tc_mma_pair<NV>(tmem + ACC_COL, desc_sw128(a0 + 32 * t), desc_sw128(b0 + 32 * t),
                            idesc_pair(NV, sf_id, sf_id), sfa + 4 * atom, sfb + 8 * atom,
                            (kt > 0 || t > 0) ? 1u : 0u);
          }
          tc_commit_pair(empty0 + 8 * s);                               // frees stage s in both CTAs
          tc_commit_local_pair(sf_empty0 + 8 * b);                      // scale buffer b may be refilled
          if (kt == (uint32_t)kt_count - 1) tc_commit_pair(tmem_full);  // accumulator ready in both CTAs
        }
      }
      j = my_tiles;
      if (ok) {
        // both epilogues have released the last accumulator (all their arrivals have landed)
        mbar_wait(tmem_empty, (j & 1) ^ 1, abort_flag, p.status, 5, p.wait_ns);
      }
      if (lane == 0) {
        // on every path: arrives once every MMA issued has completed (an epilogue that gave up may
        // have left a tile's MMAs running)
        tc_commit_local_pair(drain0);
        mbar_drain(drain0, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------------ epilogue (warps 4..11, both CTAs)
    // Warp w reads tensor-memory lanes 32 (w % 4).. (its rows) and accumulator columns
    // 128 (w >= 8).. : four 32-column loads, one wait, then the accumulator is released to the MMA
    // warp before the conversion and the stores, so the next tile's MMAs wait only for the loads.
    const int q = warp & 3, half = warp >= 8 ? 1 : 0;
    const float alpha = p.nv ? __fmul_rn(*p.Ag, *p.Bg) : 1.0f;
    const uint32_t empty_leader = map_rank(tmem_empty, 0);
    uint32_t j = 0;
    for (int tile = cid; tile < num_tiles; tile += ncl, ++j) {
      int tm, tn;
      tile_coords(tile, tiles_m, tiles_n, p.group_m, tm, tn);
      if (!warp_wait(tmem_full, j & 1, abort_flag, p.status, 3, p.wait_ns)) break;
      tc_fence_after();
      const uint32_t taddr = tmem + ACC_COL + ((uint32_t)(q * 32) << 16) + (uint32_t)(half * 128);
      uint32_t r0[32], r1[32], r2[32], r3[32];
      TC_LD32(taddr, r0);
      TC_LD32(taddr + 32, r1);
      TC_LD32(taddr + 64, r2);
      TC_LD32(taddr + 96, r3);
      asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(empty_leader);  // this warp's part of the accumulator is read
      uint32_t pk[64];
#pragma unroll
      for (int i = 0; i < 16; ++i) {
        pk[i] = bf16x2_scaled(r0[2 * i], r0[2 * i + 1], alpha);
        pk[16 + i] = bf16x2_scaled(r1[2 * i], r1[2 * i + 1], alpha);
        pk[32 + i] = bf16x2_scaled(r2[2 * i], r2[2 * i + 1], alpha);
        pk[48 + i] = bf16x2_scaled(r3[2 * i], r3[2 * i + 1], alpha);
      }
      const int row = tm * 256 + (int)rank * 128 + q * 32 + lane;
      uint4* crow = reinterpret_cast<uint4*>(p.C + (size_t)row * p.ldc + (size_t)tn * BN + half * 128);
#pragma unroll
      for (int v = 0; v < 16; ++v) crow[v] = make_uint4(pk[4 * v], pk[4 * v + 1], pk[4 * v + 2], pk[4 * v + 3]);
    }
  }

  tc_fence_before();
  cluster_sync();
  tc_fence_after();
  if (warp == 1) {
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(TMEM_COLS));
  }
}

// ---------------------------------------------------------------------------------------------
// Host side: tensor maps through the driver entry point (no link against libcuda).

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  if (!fn) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  }
  return fn;
}

static bool make_map(CUtensorMap* m, const void* base, uint64_t row_bytes, uint64_t rows, uint32_t box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {row_bytes, rows};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {(cuuint32_t)BKB, box_rows};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

// Scale tiles in the MMA tile layout viewed as a 3-D tensor of 32-bit words: 128 words (one
// 512-byte 128x4 atom) x atoms per 128-row group x row groups.  A box of `atoms` atoms x
// `groups` row groups lands in shared memory as consecutive atoms, group-major.
static bool make_sf_map(CUtensorMap* m, const void* base, uint64_t atoms_row, uint64_t groups, uint32_t atoms,
                        uint32_t box_groups) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[3] = {128, atoms_row, groups};
  cuuint64_t strides[2] = {512, atoms_row * 512};
  cuuint32_t box[3] = {128, atoms, box_groups};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<void*>(base), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

}  // namespace gemm

static std::atomic<unsigned long long> g_wait_ns{gemm::kTimeoutNs};

unsigned long long set_gemm_wait_limit(unsigned long long ns) { return g_wait_ns.exchange(ns); }

static cudaError_t launch_gemm_pair(const GemmLaunch& L, const gemm::Params& p, cudaStream_t s) {
  using namespace gemm;
  const uint32_t atoms = L.nv ? 4 : 2;
  CUtensorMap ta, tb, tsa, tsb;
  if (!make_map(&ta, L.Aq, (uint64_t)L.K / 2, (uint64_t)L.M, 128) ||
      !make_map(&tb, L.Bq, (uint64_t)L.K / 2, (uint64_t)L.N, 128) ||
      !make_sf_map(&tsa, L.As, (uint64_t)p.atoms_row, (uint64_t)L.M / 128, atoms, 1) ||
      !make_sf_map(&tsb, L.Bs, (uint64_t)p.atoms_row, (uint64_t)L.N / 128, atoms, 2))
    return cudaErrorInvalidValue;
  const int tiles = (L.M / 256) * (L.N / 256);
  const int pairs = num_sms() / 2;
  const int grid = 2 * (tiles < pairs ? tiles : pairs);
  if (L.nv) {
    auto k = gemm_pair_kernel<true>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg<true>::SMEM);
    k<<<grid, PAIR_THREADS, PairCfg<true>::SMEM, s>>>(ta, tb, tsa, tsb, p);
  } else {
    auto k = gemm_pair_kernel<false>;
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, PairCfg<false>::SMEM);
    k<<<grid, PAIR_THREADS, PairCfg<false>::SMEM, s>>>(ta, tb, tsa, tsb, p);
  }
  return cudaGetLastError();
}

cudaError_t launch_gemm(const GemmLaunch& L, cudaStream_t s) {
  using namespace gemm;
  Params p;
  p.M = L.M; p.N = L.N; p.K = L.K; p.nv = L.nv ? 1 : 0;
  p.atoms = L.nv ? 4 : (L.e4m3 ? 1 : 2);
  p.atoms_row = L.K / (L.nv ? 16 : 32) / 4;
  p.As = L.As; p.Bs = L.Bs; p.Ag = L.Ag; p.Bg = L.Bg;
  p.C = reinterpret_cast<__nv_bfloat16_raw*>(L.C);
  p.ldc = L.ldc;
  p.status = L.status;
  p.wait_ns = g_wait_ns.load();
  // Tile walk.  When all of B fits in 40 MB of L2 (a little under a third of it), N goes fastest:
  // a wave then spans a few bands of A rows and all of B, which stays resident, and it writes
  // whole rows of C (NVFP4 8192^3: 1.3% faster than banding M).  Otherwise the walk takes the
  // largest power-of-two band of M tiles whose A rows fit in those 40 MB, so A stays resident
  // while B streams past (B is 117-235 MB in the down_proj GEMMs and 134 MB as fp16 in the IF4
  // one, where walking N fastest cost 10%).  Tiles are 256 rows in the 2-SM kernel and 128 in the
  // 1-SM one; operand rows hold K/2 bytes (FP4), K (E4M3) or 2K (fp16).
  {
    const bool pair = !L.e4m3 && !L.f16 && L.M % 256 == 0 && num_sms() >= 2;
    const int tile_rows = pair ? 256 : BM;
    const unsigned long long row_bytes = L.f16 ? 2ull * L.K : (L.e4m3 ? (unsigned long long)L.K : L.K / 2ull);
    const unsigned long long band = (unsigned long long)tile_rows * row_bytes;
    const int tiles_m = L.M / tile_rows;
    p.group_m = 1;
    if ((unsigned long long)L.N * row_bytes > (40ull << 20))
      while (tiles_m % (2 * p.group_m) == 0 && 2ull * p.group_m * band <= (40ull << 20)) p.group_m *= 2;
  }
  if (!L.e4m3 && !L.f16 && L.M % 256 == 0 && num_sms() >= 2) return launch_gemm_pair(L, p, s);
  // operand rows: K/2 packed bytes (FP4), K bytes (E4M3 expansion) or 2K bytes (fp16)
  const uint64_t row_bytes = L.f16 ? 2 * (uint64_t)L.K : (L.e4m3 ? (uint64_t)L.K : (uint64_t)L.K / 2);
  CUtensorMap ta, tb;
  if (!make_map(&ta, L.Aq, row_bytes, (uint64_t)L.M, BM) || !make_map(&tb, L.Bq, row_bytes, (uint64_t)L.N, BN))
    return cudaErrorInvalidValue;
  const int tiles = (L.M / BM) * (L.N / BN);
  const int grid = tiles < num_sms() ? tiles : num_sms();
  auto go = [&](auto k, int smem) {
    cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    k<<<grid, NUM_THREADS, smem, s>>>(ta, tb, p);
  };
  if (L.f16) go(gemm_kernel<kF16>, smem_bytes<kF16>());
  else if (L.e4m3) go(gemm_kernel<kMxE4m3>, smem_bytes<kMxE4m3>());
  else if (L.nv) go(gemm_kernel<kNvFp4>, smem_bytes<kNvFp4>());
  else go(gemm_kernel<kMxFp4>, smem_bytes<kMxFp4>());
  return cudaGetLastError();
}

}  // namespace fp4k
