// capi_noalloc.cu — nvfp4_quantize for callers that cannot allocate device memory.
//
// nvfp4_quantize needs a small device workspace (the per-CTA partial maxima that carry the tensor
// amax between its two passes).  Some callers cannot provide one: a plugin running inside another runtime that
// hands it only its input and output buffers, or a latency-critical loop in which a cudaMalloc
// (which may synchronise the device) is not acceptable.  This entry point takes the workspace from
// a fixed array in this library's device memory instead, and otherwise runs exactly the
// nvfp4_quantize path.
//
// The array is a file-scope __device__ variable.  Its host-side name is only a stand-in, so its
// device address is looked up with cudaGetSymbolAddress — once per device, with that device
// current, on the first call made on it — and that address is what the kernels receive.
#include <cstdio>
#include <mutex>

#include "../../include/fp4mx.h"
#include "launch.h"

namespace {

// holds the amax pass's partial maxima (fp4_workspace_size's need for every shape)
constexpr size_t kNoallocScratchBytes = fp4k::kAmaxSlots * sizeof(uint32_t);
constexpr int kMaxDevices = 64;

static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

std::mutex g_scratch_mu;
void* g_scratch_ptr[kMaxDevices] = {nullptr};

fp4_status noalloc_fail(fp4_status s, const char* msg) {
  fp4k::set_last_error(msg);
  return s;
}

}  // namespace

extern "C" fp4_status nvfp4_quantize_noalloc(const void* x, fp4_dtype dtype, long rows, long cols, int block,
                                             fp4_round round, int mode, unsigned long long seed,
                                             fp4_scale_layout layout, const float* global_in, float* global_out,
                                             unsigned char* q, unsigned char* scales, fp4_counts* counts,
                                             void* stream) {
  const size_t need = fp4_workspace_size(FP4_OP_NVFP4_QUANTIZE, rows, cols);
  if (need > kNoallocScratchBytes) {
    char msg[160];
    snprintf(msg, sizeof(msg),
             "nvfp4_quantize_noalloc: this shape needs %zu bytes of scratch, the built-in area holds %zu",
             need, kNoallocScratchBytes);
    return noalloc_fail(FP4_EUNSUPPORTED, msg);
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return noalloc_fail(FP4_ECUDA, "nvfp4_quantize_noalloc: cudaGetDevice failed");
  if (dev < 0 || dev >= kMaxDevices) return noalloc_fail(FP4_EUNSUPPORTED, "nvfp4_quantize_noalloc: device index out of range");
  void* scratch = nullptr;
  {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        char msg[160];
        snprintf(msg, sizeof(msg), "nvfp4_quantize_noalloc: cudaGetSymbolAddress failed: %s", cudaGetErrorString(e));
        return noalloc_fail(FP4_ECUDA, msg);
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  // the amax pass overwrites every slot the quantise pass reads, so the contents left by the
  // previous call do not leak into this one.
  return nvfp4_quantize(x, dtype, rows, cols, block, round, mode, seed, layout, global_in, global_out, q, scales,
                        counts, scratch, kNoallocScratchBytes, stream);
}
