// A forward entry point that allocates nothing.
//
// svdq_linear_forward asks its caller for a workspace (the activation codes,
// group scales and the branch input T that its first kernel writes and its
// second kernel reads). Some callers cannot hand one over: hosts whose device
// memory is owned by their own allocator and may not be grown behind its back
// (a framework's caching allocator, a plugin host with a fixed budget), and
// latency-critical loops where a cudaMalloc may synchronize the device. For
// them this file keeps the workspace in a fixed scratch array that is part of
// the library's device image, so the call needs no allocation at all: every
// GPU that loads the library holds kScratchBytes of it until the process ends.
//
// Sharing rules: all calls on a device use the same array and it keeps what
// the previous call left there. Nothing in it has to start at zero, because
// the activation kernel writes every byte the GEMM reads. Calls whose work
// overlaps on the GPU (different streams, or different layers run
// concurrently) race on the array; serialize them on one stream.
#include <cuda_runtime.h>

#include <mutex>
#include <string>

#include "svdq.h"

namespace svdq {
void set_last_error(const std::string& msg);
}

namespace {

// Largest workspace the array holds. What a call needs is svdq_workspace_size:
// the activation codes and scales, T, and the activation kernel's float
// partials of T, whose count is the kernel's K split (SMs x resident CTAs per
// SM / 128-row blocks, at most 16). With one resident CTA per SM that split is
// 4 at 4608 rows on 148 SMs, and the 4608 x 3072 attention projection then
// needs about 25 MiB (INT4) or 18 MiB (NVFP4) at rank 128, 17 / 10 MiB at
// rank 32. Anything larger is refused below, whatever the shape.
constexpr size_t kScratchBytes = size_t(32) << 20;

constexpr int kMaxDevices = 64;
std::mutex g_mutex;
void* g_scratch_ptr[kMaxDevices] = {};

}  // namespace

// File-scope device array; device code could name it directly, host code only
// through the address cudaGetSymbolAddress returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes];

extern "C" svdq_status svdq_linear_forward_noalloc(svdq_layer_t layer, const void* X, int M, void* Y, void* stream) {
  size_t need = 0;
  svdq_status st = svdq_workspace_size(layer, M, &need);
  if (st != SVDQ_OK) return st;
  if (need > kScratchBytes) {
    svdq::set_last_error("svdq_linear_forward_noalloc: this layer needs " + std::to_string(need) +
                         " bytes of workspace for M = " + std::to_string(M) + ", above the fixed " +
                         std::to_string(kScratchBytes) + "-byte scratch; use svdq_linear_forward");
    return SVDQ_ERR_INVALID_ARG;
  }
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess || dev < 0 || dev >= kMaxDevices) {
    svdq::set_last_error(std::string("svdq_linear_forward_noalloc: no usable current device: ") +
                         cudaGetErrorString(e));
    return SVDQ_ERR_CUDA;
  }
  void* scratch = nullptr;
  {
    // one-time set-up per device, done with that device current
    std::lock_guard<std::mutex> lock(g_mutex);
    if (!g_scratch_ptr[dev]) {
      void* p = nullptr;
      e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || !p) {
        svdq::set_last_error(std::string("svdq_linear_forward_noalloc: cudaGetSymbolAddress failed: ") +
                             cudaGetErrorString(e));
        return SVDQ_ERR_CUDA;
      }
      g_scratch_ptr[dev] = p;
    }
    scratch = g_scratch_ptr[dev];
  }
  return svdq_linear_forward(layer, X, M, Y, scratch, kScratchBytes, stream);
}
