// quantize_noalloc.cu -- nvfp4_quantize for callers that cannot allocate device memory.
//
// nvfp4_quantize needs a small device workspace (the word that collects the
// tensor's absolute maximum when the caller supplies no global scale).  Some
// callers have no way to provide one: code that runs inside a framework or
// server that owns every device allocation and offers no workspace hook, and
// latency-critical loops where a cudaMalloc would synchronize the device.
// nvfp4_quantize_noalloc takes the same inputs and outputs and uses instead a
// fixed scratch block compiled into this library.
//
// The scratch block is a file-scope __device__ array: every GPU that loads the
// library holds its own copy until the process exits.  Host code cannot pass the
// array's name to a kernel (on the host it only names a stand-in), so the first
// call on each device looks up the array's device address with
// cudaGetSymbolAddress, with that device current, and caches it.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nvfp4.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

std::mutex g_scratch_mutex;
void* g_scratch_addr[kMaxDevices] = {};

// Device address of this device's scratch block (looked up once per device).
nvfp4_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
  if (dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  if (g_scratch_addr[dev] == nullptr) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) return NVFP4_ERR_CUDA;
    g_scratch_addr[dev] = p;
  }
  *out = g_scratch_addr[dev];
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                               nvfp4_scale_mode mode, nvfp4_sf_layout layout,
                                               const float* global_scale_in, uint8_t* codes, uint8_t* scales,
                                               float* global_scale_out, float* block_err, void* stream) {
  if (rows >= 0 && cols >= 0 && nvfp4_quantize_workspace_bytes(rows, cols) > kNoAllocScratchBytes)
    return NVFP4_ERR_WORKSPACE;
  void* scratch = nullptr;
  if (global_scale_in == nullptr) {
    const nvfp4_status st = scratch_for_current_device(&scratch);
    if (st != NVFP4_OK) return st;
  }
  // nvfp4_quantize clears the amax word of the scratch block before it uses it.
  return nvfp4_quantize(x, rows, cols, ld_x, mode, layout, global_scale_in, codes, scales, global_scale_out,
                        block_err, scratch, scratch ? kNoAllocScratchBytes : 0, stream);
}
