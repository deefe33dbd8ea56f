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
// cudaGetSymbolAddress, with that device current, and caches it together with the
// identity of the device's CUDA context.  A context destroyed by cudaDeviceReset
// takes the array with it; the next call sees a new context and looks the address
// up again.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/nvfp4.h"
#include "internal.h"

namespace {

constexpr size_t kNoAllocScratchBytes = 256;
constexpr int kMaxDevices = 64;

__device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct ScratchEntry {
  void* addr = nullptr;
  unsigned long long ctx_id = 0;  // context the address belongs to (0: none yet)
};

std::mutex g_scratch_mutex;
ScratchEntry g_scratch[kMaxDevices];

using CtxGetCurrentFn = CUresult (*)(CUcontext*);
using CtxGetIdFn = CUresult (*)(CUcontext, unsigned long long*);

template <typename Fn>
Fn driver_entry(const char* name) {
  void* p = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint(name, &p, cudaEnableDefault, &q) != cudaSuccess || q != cudaDriverEntryPointSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return reinterpret_cast<Fn>(p);
}

// Unique id of the calling thread's current CUDA context, 0 if none is current
// (or the driver cannot say).
unsigned long long current_context_id() {
  static CtxGetCurrentFn get_current = driver_entry<CtxGetCurrentFn>("cuCtxGetCurrent");
  static CtxGetIdFn get_id = driver_entry<CtxGetIdFn>("cuCtxGetId");
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of this device's scratch block, looked up once per device and
// context (the lookup creates the device's primary context if there is none yet).
nvfp4_status scratch_for_current_device(void** out) {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) {
    cudaGetLastError();
    return NVFP4_ERR_CUDA;
  }
  if (dev >= kMaxDevices) return NVFP4_ERR_UNSUPPORTED_DEVICE;
  std::lock_guard<std::mutex> lock(g_scratch_mutex);
  ScratchEntry& e = g_scratch[dev];
  const unsigned long long id = current_context_id();
  if (e.addr == nullptr || id == 0 || id != e.ctx_id) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();  // leave no pending error for the caller's next CUDA call
      e = ScratchEntry{};
      return NVFP4_ERR_CUDA;
    }
    e.addr = p;
    e.ctx_id = id != 0 ? id : current_context_id();  // the lookup made a context current
  }
  *out = e.addr;
  return NVFP4_OK;
}

}  // namespace

extern "C" nvfp4_status nvfp4_quantize_noalloc(const void* x, int64_t rows, int64_t cols, int64_t ld_x,
                                               nvfp4_scale_mode mode, nvfp4_sf_layout layout,
                                               const float* global_scale_in, uint8_t* codes, uint8_t* scales,
                                               float* global_scale_out, float* block_err, void* stream) {
  if (rows >= 0 && cols >= 0 && nvfp4_quantize_workspace_bytes(rows, cols) > kNoAllocScratchBytes)
    return NVFP4_ERR_WORKSPACE;
  // the arguments first, then the device, so that an unsupported device is reported
  // as such before any lookup on it
  nvfp4_status st = nvfp4::validate_quantize(x, rows, cols, ld_x, mode, layout, global_scale_in, codes, scales,
                                             global_scale_out, block_err);
  if (st != NVFP4_OK) return st;
  st = nvfp4_check_device();
  if (st != NVFP4_OK) return st;
  void* scratch = nullptr;
  if (global_scale_in == nullptr) {
    st = scratch_for_current_device(&scratch);
    if (st != NVFP4_OK) return st;
  }
  // nvfp4_quantize clears the amax word of the scratch block before it uses it.
  return nvfp4_quantize(x, rows, cols, ld_x, mode, layout, global_scale_in, codes, scales, global_scale_out,
                        block_err, scratch, scratch ? kNoAllocScratchBytes : 0, stream);
}
