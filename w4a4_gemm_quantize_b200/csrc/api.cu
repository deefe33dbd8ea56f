// api.cu -- the extern "C" entry points declared in include/nvfp4.h: host-side
// validation, workspace layout and kernel launches.  No allocation, no
// synchronisation (except nvfp4_read_device_error).
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>

#include "../../include/nvfp4.h"
#include "internal.h"

namespace nvfp4 {
thread_local int g_last_launches = 0;
}

namespace {

constexpr size_t kQuantizeWorkspace = 256;  // word 0: global amax (BF16 magnitude bits)
constexpr size_t kGemmWorkspace = 256;      // word 0: device status word of bounded waits

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

nvfp4_status check_device_cached() {
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0) return NVFP4_ERR_CUDA;
  static int verdict[64] = {0};  // 0 unknown, 1 ok, 2 unsupported
  if (dev < 64 && verdict[dev] != 0) return verdict[dev] == 1 ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED_DEVICE;
  int major = 0, minor = 0;
  if (cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev) != cudaSuccess ||
      cudaDeviceGetAttribute(&minor, cudaDevAttrComputeCapabilityMinor, dev) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  const bool ok = (major == 10 && minor == 0);
  if (dev < 64) verdict[dev] = ok ? 1 : 2;
  return ok ? NVFP4_OK : NVFP4_ERR_UNSUPPORTED_DEVICE;
}

nvfp4_status from_cuda(cudaError_t e) { return e == cudaSuccess ? NVFP4_OK : NVFP4_ERR_CUDA; }

// Workspace of nvfp4_linear: [0, 256) the GEMM status word, [256, 260) the
// activation's amax word, [260, 264) its global scale (large-M path), then from
// byte 512 the GEMM's counters and partial tiles (small-M kernel or pair kernel),
// and the activation's codes (rounded up to 256 bytes) and swizzled scales.
constexpr size_t kLinearHeader = 512;

size_t linear_codes_bytes(int64_t M, int64_t K) { return (static_cast<size_t>(M) * (K / 2) + 255) / 256 * 256; }


}  // namespace

extern "C" {

const char* nvfp4_status_string(nvfp4_status status) {
  switch (status) {
    case NVFP4_OK: return "ok";
    case NVFP4_ERR_INVALID_ARG: return "invalid argument";
    case NVFP4_ERR_SHAPE: return "unsupported shape";
    case NVFP4_ERR_ALIGNMENT: return "misaligned pointer or leading dimension";
    case NVFP4_ERR_UNSUPPORTED_DEVICE: return "device is not sm_100";
    case NVFP4_ERR_CUDA: return "CUDA error";
    case NVFP4_ERR_TIMEOUT: return "device-side wait timed out";
    case NVFP4_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

nvfp4_status nvfp4_check_device(void) { return check_device_cached(); }

size_t nvfp4_codes_bytes(int64_t rows, int64_t cols) {
  if (rows < 0 || cols < 0) return 0;
  return static_cast<size_t>(rows) * static_cast<size_t>(cols / 2);
}

size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout) {
  if (rows < 0 || cols < 0) return 0;
  const int64_t nblk = cols / 16;
  if (layout == NVFP4_SF_LINEAR) return static_cast<size_t>(rows * nblk);
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (nblk + 3) / 4 * 4;
  return static_cast<size_t>(rp * cp);
}

size_t nvfp4_quantize_workspace_bytes(int64_t, int64_t) { return kQuantizeWorkspace; }

}  // extern "C"

namespace nvfp4 {

nvfp4_status validate_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int mode, int layout,
                               const float* global_scale_in, const uint8_t* codes, const uint8_t* scales,
                               const float* global_scale_out, const float* block_err) {
  if (rows < 0 || cols < 0 || ld_x < cols) return NVFP4_ERR_INVALID_ARG;
  if (mode != NVFP4_SCALE_ABSMAX && mode != NVFP4_SCALE_MSE && mode != NVFP4_SCALE_FOUR_OVER_SIX)
    return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_SWIZZLED && layout != NVFP4_SF_LINEAR) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (rows > 0 && cols > 0 && (x == nullptr || codes == nullptr || scales == nullptr)) return NVFP4_ERR_INVALID_ARG;
  if ((x && !aligned16(x)) || (codes && !aligned16(codes)) || (scales && !aligned16(scales)) || ld_x % 8 != 0)
    return NVFP4_ERR_ALIGNMENT;
  if ((global_scale_in && (reinterpret_cast<uintptr_t>(global_scale_in) & 3u)) ||
      (global_scale_out && (reinterpret_cast<uintptr_t>(global_scale_out) & 3u)) ||
      (block_err && (reinterpret_cast<uintptr_t>(block_err) & 3u)))
    return NVFP4_ERR_ALIGNMENT;
  return NVFP4_OK;
}

}  // namespace nvfp4

extern "C" {

nvfp4_status nvfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld_x, nvfp4_scale_mode mode,
                            nvfp4_sf_layout layout, const float* global_scale_in, uint8_t* codes, uint8_t* scales,
                            float* global_scale_out, float* block_err, void* workspace, size_t workspace_bytes,
                            void* stream) {
  nvfp4::g_last_launches = 0;
  nvfp4_status st = nvfp4::validate_quantize(x, rows, cols, ld_x, mode, layout, global_scale_in, codes, scales,
                                             global_scale_out, block_err);
  if (st != NVFP4_OK) return st;
  if (global_scale_in == nullptr && (workspace == nullptr || workspace_bytes < kQuantizeWorkspace))
    return NVFP4_ERR_WORKSPACE;
  if (workspace && !aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
  st = check_device_cached();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);

  const bool swz = layout == NVFP4_SF_SWIZZLED;
  uint32_t* amax_word = static_cast<uint32_t*>(workspace);
  if (global_scale_in == nullptr && rows > 0 && cols > 0 && nvfp4::quantize_fuses_amax(rows, cols, mode)) {
    // a small tensor: one launch computes the amax and encodes
    st = from_cuda(nvfp4::launch_quantize_fused(static_cast<const uint16_t*>(x), rows, cols, ld_x, swz, codes,
                                                scales, global_scale_out, block_err, s));
    if (st == NVFP4_OK) ++nvfp4::g_last_launches;
    return st;
  }
  if (global_scale_in == nullptr) {
    if (cudaMemsetAsync(amax_word, 0, sizeof(uint32_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
    if (rows > 0 && cols > 0) {
      st = from_cuda(nvfp4::launch_amax(static_cast<const uint16_t*>(x), rows, cols, ld_x, amax_word, s));
      if (st != NVFP4_OK) return st;
      ++nvfp4::g_last_launches;
    }
  }
  if (rows == 0 || cols == 0) {
    // Nothing to encode; still publish s_g (1.0 for an empty tensor, or the given one).
    if (global_scale_out) {
      if (global_scale_in) {
        if (cudaMemcpyAsync(global_scale_out, global_scale_in, sizeof(float), cudaMemcpyDeviceToDevice, s) !=
            cudaSuccess)
          return NVFP4_ERR_CUDA;
      } else {
        static const float one = 1.0f;
        if (cudaMemcpyAsync(global_scale_out, &one, sizeof(float), cudaMemcpyHostToDevice, s) != cudaSuccess)
          return NVFP4_ERR_CUDA;
      }
    }
    return NVFP4_OK;
  }
  // (the quantize kernel also zeroes the padding of a swizzled scale buffer)
  st = from_cuda(nvfp4::launch_quantize(static_cast<const uint16_t*>(x), rows, cols, ld_x, static_cast<int>(mode),
                                        swz, global_scale_in, amax_word, codes, scales, global_scale_out, block_err,
                                        s));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

nvfp4_status nvfp4_dequantize(const uint8_t* codes, const uint8_t* scales, nvfp4_sf_layout layout,
                              const float* global_scale, int64_t rows, int64_t cols, void* out, int64_t ld_out,
                              void* stream) {
  nvfp4::g_last_launches = 0;
  if (rows < 0 || cols < 0 || ld_out < cols) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_SWIZZLED && layout != NVFP4_SF_LINEAR) return NVFP4_ERR_INVALID_ARG;
  if (cols % 16 != 0) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !scales || !global_scale || !out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || ld_out % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(global_scale) & 3u))
    return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  st = from_cuda(nvfp4::launch_dequantize(codes, scales, layout == NVFP4_SF_SWIZZLED, global_scale, rows, cols,
                                          static_cast<uint16_t*>(out), ld_out, static_cast<cudaStream_t>(stream)));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1) return kGemmWorkspace;
  return kGemmWorkspace + nvfp4::gemm_scratch_bytes(M, N, K);
}

nvfp4_status nvfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, const float* a_global_scale, int64_t M,
                        const uint8_t* b_codes, const uint8_t* b_scales, const float* b_global_scale, int64_t N,
                        int64_t K, void* c, int64_t ldc, void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4::g_last_launches = 0;
  if (M < 1 || N < 1 || K < 1 || ldc < N) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return NVFP4_ERR_SHAPE;
  if (!a_codes || !a_scales || !a_global_scale || !b_codes || !b_scales || !b_global_scale || !c)
    return NVFP4_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nvfp4_gemm_workspace_bytes(M, N, K)) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) ||
      !aligned16(c) || !aligned16(workspace) || ldc % 8 != 0 ||
      (reinterpret_cast<uintptr_t>(a_global_scale) & 3u) || (reinterpret_cast<uintptr_t>(b_global_scale) & 3u))
    return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t* status = static_cast<uint32_t*>(workspace);
  const size_t zero = nvfp4::gemm_zero_bytes(M, N, K);
  if (zero > 0 && cudaMemsetAsync(status, 0, zero, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  const cudaError_t e = nvfp4::launch_gemm(a_codes, a_scales, a_global_scale, M, b_codes, b_scales, b_global_scale,
                                           N, K, static_cast<uint16_t*>(c), ldc, status, s);
  if (e == cudaErrorInvalidValue) return NVFP4_ERR_CUDA;
  st = from_cuda(e);
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

namespace {

// Workspace of nvfp4_linear: the 512-byte header (status word, amax word, the
// activation's global scale), the GEMM's counters and partial tiles, then the
// activation's codes and swizzled scales.  The memset clears the header and the
// counters (the `zero` bytes).
struct LinearLayout {
  size_t gemm_scratch, x_codes, x_scales, zero, total;
};

LinearLayout linear_layout(int64_t M, int64_t N, int64_t K) {
  LinearLayout l{};
  l.gemm_scratch = kLinearHeader;
  const size_t scratch = nvfp4::gemm_scratch_bytes(M, N, K);
  l.zero = kLinearHeader + nvfp4::gemm_counter_bytes(M, N, K);
  l.x_codes = (kLinearHeader + scratch + 255) / 256 * 256;
  l.x_scales = l.x_codes + linear_codes_bytes(M, K);
  l.total = l.x_scales + nvfp4_scales_bytes(M, K, NVFP4_SF_SWIZZLED);
  return l;
}

nvfp4_status validate_linear(const void* x, int64_t M, int64_t K, int64_t ld_x, const float* x_global_scale,
                             const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global_scale, int64_t N,
                             void* c, int64_t ldc, void* workspace, size_t workspace_bytes, size_t need) {
  if (M < 1 || N < 1 || K < 1 || ld_x < K || ldc < N) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return NVFP4_ERR_SHAPE;
  if (!x || !w_codes || !w_scales || !w_global_scale || !c) return NVFP4_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < need) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(c) || !aligned16(workspace) ||
      ld_x % 8 != 0 || ldc % 8 != 0 || (reinterpret_cast<uintptr_t>(w_global_scale) & 3u) ||
      (x_global_scale && (reinterpret_cast<uintptr_t>(x_global_scale) & 3u)))
    return NVFP4_ERR_ALIGNMENT;
  return check_device_cached();
}

}  // namespace

size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K) {
  if (M < 1 || N < 1 || K < 1) return kLinearHeader;
  return linear_layout(M, N, K).total;
}

nvfp4_status nvfp4_linear(const void* x, int64_t M, int64_t K, int64_t ld_x, const float* x_global_scale,
                          const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global_scale, int64_t N,
                          void* c, int64_t ldc, void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4::g_last_launches = 0;
  nvfp4_status st = validate_linear(x, M, K, ld_x, x_global_scale, w_codes, w_scales, w_global_scale, N, c, ldc,
                                    workspace, workspace_bytes,
                                    M >= 1 && N >= 1 && K >= 1 ? nvfp4_linear_workspace_bytes(M, N, K) : 0);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const LinearLayout l = linear_layout(M, N, K);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  uint32_t* amax_word = reinterpret_cast<uint32_t*>(ws + 256);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  // one memset ahead of the chain: the status word, the amax word and (small M) the
  // tile counters, so that the kernels after it follow one another with programmatic
  // dependent launch
  if (cudaMemsetAsync(ws, 0, l.zero, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  // a small activation without a given s_g: one launch computes its amax and encodes it
  const bool fused_amax = x_global_scale == nullptr && nvfp4::quantize_fuses_amax(M, K, NVFP4_SCALE_ABSMAX);
  if (x_global_scale == nullptr && !fused_amax) {
    st = from_cuda(nvfp4::launch_amax(xb, M, K, ld_x, amax_word, s));
    if (st != NVFP4_OK) return st;
    ++nvfp4::g_last_launches;
  }
  uint8_t* a_codes = ws + l.x_codes;
  uint8_t* a_scales = ws + l.x_scales;
  float* a_gs = x_global_scale ? nullptr : reinterpret_cast<float*>(ws + 260);
  st = from_cuda(fused_amax ? nvfp4::launch_quantize_fused(xb, M, K, ld_x, true, a_codes, a_scales, a_gs, nullptr, s)
                            : nvfp4::launch_quantize(xb, M, K, ld_x, NVFP4_SCALE_ABSMAX, true, x_global_scale,
                                                     amax_word, a_codes, a_scales, a_gs, nullptr, s));
  if (st != NVFP4_OK) return st;
  ++nvfp4::g_last_launches;
  st = from_cuda(nvfp4::launch_gemm(a_codes, a_scales, x_global_scale ? x_global_scale : a_gs, M, w_codes, w_scales,
                                    w_global_scale, N, K, static_cast<uint16_t*>(c), ldc, status, s,
                                    ws + l.gemm_scratch));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

nvfp4_status nvfp4_linear_fused(const void* x, int64_t M, int64_t K, int64_t ld_x, const float* x_global_scale,
                                const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global_scale,
                                int64_t N, void* c, int64_t ldc, void* workspace, size_t workspace_bytes,
                                void* stream) {
  nvfp4::g_last_launches = 0;
  if (M > 32) return NVFP4_ERR_SHAPE;
  nvfp4_status st = validate_linear(x, M, K, ld_x, x_global_scale, w_codes, w_scales, w_global_scale, N, c, ldc,
                                    workspace, workspace_bytes,
                                    M >= 1 && N >= 1 && K >= 1 ? nvfp4_linear_workspace_bytes(M, N, K) : 0);
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const LinearLayout l = linear_layout(M, N, K);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  uint32_t* amax_word = reinterpret_cast<uint32_t*>(ws + 256);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  if (cudaMemsetAsync(ws, 0, l.zero, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (x_global_scale == nullptr) {
    st = from_cuda(nvfp4::launch_amax(xb, M, K, ld_x, amax_word, s));
    if (st != NVFP4_OK) return st;
    ++nvfp4::g_last_launches;
  }
  st = from_cuda(nvfp4::launch_decode_quantize_x(xb, M, K, ld_x, x_global_scale,
                                                 x_global_scale ? nullptr : amax_word, w_codes, w_scales,
                                                 w_global_scale, N, static_cast<uint16_t*>(c), ldc, status,
                                                 ws + l.gemm_scratch, s));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

namespace {

// Workspace of nvfp4_linear_lora: the 512-byte header of nvfp4_linear, the
// down-projection's counters, the small-M kernel's counters (one zeroed range) and
// partial tiles, then the down-projection's partial tiles, t / alpha hi and lo, and
// the activation's codes and scales.
struct LoraLayout {
  size_t lora_counters, gemm_scratch, lora_partial, thi, tlo, x_codes, x_scales, zero, total;
};

LoraLayout lora_layout(int64_t M, int64_t N, int64_t K, int64_t R) {
  auto up = [](size_t b) { return (b + 255) / 256 * 256; };
  LoraLayout l{};
  size_t off = kLinearHeader;
  l.lora_counters = off;
  off += nvfp4::lora_counter_bytes(M);
  l.gemm_scratch = off;
  if (M <= 32) off += nvfp4::gemm_scratch_bytes(M, N, K);
  l.zero = M <= 32 ? l.gemm_scratch + (nvfp4::gemm_zero_bytes(M, N, K) - 256) : l.gemm_scratch;
  off = up(off);
  l.lora_partial = off;
  off = up(off + nvfp4::lora_partial_bytes(M, K, R));
  l.thi = off;
  off = up(off + static_cast<size_t>(M * R * 2));
  l.tlo = off;
  off = up(off + static_cast<size_t>(M * R * 2));
  l.x_codes = off;
  off += linear_codes_bytes(M, K);
  l.x_scales = off;
  off += nvfp4_scales_bytes(M, K, NVFP4_SF_SWIZZLED);
  l.total = off;
  return l;
}

}  // namespace

size_t nvfp4_linear_lora_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t R) {
  if (M < 1 || N < 1 || K < 1 || R < 1) return kLinearHeader;
  return lora_layout(M, N, K, R).total;
}

nvfp4_status nvfp4_linear_lora(const void* x, int64_t M, int64_t K, int64_t ld_x, const float* x_global_scale,
                               const uint8_t* w_codes, const uint8_t* w_scales, const float* w_global_scale,
                               int64_t N, const void* lora_a, const void* lora_b, int64_t R, void* c, int64_t ldc,
                               void* t_out, void* workspace, size_t workspace_bytes, void* stream) {
  nvfp4::g_last_launches = 0;
  if (M < 1 || N < 1 || K < 1 || ld_x < K || ldc < N || R < 1) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || R % 16 != 0 || R > 64 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX)
    return NVFP4_ERR_SHAPE;
  if (!x || !w_codes || !w_scales || !w_global_scale || !c || !lora_a || !lora_b) return NVFP4_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nvfp4_linear_lora_workspace_bytes(M, N, K, R)) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(x) || !aligned16(w_codes) || !aligned16(w_scales) || !aligned16(c) || !aligned16(workspace) ||
      !aligned16(lora_a) || !aligned16(lora_b) || (t_out && !aligned16(t_out)) || ld_x % 8 != 0 ||
      ldc % 8 != 0 || (reinterpret_cast<uintptr_t>(w_global_scale) & 3u) ||
      (x_global_scale && (reinterpret_cast<uintptr_t>(x_global_scale) & 3u)))
    return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const LoraLayout l = lora_layout(M, N, K, R);
  uint32_t* status = reinterpret_cast<uint32_t*>(ws);
  uint32_t* amax_word = reinterpret_cast<uint32_t*>(ws + 256);
  const uint16_t* xb = static_cast<const uint16_t*>(x);
  uint16_t* thi = reinterpret_cast<uint16_t*>(ws + l.thi);
  uint16_t* tlo = reinterpret_cast<uint16_t*>(ws + l.tlo);
  if (cudaMemsetAsync(ws, 0, l.zero, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (x_global_scale == nullptr) {
    st = from_cuda(nvfp4::launch_amax(xb, M, K, ld_x, amax_word, s));
    if (st != NVFP4_OK) return st;
    ++nvfp4::g_last_launches;
  }
  st = from_cuda(nvfp4::launch_lora_down(xb, M, K, ld_x, x_global_scale, x_global_scale ? nullptr : amax_word,
                                         w_global_scale, static_cast<const uint16_t*>(lora_a), R,
                                         static_cast<uint16_t*>(t_out), thi, tlo,
                                         reinterpret_cast<uint32_t*>(ws + l.lora_counters),
                                         reinterpret_cast<float*>(ws + l.lora_partial), status, s));
  if (st != NVFP4_OK) return st;
  ++nvfp4::g_last_launches;
  const uint16_t* lb = static_cast<const uint16_t*>(lora_b);
  float* a_gs = x_global_scale ? nullptr : reinterpret_cast<float*>(ws + 260);
  st = from_cuda(nvfp4::launch_quantize(xb, M, K, ld_x, NVFP4_SCALE_ABSMAX, true, x_global_scale, amax_word,
                                        ws + l.x_codes, ws + l.x_scales, a_gs, nullptr, s));
  if (st != NVFP4_OK) return st;
  ++nvfp4::g_last_launches;
  const float* gs = x_global_scale ? x_global_scale : a_gs;
  if (M <= 32)
    st = from_cuda(nvfp4::launch_decode_lora(ws + l.x_codes, ws + l.x_scales, gs, M, w_codes, w_scales,
                                             w_global_scale, N, K, lb, thi, tlo, R, static_cast<uint16_t*>(c), ldc,
                                             status, ws + l.gemm_scratch, s));
  else
    st = from_cuda(nvfp4::launch_gemm_lora(ws + l.x_codes, ws + l.x_scales, gs, M, w_codes, w_scales,
                                           w_global_scale, N, K, static_cast<uint16_t*>(c), ldc, status, lb, thi, tlo,
                                           R, s));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

size_t mxfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout) {
  if (rows < 0 || cols < 0) return 0;
  const int64_t nblk = cols / 32;
  if (layout == NVFP4_SF_LINEAR) return static_cast<size_t>(rows * nblk);
  return static_cast<size_t>((rows + 127) / 128 * 128 * ((nblk + 3) / 4 * 4));
}

nvfp4_status mxfp4_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld_x, nvfp4_sf_layout layout,
                            uint8_t* codes, uint8_t* scales, void* stream) {
  nvfp4::g_last_launches = 0;
  if (rows < 0 || cols < 0 || ld_x < cols) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_SWIZZLED && layout != NVFP4_SF_LINEAR) return NVFP4_ERR_INVALID_ARG;
  if (cols % 32 != 0) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!x || !codes || !scales) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(x) || !aligned16(codes) || !aligned16(scales) || ld_x % 8 != 0) return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  st = from_cuda(nvfp4::launch_quantize_mx(static_cast<const uint16_t*>(x), rows, cols, ld_x,
                                           layout == NVFP4_SF_SWIZZLED, codes, scales,
                                           static_cast<cudaStream_t>(stream)));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

nvfp4_status mxfp4_dequantize(const uint8_t* codes, const uint8_t* scales, nvfp4_sf_layout layout, int64_t rows,
                              int64_t cols, void* out, int64_t ld_out, void* stream) {
  nvfp4::g_last_launches = 0;
  if (rows < 0 || cols < 0 || ld_out < cols) return NVFP4_ERR_INVALID_ARG;
  if (layout != NVFP4_SF_SWIZZLED && layout != NVFP4_SF_LINEAR) return NVFP4_ERR_INVALID_ARG;
  if (cols % 32 != 0) return NVFP4_ERR_SHAPE;
  if (rows == 0 || cols == 0) return NVFP4_OK;
  if (!codes || !scales || !out) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(codes) || !aligned16(scales) || !aligned16(out) || ld_out % 8 != 0) return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  st = from_cuda(nvfp4::launch_dequantize_mx(codes, scales, layout == NVFP4_SF_SWIZZLED, rows, cols,
                                             static_cast<uint16_t*>(out), ld_out, static_cast<cudaStream_t>(stream)));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

nvfp4_status mxfp4_gemm(const uint8_t* a_codes, const uint8_t* a_scales, int64_t M, const uint8_t* b_codes,
                        const uint8_t* b_scales, int64_t N, int64_t K, void* c, int64_t ldc, void* workspace,
                        size_t workspace_bytes, void* stream) {
  nvfp4::g_last_launches = 0;
  if (M < 1 || N < 1 || K < 1 || ldc < N) return NVFP4_ERR_INVALID_ARG;
  if (K % 32 != 0 || M > INT32_MAX || N > INT32_MAX || K > INT32_MAX) return NVFP4_ERR_SHAPE;
  if (!a_codes || !a_scales || !b_codes || !b_scales || !c) return NVFP4_ERR_INVALID_ARG;
  if (!workspace || workspace_bytes < nvfp4_gemm_workspace_bytes(M, N, K)) return NVFP4_ERR_WORKSPACE;
  if (!aligned16(a_codes) || !aligned16(a_scales) || !aligned16(b_codes) || !aligned16(b_scales) || !aligned16(c) ||
      !aligned16(workspace) || ldc % 8 != 0)
    return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word (and the small-M kernel's counters) cleared before the kernel
  if (cudaMemsetAsync(workspace, 0, M <= 32 ? nvfp4::gemm_zero_bytes(M, N, K) : 256, s) != cudaSuccess)
    return NVFP4_ERR_CUDA;
  st = from_cuda(nvfp4::launch_gemm_mx(a_codes, a_scales, M, b_codes, b_scales, N, K, static_cast<uint16_t*>(c), ldc,
                                       static_cast<uint32_t*>(workspace), s));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

nvfp4_status nvfp4_read_device_error(const void* workspace, void* stream, uint32_t* word) {
  if (!workspace) return NVFP4_ERR_INVALID_ARG;
  uint32_t w = 0;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemcpyAsync(&w, workspace, sizeof(w), cudaMemcpyDeviceToHost, s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return NVFP4_ERR_CUDA;
  if (word) *word = w;
  return w == 0 ? NVFP4_OK : NVFP4_ERR_TIMEOUT;
}

nvfp4_status nvfp4_selftest_wait_timeout(void* workspace, uint32_t timeout_us, void* stream) {
  nvfp4::g_last_launches = 0;
  if (!workspace || timeout_us == 0 || timeout_us > 2000000u) return NVFP4_ERR_INVALID_ARG;
  if (!aligned16(workspace)) return NVFP4_ERR_ALIGNMENT;
  nvfp4_status st = check_device_cached();
  if (st != NVFP4_OK) return st;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(workspace, 0, sizeof(uint32_t), s) != cudaSuccess) return NVFP4_ERR_CUDA;
  st = from_cuda(nvfp4::launch_selftest_wait(static_cast<uint32_t*>(workspace), uint64_t(timeout_us) * 1000u, s));
  if (st == NVFP4_OK) ++nvfp4::g_last_launches;
  return st;
}

// Kernels the most recent call on this thread enqueued (benchmark bookkeeping).
int nvfp4_last_launch_count(void) { return nvfp4::g_last_launches; }

}  // extern "C"
