// internal.h -- host-side declarations shared by the library's translation units.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

#include "../../include/nvfp4.h"

namespace nvfp4 {

// Host-side checks of nvfp4_quantize's arguments other than the workspace (api.cu),
// made before any CUDA call: NVFP4_OK or the status the entry point returns.
nvfp4_status validate_quantize(const void* x, int64_t rows, int64_t cols, int64_t ld_x, int mode, int layout,
                               const float* global_scale_in, const uint8_t* codes, const uint8_t* scales,
                               const float* global_scale_out, const float* block_err);

// Quantizer launchers (quantize.cu).  All pointers are device pointers that the
// API layer has already validated.
cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax_bits,
                        cudaStream_t stream);
// Absmax quantization of a small tensor (quantize_fuses_amax) in one launch that also
// computes the amax: s_g = amax / 2688 by the same rule as the two-pass path.
bool quantize_fuses_amax(int64_t rows, int64_t cols, int mode);
cudaError_t launch_quantize_fused(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool swizzled,
                                  uint8_t* codes, uint8_t* scales, float* gs_out, float* block_err,
                                  cudaStream_t stream);
cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int mode,
                            bool swizzled, const float* gs_in, const uint32_t* amax_bits, uint8_t* codes,
                            uint8_t* scales, float* gs_out, float* block_err, cudaStream_t stream);
cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, bool swizzled, const float* gs,
                              int64_t rows, int64_t cols, uint16_t* out, int64_t ld_out, cudaStream_t stream);

// MXFP4 quantizer and reconstruction (quantize.cu): blocks of 32, E8M0 scales (the
// swizzled layout has the same 128 x 4 atoms, one byte per 32-value block).
cudaError_t launch_quantize_mx(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool swizzled,
                               uint8_t* codes, uint8_t* scales, cudaStream_t stream);
cudaError_t launch_dequantize_mx(const uint8_t* codes, const uint8_t* scales, bool swizzled, int64_t rows,
                                 int64_t cols, uint16_t* out, int64_t ld_out, cudaStream_t stream);

// Bounded-wait self test (quantize.cu).
cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t stream);

// GEMM launcher (gemm_sm100.cu).  Returns cudaErrorInvalidValue when a tensor
// map cannot be encoded.  scratch (M <= 32 only): the small-M kernel's tile counters
// (zeroed before the launch) and partial tiles; null means status + 256 bytes.
cudaError_t launch_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                        uint16_t* c, int64_t ldc, uint32_t* status, cudaStream_t stream, uint8_t* scratch = nullptr);

// The small-M GEMM (M <= 32) that quantizes its BF16 activation x (M x K, row stride
// ld_x) itself, absmax block scales under the global scale *x_gs_in, or, when x_gs_in
// is null, RN32(amax / 2688) from the amax word x_amax written by launch_amax.
// scratch: the decode kernel's counters (zeroed) and partial tiles.
cudaError_t launch_decode_quantize_x(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* x_gs_in,
                                     const uint32_t* x_amax, const uint8_t* b_codes, const uint8_t* b_sf,
                                     const float* b_gs, int64_t N, uint16_t* c, int64_t ldc, uint32_t* status,
                                     uint8_t* scratch, cudaStream_t stream);

// The small-M GEMM (M <= 32) on quantized operands with the low-rank branch added to
// the accumulator: lora_b (N x R BF16) and t / alpha as BF16 hi and lo parts (M x R
// each, from launch_lora_down), R <= 64; scratch as launch_gemm's.
cudaError_t launch_decode_lora(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                               const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                               const uint16_t* lora_b, const uint16_t* thi, const uint16_t* tlo, int64_t R,
                               uint16_t* c, int64_t ldc, uint32_t* status, uint8_t* scratch, cudaStream_t stream);

// The MXFP4 GEMM C = A B^T (E8M0 block-32 scales, swizzled, no per-tensor scales):
// the small-M kernel for M <= 32 (workspace as nvfp4_gemm's), the CTA-pair kernel above.
cudaError_t launch_gemm_mx(const uint8_t* a_codes, const uint8_t* a_sf, int64_t M, const uint8_t* b_codes,
                           const uint8_t* b_sf, int64_t N, int64_t K, uint16_t* c, int64_t ldc, uint32_t* status,
                           cudaStream_t stream);

// The CTA-pair GEMM (any M, N; meant for M > 32) with the low-rank branch: lora_b
// (N x R BF16) and t / alpha as BF16 hi and lo parts (M x R each), R <= 64.
cudaError_t launch_gemm_lora(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                             const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                             uint16_t* c, int64_t ldc, uint32_t* status, const uint16_t* lora_b, const uint16_t* thi,
                             const uint16_t* tlo, int64_t R, cudaStream_t stream);

// The low-rank down-projection t = BF16(x A^T) (x M x K, A R x K BF16, R % 16 == 0,
// R <= 64), with t / alpha as BF16 hi and lo parts (alpha = s_gA s_gB, s_gA from
// x_gs_in or the amax word x_amax); t_out may be null.  counters: lora_counter_bytes(M)
// zeroed bytes (left zeroed); partial: lora_partial_bytes(M, K, R) bytes.
cudaError_t launch_lora_down(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* x_gs_in,
                             const uint32_t* x_amax, const float* w_gs, const uint16_t* lora_a, int64_t R,
                             uint16_t* t_out, uint16_t* thi, uint16_t* tlo, uint32_t* counters, float* partial,
                             uint32_t* status, cudaStream_t stream);
size_t lora_partial_bytes(int64_t M, int64_t K, int64_t R);
size_t lora_counter_bytes(int64_t M);

// Bytes the GEMM needs in its workspace after the 256-byte status block: the
// small-M kernel's tile counters and split partial tiles, or the pair kernel's
// shared-tile counters and partial tiles; 0 when none.
size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K);

// Bytes at the start of the workspace that must be zero when the GEMM launches
// (cleared with one memset before the kernel): the status word, and the counters at
// the start of the scratch after the 256-byte status block.
size_t gemm_zero_bytes(int64_t M, int64_t N, int64_t K);

// The counter bytes at the start of the GEMM scratch (0 when none).
size_t gemm_counter_bytes(int64_t M, int64_t N, int64_t K);

// Number of kernel launches the last call of each entry point enqueued (for
// the benchmark's launch count); host-side bookkeeping only.
extern thread_local int g_last_launches;

}  // namespace nvfp4
