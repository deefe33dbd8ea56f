/*
 * nvfp4.h -- C ABI of the NVFP4 quantizer and the W4A4 block-scaled GEMM for
 * NVIDIA B200 (sm_100a).
 *
 * Format (web page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de
 * laptop", section 2 "Qué es realmente NVFP4", box "Fundamento matemático:
 * bitfield E2M1 y cuantización jerárquica"): every value is a 4-bit E2M1 code
 * (1 sign, 2 exponent bits with bias 1, 1 mantissa bit; grid 0, ±0.5, ±1, ±1.5,
 * ±2, ±3, ±4, ±6) times an E4M3 scale shared by 16 consecutive values along the
 * row (the K / input dimension) times one FP32 scale for the whole tensor:
 * W^ = q * s_b * s_g.
 *
 * Conventions for every entry point:
 *  - Pointers marked "device" point to GPU global memory on the current CUDA
 *    device; the caller allocates and owns all of it.  The library never
 *    allocates or frees memory and keeps no pointer after a call returns.
 *  - `stream` is a cudaStream_t passed as void* (NULL = the legacy default
 *    stream).  Calls enqueue work and return without synchronizing, except
 *    nvfp4_read_device_error.
 *  - Arguments are validated on the host before anything is launched; a
 *    failed check returns an error status and enqueues nothing.  Launch
 *    failures return NVFP4_ERR_CUDA.
 *  - Every device pointer must be 16-byte aligned (NVFP4_ERR_ALIGNMENT).
 *  - Only sm_100 devices are accepted (NVFP4_ERR_UNSUPPORTED_DEVICE).
 *  - Matrices are row-major.  BF16 is IEEE binary16-brain (8 exponent bits).
 */
#ifndef NVFP4_B200_H
#define NVFP4_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
    NVFP4_OK = 0,
    NVFP4_ERR_INVALID_ARG = 1,        /* NULL where a pointer is required, negative size, bad enum */
    NVFP4_ERR_SHAPE = 2,              /* a size constraint below is not met */
    NVFP4_ERR_ALIGNMENT = 3,          /* a device pointer or leading dimension is misaligned */
    NVFP4_ERR_UNSUPPORTED_DEVICE = 4, /* current device is not sm_100 */
    NVFP4_ERR_CUDA = 5,               /* a CUDA runtime/driver call failed */
    NVFP4_ERR_TIMEOUT = 6,            /* a bounded device-side wait gave up (see nvfp4_read_device_error) */
    NVFP4_ERR_WORKSPACE = 7           /* workspace missing or smaller than the *_workspace_bytes query */
} nvfp4_status;

/* How a block's E4M3 scale is chosen.  The flags `--qformat nvfp4` and
 * `--qformat nvfp4_mse` of the same page, section 2, box "Derivación del
 * objetivo de optimización MSE vs Absmax":
 *  ABSMAX: s_b = E4M3(amax_b / (6 s_g)) -- the block's largest value lands on 6;
 *  MSE:    the candidates f * amax_b / (6 s_g), f = 0.3, 0.4, ..., 1.0, each
 *          rounded to E4M3; keep the one with the least squared reconstruction
 *          error sum_k (x_k - q_k s_b s_g)^2 (ties keep the larger scale);
 *  FOUR_OVER_SIX: the same page's table of block-scale algorithms (section 2):
 *          each block picks one of two maxima, 4 or 6, by least error -- the
 *          absmax scale, then E4M3(amax_b / (4 s_g)) kept only on a strictly
 *          smaller squared error (ties keep the absmax scale). */
typedef enum { NVFP4_SCALE_ABSMAX = 0, NVFP4_SCALE_MSE = 1, NVFP4_SCALE_FOUR_OVER_SIX = 2 } nvfp4_scale_mode;

/* Layout of the E4M3 block-scale buffer of a rows x cols tensor (nblk = cols/16).
 *  SWIZZLED: the 128 x 4 tiled layout that the tcgen05 block-scaled MMA reads
 *            (rows padded to 128, block columns padded to 4, padding zero):
 *            byte (r, c) at ((r/128)*(Cp/4) + c/4)*512 + (r%32)*16 + ((r%128)/32)*4 + c%4,
 *            Cp = ceil(nblk/4)*4.  Required by nvfp4_gemm.
 *  LINEAR:   (rows, nblk) row-major, the checkpoint layout of the page "NVFP4 en
 *            difusión: la misma cuantización, un motor completamente distinto",
 *            section 2 (weight_scale of shape (out, in // 16), float8_e4m3fn). */
typedef enum { NVFP4_SF_SWIZZLED = 0, NVFP4_SF_LINEAR = 1 } nvfp4_sf_layout;

/* Human-readable name of a status code (static string, never NULL). */
const char *nvfp4_status_string(nvfp4_status status);

/* NVFP4_OK when the current CUDA device is an sm_100 GPU. */
nvfp4_status nvfp4_check_device(void);

/* Bytes of the packed code buffer of a rows x cols tensor: rows * cols / 2.
 * Two codes per byte, element 2j in bits 3:0 and element 2j+1 in bits 7:4
 * (the (out, in // 2) uint8 buffer of "NVFP4 en difusión ...", section 2). */
size_t nvfp4_codes_bytes(int64_t rows, int64_t cols);

/* Bytes of the scale buffer in the given layout (SWIZZLED includes padding). */
size_t nvfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout);

/* Workspace nvfp4_quantize needs (device memory, any content on entry; the
 * call overwrites it).  Constant: 256 bytes. */
size_t nvfp4_quantize_workspace_bytes(int64_t rows, int64_t cols);

/* Quantize a BF16 matrix to NVFP4.
 *   x            device, BF16, rows x cols, row stride ld_x elements (ld_x >= cols, ld_x % 8 == 0).
 *   rows, cols   rows >= 0, cols % 16 == 0 (one scale per 16 values along a row).
 *   mode         NVFP4_SCALE_ABSMAX, NVFP4_SCALE_MSE or NVFP4_SCALE_FOUR_OVER_SIX.
 *   layout       layout of `scales`.
 *   global_scale_in  device float or NULL.  NULL: s_g = amax(|x|) / 2688 (an
 *                all-zero tensor gets 1.0), computed on the device by a first
 *                pass over x -- for an ABSMAX tensor of at most 262144 elements
 *                inside the quantizing launch itself (one cluster of CTAs), the
 *                same value.  Non-NULL: use *global_scale_in (> 0) and skip
 *                that pass.
 *   codes        device, nvfp4_codes_bytes(rows, cols) bytes, dense (row stride cols/2).
 *   scales       device, nvfp4_scales_bytes(rows, cols, layout) bytes; every byte
 *                is written, padding included.
 *   global_scale_out device float or NULL: receives s_g.
 *   block_err    device float[rows * cols/16] or NULL: the squared error
 *                sum_k (x_k - q_k s_b s_g)^2 of each block, row-major (rows, cols/16).
 *   workspace    device, >= nvfp4_quantize_workspace_bytes(); may be NULL only
 *                when global_scale_in is non-NULL.
 * Codes and scales are a deterministic function of x and s_g (bit-exact with
 * the CPU definition shipped with the tests).  Errors: INVALID_ARG, SHAPE,
 * ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE, CUDA. */
nvfp4_status nvfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                            nvfp4_scale_mode mode, nvfp4_sf_layout layout,
                            const float *global_scale_in, uint8_t *codes, uint8_t *scales,
                            float *global_scale_out, float *block_err, void *workspace,
                            size_t workspace_bytes, void *stream);

/* Reconstruct BF16 values W^ = q * s_b * s_g (same page, same box), evaluated as
 * RN32(q * RN32(s_b * s_g)) and rounded to BF16 (round-to-nearest-even).
 *   codes, scales  device, as written by nvfp4_quantize with `layout`.
 *   global_scale   device float (s_g).
 *   out            device BF16, rows x cols, row stride ld_out elements (ld_out % 8 == 0).
 * Errors: INVALID_ARG, SHAPE (cols % 16), ALIGNMENT, UNSUPPORTED_DEVICE, CUDA. */
nvfp4_status nvfp4_dequantize(const uint8_t *codes, const uint8_t *scales, nvfp4_sf_layout layout,
                              const float *global_scale, int64_t rows, int64_t cols, void *out,
                              int64_t ld_out, void *stream);

/* Workspace nvfp4_gemm needs (device memory, any content on entry): 256 bytes
 * for the status word, plus
 *  - when M <= 32, the small-M kernel's per-tile counters and FP32 partial tiles
 *    (the weight stream is split evenly over the SMs, so a 128-row weight tile can
 *    be cut into a few K segments: about N * 128 * segments bytes, a few MB for
 *    8B-class layers);
 *  - when M > 128 and N > 128, the 256 x 256-tile kernel's shared-tile counters and
 *    FP32 partial tiles (when the tile count is not a multiple of the CTA pairs and
 *    K is long, the last round's work is spread over all pairs, a tile split along K
 *    between two of them; 74 slots of 512 KB, about 38.8 MB).
 * nvfp4_gemm clears the status word and the counters itself (one memset on
 * `stream`). */
size_t nvfp4_gemm_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* Block-scaled W4A4 GEMM, C = (A s_a)(B s_b)^T * s_gA * s_gB, FP32 accumulation,
 * BF16 output ("NVFP4 en difusión ...", section 2: out = (A·s_a)(B·s_b)ᵀ with the
 * scales applied per block inside the kernel and out_dtype BF16).
 *   A: M x K activations -- a_codes (M, K/2) bytes, a_scales SWIZZLED for (M, K/16),
 *      a_global_scale device float.
 *   B: N x K weights (out x in, the checkpoint orientation) -- b_codes (N, K/2),
 *      b_scales SWIZZLED for (N, K/16), b_global_scale device float.
 *   C: device BF16, M x N, row stride ldc elements (ldc >= N, ldc % 8 == 0).
 *   M, N >= 1; K >= 32 and K % 32 == 0.
 *   workspace: device, >= nvfp4_gemm_workspace_bytes(M, N, K) bytes; holds the
 *      status word that bounded device-side waits write on a timeout.
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE, CUDA. */
nvfp4_status nvfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, const float *a_global_scale,
                        int64_t M, const uint8_t *b_codes, const uint8_t *b_scales,
                        const float *b_global_scale, int64_t N, int64_t K, void *c, int64_t ldc,
                        void *workspace, size_t workspace_bytes, void *stream);

/* Workspace nvfp4_linear and nvfp4_linear_fused need (device memory, any content
 * on entry): 512 bytes (status word, the activation's amax and global scale), for
 * M <= 32 the small-M kernel's tile counters and partial tiles, then the
 * activation's codes and swizzled scales. */
size_t nvfp4_linear_workspace_bytes(int64_t M, int64_t N, int64_t K);

/* The W4A4 linear layer: the BF16 activation X is quantized on this call (absmax
 * block scales) and multiplied by the pre-quantized weight W, C = Q(X) W^T in BF16
 * -- the page "NVFP4 en difusión: la misma cuantización, un motor completamente
 * distinto", section 2 "NVFP4 sin vLLM: torch._scaled_mm a mano" (the activation
 * is quantized on every forward, 16-block by 16-block, while the weights come
 * quantized from the checkpoint; out = (A s_a)(B s_b)^T in BF16).
 *   x            device, BF16, M x K, row stride ld_x elements (ld_x >= K, ld_x % 8 == 0).
 *   x_global_scale  device float or NULL: the activation's per-tensor FP32 scale.
 *                Given (a calibrated activation scale: "Tu pipeline NVFP4 ...",
 *                section 2, the third of the "three questions" every quantization
 *                scheme answers -- activation scales come from calibration on real
 *                activations), nothing reads the whole of x first.  NULL:
 *                s_g = amax(|x|) / 2688 computed on the device as nvfp4_quantize
 *                does (for M x K <= 262144 inside the quantizing launch).
 *   w_codes, w_scales, w_global_scale  the weight N x K as nvfp4_quantize writes it
 *                (scales SWIZZLED).
 *   c            device BF16, M x N, row stride ldc (ldc >= N, ldc % 8 == 0).
 *   M, N >= 1; K >= 32, K % 32 == 0.
 * The result equals nvfp4_quantize(x, ABSMAX, SWIZZLED, x_global_scale) followed by
 * nvfp4_gemm bit for bit, and that is what runs: one memset of the workspace's
 * counters, the amax pass (x_global_scale NULL), the quantizer writing the
 * activation's codes into the workspace and the GEMM, chained with programmatic
 * dependent launch (the small-M GEMM starts its weight stream before the quantizer
 * has finished).
 * Errors: INVALID_ARG, SHAPE, ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE, CUDA; a
 * device-side timeout is read with nvfp4_read_device_error(workspace, ...). */
nvfp4_status nvfp4_linear(const void *x, int64_t M, int64_t K, int64_t ld_x, const float *x_global_scale,
                          const uint8_t *w_codes, const uint8_t *w_scales, const float *w_global_scale,
                          int64_t N, void *c, int64_t ldc, void *workspace, size_t workspace_bytes,
                          void *stream);

/* nvfp4_linear for M <= 32 with the quantization inside the GEMM kernel, as the same
 * page's section 3 describes for nunchaku's fused kernel: every CTA quantizes the
 * activation K-tiles it consumes (absmax, the quantizer's arithmetic) instead of
 * reading codes a separate pass wrote.  Same arguments, workspace
 * (nvfp4_linear_workspace_bytes) and result bit for bit as nvfp4_linear; M > 32
 * returns SHAPE.  Every CTA of the small-M GEMM needs the whole activation, so each
 * quantizes all of it: on B200 this is slower than nvfp4_linear for the shapes
 * measured (decode M = 1, 8, 32 against a 14336 x 4096 weight). */
nvfp4_status nvfp4_linear_fused(const void *x, int64_t M, int64_t K, int64_t ld_x, const float *x_global_scale,
                                const uint8_t *w_codes, const uint8_t *w_scales, const float *w_global_scale,
                                int64_t N, void *c, int64_t ldc, void *workspace, size_t workspace_bytes,
                                void *stream);

/* Workspace nvfp4_linear_lora needs (device memory, any content on entry). */
size_t nvfp4_linear_lora_workspace_bytes(int64_t M, int64_t N, int64_t K, int64_t R);

/* The W4A4 linear layer with a low-rank (LoRA) branch, y = Q(x) W^T + (x A^T) B^T --
 * the page "NVFP4 en difusión: la misma cuantización, un motor completamente
 * distinto", section 3 ("¿Cómo fine-tuneás algo que ya está en 4 bits?"): a LoRA
 * cannot be merged into NVFP4 weights, so the kernel computes y = W_4bit x + B (A x),
 * the low-rank term in 16 bits, added to the quantized matmul before the result
 * is returned.  Here t = x A^T (M x R) is accumulated in FP32 on the tensor cores
 * and rounded to BF16 (the 16-bit intermediate); t B^T is added to the W4A4 GEMM's
 * FP32 accumulator by tensor-core MMAs, and the sum is rounded to BF16 once.
 *   x, M, K, ld_x, x_global_scale, w_codes, w_scales, w_global_scale, N, c, ldc:
 *                as nvfp4_linear (the activation is quantized on the call, absmax).
 *   lora_a       device BF16, R x K, row-major (row stride K).
 *   lora_b       device BF16, N x R, row-major (row stride R).
 *   R            the rank: 16, 32, 48 or 64.
 *   t_out        device BF16 M x R (row stride R) or NULL: receives t.
 * The order of t's FP32 accumulation is the tensor cores' (t can differ by one BF16
 * ulp from a differently ordered sum).  The GEMM consumes t / (s_gA s_gB) as two
 * BF16 parts (about 2^-16 relative), so alpha = s_gA s_gB must be a normal float.
 * Errors: INVALID_ARG, SHAPE (K % 32, R), ALIGNMENT, WORKSPACE, UNSUPPORTED_DEVICE,
 * CUDA; device-side timeouts as for nvfp4_linear. */
nvfp4_status nvfp4_linear_lora(const void *x, int64_t M, int64_t K, int64_t ld_x, const float *x_global_scale,
                               const uint8_t *w_codes, const uint8_t *w_scales, const float *w_global_scale,
                               int64_t N, const void *lora_a, const void *lora_b, int64_t R, void *c, int64_t ldc,
                               void *t_out, void *workspace, size_t workspace_bytes, void *stream);

/* ---------------------------------------------------------------------------------
 * MXFP4 -- the microscaled 4-bit format that "Cuantización en Producción: AWQ, GPTQ,
 * GGUF K-quants, FP8, MXFP4/NVFP4" (section "MXFP4 / NVFP4: Blackwell agresivo")
 * names next to NVFP4 without giving its block size or scale type.  These calls
 * follow the public OCP Microscaling Formats (MX) v1.0 specification: E2M1 codes in
 * blocks of 32 along K, one E8M0 scale (a power of two, 2^(byte - 127)) per block, no
 * per-tensor scale.  Codes are packed as for NVFP4; the SWIZZLED scale layout is
 * NVFP4's 128 x 4 atom layout with one byte per 32-value block.
 * --------------------------------------------------------------------------------- */

/* Bytes of an MXFP4 scale buffer: rows x cols/32 (LINEAR) or padded to 128 rows and
 * 4 block columns (SWIZZLED). */
size_t mxfp4_scales_bytes(int64_t rows, int64_t cols, nvfp4_sf_layout layout);

/* Quantize a BF16 matrix to MXFP4: per 32-value block, the scale 2^e with
 * e = floor(log2 amax) - 2 clamped to [-127, 127] (byte e + 127; byte 0 for an
 * all-zero block), codes E2M1(x / 2^e) rounded to nearest (ties to even),
 * saturating at 6, the sign kept.
 *   x      device BF16, rows x cols, row stride ld_x (ld_x % 8 == 0); cols % 32 == 0.
 *   codes  device, nvfp4_codes_bytes(rows, cols) bytes.
 *   scales device, mxfp4_scales_bytes(rows, cols, layout) bytes (padding zeroed).
 * Bit-exact with the CPU definition shipped with the tests.  Errors: INVALID_ARG,
 * SHAPE, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA. */
nvfp4_status mxfp4_quantize(const void *x, int64_t rows, int64_t cols, int64_t ld_x, nvfp4_sf_layout layout,
                            uint8_t *codes, uint8_t *scales, void *stream);

/* BF16 reconstruction q * 2^(s - 127) (exact in binary32, rounded to BF16). */
nvfp4_status mxfp4_dequantize(const uint8_t *codes, const uint8_t *scales, nvfp4_sf_layout layout, int64_t rows,
                              int64_t cols, void *out, int64_t ld_out, void *stream);

/* The MXFP4 x MXFP4 GEMM, C = A B^T with the block scales applied inside the kernel
 * (tcgen05 block-scaled MMA with 32-value UE8M0 scales), FP32 accumulation, BF16 out.
 *   A: M x K (codes, SWIZZLED scales), B: N x K (the weight, out x in), C: M x N, ldc.
 *   M, N >= 1; K % 32 == 0.  workspace: nvfp4_gemm_workspace_bytes(M, N, K) bytes.
 * Errors as nvfp4_gemm. */
nvfp4_status mxfp4_gemm(const uint8_t *a_codes, const uint8_t *a_scales, int64_t M, const uint8_t *b_codes,
                        const uint8_t *b_scales, int64_t N, int64_t K, void *c, int64_t ldc, void *workspace,
                        size_t workspace_bytes, void *stream);

/* Synchronize `stream` and read the device status word at the start of a GEMM
 * (or nvfp4_linear, nvfp4_linear_lora) workspace.  Returns NVFP4_OK when no bounded wait gave up, NVFP4_ERR_TIMEOUT
 * otherwise (and stores the raw word, which names the wait, in *word if non-NULL),
 * NVFP4_ERR_CUDA if the copy fails.  Clears nothing: a workspace is reset by the
 * next nvfp4_gemm that uses it. */
nvfp4_status nvfp4_read_device_error(const void *workspace, void *stream, uint32_t *word);

/* Diagnostic for the bounded device-side waits (library plumbing; no
 * counterpart on the pages).  Launches one thread that waits, with the same
 * bounded wait the GEMM kernels use, on a barrier that nothing completes; after
 * timeout_us microseconds (1 .. 2,000,000) it gives up and writes its status
 * word into the first word of `workspace` (device, >= 256 bytes).  A following
 * nvfp4_read_device_error(workspace, ...) must report NVFP4_ERR_TIMEOUT; the
 * context stays usable.  Errors: INVALID_ARG, ALIGNMENT, UNSUPPORTED_DEVICE, CUDA. */
nvfp4_status nvfp4_selftest_wait_timeout(void *workspace, uint32_t timeout_us, void *stream);

/* nvfp4_quantize for callers that cannot allocate device memory: a framework or
 * server plugin that owns no allocator and gets no workspace from its host, or a
 * latency-critical loop where cudaMalloc would synchronize the device.  Same
 * arguments and results as nvfp4_quantize, minus the workspace: it uses a
 * 256-byte scratch block compiled into the library (one per GPU, held until the
 * process exits).  The pages have no counterpart; this is an interface of this
 * library only.
 *  - It allocates nothing (no cudaMalloc/cudaFree, no allocating library call).
 *  - The first call on a device, with that device current, looks up the scratch
 *    block's device address (cudaGetSymbolAddress); make that first call before
 *    any stream capture.  The address is cached per device and CUDA context: after
 *    cudaDeviceReset (which frees the block with the context) the next call looks
 *    it up again in the new context, so make that call outside a capture too.
 *  - Every call shares the one scratch block per device and clears what it needs
 *    zeroed before use; calls whose work overlaps on the GPU (other streams, or
 *    other host threads) race on it -- serialize them.
 *  - Returns NVFP4_ERR_WORKSPACE if the quantizer would need more scratch than
 *    the 256 bytes (nvfp4_quantize_workspace_bytes(rows, cols) > 256); otherwise
 *    the errors of nvfp4_quantize. */
nvfp4_status nvfp4_quantize_noalloc(const void *x, int64_t rows, int64_t cols, int64_t ld_x,
                                    nvfp4_scale_mode mode, nvfp4_sf_layout layout,
                                    const float *global_scale_in, uint8_t *codes, uint8_t *scales,
                                    float *global_scale_out, float *block_err, void *stream);

/* Number of kernels the most recent nvfp4_quantize / nvfp4_dequantize /
 * nvfp4_gemm call on the calling host thread enqueued (library bookkeeping for
 * launch counting; no counterpart on the pages). */
int nvfp4_last_launch_count(void);

#ifdef __cplusplus
}
#endif

#endif /* NVFP4_B200_H */
