// quant_block.cuh -- the encoding of one 16-value NVFP4 block, shared by the
// quantizer kernels and the GEMM that quantizes its activation operand itself.
//
// Method (web page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop",
// section 2 "Qué es realmente NVFP4", box "Fundamento matemático: bitfield E2M1 y
// cuantización jerárquica"): q = the E2M1 grid value nearest to x / (s_b s_g), the
// sign of x kept; every operation binary32 round-to-nearest-even, in this order:
//   eff = dec(s_b) s_g, r = 1/eff, y = |x| r, q = E2M1_sat(y);
//   block error e = fma(d_k, d_k, e) over k with d_k = fma(-q_k, eff, x_k).
#pragma once

#include <cstdint>
#include <cuda_bf16.h>
#include <cuda_fp16.h>

#include "ptx.cuh"

namespace nvfp4 {

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

// Two binary32 values in one 64-bit register (element 2i low, 2i+1 high) for the
// packed f32x2 arithmetic of sm_100.
__device__ __forceinline__ uint64_t pack2(float lo, float hi) {
  uint64_t r;
  asm("mov.b64 %0, {%1, %2};" : "=l"(r) : "f"(lo), "f"(hi));
  return r;
}

__device__ __forceinline__ void unpack2(uint64_t v, float& lo, float& hi) {
  asm("mov.b64 {%0, %1}, %2;" : "=f"(lo), "=f"(hi) : "l"(v));
}

// RN32(a * b) on both halves.
__device__ __forceinline__ uint64_t mul2(uint64_t a, uint64_t b) {
  uint64_t d;
  asm("mul.rn.f32x2 %0, %1, %2;" : "=l"(d) : "l"(a), "l"(b));
  return d;
}

// RN32(a * b + c) on both halves (one rounding each).
__device__ __forceinline__ uint64_t fma2(uint64_t a, uint64_t b, uint64_t c) {
  uint64_t d;
  asm("fma.rn.f32x2 %0, %1, %2, %3;" : "=l"(d) : "l"(a), "l"(b), "l"(c));
  return d;
}

// Sign bit of each of the 16 values moved to bit 3 of its code nibble.
__device__ __forceinline__ void sign_codes(const uint64_t (&x2)[8], uint32_t& c0, uint32_t& c1) {
  c0 = c1 = 0u;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t lo = static_cast<uint32_t>(x2[i]) >> 31, hi = static_cast<uint32_t>(x2[i] >> 32) >> 31;
    const uint32_t nib = (lo << 3) | (hi << 7);
    if (i < 4)
      c0 |= nib << (8 * i);
    else
      c1 |= nib << (8 * (i - 4));
  }
}

// Signed 4-bit codes of 16 values (packed pairs x2) for effective scale eff with
// rcp = RN32(1/eff): y = RN32(x * rcp) rounded to the E2M1 grid (RNE, saturating),
// the sign of x kept by the conversion (-0 and small negatives give code 0x8).
__device__ __forceinline__ void encode_codes(const uint64_t (&x2)[8], float eff, float rcp, uint32_t& c0,
                                             uint32_t& c1) {
  if (eff == 0.0f) {  // zero scale: every magnitude is 0, only the signs remain
    sign_codes(x2, c0, c1);
    return;
  }
  const uint64_t r2 = pack2(rcp, rcp);
  float y[16];
#pragma unroll
  for (int i = 0; i < 8; ++i) unpack2(mul2(x2[i], r2), y[2 * i], y[2 * i + 1]);
  if (isinf(rcp)) {
    // 1/eff overflowed: +-0 * inf is NaN; a zero input keeps its own (signed) zero
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float lo, hi;
      unpack2(x2[i], lo, hi);
      if (lo == 0.0f) y[2 * i] = lo;
      if (hi == 0.0f) y[2 * i + 1] = hi;
    }
  }
  c0 = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
  c1 = cvt_e2m1x8(y[8], y[9], y[10], y[11], y[12], y[13], y[14], y[15]);
}

// Squared reconstruction error of the block in element order:
// d_k = RN32(x_k - q_k * eff) (one fma), e = fma(d_k, d_k, e), k = 0..15.
__device__ __forceinline__ float block_sse(const uint64_t (&x2)[8], uint32_t c0, uint32_t c1, float eff) {
  const uint64_t neff2 = pack2(-eff, -eff);
  float e = 0.0f;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const uint32_t h2 = e2m1x2_to_half2(i < 4 ? c0 : c1, i & 3);
    const float q_lo = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xFFFFu)));
    const float q_hi = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 >> 16)));
    float d_lo, d_hi;
    unpack2(fma2(pack2(q_lo, q_hi), neff2, x2[i]), d_lo, d_hi);
    e = __fmaf_rn(d_lo, d_lo, e);
    e = __fmaf_rn(d_hi, d_hi, e);
  }
  return e;
}

__device__ __forceinline__ float global_scale(const float* gs_in, const uint32_t* amax_bits) {
  if (gs_in) return *gs_in;
  const float amax = bf16_bits_to_float(*amax_bits);
  return amax == 0.0f ? 1.0f : __fdiv_rn(amax, 2688.0f);
}

// The 127 finite non-negative E4M3 scale bytes of one tensor, decoded: eff =
// RN32(dec(s) s_g) and RN32(1/eff) (0 for eff = 0).  Every CTA builds them once, so
// each candidate scale costs two shared-memory reads instead of a conversion, a
// product and a correctly rounded reciprocal.
struct ScaleTables {
  float eff[128];
  float rcp[128];
};

}  // namespace nvfp4
