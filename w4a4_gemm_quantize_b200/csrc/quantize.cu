// quantize.cu -- NVFP4 block quantization and reconstruction kernels for sm_100a.
//
// Method (web page "Tu pipeline NVFP4: meter 62 GB de modelo en 24 GB de laptop",
// section 2 "Qué es realmente NVFP4"):
//  * box "Fundamento matemático: bitfield E2M1 y cuantización jerárquica": each
//    value becomes q = argmin over the E2M1 grid of |x / (s_b s_g) - q|, with s_b an
//    E4M3 scale per 16 consecutive values and s_g one FP32 scale per tensor;
//    reconstruction W^ = q s_b s_g;
//  * box "Derivación del objetivo de optimización MSE vs Absmax": absmax scale
//    s = max|x| / 6, or the MSE scale that minimises sum_k (x_k - s s_g Q(x_k/(s s_g)))^2
//    over candidates below the absmax scale (the search of section 8 "Para
//    practicar" of "NVFP4 en difusión: la misma cuantización, un motor
//    completamente distinto", with 8 factors 0.3, 0.4, ..., 1.0);
//  * the section's table of block-scale algorithms, row "Four-over-six": each
//    block picks one of two maxima, 4 or 6, by least error -- the absmax scale,
//    then s_b = E4M3(amax_b / (4 s_g)) kept only on a strictly smaller error.
//
// Arithmetic, in this order and all binary32 round-to-nearest-even:
//   s_g = amax_t / 2688 (1 for an all-zero tensor); d6 = 6 s_g; v_b = amax_b / d6;
//   per candidate f: u = f v_b, s_b = E4M3_sat(u), eff = dec(s_b) s_g, r = 1/eff,
//   y_k = |x_k| r, mag_k = E2M1_sat(y_k) (RNE), code_k = sign(x_k) | mag_k;
//   block error e = fma(d_k, d_k, e) over k with d_k = fma(-|q_k|, eff, |x_k|);
//   candidates walked from f = 1 down, kept on a strict improvement.
//
// Kernels: the absmax pass is HBM-bound, the MSE search issue-bound.  One thread
// per 16-value block (2 x 128-bit loads, packed 8-byte code stores), one warp per
// 32 consecutive blocks of a row, per-CTA tables of the decoded scales and their
// reciprocals, hardware cvt for E4M3 and E2M1 rounding, swizzled scale bytes
// stored four at a time; the encode kernel also zeroes the swizzled padding.  The
// MSE search queues the blocks whose walk goes past f = 0.9 per warp and resumes
// them 32 at a time; a small absmax tensor computes its amax inside the encode
// launch (one cluster).  Every kernel is launched with programmatic dependent launch
// and waits for its predecessor before reading its inputs.
#include <cuda_runtime.h>

#include "internal.h"
#include "ptx.cuh"
#include "quant_block.cuh"

namespace nvfp4 {

namespace {

constexpr int kThreads = 256;
// CTAs (one cluster) of the quantizer that computes the amax itself; used for tensors of
// at most kFusedMaxElems elements, where the separate amax pass is mostly launch cost.
constexpr int kFusedCtas = 8;
constexpr int64_t kFusedMaxElems = 256 * 1024;

// Streaming 16-byte load: read-only path, no L1 allocation, 256-byte L2 fetches.
__device__ __forceinline__ uint4 ld_nc_v4(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::256B.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// max over the eight BF16 magnitudes of a 16-byte vector, as 16-bit patterns in both halves
__device__ __forceinline__ uint32_t vmax_mag(uint32_t m, uint4 v) {
  m = __vmaxu2(m, v.x & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.y & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.z & 0x7FFF7FFFu);
  m = __vmaxu2(m, v.w & 0x7FFF7FFFu);
  return m;
}

// Global amax: the largest |x| as the 15-bit magnitude pattern of a BF16 value
// (for non-negative BF16 values the integer order of the bit patterns is the
// numeric order).  One atomicMax per CTA into a zero-initialised word.
__global__ void __launch_bounds__(kThreads) amax_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                        int64_t cols, int64_t ld,
                                                        uint32_t* __restrict__ amax_bits) {
  grid_dependents_launch();  // the quantizer behind this pass may set up meanwhile
  uint32_t m = 0;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (ld == cols) {
    const int64_t nvec = rows * cols / 8;
    const uint4* v = reinterpret_cast<const uint4*>(x);
    int64_t i = tid;
    for (; i + 3 * stride < nvec; i += 4 * stride) {
      uint4 a = ld_nc_v4(v + i), b = ld_nc_v4(v + i + stride), c = ld_nc_v4(v + i + 2 * stride),
            d = ld_nc_v4(v + i + 3 * stride);
      m = vmax_mag(m, a);
      m = vmax_mag(m, b);
      m = vmax_mag(m, c);
      m = vmax_mag(m, d);
    }
    for (; i < nvec; i += stride) m = vmax_mag(m, ld_nc_v4(v + i));
  } else {
    const int64_t vpr = cols / 8;
    const int64_t nvec = rows * vpr;
    for (int64_t i = tid; i < nvec; i += stride) {
      const int64_t r = i / vpr, c = i - r * vpr;
      m = vmax_mag(m, ld_nc_v4(x + r * ld + c * 8));
    }
  }
  m = max(m & 0xFFFFu, m >> 16);
  m = __reduce_max_sync(0xFFFFFFFFu, m);
  __shared__ uint32_t warp_max[kThreads / 32];
  if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
  __syncthreads();
  if (threadIdx.x < 32) {
    m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
    m = __reduce_max_sync(0xFFFFFFFFu, m);
    if (threadIdx.x == 0 && m != 0) atomicMax(amax_bits, m);
  }
}

__device__ __forceinline__ int64_t swizzled_offset(int64_t r, int64_t c, int64_t atoms_per_group) {
  return ((r >> 7) * atoms_per_group + (c >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 + (c & 3);
}

// Zero the padding of a swizzled scale buffer (rows [rows, Rp) and block columns
// [nblk, Cp) of rows [0, rows)), grid-strided over all threads of the launch.
__device__ __forceinline__ void zero_scale_padding(uint8_t* __restrict__ scales, int64_t rows, int64_t nblk) {
  const int64_t rp = (rows + 127) / 128 * 128;
  const int64_t cp = (nblk + 3) / 4 * 4;
  const int64_t n_row_pad = (rp - rows) * cp;
  const int64_t n_col_pad = rows * (cp - nblk);
  if (n_row_pad + n_col_pad == 0) return;
  const int64_t atoms_per_group = cp / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n_row_pad + n_col_pad;
       i += stride) {
    int64_t r, c;
    if (i < n_row_pad) {
      r = rows + i / cp;
      c = i % cp;
    } else {
      const int64_t j = i - n_row_pad;
      const int64_t wdt = cp - nblk;
      r = j / wdt;
      c = nblk + j % wdt;
    }
    scales[swizzled_offset(r, c, atoms_per_group)] = 0;
  }
}

// Load one 16-value block: its binary32 pairs, its maximum magnitude and
// v_b = amax_b / (6 s_g).
__device__ __forceinline__ void load_x2(uint4 lo, uint4 hi, float d6, uint64_t (&x2)[8], float& amax_b,
                                        float& vb) {
  const uint32_t wd[8] = {lo.x, lo.y, lo.z, lo.w, hi.x, hi.y, hi.z, hi.w};
  uint32_t mb = 0;
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    x2[i] = pack2(__uint_as_float(wd[i] << 16), __uint_as_float(wd[i] & 0xFFFF0000u));  // exact widening
    mb = __vmaxu2(mb, wd[i] & 0x7FFF7FFFu);
  }
  amax_b = bf16_bits_to_float(max(mb & 0xFFFFu, mb >> 16));
  vb = __fdiv_rn(amax_b, d6);
}

// Clip bound of the MSE walk: if the block maximum lands above the 4|6 midpoint it
// is coded as 6, and its term alone makes e >= RN(d*d) with d = fma(-6, eff, amax_b):
// each fma of the error sum adds a non-negative term to a non-negative sum, and
// rounding is monotone.  Such a candidate cannot strictly improve when RN(d*d) >=
// best_e.  When d >= 0 (the maximum is clipped) later candidates, with smaller eff,
// have a larger d and cannot either, so the walk stops.
enum Verdict { kEvaluate, kSkip, kStop };
__device__ __forceinline__ Verdict clip_verdict(float amax_b, float eff, float rcp, float best_e) {
  if (eff != 0.0f && __fmul_rn(amax_b, rcp) > 5.0f) {
    const float d = __fmaf_rn(-6.0f, eff, amax_b);
    if (__fmul_rn(d, d) >= best_e) return d >= 0.0f ? kStop : kSkip;
  }
  return kEvaluate;
}

// Evaluate scale s in full and keep it on a strict improvement.
__device__ __forceinline__ void mse_try(const uint64_t (&x2)[8], uint32_t s, float eff, float rcp, uint32_t& best_s,
                                        float& best_e, uint32_t& best_c0, uint32_t& best_c1) {
  uint32_t c0w, c1w;
  encode_codes(x2, eff, rcp, c0w, c1w);
  const float e = block_sse(x2, c0w, c1w, eff);
  if (e < best_e) {
    best_e = e;
    best_s = s;
    best_c0 = c0w;
    best_c1 = c1w;
  }
}

// The MSE walk over the candidates f = 0.9, 0.8, ..., 0.3 (index i = 0..6) from
// index i0, with prev_s the scale of the candidate before it.
__device__ __forceinline__ void mse_walk(const uint64_t (&x2)[8], float amax_b, float vb, int i0, uint32_t prev_s,
                                         const ScaleTables& tab, uint32_t& best_s, float& best_e, uint32_t& best_c0,
                                         uint32_t& best_c1) {
#pragma unroll 1
  for (int i = i0; i < 7; ++i) {
    // the factor of candidate i, selected in registers (an indexed array would live in
    // local memory)
    const float fi = i == 0 ? 0.9f : i == 1 ? 0.8f : i == 2 ? 0.7f : i == 3 ? 0.6f : i == 4 ? 0.5f : i == 5 ? 0.4f : 0.3f;
    const uint32_t s = cvt_e4m3_satfinite(__fmul_rn(fi, vb));
    if (s == prev_s) continue;  // same scale, same error: never a strict improvement
    prev_s = s;
    const float eff = tab.eff[s], rcp = tab.rcp[s];
    const Verdict v = clip_verdict(amax_b, eff, rcp, best_e);
    if (v == kStop) return;
    if (v == kEvaluate) mse_try(x2, s, eff, rcp, best_s, best_e, best_c0, best_c1);
  }
}

// One warp handles 32 consecutive blocks of one row (lane = block); warps walk a
// fixed column chunk down the rows, so block coordinates and output offsets need
// no division.
// FUSED: the tensor's amax is computed by the launch itself -- one cluster of
// kFusedCtas CTAs, each CTA's maximum in shared memory, combined over the cluster
// through distributed shared memory -- so a small tensor needs neither the amax pass
// nor its cleared word (s_g from the same rule and arithmetic as the two-pass path).
template <int MODE, bool SWZ, bool FUSED = false>
__global__ void __launch_bounds__(kThreads, 4) quantize_kernel(
    const uint16_t* __restrict__ x, int64_t rows, int64_t cols, int64_t ld, const float* __restrict__ gs_in,
    const uint32_t* __restrict__ amax_bits, uint8_t* __restrict__ codes, uint8_t* __restrict__ scales,
    float* __restrict__ gs_out, float* __restrict__ block_err) {
  __shared__ ScaleTables tab;
  // MSE: per-warp ring of blocks whose walk goes on past f = 0.9 (about one block in
  // seven, but nearly every warp has one).  They are resumed 32 at a time, one per
  // lane, so the longer walks no longer hold the other 31 lanes of a warp.  An entry
  // is three 16-byte words: {row r, block column cb, the scales (current best, last
  // candidate) with bits 32..39 of cb and of r, error}, then the block's 16 BF16 values
  // (a tensor in device memory has fewer than 2^40 rows and blocks per row).  A resumed block that
  // finds no better scale keeps the outputs already stored, so its codes are not kept.
  constexpr int kRing = MODE == 1 ? 64 : 1;
  __shared__ uint4 ring[3][kThreads / 32][kRing];
  grid_dependents_launch();  // the GEMM behind this pass may set up and start its weight stream
  grid_dependency_wait();    // launched behind the amax pass or the producer of x (programmatic launch)
  const int64_t nblk = cols / 16;
  const int64_t atoms_per_group = (nblk + 3) / 4;
  float sg;
  if constexpr (FUSED) {
    __shared__ uint32_t cta_max;
    uint32_t m = 0;
    const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
    const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
    const int64_t vpr = cols / 8, nvec = rows * vpr;
    if (ld == cols) {
      for (int64_t i = tid; i < nvec; i += stride) m = vmax_mag(m, ld_nc_v4(x + i * 8));
    } else {
      for (int64_t i = tid; i < nvec; i += stride) {
        const int64_t r = i / vpr, c = i - r * vpr;
        m = vmax_mag(m, ld_nc_v4(x + r * ld + c * 8));
      }
    }
    m = __reduce_max_sync(0xFFFFFFFFu, max(m & 0xFFFFu, m >> 16));
    __shared__ uint32_t warp_max[kThreads / 32];
    if ((threadIdx.x & 31) == 0) warp_max[threadIdx.x >> 5] = m;
    __syncthreads();
    if (threadIdx.x < 32) {
      m = threadIdx.x < kThreads / 32 ? warp_max[threadIdx.x] : 0u;
      m = __reduce_max_sync(0xFFFFFFFFu, m);
      if (threadIdx.x == 0) cta_max = m;
    }
    cluster_sync();  // every CTA's maximum is in its shared memory
    uint32_t g = 0;
    for (uint32_t r = 0; r < static_cast<uint32_t>(kFusedCtas); ++r)
      g = max(g, ld_shared_cluster_u32(mapa_shared(smem_u32(&cta_max), r)));
    cluster_sync();  // no CTA leaves while another still reads its word
    sg = global_scale(nullptr, &g);
  } else {
    sg = global_scale(gs_in, amax_bits);
  }
  if (gs_out && blockIdx.x == 0 && threadIdx.x == 0) *gs_out = sg;
  const float d6 = __fmul_rn(6.0f, sg);
  if (threadIdx.x < 128) {
    const float eff = __fmul_rn(e4m3_to_float(threadIdx.x), sg);
    tab.eff[threadIdx.x] = eff;
    tab.rcp[threadIdx.x] = eff == 0.0f ? 0.0f : __frcp_rn(eff);
  }
  __syncthreads();

  const int64_t chunks = (nblk + 31) / 32;  // warp tasks per row
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  int64_t r0, r_step, c0, c_step;
  if (nwarps >= chunks) {
    r_step = nwarps / chunks;
    r0 = w / chunks;
    c0 = w % chunks;
    c_step = chunks;
    if (r0 >= r_step) r0 = rows;  // the few warps past the last whole set of chunks encode nothing
  } else {
    r0 = 0;
    r_step = 1;
    c0 = w;
    c_step = nwarps;
  }
  const int lane = threadIdx.x & 31;
  const int wid = threadIdx.x >> 5;
  uint32_t ring_head = 0, ring_tail = 0;  // warp-uniform
  // resume the walks of the n oldest queued blocks (lane j takes the j-th) and rewrite
  // the outputs of those whose best candidate changed
  auto resume = [&](uint32_t n) {
    __syncwarp();
    const uint32_t slot = (ring_head + lane) & (kRing - 1);
    const uint4 f = ring[0][wid][slot], lo = ring[1][wid][slot], hi = ring[2][wid][slot];
    __syncwarp();  // the slots may be refilled once every lane has read its entry
    ring_head += n;
    if (static_cast<uint32_t>(lane) >= n) return;
    const int64_t r = static_cast<int64_t>((static_cast<uint64_t>(f.z >> 24) << 32) | f.x);
    const int64_t cb = static_cast<int64_t>((static_cast<uint64_t>((f.z >> 16) & 0xFFu) << 32) | f.y);
    uint64_t x2[8];
    float amax_b, vb;
    load_x2(lo, hi, d6, x2, amax_b, vb);
    uint32_t best_s = f.z & 0xFFu;
    const uint32_t queued_s = best_s;
    float best_e = __uint_as_float(f.w);
    uint32_t best_c0 = 0, best_c1 = 0;
    mse_walk(x2, amax_b, vb, 1, (f.z >> 8) & 0xFFu, tab, best_s, best_e, best_c0, best_c1);
    if (best_s == queued_s) return;  // a strict improvement always changes the scale
    *reinterpret_cast<uint2*>(codes + r * (cols / 2) + cb * 8) = make_uint2(best_c0, best_c1);
    scales[SWZ ? swizzled_offset(r, cb, atoms_per_group) : r * nblk + cb] = static_cast<uint8_t>(best_s);
    if (block_err) block_err[r * nblk + cb] = best_e;
  };
  // absmax and four-over-six: the warp's next 32 blocks are requested before these are
  // encoded, so two blocks' loads per lane are in flight (the MSE search is issue-bound
  // and keeps its registers)
  constexpr bool kPrefetch = MODE != 1;
  auto load_block = [&](int64_t r, int64_t c, uint4& lo, uint4& hi) {
    const int64_t cb = c * 32 + lane;
    if (r < rows && cb < nblk) {
      const uint16_t* p = x + r * ld + cb * 16;
      lo = ld_nc_v4(p);
      hi = ld_nc_v4(p + 8);
    }
  };
  uint4 next_lo = make_uint4(0u, 0u, 0u, 0u), next_hi = next_lo;
  if (c0 >= chunks) r0 = rows;
  if (kPrefetch) load_block(r0, c0, next_lo, next_hi);
  // (r, c) walks the warp's tasks in order: c = c0, c0 + c_step, ... below `chunks` for
  // r = r0, r0 + r_step, ...
  for (int64_t r = r0, c = c0; r < rows;) {
    int64_t rn = r, cn = c + c_step;
    if (cn >= chunks) {
      cn = c0;
      rn = r + r_step;
    }
    uint4 lo = next_lo, hi = next_hi;
    if (kPrefetch) load_block(rn, cn, next_lo, next_hi);
    const uint16_t* xrow = x + r * ld;
    uint8_t* crow = codes + r * (cols / 2);
    const int64_t sf_row = SWZ ? (r >> 7) * atoms_per_group * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4 : r * nblk;
    {
      const int64_t cb = c * 32 + lane;
      const bool active = cb < nblk;
      uint32_t best_s = 0;
      uint32_t n_queued = 0;  // MSE: blocks of this task queued (valid in lane 0)
      const uint32_t active_mask = MODE == 1 ? __ballot_sync(0xFFFFFFFFu, active) : 0u;
      if (active) {
        if (!kPrefetch) {
          lo = ld_nc_v4(xrow + cb * 16);
          hi = ld_nc_v4(xrow + cb * 16 + 8);
        }
        uint64_t x2[8];  // the block as signed binary32 pairs
        float amax_b, vb;
        load_x2(lo, hi, d6, x2, amax_b, vb);

        // candidate f = 1: the absmax scale
        best_s = cvt_e4m3_satfinite(vb);
        const float best_eff = tab.eff[best_s];
        uint32_t best_c0, best_c1;
        encode_codes(x2, best_eff, tab.rcp[best_s], best_c0, best_c1);
        float best_e = 0.0f;
        if (MODE != 0 || block_err) best_e = block_sse(x2, best_c0, best_c1, best_eff);

        if (MODE == 1) {
          // f = 0.9 here, and the clip test of f = 0.8; a block whose walk goes on is
          // queued with its state and resumes at f = 0.8
          uint32_t prev_s = best_s;
          bool more = true;
          uint32_t s = cvt_e4m3_satfinite(__fmul_rn(0.9f, vb));
          if (s != prev_s) {
            prev_s = s;
            const float eff = tab.eff[s], rcp = tab.rcp[s];
            const Verdict v = clip_verdict(amax_b, eff, rcp, best_e);
            more = v != kStop;
            if (v == kEvaluate) mse_try(x2, s, eff, rcp, best_s, best_e, best_c0, best_c1);
          }
          if (more) {
            s = cvt_e4m3_satfinite(__fmul_rn(0.8f, vb));
            if (s != prev_s) more = clip_verdict(amax_b, tab.eff[s], tab.rcp[s], best_e) != kStop;
          }
          // the outputs below hold the best so far; a queued block's are rewritten when
          // it is resumed (active lanes are a prefix of the warp, lane 0 among them)
          const uint32_t queued = __ballot_sync(active_mask, more);
          if (more) {
            const uint32_t slot = (ring_tail + __popc(queued & ((1u << lane) - 1u))) & (kRing - 1);
            const uint32_t hi_bits = ((static_cast<uint32_t>(static_cast<uint64_t>(cb) >> 32) & 0xFFu) << 16) |
                                     (static_cast<uint32_t>(static_cast<uint64_t>(r) >> 32) << 24);
            ring[0][wid][slot] = make_uint4(static_cast<uint32_t>(r), static_cast<uint32_t>(cb),
                                            best_s | (prev_s << 8) | hi_bits, __float_as_uint(best_e));
            // each BF16 pair back from its exact binary32 widening: the high halves
            uint32_t wd[8];
#pragma unroll
            for (int j = 0; j < 8; ++j)
              wd[j] = __byte_perm(static_cast<uint32_t>(x2[j]), static_cast<uint32_t>(x2[j] >> 32), 0x7632);
            ring[1][wid][slot] = make_uint4(wd[0], wd[1], wd[2], wd[3]);
            ring[2][wid][slot] = make_uint4(wd[4], wd[5], wd[6], wd[7]);
          }
          n_queued = __popc(queued);
        }
        if (MODE == 2) {
          // four-over-six: the block maximum mapped to 4 instead of 6, kept only on a
          // strictly smaller error (4 s_g is exact: a power-of-two multiple)
          const uint32_t s = cvt_e4m3_satfinite(__fdiv_rn(amax_b, __fmul_rn(4.0f, sg)));
          if (s != best_s) {
            uint32_t c0w, c1w;
            encode_codes(x2, tab.eff[s], tab.rcp[s], c0w, c1w);
            const float e = block_sse(x2, c0w, c1w, tab.eff[s]);
            if (e < best_e) {
              best_e = e;
              best_s = s;
              best_c0 = c0w;
              best_c1 = c1w;
            }
          }
        }
        *reinterpret_cast<uint2*>(crow + cb * 8) = make_uint2(best_c0, best_c1);
        if (!SWZ) scales[sf_row + cb] = static_cast<uint8_t>(best_s);
        if (block_err) block_err[r * nblk + cb] = best_e;
      }
      if (SWZ) {
        // lanes 4j..4j+3 hold four consecutive blocks of the row: one 32-bit store of
        // their scale bytes (a lane past the row end contributes the padding's 0)
        const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, best_s, 1);
        const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, best_s, 2);
        const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, best_s, 3);
        if (active && (lane & 3) == 0)
          *reinterpret_cast<uint32_t*>(scales + sf_row + (cb >> 2) * 512) =
              best_s | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
      if (MODE == 1) {
        ring_tail += __shfl_sync(0xFFFFFFFFu, n_queued, 0);
        if (ring_tail - ring_head >= 32) resume(32);  // at most 63 queued before this
      }
    }
    r = rn;
    c = cn;
  }
  if (MODE == 1 && ring_tail != ring_head) resume(ring_tail - ring_head);
  if (SWZ) zero_scale_padding(scales, rows, nblk);
}

template <bool SWZ>
__global__ void __launch_bounds__(kThreads) dequantize_kernel(const uint8_t* __restrict__ codes,
                                                              const uint8_t* __restrict__ scales,
                                                              const float* __restrict__ gs, int64_t rows,
                                                              int64_t cols, uint16_t* __restrict__ out,
                                                              int64_t ld_out) {
  grid_dependency_wait();  // launched behind the kernel that wrote the codes (programmatic launch)
  const int64_t nblk = cols / 16;
  const int64_t total = rows * nblk;
  const int64_t atoms_per_group = (nblk + 3) / 4;
  const float sg = *gs;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < total; b += stride) {
    const int64_t r = b / nblk, cb = b - r * nblk;
    const uint2 cw = *reinterpret_cast<const uint2*>(codes + r * (cols / 2) + cb * 8);
    const uint32_t s = SWZ ? scales[swizzled_offset(r, cb, atoms_per_group)] : scales[b];
    const float eff = __fmul_rn(e4m3_to_float(s), sg);
    uint32_t o[8];
#pragma unroll
    for (int w = 0; w < 2; ++w) {
      const uint32_t word = w ? cw.y : cw.x;
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t h2 = e2m1x2_to_half2(word, k);
        const float q_lo = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xFFFFu)));
        const float q_hi = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 >> 16)));
        const __nv_bfloat16 lo = __float2bfloat16_rn(__fmul_rn(q_lo, eff));
        const __nv_bfloat16 hi = __float2bfloat16_rn(__fmul_rn(q_hi, eff));
        o[4 * w + k] = static_cast<uint32_t>(__bfloat16_as_ushort(lo)) |
                       (static_cast<uint32_t>(__bfloat16_as_ushort(hi)) << 16);
      }
    }
    uint4* dst = reinterpret_cast<uint4*>(out + r * ld_out + cb * 16);
    dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
    dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
  }
}

// ---------------------------------------------------------------------------------------------
// MXFP4: blocks of 32 values along the row, an E8M0 (power-of-two) scale per block, no
// per-tensor scale -- the OCP Microscaling Formats (MX) v1.0 rule, the outside reading
// for the format that "Cuantización en Producción: AWQ, GPTQ, GGUF K-quants, FP8,
// MXFP4/NVFP4" names without its block size or scale type: shared = floor(log2 amax)
// - 2 clamped to [-127, 127], scale byte shared + 127 (0 for an all-zero block), codes
// = E2M1_sat(x * 2^-shared) (RNE, the sign kept).
// ---------------------------------------------------------------------------------------------

// floor(log2 a) of a positive finite float from its bits (subnormals included).
__device__ __forceinline__ int floor_log2_bits(uint32_t bits) {
  const int e = static_cast<int>(bits >> 23);
  if (e > 0) return e - 127;
  return (31 - __clz(static_cast<int>(bits & 0x7FFFFFu))) - 149;
}

// 2^k as a float for k in [-127, 127] (2^-127 is subnormal).
__device__ __forceinline__ float pow2f(int k) {
  return k >= -126 ? __uint_as_float(static_cast<uint32_t>(k + 127) << 23) : __uint_as_float(0x00400000u);
}

// One thread per 32-value block, one warp per 32 consecutive blocks of a row.
template <bool SWZ>
__global__ void __launch_bounds__(kThreads) quantize_mx_kernel(const uint16_t* __restrict__ x, int64_t rows,
                                                               int64_t cols, int64_t ld, uint8_t* __restrict__ codes,
                                                               uint8_t* __restrict__ scales) {
  grid_dependency_wait();
  const int64_t nblk = cols / 32;
  const int64_t atoms_per_group = (nblk + 3) / 4;
  const int64_t chunks = (nblk + 31) / 32;
  const int64_t nwarps = static_cast<int64_t>(gridDim.x) * (kThreads / 32);
  const int64_t w = static_cast<int64_t>(blockIdx.x) * (kThreads / 32) + (threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  for (int64_t task = w; task < rows * chunks; task += nwarps) {
    const int64_t r = task / chunks, cb = (task - r * chunks) * 32 + lane;
    const bool active = cb < nblk;
    uint32_t sbyte = 0;
    if (active) {
      const uint16_t* src = x + r * ld + cb * 32;
      uint4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = ld_nc_v4(src + 8 * i);
      uint32_t m = 0;
#pragma unroll
      for (int i = 0; i < 4; ++i) m = vmax_mag(m, v[i]);
      const uint32_t amax_bits = max(m & 0xFFFFu, m >> 16) << 16;
      int shared = amax_bits == 0 ? -127 : floor_log2_bits(amax_bits) - 2;
      shared = max(-127, min(127, shared));
      sbyte = static_cast<uint32_t>(shared + 127);
      const float inv = pow2f(-shared);
      uint32_t out[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {  // eight values per 32-bit word of codes
        const uint4 q = v[h];
        const uint32_t wd[4] = {q.x, q.y, q.z, q.w};
        float y[8];
#pragma unroll
        for (int k = 0; k < 4; ++k) {
          y[2 * k] = __fmul_rn(__uint_as_float(wd[k] << 16), inv);
          y[2 * k + 1] = __fmul_rn(__uint_as_float(wd[k] & 0xFFFF0000u), inv);
        }
        out[h] = cvt_e2m1x8(y[0], y[1], y[2], y[3], y[4], y[5], y[6], y[7]);
      }
      *reinterpret_cast<uint4*>(codes + r * (cols / 2) + cb * 16) = make_uint4(out[0], out[1], out[2], out[3]);
      if (!SWZ) scales[r * nblk + cb] = static_cast<uint8_t>(sbyte);
    }
    if (SWZ) {
      const uint32_t s1 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 1);
      const uint32_t s2 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 2);
      const uint32_t s3 = __shfl_down_sync(0xFFFFFFFFu, sbyte, 3);
      if (active && (lane & 3) == 0) {
        const int64_t off = ((r >> 7) * atoms_per_group + (cb >> 2)) * 512 + (r & 31) * 16 + ((r >> 5) & 3) * 4;
        *reinterpret_cast<uint32_t*>(scales + off) = sbyte | (s1 << 8) | (s2 << 16) | (s3 << 24);
      }
    }
  }
  if (SWZ) zero_scale_padding(scales, rows, nblk);
}

// BF16 reconstruction q * 2^(s - 127), one thread per 32-value block.
template <bool SWZ>
__global__ void __launch_bounds__(kThreads) dequantize_mx_kernel(const uint8_t* __restrict__ codes,
                                                                 const uint8_t* __restrict__ scales, int64_t rows,
                                                                 int64_t cols, uint16_t* __restrict__ out,
                                                                 int64_t ld_out) {
  grid_dependency_wait();
  const int64_t nblk = cols / 32;
  const int64_t atoms_per_group = (nblk + 3) / 4;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t b = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; b < rows * nblk; b += stride) {
    const int64_t r = b / nblk, cb = b - r * nblk;
    const uint4 cw = *reinterpret_cast<const uint4*>(codes + r * (cols / 2) + cb * 16);
    const uint32_t s = SWZ ? scales[swizzled_offset(r, cb, atoms_per_group)] : scales[b];
    const float scale = pow2f(static_cast<int>(s) - 127);
    const uint32_t words[4] = {cw.x, cw.y, cw.z, cw.w};
    uint4* dst = reinterpret_cast<uint4*>(out + r * ld_out + cb * 32);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      uint32_t o[4];
#pragma unroll
      for (int k = 0; k < 4; ++k) {
        const uint32_t h2 = e2m1x2_to_half2(words[h], k);
        const float q_lo = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 & 0xFFFFu)));
        const float q_hi = __half2float(__ushort_as_half(static_cast<uint16_t>(h2 >> 16)));
        o[k] = static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(q_lo, scale)))) |
               (static_cast<uint32_t>(__bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(q_hi, scale)))) << 16);
      }
      dst[h] = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

// One thread waits, with the kernels' bounded wait, on an mbarrier that nothing
// completes; it gives up after timeout_ns and records kErrSelfTest.
__global__ void selftest_wait_kernel(uint32_t* status, uint64_t timeout_ns) {
  __shared__ uint64_t bar;
  __shared__ uint32_t abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_flag = 0u;
    fence_mbarrier_init();
    mbar_wait(&bar, 0u, &abort_flag, status, kErrSelfTest, timeout_ns);
  }
}

int grid_for(int64_t work, int threads) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t need = (work + threads - 1) / threads;
  const int64_t cap = static_cast<int64_t>(sms) * 16;  // grid-stride beyond 16 CTAs per SM
  return static_cast<int>(need < 1 ? 1 : (need < cap ? need : cap));
}

}  // namespace

cudaError_t launch_amax(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, uint32_t* amax_bits,
                        cudaStream_t stream) {
  const int64_t vecs = rows * cols / 8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t blocks = (vecs + kThreads * 4 - 1) / (kThreads * 4);
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  amax_kernel<<<static_cast<int>(blocks), kThreads, 0, stream>>>(x, rows, cols, ld, amax_bits);
  return cudaGetLastError();
}

cudaError_t launch_quantize(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, int mode,
                            bool swizzled, const float* gs_in, const uint32_t* amax_bits, uint8_t* codes,
                            uint8_t* scales, float* gs_out, float* block_err, cudaStream_t stream) {
  const int64_t blocks16 = rows * (cols / 16);
  // enough threads for the larger of the blocks to encode and the padding to zero
  // (a few activation rows pad their scales to 128 rows)
  const int64_t nblk = cols / 16;
  const int64_t pads = swizzled ? ((rows + 127) / 128 * 128) * ((nblk + 3) / 4 * 4) - blocks16 : 0;
  const int grid = grid_for(blocks16 > pads ? blocks16 : pads, kThreads);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
#define NVFP4_Q(MODE, SWZ) \
  cudaLaunchKernelEx(&cfg, quantize_kernel<MODE, SWZ>, x, rows, cols, ld, gs_in, amax_bits, codes, scales, gs_out, block_err)
  cudaError_t e;
  if (mode == 2)
    e = swizzled ? NVFP4_Q(2, true) : NVFP4_Q(2, false);
  else if (mode == 1)
    e = swizzled ? NVFP4_Q(1, true) : NVFP4_Q(1, false);
  else
    e = swizzled ? NVFP4_Q(0, true) : NVFP4_Q(0, false);
#undef NVFP4_Q
  return e != cudaSuccess ? e : cudaGetLastError();
}

bool quantize_fuses_amax(int64_t rows, int64_t cols, int mode) {
  return mode == 0 && rows * cols <= kFusedMaxElems;
}

cudaError_t launch_quantize_fused(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool swizzled,
                                  uint8_t* codes, uint8_t* scales, float* gs_out, float* block_err,
                                  cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(kFusedCtas);
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = kFusedCtas;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  const cudaError_t e =
      swizzled ? cudaLaunchKernelEx(&cfg, quantize_kernel<0, true, true>, x, rows, cols, ld,
                                    static_cast<const float*>(nullptr), static_cast<const uint32_t*>(nullptr), codes,
                                    scales, gs_out, block_err)
               : cudaLaunchKernelEx(&cfg, quantize_kernel<0, false, true>, x, rows, cols, ld,
                                    static_cast<const float*>(nullptr), static_cast<const uint32_t*>(nullptr), codes,
                                    scales, gs_out, block_err);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_quantize_mx(const uint16_t* x, int64_t rows, int64_t cols, int64_t ld, bool swizzled,
                               uint8_t* codes, uint8_t* scales, cudaStream_t stream) {
  const int64_t nblk = cols / 32;
  const int64_t pads = swizzled ? ((rows + 127) / 128 * 128) * ((nblk + 3) / 4 * 4) - rows * nblk : 0;
  const int64_t work = rows * ((nblk + 31) / 32) * 32;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_for(work > pads ? work : pads, kThreads));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e = swizzled ? cudaLaunchKernelEx(&cfg, quantize_mx_kernel<true>, x, rows, cols, ld, codes, scales)
                                 : cudaLaunchKernelEx(&cfg, quantize_mx_kernel<false>, x, rows, cols, ld, codes, scales);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_dequantize_mx(const uint8_t* codes, const uint8_t* scales, bool swizzled, int64_t rows,
                                 int64_t cols, uint16_t* out, int64_t ld_out, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_for(rows * (cols / 32), kThreads));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      swizzled ? cudaLaunchKernelEx(&cfg, dequantize_mx_kernel<true>, codes, scales, rows, cols, out, ld_out)
               : cudaLaunchKernelEx(&cfg, dequantize_mx_kernel<false>, codes, scales, rows, cols, out, ld_out);
  return e != cudaSuccess ? e : cudaGetLastError();
}

cudaError_t launch_selftest_wait(uint32_t* status, uint64_t timeout_ns, cudaStream_t stream) {
  selftest_wait_kernel<<<1, 32, 0, stream>>>(status, timeout_ns);
  return cudaGetLastError();
}

cudaError_t launch_dequantize(const uint8_t* codes, const uint8_t* scales, bool swizzled, const float* gs,
                              int64_t rows, int64_t cols, uint16_t* out, int64_t ld_out, cudaStream_t stream) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid_for(rows * (cols / 16), kThreads));
  cfg.blockDim = dim3(kThreads);
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const cudaError_t e =
      swizzled ? cudaLaunchKernelEx(&cfg, dequantize_kernel<true>, codes, scales, gs, rows, cols, out, ld_out)
               : cudaLaunchKernelEx(&cfg, dequantize_kernel<false>, codes, scales, gs, rows, cols, out, ld_out);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

}  // namespace nvfp4
