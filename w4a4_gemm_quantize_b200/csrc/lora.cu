// lora.cu -- the low-rank branch of the W4A4 linear layer: t = A x on the tensor cores.
//
// Page "NVFP4 en difusión: la misma cuantización, un motor completamente distinto",
// section 3 ("¿Cómo fine-tuneás algo que ya está en 4 bits?"): a LoRA cannot be
// merged into NVFP4 weights, so the kernel computes y = W_4bit x + B (A x), the
// low-rank term in 16 bits, added to the quantized matmul before the result is
// returned.  Here the term's first product t = A x (M x R, R the rank) is a BF16
// GEMM on the tensor cores (tcgen05.mma kind::f16, FP32 accumulation, TMA-fed,
// TMEM accumulator); t is rounded to BF16 -- the 16-bit intermediate -- and the
// W4A4 GEMM adds B t to its FP32 accumulator with more kind::f16 MMAs before its
// single BF16 rounding.  Because that accumulator is scaled by alpha = s_gA s_gB in
// the GEMM's epilogue, this kernel also writes t / alpha as a pair of BF16 values
// (hi = BF16(RN32(t / alpha)), lo = BF16(RN32(t / alpha) - hi)), which the GEMM
// multiplies by B; the pair carries t / alpha to about 2^-16 relative.
//
// One CTA per 128-row tile of x and K-split (the split lets a few rows spread over
// many SMs): warp 0 loads 64-value K-steps of x (128 rows) and of A (R rows) with
// TMA into a 6-stage ring, warp 1 issues four 128 x R x 16 MMAs per K-step, warps
// 2-5 read the accumulator.  With more than one split each CTA stores an FP32
// partial tile; the last CTA of a row tile (acquire-release counter) sums the
// partials in split order, so the result does not depend on arrival order.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "quant_block.cuh"

namespace nvfp4 {

namespace {

struct LoraCfg {
  static constexpr int BM = 128;
  static constexpr int KSTEP_BYTES = 128;            // 64 BF16 values per row per stage
  static constexpr int X_BYTES = BM * KSTEP_BYTES;   // 16 KB
  static constexpr int A_BYTES = 64 * KSTEP_BYTES;   // up to 64 rank rows: 8 KB
  static constexpr int STAGE_BYTES = X_BYTES + A_BYTES;
  static constexpr int STAGES = 6;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + 256;
  static constexpr int THREADS = 192;                // warp 0 producer, 1 MMA, 2-5 epilogue
  static constexpr int TMEM_COLS = 128;
  static constexpr int MAX_RANK = 64;
};

__device__ __forceinline__ bool lora_wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status) {
  const uint32_t addr = smem_u32(bar);
  const uint64_t t0 = globaltimer_ns();
  while (!mbar_try_wait(addr, parity)) {
    if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
      if (status) atomicCAS(status, 0u, static_cast<uint32_t>(kErrWaitDrain));
      return false;
    }
  }
  return true;
}

__device__ __forceinline__ uint16_t bf16_bits(float f) { return __bfloat16_as_ushort(__float2bfloat16_rn(f)); }

// Row `row` of the finished tile (acc[0..R)): t = BF16(acc), hi / lo of t / alpha.
__device__ __forceinline__ void lora_finish_row(const float* acc, int R, float alpha, int64_t row,
                                                uint16_t* __restrict__ t_out, uint16_t* __restrict__ thi,
                                                uint16_t* __restrict__ tlo) {
  for (int j = 0; j < R; j += 8) {
    uint32_t pt[4], ph[4], pl[4];
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      uint16_t tb[2], hb[2], lb[2];
#pragma unroll
      for (int h = 0; h < 2; ++h) {
        tb[h] = bf16_bits(acc[j + e + h]);
        const float q = __fdiv_rn(__uint_as_float(static_cast<uint32_t>(tb[h]) << 16), alpha);
        hb[h] = bf16_bits(q);
        lb[h] = bf16_bits(__fsub_rn(q, __uint_as_float(static_cast<uint32_t>(hb[h]) << 16)));
      }
      pt[e / 2] = tb[0] | (static_cast<uint32_t>(tb[1]) << 16);
      ph[e / 2] = hb[0] | (static_cast<uint32_t>(hb[1]) << 16);
      pl[e / 2] = lb[0] | (static_cast<uint32_t>(lb[1]) << 16);
    }
    const int64_t off = row * R + j;
    if (t_out) *reinterpret_cast<uint4*>(t_out + off) = make_uint4(pt[0], pt[1], pt[2], pt[3]);
    *reinterpret_cast<uint4*>(thi + off) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
    *reinterpret_cast<uint4*>(tlo + off) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
  }
}

__global__ void __launch_bounds__(LoraCfg::THREADS, 1)
    lora_down_kernel(const __grid_constant__ CUtensorMap tmap_x, const __grid_constant__ CUtensorMap tmap_a, int M,
                     int K, int R, int splits, const float* __restrict__ x_gs_in, const uint32_t* __restrict__ x_amax,
                     const float* __restrict__ w_gs, uint16_t* __restrict__ t_out, uint16_t* __restrict__ thi,
                     uint16_t* __restrict__ tlo, float* __restrict__ partial, uint32_t* __restrict__ counters,
                     uint32_t* __restrict__ status) {
  using Cfg = LoraCfg;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sX = smem;
  uint8_t* sA = sX + STAGES * Cfg::X_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sA + STAGES * Cfg::A_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* drain = acc_full + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* decision = tmem_slot + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int rt = blockIdx.x / splits, sp = blockIdx.x % splits;
  const int ksteps = (K + 63) / 64;
  const int k0 = sp * ksteps / splits, k1 = (sp + 1) * ksteps / splits;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == 0 && lane == 0) {
    prefetch_tmap(&tmap_x);
    prefetch_tmap(&tmap_a);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  grid_dependents_launch();  // the quantizer and GEMM behind this kernel may set up meanwhile
  grid_dependency_wait();    // x and the activation's amax word come from earlier kernels

  if (warp == 0) {
    if (lane == 0) {
      // ---------------- producer ----------------
      int issued_last[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_last[s] = -1;
      for (int ks = k0, i = 0; ks < k1; ++ks, ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&empty[s], (static_cast<uint32_t>(i / STAGES) & 1u) ^ 1u, abort_flag, status,
                       kErrLora + 1))
          break;
        const int rows16 = (R + 15) / 16 * 16;
        mbar_arrive_expect_tx(&full[s], Cfg::X_BYTES + rows16 * Cfg::KSTEP_BYTES);
        tma_load_2d(sX + s * Cfg::X_BYTES, &tmap_x, &full[s], ks * 64, rt * Cfg::BM);
        tma_load_2d(sA + s * Cfg::A_BYTES, &tmap_a, &full[s], ks * 64, 0);
        issued_last[s] = i;
      }
      if (*abort_flag)
        for (int s = 0; s < STAGES; ++s)
          if (issued_last[s] >= 0) lora_wait_drain(&full[s], static_cast<uint32_t>(issued_last[s] / STAGES) & 1u, status);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_bf16(Cfg::BM, (R + 15) / 16 * 16);
      bool ok = true;
      for (int ks = k0, i = 0; ks < k1; ++ks, ++i) {
        const int s = i % STAGES;
        if (!mbar_wait(&full[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, status, kErrLora + 2)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t xb = smem_u32(sX + s * Cfg::X_BYTES), ab = smem_u32(sA + s * Cfg::A_BYTES);
#pragma unroll
        for (int j = 0; j < 4; ++j)  // 16 BF16 values (32 bytes) of K per instruction
          mma_bf16(tmem_base, sdesc_kmajor_sw128(xb + 32 * j), sdesc_kmajor_sw128(ab + 32 * j), idesc,
                   (ks != k0 || j != 0) ? 1u : 0u);
        tc_commit(&empty[s]);
      }
      if (ok) {
        tc_commit(acc_full);
      } else {
        tc_commit(drain);
        lora_wait_drain(drain, 0u, status);
      }
    }
  } else {
    // ---------------- epilogue (warps 2-5): lane = row of the tile ----------------
    const int quarter = warp & 3;
    const int64_t row = static_cast<int64_t>(rt) * Cfg::BM + quarter * 32 + lane;
    const bool got = warp_wait(acc_full, 0u, abort_flag, status, kErrLora + 3);
    float acc[Cfg::MAX_RANK];
    if (got) {
      tc_fence_after();
      for (int c = 0; c < R; c += 16) {
        uint32_t v[16];
        tmem_ld_32x32b_x16(tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int e = 0; e < 16; ++e) acc[c + e] = __uint_as_float(v[e]);
      }
      tc_fence_before();
    }
    // one decision for the four warps
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (threadIdx.x == 64) *decision = *abort_flag ? 0u : 1u;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    const bool go = *decision == 1u;
    asm volatile("bar.sync 1, 128;" ::: "memory");
    if (go) {
      const float alpha = __fmul_rn(global_scale(x_gs_in, x_amax), *w_gs);
      if (splits == 1) {
        if (row < M) lora_finish_row(acc, R, alpha, row, t_out, thi, tlo);
      } else {
        float* mine = partial + ((static_cast<int64_t>(rt) * splits + sp) * Cfg::BM + quarter * 32 + lane) * R;
        if (row < M)
          for (int j = 0; j < R; j += 4)
            *reinterpret_cast<float4*>(mine + j) = make_float4(acc[j], acc[j + 1], acc[j + 2], acc[j + 3]);
        // the four warps' rows are ordered before the release by the barrier; the
        // split that arrives last acquires every other split's rows
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 64)
          *decision = atom_add_acq_rel_gpu(&counters[rt], 1u) == static_cast<uint32_t>(splits - 1) ? 2u : 1u;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool last = *decision == 2u;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (last) {
          if (row < M) {
            for (int j = 0; j < R; ++j) acc[j] = 0.0f;
            for (int p = 0; p < splits; ++p) {
              const float* src = partial + ((static_cast<int64_t>(rt) * splits + p) * Cfg::BM + quarter * 32 + lane) * R;
              for (int j = 0; j < R; j += 4) {
                const float4 f = __ldcg(reinterpret_cast<const float4*>(src + j));
                acc[j] = __fadd_rn(acc[j], f.x);
                acc[j + 1] = __fadd_rn(acc[j + 1], f.y);
                acc[j + 2] = __fadd_rn(acc[j + 2], f.z);
                acc[j + 3] = __fadd_rn(acc[j + 3], f.w);
              }
            }
            lora_finish_row(acc, R, alpha, row, t_out, thi, tlo);
          }
          if (threadIdx.x == 64) counters[rt] = 0u;  // ready for the next call
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn lora_encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess) {
      cudaGetLastError();
      p = nullptr;
    }
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// BF16 rows x cols matrix (row stride ld elements), box = box_rows x 64 values
// (128 bytes), 128-byte swizzle; rows and values past the edge read as zero.
bool encode_bf16_kmajor_map(CUtensorMap* map, const void* base, int64_t rows, int64_t cols, int64_t ld,
                            int box_rows) {
  EncodeTiledFn enc = lora_encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ld * 2)};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

}  // namespace

int lora_splits(int64_t M, int64_t K, int sms) {
  const int64_t tiles = (M + LoraCfg::BM - 1) / LoraCfg::BM;
  const int64_t ksteps = (K + 63) / 64;
  int64_t s = sms / tiles;
  const int64_t most = ksteps / 4 > 0 ? ksteps / 4 : 1;  // at least four K-steps per CTA
  if (s > most) s = most;
  return static_cast<int>(s < 1 ? 1 : s);
}

size_t lora_partial_bytes(int64_t M, int64_t K, int64_t R) {
  const int64_t tiles = (M + LoraCfg::BM - 1) / LoraCfg::BM;
  const int64_t splits = lora_splits(M, K, 296);  // the largest grid the launcher uses
  return splits > 1 ? static_cast<size_t>(tiles * splits) * LoraCfg::BM * R * 4 : 0;
}

size_t lora_counter_bytes(int64_t M) {
  const int64_t tiles = (M + LoraCfg::BM - 1) / LoraCfg::BM;
  return static_cast<size_t>((tiles * 4 + 255) / 256 * 256);
}

cudaError_t launch_lora_down(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* x_gs_in,
                             const uint32_t* x_amax, const float* w_gs, const uint16_t* lora_a, int64_t R,
                             uint16_t* t_out, uint16_t* thi, uint16_t* tlo, uint32_t* counters, float* partial,
                             uint32_t* status, cudaStream_t stream) {
  CUtensorMap tx, ta;
  if (!encode_bf16_kmajor_map(&tx, x, M, K, ld_x, LoraCfg::BM) ||
      !encode_bf16_kmajor_map(&ta, lora_a, R, K, K, static_cast<int>((R + 15) / 16 * 16)))
    return cudaErrorInvalidValue;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  std::call_once(once[dev & 63], [&] {
    attr_err[dev & 63] =
        cudaFuncSetAttribute(lora_down_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, LoraCfg::SMEM_BYTES);
  });
  if (attr_err[dev & 63] != cudaSuccess) return attr_err[dev & 63];
  const int splits = lora_splits(M, K, sms > 296 ? 296 : sms);
  const int64_t tiles = (M + LoraCfg::BM - 1) / LoraCfg::BM;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(tiles * splits));
  cfg.blockDim = dim3(LoraCfg::THREADS);
  cfg.dynamicSmemBytes = LoraCfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, lora_down_kernel, tx, ta, static_cast<int>(M), static_cast<int>(K),
                            static_cast<int>(R), splits, x_gs_in, x_amax, w_gs, t_out, thi, tlo, partial, counters,
                            status);
}

}  // namespace nvfp4
