// gemm_sm100.cu -- block-scaled NVFP4 x NVFP4 GEMM on the sm_100a tensor cores.
//
// C = (A s_a)(B s_b)^T * s_gA * s_gB with FP32 accumulation and BF16 output: the
// equation out = (A·s_a) × (B·s_b)ᵀ of the web page "NVFP4 en difusión: la
// misma cuantización, un motor completamente distinto", section 2 "NVFP4 sin
// vLLM: torch._scaled_mm a mano" -- the per-16 E4M3 scales travel as separate
// tensors and are applied per block inside the kernel; the result is BF16.
//
// Three kernels, chosen by launch_gemm from the shape: gemm_pair_kernel (M > 128
// and N > 128: CTA pairs on 256 x 256 tiles, with a stream-K instantiation for the
// last round of long-K shapes), gemm_decode_kernel (M <= 32: the weight stream
// split evenly over the SMs) and gemm_kernel<BN> (the other shapes), each described
// where it is defined.  All are launched with programmatic dependent launch.
//
// gemm_kernel<BN>: a persistent kernel, one CTA per SM, each CTA walking 128 x BN output
// tiles in a grouped order (GROUP_M row-tiles at a time, so the CTAs running at
// the same moment share A and B tiles through L2).  Ten warps:
//   warp 8  TMA producer: per K-tile of 256 values, a 128 x 128-byte A tile and a
//           BN x 128-byte B tile (tensor maps, 128-byte swizzle) plus the scale
//           tiles (plain bulk copies of the 512-byte 128x4 atoms), into a
//           STAGES-deep shared-memory ring guarded by full/empty mbarriers; the
//           ring keeps flowing across tile boundaries;
//   warp 9  allocates TMEM and issues, from one thread, tcgen05.cp of the scale
//           atoms into TMEM and tcgen05.mma.kind::mxf4nvf4.block_scale.block16
//           (128 x BN x 64 per instruction) into the TMEM accumulator;
//           tcgen05.commit frees each stage and signals the finished tile;
//   warps 0-7 epilogue: warp w reads TMEM lanes 32(w%4).. (tile rows) and half of
//           the columns, converts to BF16 in registers, releases the accumulator
//           (so the next tile's MMAs start) and then stores its rows.
// Every mbarrier wait is bounded; on a timeout the kernel writes the status word,
// drains its in-flight copies and MMAs (again bounded), frees TMEM and returns.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "internal.h"
#include "ptx.cuh"
#include "quant_block.cuh"

namespace nvfp4 {

namespace {

template <int BN_>
struct GemmCfg {
  static constexpr int BM = 128;
  static constexpr int BN = BN_;
  static constexpr int KTILE_BYTES = 128;             // 256 FP4 values per row per stage
  static constexpr int A_BYTES = BM * KTILE_BYTES;    // 16 KB
  static constexpr int B_BYTES = BN * KTILE_BYTES;
  static constexpr int SF_ATOM = 512;                 // 128 rows x 4 scales (64 values of K)
  static constexpr int SFA_BYTES = 4 * SF_ATOM;       // one row group, 4 K-steps
  static constexpr int SFB_BYTES = (BN / 128) * 4 * SF_ATOM;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = (220 * 1024) / STAGE_BYTES;
  static constexpr int BAR_BYTES = 256;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + BAR_BYTES;
  static constexpr int EPI_WARPS = 8;
  static constexpr int PRODUCER_WARP = EPI_WARPS;
  static constexpr int MMA_WARP = EPI_WARPS + 1;
  static constexpr int THREADS = (EPI_WARPS + 2) * 32;
  static constexpr int GROUP_M = 8;
  // TMEM columns: accumulator [0, BN), then two scale regions (A 16 + B BN/8 each).
  static constexpr int TMEM_SFA = BN;
  static constexpr int TMEM_SFB = BN + 16;
  static constexpr int TMEM_SF_STRIDE = 16 + BN / 8;
  static constexpr int TMEM_USED = BN + 2 * TMEM_SF_STRIDE;
  static constexpr int TMEM_COLS = TMEM_USED <= 256 ? 256 : 512;
  static_assert(BN == 128 || BN == 256, "tile width");
  static_assert(STAGES >= 2, "pipeline depth");
  static_assert(TMEM_USED <= TMEM_COLS, "TMEM budget");
};

// Wait with a timeout that ignores the abort flag (teardown after an abort).
__device__ __forceinline__ bool mbar_wait_drain(uint64_t* bar, uint32_t parity, uint32_t* status) {
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

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  const __nv_bfloat16 a = __float2bfloat16_rn(lo), b = __float2bfloat16_rn(hi);
  return static_cast<uint32_t>(__bfloat16_as_ushort(a)) | (static_cast<uint32_t>(__bfloat16_as_ushort(b)) << 16);
}

// Tile t -> (row tile, column tile): groups of GROUP_M row tiles, column-major
// inside a group, so that consecutive tiles reuse the same few A and B tiles.
template <int GROUP_M>
__device__ __forceinline__ void tile_coords(int t, int num_m, int num_n, int& tm, int& tn) {
  const int per_group = GROUP_M * num_n;
  const int g = t / per_group;
  const int first_m = g * GROUP_M;
  const int gm = min(GROUP_M, num_m - first_m);
  const int local = t - g * per_group;
  tm = first_m + local % gm;
  tn = local / gm;
}

template <int BN>
__global__ void __launch_bounds__(GemmCfg<BN>::THREADS, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                const uint8_t* __restrict__ sfa, const uint8_t* __restrict__ sfb, const float* __restrict__ a_gs,
                const float* __restrict__ b_gs, uint16_t* __restrict__ C, int M, int N, int K, int64_t ldc,
                uint32_t* __restrict__ status) {
  using Cfg = GemmCfg<BN>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * Cfg::A_BYTES;
  uint8_t* sSFA = sB + STAGES * Cfg::B_BYTES;
  uint8_t* sSFB = sSFA + STAGES * Cfg::SFA_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * Cfg::SFB_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* acc_full = empty + STAGES;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_atoms = (K + 63) / 64;  // 64-value K steps = scale atoms per 128-row group
  const int k_tiles = (k_atoms + 3) / 4;
  const int n_groups_b = (N + 127) / 128;
  const int num_m = (M + Cfg::BM - 1) / Cfg::BM;
  const int num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, Cfg::EPI_WARPS);
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  if (warp == Cfg::PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The set-up above overlaps the previous kernel's tail (programmatic launch);
  // from here on the operands it wrote are visible.  (The status word was cleared
  // by a memset before the launch, so no CTA can erase another's timeout code.)
  grid_dependency_wait();

  if (warp == Cfg::PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- TMA producer ----------------
      int issued_last[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_last[s] = -1;
      int kc = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x) {
        int tm, tn;
        tile_coords<Cfg::GROUP_M>(t, num_m, num_n, tm, tn);
        int valid_b_groups = 0;
        for (int g = 0; g < BN / 128; ++g)
          if (tn * (BN / 128) + g < n_groups_b) ++valid_b_groups;
        for (int kt = 0; kt < k_tiles; ++kt, ++kc) {
          const int s = kc % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kc / STAGES) & 1u;
          if (!mbar_wait(&empty[s], ph ^ 1u, abort_flag, status, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          const int ka0 = kt * 4;
          const int na = min(4, k_atoms - ka0);
          const uint32_t sf_bytes = static_cast<uint32_t>(na) * Cfg::SF_ATOM;
          mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + Cfg::B_BYTES + sf_bytes * (1 + valid_b_groups));
          tma_load_2d(sA + s * Cfg::A_BYTES, &tmap_a, &full[s], kt * Cfg::KTILE_BYTES, tm * Cfg::BM);
          tma_load_2d(sB + s * Cfg::B_BYTES, &tmap_b, &full[s], kt * Cfg::KTILE_BYTES, tn * BN);
          bulk_load(sSFA + s * Cfg::SFA_BYTES, sfa + (static_cast<size_t>(tm) * k_atoms + ka0) * Cfg::SF_ATOM,
                    sf_bytes, &full[s]);
          for (int g = 0; g < valid_b_groups; ++g)
            bulk_load(sSFB + s * Cfg::SFB_BYTES + g * 4 * Cfg::SF_ATOM,
                      sfb + (static_cast<size_t>(tn * (BN / 128) + g) * k_atoms + ka0) * Cfg::SF_ATOM, sf_bytes,
                      &full[s]);
          issued_last[s] = kc;
        }
      }
      if (*abort_flag) {
        // Let every copy this thread started land before the CTA exits.
        for (int s = 0; s < STAGES; ++s)
          if (issued_last[s] >= 0)
            mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_last[s] / STAGES) & 1u, status);
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = idesc_mxf4nvf4(Cfg::BM, BN);
      const uint32_t t_acc = tmem_base;
      const uint32_t t_sfa = tmem_base + Cfg::TMEM_SFA;
      const uint32_t t_sfb = tmem_base + Cfg::TMEM_SFB;
      bool ok = true;
      int kc = 0, it = 0;
      for (int t = blockIdx.x; t < num_tiles && ok; t += gridDim.x, ++it) {
        // the epilogue must have drained the previous tile's accumulator
        if (!mbar_wait(acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag, status, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        for (int kt = 0; kt < k_tiles; ++kt, ++kc) {
          const int s = kc % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kc / STAGES) & 1u;
          if (!mbar_wait(&full[s], ph, abort_flag, status, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int na = min(4, k_atoms - kt * 4);
          const uint32_t a_base = smem_u32(sA + s * Cfg::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * Cfg::B_BYTES);
          const uint32_t sfa_base = smem_u32(sSFA + s * Cfg::SFA_BYTES);
          const uint32_t sfb_base = smem_u32(sSFB + s * Cfg::SFB_BYTES);
          // scale factors go to one of two TMEM regions by K-tile parity, so these
          // copies need not wait for the previous K-tile's MMAs to finish reading
          const uint32_t sf_off = (kc & 1) ? Cfg::TMEM_SF_STRIDE : 0u;
          for (int j = 0; j < na; ++j) {
            tc_cp_sf(t_sfa + sf_off + 4 * j, sdesc_sf_tile(sfa_base + j * Cfg::SF_ATOM));
#pragma unroll
            for (int g = 0; g < BN / 128; ++g)
              tc_cp_sf(t_sfb + sf_off + (BN / 32) * j + 4 * g,
                       sdesc_sf_tile(sfb_base + (g * 4 + j) * Cfg::SF_ATOM));
            mma_mxf4nvf4(t_acc, sdesc_kmajor_sw128(a_base + 32 * j), sdesc_kmajor_sw128(b_base + 32 * j), idesc,
                         t_sfa + sf_off + 4 * j, t_sfb + sf_off + (BN / 32) * j, (kt | j) != 0 ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(acc_full);
      }
      if (!ok) {
        tc_commit(drain);
        mbar_wait_drain(drain, 0u, status);
      }
    }
  } else {
    // ---------------- epilogue (warps 0-7) ----------------
    constexpr int HALF = BN / 2;  // columns per epilogue warp
    const int quarter = warp & 3, half = warp >> 2;
    const float alpha = __fmul_rn(*a_gs, *b_gs);
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * HALF;
    int it = 0;
    for (int t = blockIdx.x; t < num_tiles; t += gridDim.x, ++it) {
      int tm, tn;
      tile_coords<Cfg::GROUP_M>(t, num_m, num_n, tm, tn);
      if (!warp_wait(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, kErrWaitAccFull)) break;
      tc_fence_after();
      uint32_t p[HALF / 2];
#pragma unroll
      for (int c = 0; c < HALF; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          p[c / 2 + i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * i]), alpha),
                                     __fmul_rn(__uint_as_float(v[2 * i + 1]), alpha));
      }
      // accumulator drained: let the MMA warp start the next tile
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(acc_empty);
      const int row = tm * Cfg::BM + quarter * 32 + lane;
      const int col0 = tn * BN + half * HALF;
      if (row < M && col0 < N) {
        uint16_t* dst = C + static_cast<int64_t>(row) * ldc + col0;
        if (col0 + HALF <= N) {
          uint4* d4 = reinterpret_cast<uint4*>(dst);
#pragma unroll
          for (int i = 0; i < HALF / 8; ++i) d4[i] = make_uint4(p[4 * i], p[4 * i + 1], p[4 * i + 2], p[4 * i + 3]);
        } else {
#pragma unroll
          for (int i = 0; i < HALF; ++i)
            if (col0 + i < N) dst[i] = static_cast<uint16_t>((i & 1) ? (p[i >> 1] >> 16) : (p[i >> 1] & 0xFFFFu));
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == Cfg::MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// CTA-pair kernel: tcgen05 cta_group::2, 256 x 256 output tile per pair of SMs
// ---------------------------------------------------------------------------------------------
//
// The two CTAs of a cluster share one MMA: CTA r holds rows 128r..128r+127 of the
// tile's A block and rows 128r..128r+127 of its B block in shared memory; the
// leader (rank 0) issues every tcgen05.mma for the pair and each CTA's TMEM holds
// its 128 accumulator rows.  Each CTA's producer loads its A/B halves with pair
// TMA loads that complete on the leader's `full` barrier (the leader expects the
// pair's bytes); the leader's commits arrive on both CTAs' barriers.
//
// Scale factors: each CTA loads its own 128 rows of A scales and all 256 rows of B
// scales (one K-tile: 4 + 8 atoms of 512 bytes) with single-CTA TMA loads, and
// "scale warps" copy them from shared memory into the TMEM scale region of that
// pipeline stage with tcgen05.st: the four warps of a set cover the four 32-lane
// TMEM sub-partitions and every lane writes the same 16-byte atom line, which is
// the 4-way replication the block-scaled MMA reads.  This keeps the copy off the
// tensor pipe (tcgen05.cp of the same bytes, even one copy per MMA, serialises with
// the MMAs).  Three sets rotate over K-tiles so that one set's barrier round trip
// overlaps the others' copies.  The leader's set also waits for the stage's A/B
// bytes before it arrives, so the MMA issuer waits on one barrier per K-tile: every
// wait in the issuing thread lets the tensor pipe's queue run dry (with four MMAs
// per wait the pipe already runs at about 85 % of its rate).  The peer's set
// gathers its four warps on a local barrier -- every warp waits for the phase, so
// that no warp's next arrival can complete it early -- and one of them arrives with
// a cluster-scope release, which orders the set's TMEM stores before the leader's
// MMA reads them (one remote release per K-tile: four of them cost ~10 % of the GEMM).
// Scale factors have their own producer and shared-memory slots, refilled as soon
// as a set has moved them to TMEM, so they land several K-tiles ahead of their MMAs.  A stage's region is free again when its shared-memory
// slot is: the producer reloads stage s only after the MMAs that read it
// completed, so no separate release barrier is needed.  Each K-tile's MMAs end with
// one commit that arrives on both CTAs' `empty` barriers.
//
// Epilogue: 8 warps (2 per sub-partition) read the accumulator, release it (the
// peer's warps with a relaxed arrive: they have only read TMEM, and waited for the
// reads), and write BF16 through 128-byte-swizzled shared-memory boxes with TMA
// stores.

// The work of one CTA pair, as a sequence of items: an item is one 256 x 256 output tile
// over a range of its K-tiles.  Tiles are done whole (data-parallel), except that, when
// the tile count T is not a multiple of the pair count P and partial tiles are enabled,
// the first P + T mod P tiles are done "stream-K": their K-tiles form one sequence of
// units, tile-major, split evenly over the pairs, so that no pair idles through a last,
// partial round.  A pair's stream-K range holds at least one tile's K-tiles, so a tile
// is shared by at most two pairs: piece 0 (from K-tile 0) and piece 1 (up to the last
// K-tile).  Both pieces store their FP32 partial tile in the slot of the later piece's
// pair; the piece that finishes second sums the two, piece 0 plus piece 1, and writes C.
// A pair does its pieces first, then its whole stream-K tiles, then its data-parallel
// tiles, so that the sums overlap the remaining work.
// Pair kernel: shapes it takes, and its shared-tile scratch -- a ticket counter and a
// ready flag per slot, CTA and epilogue warp, then two pieces x two CTAs x 8 warps x
// 32 x 128 FP32 per slot --
// for up to kMaxPairSlots pairs (148 SMs); a larger grid runs without partial tiles.
constexpr int kMaxPairSlots = 74;
inline bool uses_pair_kernel(int64_t M, int64_t N) { return M > 128 && N > 128; }
constexpr int kPairFlagOffset = kMaxPairSlots * 2 * 8;  // flags follow the counters (words)
inline size_t pair_counter_bytes() { return (static_cast<size_t>(2 * kPairFlagOffset) * 4 + 255) / 256 * 256; }
inline size_t pair_partial_bytes() { return static_cast<size_t>(kMaxPairSlots) * 2 * 2 * 8 * 32 * 128 * 4; }

// Bounded wait for a flag that another CTA of the grid sets (every CTA of the pair
// kernel is resident: one per SM, at most as many pairs as fit).
__device__ __forceinline__ bool wait_flag(const uint32_t* flag, volatile uint32_t* abort, uint32_t* status,
                                          uint32_t where) {
  const uint64_t t0 = globaltimer_ns();
  for (uint32_t n = 1;; ++n) {
    if (*reinterpret_cast<const volatile uint32_t*>(flag) != 0u) return true;
    if ((n & 63u) == 0) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > kWaitTimeoutNs) {
        *abort = 1u;
        if (status) atomicCAS(status, 0u, where);
        return false;
      }
    }
  }
}

struct PairItem {
  int tile;      // tile index, in tile_coords order
  int kt0, kt1;  // K-tiles [kt0, kt1)
  int slot;      // partial-tile slot of a shared tile; -1 for a whole tile
  int piece;     // 0 or 1 for a shared tile
};

// Stream-K tiles (the first n_sk).  A shared tile costs its two pieces' epilogues
// (the FP32 partial sums out, then in again while the accumulator is held) and the
// stream-K part reads A and B with less reuse between neighbouring pairs; measured on
// B200 this pays only when the last round would leave the pairs idle for at least ~40
// K-tiles on average (e.g. K = 21504 with 672 tiles on 74 pairs, not K = 5376).
__host__ __device__ __forceinline__ int pair_sk_tiles(int P, int T, int KT, bool partial_tiles) {
  const int rem = T % P;
  if (!partial_tiles || rem == 0 || T < P) return 0;
  if (static_cast<int64_t>(P - rem) * KT < 40LL * P) return 0;
  return P + rem;
}

__device__ __forceinline__ int pair_item_count(int pair, int P, int T, int KT, bool partial_tiles) {
  const int n_sk = pair_sk_tiles(P, T, KT, partial_tiles);
  const int64_t U = static_cast<int64_t>(n_sk) * KT;
  const int64_t b0 = static_cast<int64_t>(pair) * U / P, b1 = static_cast<int64_t>(pair + 1) * U / P;
  int n = 0;
  if (n_sk > 0) n = static_cast<int>(b0 % KT != 0) + static_cast<int>(b1 % KT != 0) +
                    static_cast<int>(b1 / KT - (b0 + KT - 1) / KT);
  const int first = n_sk + pair;
  return n + (first < T ? (T - first + P - 1) / P : 0);
}

// Item i of the pair: [start piece][end piece][whole stream-K tiles][data-parallel tiles].
__device__ __forceinline__ PairItem pair_item(int i, int pair, int P, int T, int KT, bool partial_tiles) {
  PairItem it;
  it.slot = -1;
  it.piece = 0;
  it.kt0 = 0;
  it.kt1 = KT;
  const int n_sk = pair_sk_tiles(P, T, KT, partial_tiles);
  if (n_sk > 0) {
    const int64_t U = static_cast<int64_t>(n_sk) * KT;
    const int64_t b0 = static_cast<int64_t>(pair) * U / P, b1 = static_cast<int64_t>(pair + 1) * U / P;
    if (b0 % KT != 0) {
      if (i == 0) {  // the end of a tile begun by the pair before
        it.tile = static_cast<int>(b0 / KT);
        it.kt0 = static_cast<int>(b0 % KT);
        it.slot = pair;
        it.piece = 1;
        return it;
      }
      --i;
    }
    if (b1 % KT != 0) {
      if (i == 0) {  // the start of a tile that the next pair finishes
        it.tile = static_cast<int>(b1 / KT);
        it.kt1 = static_cast<int>(b1 % KT);
        it.slot = pair + 1;
        it.piece = 0;
        return it;
      }
      --i;
    }
    const int w0 = static_cast<int>((b0 + KT - 1) / KT), w1 = static_cast<int>(b1 / KT);
    if (i < w1 - w0) {
      it.tile = w0 + i;
      return it;
    }
    i -= w1 - w0;
  }
  it.tile = n_sk + pair + i * P;
  return it;
}

template <bool LR = false>
struct PairCfg {
  static constexpr int BM = 128;                      // rows of A per CTA (256 per pair)
  static constexpr int BN = 256;                      // columns of the pair's tile
  static constexpr int KTILE_BYTES = 128;             // 256 FP4 values per row per stage
  static constexpr int A_BYTES = BM * KTILE_BYTES;    // 16 KB
  static constexpr int B_BYTES = 128 * KTILE_BYTES;   // this CTA's half of B: 16 KB
  static constexpr int SF_ATOM = 512;
  static constexpr int SFA_BYTES = 4 * SF_ATOM;       // own 128 rows, 4 K-steps
  static constexpr int SFB_BYTES = 2 * 4 * SF_ATOM;   // all 256 rows, 4 K-steps
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  // LR (low-rank branch): four stages, C staged through 32 x 32 boxes (64-byte swizzle)
  // instead of 32 x 64, and the tile's low-rank operands -- t / alpha hi and lo (this
  // CTA's 128 rows) and B's rows (this CTA's 128 columns), 128-byte K-major rows
  // (rank up to 64)
  static constexpr int STAGES = LR ? 4 : 5;
  static constexpr int EPI_WARPS = 8;
  static constexpr int C_BOX_COLS = LR ? 32 : 64;     // BF16 columns of one staging box
  static constexpr int C_BOX_BYTES = 32 * C_BOX_COLS * 2;
  static constexpr int C_BYTES = EPI_WARPS * C_BOX_BYTES;
  static constexpr int LORA_BYTES = LR ? 3 * 128 * 128 : 0;
  static constexpr int BAR_BYTES = 512;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + C_BYTES + LORA_BYTES + BAR_BYTES;
  static constexpr int PRODUCER_WARP = EPI_WARPS;     // 8
  static constexpr int MMA_WARP = EPI_WARPS + 1;      // 9
  static constexpr int SF_WARP0 = EPI_WARPS + 2;      // 10..
  static constexpr int SF_SETS = 3;                   // sets of 4 scale warps, rotating over K-tiles
  static constexpr int SF_PRODUCER_WARP = SF_WARP0 + 4 * SF_SETS;  // 22
  static constexpr int THREADS = (SF_PRODUCER_WARP + 1) * 32;
  static constexpr int GROUP_M = 8;                   // in 256-row tiles
  static constexpr int SF_REGIONS = STAGES;           // one TMEM scale region per pipeline stage
  static constexpr int SF_COLS = 48;                  // A: 16 columns, B: 32 columns per K-tile
  static constexpr int TMEM_SF = BN;
  static constexpr int TMEM_COLS = 512;
  static_assert(SMEM_BYTES <= 232448, "shared memory");
  static_assert(BN + SF_REGIONS * SF_COLS <= TMEM_COLS, "TMEM budget");
};

template <bool LR, bool MX, bool SK = false>
__global__ void __launch_bounds__(PairCfg<LR>::THREADS, 1)
    gemm_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                     const __grid_constant__ CUtensorMap tmap_sfa, const __grid_constant__ CUtensorMap tmap_sfb,
                     const __grid_constant__ CUtensorMap tmap_c, const __grid_constant__ CUtensorMap tmap_lb,
                     const __grid_constant__ CUtensorMap tmap_thi, const __grid_constant__ CUtensorMap tmap_tlo,
                     int rank_lr, uint16_t* __restrict__ C, int64_t ldc, const float* __restrict__ a_gs,
                     const float* __restrict__ b_gs, int M, int N, int K, uint32_t* __restrict__ status,
                     uint32_t* __restrict__ piece_counters, float* __restrict__ piece_partials) {
  using Cfg = PairCfg<LR>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int R = Cfg::SF_REGIONS;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * Cfg::A_BYTES;
  uint8_t* sLB = sB + STAGES * Cfg::B_BYTES;            // LR: B's rows, then t / alpha hi and lo
  uint8_t* sTH = sLB + Cfg::LORA_BYTES / 3;
  uint8_t* sTL = sTH + Cfg::LORA_BYTES / 3;
  uint8_t* sSFA = sLB + Cfg::LORA_BYTES;
  uint8_t* sSFB = sSFA + STAGES * Cfg::SFA_BYTES;
  uint8_t* sC = sSFB + STAGES * Cfg::SFB_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sC + Cfg::C_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_full = empty + STAGES;
  uint64_t* sf_empty = sf_full + STAGES;
  uint64_t* sf_ready = sf_empty + STAGES;
  uint64_t* set_done = sf_ready + STAGES;  // [SF_SETS]: the four warps of a set (peer CTA)
  uint64_t* acc_full = set_done + Cfg::SF_SETS;
  uint64_t* acc_empty = acc_full + 1;
  uint64_t* drain = acc_empty + 1;
  uint64_t* lora_full = drain + 1;    // LR, leader: the tile's low-rank operands landed (both CTAs)
  uint64_t* lora_empty = lora_full + 1;  // LR, both CTAs: the low-rank MMAs completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lora_empty + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const int pair = static_cast<int>(cluster_id_x());
  const int npairs = static_cast<int>(num_clusters_x());
  const int k_atoms = (K + 63) / 64;
  const int k_tiles = (k_atoms + 3) / 4;
  const int num_m = (M + 2 * Cfg::BM - 1) / (2 * Cfg::BM);
  const int num_n = (N + Cfg::BN - 1) / Cfg::BN;
  const int num_tiles = num_m * num_n;
  // partial tiles (the stream-K part): a separate instantiation, launched when the
  // schedule uses them (never with the low-rank branch, which adds its term once per tile)
  const bool partial_tiles = SK && !LR && piece_partials != nullptr;
  const int n_items = pair_item_count(pair, npairs, num_tiles, k_tiles, partial_tiles);

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_full[s], 1);
      mbar_init(&sf_empty[s], 4);  // the four warps of the set that read the slot
    }
    for (int r = 0; r < R; ++r) mbar_init(&sf_ready[r], 5);  // 4 leader warps + 1 arrival from the peer
    for (int q = 0; q < Cfg::SF_SETS; ++q) mbar_init(&set_done[q], 4);
    mbar_init(acc_full, 1);
    mbar_init(acc_empty, 2 * Cfg::EPI_WARPS);
    mbar_init(drain, 1);
    mbar_init(lora_full, 1);
    mbar_init(lora_empty, 1);
    *abort_flag = 0u;
    fence_mbarrier_init();
  }
  if (warp == Cfg::MMA_WARP) {
    tmem_alloc_pair(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish_pair();
  }
  if (warp == Cfg::PRODUCER_WARP && lane == 0) {
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
    prefetch_tmap(&tmap_sfa);
    prefetch_tmap(&tmap_sfb);
    prefetch_tmap(&tmap_c);
    if (LR) {
      prefetch_tmap(&tmap_lb);
      prefetch_tmap(&tmap_thi);
      prefetch_tmap(&tmap_tlo);
    }
  }
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // set-up overlapped the previous kernel's tail; its outputs are visible from here
  // (the status word was cleared by a memset before the launch)
  grid_dependency_wait();

  if (warp == Cfg::PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- TMA producer (both CTAs) ----------------
      int issued_last[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_last[s] = -1;
      int kc = 0, it = 0;
      bool ok = true;
      for (; it < n_items && ok; ++it) {
        const PairItem item = pair_item(it, pair, npairs, num_tiles, k_tiles, partial_tiles);
        int tm, tn;
        tile_coords<Cfg::GROUP_M>(item.tile, num_m, num_n, tm, tn);
        if (LR) {
          // the tile's low-rank operands, once the previous tile's low-rank MMAs are done
          if (!mbar_wait_cluster(lora_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag, status,
                                 kErrWaitEmpty + 3)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(lora_full, 2u * Cfg::LORA_BYTES);
          const uint32_t lbar = mapa_shared(smem_u32(lora_full), 0u);
          tma_load_2d_pair(sLB, &tmap_lb, lbar, 0, tn * Cfg::BN + static_cast<int>(rank) * 128);
          tma_load_2d_pair(sTH, &tmap_thi, lbar, 0, tm * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM);
          tma_load_2d_pair(sTL, &tmap_tlo, lbar, 0, tm * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM);
        }
        for (int kt = item.kt0; kt < item.kt1; ++kt, ++kc) {
          const int s = kc % STAGES;
          const uint32_t ph = static_cast<uint32_t>(kc / STAGES) & 1u;
          if (!mbar_wait_cluster(&empty[s], ph ^ 1u, abort_flag, status, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (rank == 0) mbar_arrive_expect_tx(&full[s], 2u * (Cfg::A_BYTES + Cfg::B_BYTES));
          const uint32_t bar = mapa_shared(smem_u32(&full[s]), 0u);
          tma_load_2d_pair(sA + s * Cfg::A_BYTES, &tmap_a, bar, kt * Cfg::KTILE_BYTES,
                           tm * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM);
          tma_load_2d_pair(sB + s * Cfg::B_BYTES, &tmap_b, bar, kt * Cfg::KTILE_BYTES,
                           tn * Cfg::BN + static_cast<int>(rank) * 128);
          issued_last[s] = kc;
        }
      }
      if (*abort_flag) {
        for (int s = 0; s < STAGES; ++s)
          if (issued_last[s] >= 0) {
            const uint32_t par = static_cast<uint32_t>(issued_last[s] / STAGES) & 1u;
            if (rank == 0) mbar_wait_drain(&full[s], par, status);
          }
        if (LR && rank == 0 && it > 0) mbar_wait_drain(lora_full, static_cast<uint32_t>(it - 1) & 1u, status);
      }
    }
  } else if (warp == Cfg::MMA_WARP) {
    if (lane == 0 && rank == 0) {
      // ---------------- MMA issuer (leader CTA only) ----------------
      const uint32_t idesc = MX ? idesc_mxf4_e8m0(2 * Cfg::BM, Cfg::BN) : idesc_mxf4nvf4(2 * Cfg::BM, Cfg::BN);
      const uint32_t t_acc = tmem_base;
      const uint32_t acc_full_own = smem_u32(acc_full);
      bool ok = true;
      int kc = 0, it = 0;
      for (; it < n_items && ok; ++it) {
        const PairItem item = pair_item(it, pair, npairs, num_tiles, k_tiles, partial_tiles);
        if (!mbar_wait_cluster(acc_empty, (static_cast<uint32_t>(it) & 1u) ^ 1u, abort_flag, status,
                               kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (LR) {
          // D += (t / alpha)(B rows)^T, hi then lo: 256 x 256 x 16 BF16 MMAs over the rank
          if (!mbar_wait_cluster(lora_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, kErrWaitFull + 8)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t idesc_lr = idesc_bf16(2 * Cfg::BM, Cfg::BN);
          const uint32_t lb = smem_u32(sLB), th = smem_u32(sTH), tl = smem_u32(sTL);
          for (int kk = 0; kk < (rank_lr + 15) / 16; ++kk)
            mma_bf16_pair(t_acc, sdesc_kmajor_sw128(th + 32 * kk), sdesc_kmajor_sw128(lb + 32 * kk), idesc_lr,
                          kk != 0 ? 1u : 0u);
          for (int kk = 0; kk < (rank_lr + 15) / 16; ++kk)
            mma_bf16_pair(t_acc, sdesc_kmajor_sw128(tl + 32 * kk), sdesc_kmajor_sw128(lb + 32 * kk), idesc_lr, 1u);
          tc_commit_pair_both(smem_u32(lora_empty));
          // MMAs of different shapes on one accumulator are not ordered by issue: the
          // 256 x 256 x 64 FP4 MMAs may start only once these K = 16 MMAs have completed
          if (!mbar_wait_cluster(lora_empty, static_cast<uint32_t>(it) & 1u, abort_flag, status, kErrWaitFull + 9)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        for (int kt = item.kt0; kt < item.kt1; ++kt, ++kc) {
          const int s = kc % STAGES;
          const int r = s;
          // one wait per K-tile: the leader's scale warps arrive on sf_ready only after
          // they have also seen the stage's A/B bytes land on full[s]
          if (!mbar_wait_cluster(&sf_ready[r], static_cast<uint32_t>(kc / STAGES) & 1u, abort_flag, status,
                                 kErrWaitFull + 1)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int na = min(4, k_atoms - kt * 4);
          const uint32_t a_base = smem_u32(sA + s * Cfg::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * Cfg::B_BYTES);
          const uint32_t t_sf = tmem_base + Cfg::TMEM_SF + r * Cfg::SF_COLS;
          for (int j = 0; j < na; ++j) {
            if constexpr (MX)
              mma_mxf4_block32_pair(t_acc, sdesc_kmajor_sw128(a_base + 32 * j), sdesc_kmajor_sw128(b_base + 32 * j),
                                    idesc, t_sf + 4 * j, t_sf + 16 + 8 * j, (LR || kt != item.kt0 || j != 0) ? 1u : 0u);
            else
              mma_mxf4nvf4_pair(t_acc, sdesc_kmajor_sw128(a_base + 32 * j), sdesc_kmajor_sw128(b_base + 32 * j),
                                idesc, t_sf + 4 * j, t_sf + 16 + 8 * j, (LR || kt != item.kt0 || j != 0) ? 1u : 0u);
          }
          tc_commit_pair_both(smem_u32(&empty[s]));
        }
        if (!ok) break;
        tc_commit_pair_both(acc_full_own);
      }
      if (!ok) {
        tc_commit_pair(smem_u32(drain));
        mbar_wait_drain(drain, 0u, status);
      }
    }
  } else if (warp == Cfg::SF_PRODUCER_WARP) {
    if (lane == 0) {
      // ---------------- scale-factor producer (both CTAs) ----------------
      // Slot s is refilled as soon as the set that copied K-tile kc-STAGES has moved it to TMEM,
      // several K-tiles before the MMAs reach kc, so the scale copy is not on the
      // critical path of a stage's reload.
      int issued_last[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_last[s] = -1;
      int kc = 0;
      bool ok = true;
      for (int it = 0; it < n_items && ok; ++it) {
        const PairItem item = pair_item(it, pair, npairs, num_tiles, k_tiles, partial_tiles);
        int tm, tn;
        tile_coords<Cfg::GROUP_M>(item.tile, num_m, num_n, tm, tn);
        for (int kt = item.kt0; kt < item.kt1; ++kt, ++kc) {
          const int s = kc % STAGES;
          if (kc >= STAGES && !mbar_wait(&sf_empty[s], (static_cast<uint32_t>(kc / STAGES) & 1u) ^ 1u, abort_flag,
                                         status, kErrWaitEmpty + 1)) {
            ok = false;
            break;
          }
          // a K-tile's scales: four 64-value atoms (NVFP4) or two 128-value atoms (MXFP4)
          constexpr int kAtoms = MX ? 2 : 4;
          mbar_arrive_expect_tx(&sf_full[s], (Cfg::SFA_BYTES + Cfg::SFB_BYTES) * kAtoms / 4);
          tma_load_3d(sSFA + s * Cfg::SFA_BYTES, &tmap_sfa, &sf_full[s], 0, kt * kAtoms,
                      tm * 2 + static_cast<int>(rank));
          tma_load_3d(sSFB + s * Cfg::SFB_BYTES, &tmap_sfb, &sf_full[s], 0, kt * kAtoms, tn * 2);
          issued_last[s] = kc;
        }
      }
      if (*abort_flag)
        for (int s = 0; s < STAGES; ++s)
          if (issued_last[s] >= 0)
            mbar_wait_drain(&sf_full[s], static_cast<uint32_t>(issued_last[s] / STAGES) & 1u, status);
    }
  } else if (warp >= Cfg::SF_WARP0) {
    // ---------------- scale warps (both CTAs): shared memory -> TMEM ----------------
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);
    const int set = (warp - Cfg::SF_WARP0) >> 2;
    const uint32_t sf_ready_leader0 = mapa_shared(smem_u32(&sf_ready[0]), 0u);
    int kc = 0, handled = 0;
    bool ok = true;
    for (int it = 0; it < n_items && ok; ++it) {
      const PairItem item = pair_item(it, pair, npairs, num_tiles, k_tiles, partial_tiles);
      for (int kt = item.kt0; kt < item.kt1; ++kt, ++kc) {
        if (kc % Cfg::SF_SETS != set) continue;
        const int s = kc % STAGES;
        const int r = s;
        const uint32_t prev = (static_cast<uint32_t>(kc / STAGES) & 1u) ^ 1u;  // parity of K-tile kc-STAGES's phase
        // A parity wait is only sound when the barrier is at most one phase behind, and
        // the sets rotate: first see K-tile kc-STAGES through slot s (its set has read the
        // slot, so those scales had landed), then wait for kc's scales.
        if (kc >= STAGES &&
            !warp_wait(&sf_empty[s], prev, abort_flag, status, kErrWaitFull + 3)) {
          ok = false;
          break;
        }
        if (!warp_wait(&sf_full[s], static_cast<uint32_t>(kc / STAGES) & 1u, abort_flag, status, kErrWaitFull + 2)) {
          ok = false;
          break;
        }
        const uint8_t* fa = sSFA + s * Cfg::SFA_BYTES + lane * 16;
        const uint8_t* fb = sSFB + s * Cfg::SFB_BYTES + lane * 16;
        uint32_t va[16], vb[32];
        if constexpr (MX) {
          // MXFP4: an atom covers two MMAs (K = 128); MMA j reads its two block-32 scale
          // bytes from the low half of its words (scale-factor id 0)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int sh = 16 * (j & 1);
            const uint4 a4 = *reinterpret_cast<const uint4*>(fa + (j >> 1) * Cfg::SF_ATOM);
            va[4 * j] = (a4.x >> sh) & 0xFFFFu;
            va[4 * j + 1] = (a4.y >> sh) & 0xFFFFu;
            va[4 * j + 2] = (a4.z >> sh) & 0xFFFFu;
            va[4 * j + 3] = (a4.w >> sh) & 0xFFFFu;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const uint4 b4 = *reinterpret_cast<const uint4*>(fb + (g * 2 + (j >> 1)) * Cfg::SF_ATOM);
              vb[8 * j + 4 * g] = (b4.x >> sh) & 0xFFFFu;
              vb[8 * j + 4 * g + 1] = (b4.y >> sh) & 0xFFFFu;
              vb[8 * j + 4 * g + 2] = (b4.z >> sh) & 0xFFFFu;
              vb[8 * j + 4 * g + 3] = (b4.w >> sh) & 0xFFFFu;
            }
          }
        } else {
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 a4 = *reinterpret_cast<const uint4*>(fa + j * Cfg::SF_ATOM);
            va[4 * j] = a4.x;
            va[4 * j + 1] = a4.y;
            va[4 * j + 2] = a4.z;
            va[4 * j + 3] = a4.w;
#pragma unroll
            for (int g = 0; g < 2; ++g) {
              const uint4 b4 = *reinterpret_cast<const uint4*>(fb + (g * 4 + j) * Cfg::SF_ATOM);
              vb[8 * j + 4 * g] = b4.x;
              vb[8 * j + 4 * g + 1] = b4.y;
              vb[8 * j + 4 * g + 2] = b4.z;
              vb[8 * j + 4 * g + 3] = b4.w;
            }
          }
        }
        // TMEM region r is free once the MMAs of K-tile kc-STAGES have completed
        if (kc >= STAGES && !warp_wait_cluster(&empty[s], prev, abort_flag, status, kErrWaitFull + 4)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t t_sf = tmem_base + (quarter * 32u << 16) + Cfg::TMEM_SF + r * Cfg::SF_COLS;
        tmem_st_32x32b_x16(t_sf, va);
        tmem_st_32x32b_x32(t_sf + 16, vb);
        tmem_st_wait();
        // Only now may the slot be refilled: the TMEM stores consumed every value this
        // warp loaded from it.  Releasing the slot right after issuing the loads let a
        // load still queued behind other memory traffic (the epilogue's stores) return
        // the next K-tile's scales, written by the refill.
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_empty[s]);
        if (rank == 0 && !warp_wait_cluster(&full[s], static_cast<uint32_t>(kc / STAGES) & 1u, abort_flag, status,
                                            kErrWaitFull)) {
          ok = false;
          break;
        }
        tc_fence_before();
        __syncwarp();
        if (rank == 0) {
          if (lane == 0) mbar_arrive(&sf_ready[r]);
        } else {
          if (lane == 0) mbar_arrive(&set_done[set]);
          // All four warps wait for the phase: a warp that went on to its next K-tile
          // without waiting could arrive inside this phase and complete it while a
          // slower warp of the set has not yet written its lanes.
          if (!warp_wait(&set_done[set], static_cast<uint32_t>(handled & 1), abort_flag, status,
                         kErrWaitFull + 5)) {
            ok = false;
            break;
          }
          if (quarter == static_cast<uint32_t>(set & 3) && lane == 0)  // one warp of the set
            mbar_arrive_cluster(sf_ready_leader0 + r * 8u);
        }
        ++handled;
      }
    }
  } else {
    // ---------------- epilogue (warps 0-7, both CTAs) ----------------
    constexpr int HALF = Cfg::BN / 2;
    const int quarter = warp & 3, half = warp >> 2;
    const float alpha = MX ? 1.0f : __fmul_rn(*a_gs, *b_gs);  // MXFP4 has no per-tensor scales
    const uint32_t t_lane = tmem_base + (static_cast<uint32_t>(quarter * 32) << 16) + half * HALF;
    const uint32_t acc_empty_leader = mapa_shared(smem_u32(acc_empty), 0u);
    uint8_t* box = sC + warp * Cfg::C_BOX_BYTES;
    bool stored = false;
    for (int it = 0; it < n_items; ++it) {
      const PairItem item = pair_item(it, pair, npairs, num_tiles, k_tiles, partial_tiles);
      int tm, tn;
      tile_coords<Cfg::GROUP_M>(item.tile, num_m, num_n, tm, tn);
      if (!warp_wait_cluster(acc_full, static_cast<uint32_t>(it) & 1u, abort_flag, status, kErrWaitAccFull)) break;
      tc_fence_after();
      // A shared tile (two pieces): the first piece to get here stores its FP32 partial
      // sums and raises a flag; the second waits for the flag and adds them to its own,
      // mine + other (FP32 addition commutes, so the sum does not depend on which piece
      // came first), then writes C.  A warp's part is its 32 rows x 128 columns, stored
      // as [column / 4][row][4] so that each store or load of the warp covers 512
      // contiguous bytes; slot, piece, CTA and warp select the part.
      constexpr size_t kPart = 32 * HALF;
      const bool split = partial_tiles && item.slot >= 0;
      bool first = false;
      float* part = nullptr;  // the first piece: its own part; the second: the other's
      const int entry = (item.slot * 2 + static_cast<int>(rank)) * 8 + warp;
      if (split) {
        uint32_t before = 0;
        if (lane == 0) before = atomicAdd(&piece_counters[entry], 1u);
        first = __shfl_sync(0xFFFFFFFFu, before, 0) == 0u;
        const int pc = first ? item.piece : 1 - item.piece;
        part = piece_partials + ((static_cast<size_t>(item.slot) * 2 + pc) * 2 + rank) * 8 * kPart +
               static_cast<size_t>(warp) * kPart;
        if (!first) {
          bool got = true;
          if (lane == 0) got = wait_flag(&piece_counters[kPairFlagOffset + entry], abort_flag, status, kErrWaitPiece);
          if (!__shfl_sync(0xFFFFFFFFu, got, 0)) break;
          __threadfence();
        }
      }
      if (split && first) {
#pragma unroll
        for (int c = 0; c < HALF; c += 32) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(t_lane + c, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            *reinterpret_cast<uint4*>(part + ((c / 4 + i) * 32 + lane) * 4) =
                make_uint4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(acc_empty);
          else
            mbar_arrive_cluster_relaxed(acc_empty_leader);
        }
        __threadfence();
        __syncwarp();
        if (lane == 0) atomicExch(&piece_counters[kPairFlagOffset + entry], 1u);
        continue;
      }
      if (split) {
        const int row0 = tm * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM + quarter * 32;
        const int col0 = tn * Cfg::BN + half * HALF;
        // the second piece: 32 columns at a time, the other piece's sums loaded before the
        // accumulator's (so that the loads overlap), summed, scaled, rounded to BF16 and
        // staged as in the whole-tile store below
#pragma unroll
        for (int chunk = 0; chunk < 2; ++chunk) {
          if (stored) {
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
#pragma unroll
          for (int sub = 0; sub < 2; ++sub) {
            const int c = chunk * 64 + sub * 32;
            float4 o[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) o[i] = __ldcg(reinterpret_cast<const float4*>(part) + (c / 4 + i) * 32 + lane);
            uint32_t v[32];
            tmem_ld_32x32b_x32(t_lane + c, v);
            tmem_ld_wait();
#pragma unroll
            for (int uu = 0; uu < 4; ++uu) {
              const float4 x = o[2 * uu], y = o[2 * uu + 1];
              const uint32_t* m = v + 8 * uu;
              const uint4 w = make_uint4(
                  pack_bf16x2(__fmul_rn(__fadd_rn(__uint_as_float(m[0]), x.x), alpha),
                              __fmul_rn(__fadd_rn(__uint_as_float(m[1]), x.y), alpha)),
                  pack_bf16x2(__fmul_rn(__fadd_rn(__uint_as_float(m[2]), x.z), alpha),
                              __fmul_rn(__fadd_rn(__uint_as_float(m[3]), x.w), alpha)),
                  pack_bf16x2(__fmul_rn(__fadd_rn(__uint_as_float(m[4]), y.x), alpha),
                              __fmul_rn(__fadd_rn(__uint_as_float(m[5]), y.y), alpha)),
                  pack_bf16x2(__fmul_rn(__fadd_rn(__uint_as_float(m[6]), y.z), alpha),
                              __fmul_rn(__fadd_rn(__uint_as_float(m[7]), y.w), alpha)));
              const int u = sub * 4 + uu;  // row `lane`, 16-byte unit u goes to u ^ (lane % 8)
              *reinterpret_cast<uint4*>(box + lane * 128 + ((u ^ (lane & 7)) << 4)) = w;
            }
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && col0 + chunk * 64 < N) {
            tma_store_2d(&tmap_c, box, col0 + chunk * 64, row0);
            bulk_commit_group();
          }
          stored = true;
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (rank == 0)
            mbar_arrive(acc_empty);
          else
            mbar_arrive_cluster_relaxed(acc_empty_leader);
        }
        continue;
      }
      uint32_t p[HALF / 2];
#pragma unroll
      for (int c = 0; c < HALF; c += 32) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(t_lane + c, v);
        tmem_ld_wait();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          p[c / 2 + i] = pack_bf16x2(__fmul_rn(__uint_as_float(v[2 * i]), alpha),
                                     __fmul_rn(__uint_as_float(v[2 * i + 1]), alpha));
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        if (rank == 0)
          mbar_arrive(acc_empty);
        else
          mbar_arrive_cluster_relaxed(acc_empty_leader);
      }
      const int row0 = tm * 2 * Cfg::BM + static_cast<int>(rank) * Cfg::BM + quarter * 32;
      const int col0 = tn * Cfg::BN + half * HALF;
      if constexpr (LR) {
        // four 32 x 32 boxes per warp, 64-byte swizzle: 16-byte unit u of row `lane` goes to
        // u ^ ((lane / 2) % 4)
#pragma unroll
        for (int chunk = 0; chunk < 4; ++chunk) {
          if (stored) {  // the previous TMA store from this box must have read it
            if (lane == 0) bulk_wait_read_all();
            __syncwarp();
          }
#pragma unroll
          for (int u = 0; u < 4; ++u) {
            const int q = chunk * 16 + 4 * u;
            *reinterpret_cast<uint4*>(box + lane * 64 + ((u ^ ((lane >> 1) & 3)) << 4)) =
                make_uint4(p[q], p[q + 1], p[q + 2], p[q + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0 && row0 < M && col0 + chunk * 32 < N) {
            tma_store_2d(&tmap_c, box, col0 + chunk * 32, row0);
            bulk_commit_group();
          }
          stored = true;
        }
      } else {
#pragma unroll
      for (int chunk = 0; chunk < 2; ++chunk) {
        // the previous TMA store from this box must have read it
        if (stored) {
          if (lane == 0) bulk_wait_read_all();
          __syncwarp();
        }
        // row `lane` of the 32 x 64 box, 128-byte swizzle: 16-byte unit u goes to u ^ (lane % 8)
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int q = chunk * 32 + 4 * u;
          const uint4 w = make_uint4(p[q], p[q + 1], p[q + 2], p[q + 3]);
          *reinterpret_cast<uint4*>(box + lane * 128 + ((u ^ (lane & 7)) << 4)) = w;
        }
        fence_proxy_async_smem();
        __syncwarp();
        if (lane == 0 && row0 < M && col0 + chunk * 64 < N) {
          tma_store_2d(&tmap_c, box, col0 + chunk * 64, row0);
          bulk_commit_group();
        }
        stored = true;
      }
      }
    }
    if (lane == 0) bulk_wait_all();
  }

  // Both CTAs stay until the pair's last remote arrival and MMA are done.
  tc_fence_before();
  __syncwarp();
  cluster_sync();
  if (warp == Cfg::MMA_WARP) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// Decode kernel (M <= 32): weights on the 128-row side of the MMA, stream-K
// ---------------------------------------------------------------------------------------------
//
// For a handful of activation rows the GEMM is a stream over the weights, so the
// weight matrix B takes the MMA's 128-row A slot (D^T = B A^T, 128 x 32 x 64 per
// instruction).  The stream is split evenly over the CTAs: the K-tiles of all
// 128-row weight tiles form one sequence of units, tile-major, and CTA c takes units
// [c U / G, (c+1) U / G).  When the tiles number between 70 % and 100 % of the SMs,
// G is the tile count and every CTA takes one whole tile; otherwise G is the SM
// count and every SM streams the same number of weight bytes whatever the number of
// tiles.  A CTA's range can cross tile boundaries; its part of one tile is a
// "segment" with its own accumulator, and TMEM holds two accumulators so that the
// MMAs of a segment overlap the epilogue of the one before.  A CTA works through its
// partial segments first and its whole tiles last, so that the reductions of the
// partial tiles overlap the streaming instead of trailing it.  A segment that
// covers a whole tile writes C.  Otherwise it stores its FP32 partial tile; the
// segment of the tile that finishes last (atomic counter) sums the tile's partials
// in segment order -- the result does not depend on arrival order -- applies
// s_gA s_gB and writes C (transposed back) in BF16, then clears the counter for
// the next call.
//
// Scale factors reach TMEM through "scale warps" (tcgen05.st of each lane's 16-byte
// atom lines into a per-stage region, as in the pair kernel), not through
// tcgen05.cp: two copies per 128 x 32 x 64 MMA made the in-order tensor pipe, not
// HBM, the limit.  The MMA issuer waits on one barrier per K-tile.
//
// QX (the activation quantized inside the GEMM, "NVFP4 en difusión ...", section 2:
// the activation is quantized on every call, per 16-block, absmax): instead of
// loading the activation's codes and scales, the scale warps quantize its BF16
// K-tile themselves.  Two groups of four warps take alternate K-tiles; in a group,
// warp q encodes K-quarter q (four blocks of each row) of the rows that exist (rows
// past M stay zero), reading the values from global memory (the activation is at
// most 32 rows and stays in L2) one K-tile ahead, writes the codes into the stage's
// B tile in the MMA's K-major 128-byte-swizzled layout and the scale bytes into a
// small per-stage array, gathers the group's scale words on an mbarrier, and then
// moves the stage's scales to TMEM.  The arithmetic is the quantizer's absmax path,
// operation for operation.

template <bool QX, bool LR = false>
struct DecodeCfg {
  static constexpr int BM = 128;                 // weight rows per tile
  static constexpr int BN = 32;                  // activation rows (padded)
  static constexpr int KTILE_BYTES = 128;
  static constexpr int A_BYTES = BM * KTILE_BYTES;   // 16 KB of weight codes
  static constexpr int B_BYTES = BN * KTILE_BYTES;   // 4 KB of activation codes
  static constexpr int SF_ATOM = 512;
  static constexpr int SFA_BYTES = 4 * SF_ATOM;
  // activation scales: 4 loaded atoms, or (QX) one 32-bit word per row and atom
  static constexpr int SFB_BYTES = QX ? 4 * BN * 4 : 4 * SF_ATOM;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES + SFA_BYTES + SFB_BYTES;
  static constexpr int STAGES = 8;
  static constexpr int TABLE_BYTES = QX ? static_cast<int>(sizeof(ScaleTables)) : 0;
  // LR (low-rank branch): the weight tile's rows of B (128 x R) and t / alpha as hi and
  // lo BF16 parts (32 x R each), K-major 128-byte rows (rank up to 64)
  static constexpr int LB_BYTES = LR ? BM * 128 : 0;
  static constexpr int LT_BYTES = LR ? BN * 128 : 0;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + LB_BYTES + 2 * LT_BYTES + TABLE_BYTES + 512;
  static constexpr int SF_WARP0 = 6;
  static constexpr int SF_GROUPS = QX ? 2 : 1;   // groups of four scale (quantizer) warps
  static constexpr int THREADS = (SF_WARP0 + 4 * SF_GROUPS) * 32;  // 0-3 epilogue, 4 producer, 5 MMA
  static constexpr int TMEM_ACC = 0;             // two accumulators of 32 columns
  static constexpr int TMEM_SF = 64;             // one scale region of 32 columns per stage
  static constexpr int TMEM_COLS = 512;
  static_assert(TMEM_SF + STAGES * 32 <= TMEM_COLS, "TMEM budget");
  static_assert(SMEM_BYTES <= 232448, "shared memory");
};

// Largest decode grid (SM count) the workspace query provisions partial-tile slots for.
constexpr int kMaxDecodeGrid = 296;

// The CTA whose unit range [c U / G, (c+1) U / G) holds unit u.
__host__ __device__ inline int64_t decode_cta_of_unit(int64_t u, int64_t U, int64_t G) {
  int64_t c = u * G / U;  // floor(c U / G) <= u for this c
  while (c + 1 < G && (c + 1) * U / G <= u) ++c;
  return c;
}

// Segments a tile of KT units can be cut into when every CTA holds at least
// U / G units (the partial-tile slots per tile in the workspace).
__host__ __device__ inline int64_t decode_max_segments(int64_t KT, int64_t U, int64_t G) {
  const int64_t per = U / G < 1 ? 1 : U / G;
  const int64_t s = (KT - 1) / per + 2;
  return s < KT ? s : KT;
}

// Segment k of a CTA's unit range [u0, u1) in processing order -- the partial
// segments first (the head of the last tile, then the tail of the first), then the
// whole tiles in order.  Returns false when the range has fewer segments.
__device__ __forceinline__ bool decode_segment(int k, int64_t u0, int64_t u1, int64_t KT, int64_t& s0,
                                               int64_t& s1) {
  if (u0 >= u1) return false;
  const int64_t t0 = u0 / KT, t1 = (u1 - 1) / KT;
  if (t0 == t1) {
    s0 = u0;
    s1 = u1;
    return k == 0;
  }
  const bool first_whole = (u0 % KT) == 0, last_whole = (u1 % KT) == 0;
  int np = 0;
  if (!last_whole) {
    if (k == np) {
      s0 = t1 * KT;
      s1 = u1;
      return true;
    }
    ++np;
  }
  if (!first_whole) {
    if (k == np) {
      s0 = u0;
      s1 = (t0 + 1) * KT;
      return true;
    }
    ++np;
  }
  const int64_t w0 = first_whole ? t0 : t0 + 1, w1 = last_whole ? t1 : t1 - 1;  // whole tiles [w0, w1]
  const int64_t t = w0 + (k - np);
  if (t > w1) return false;
  s0 = t * KT;
  s1 = s0 + KT;
  return true;
}

// The activation's global scale inside a QX launch: the caller's, or RN32(amax / 2688)
// from the amax pass (1 for an all-zero activation) -- the quantizer's rule.
__device__ __forceinline__ float decode_x_scale(const float* x_gs_in, const uint32_t* x_amax) {
  return global_scale(x_gs_in, x_amax);
}

template <bool QX, bool LR, bool MX>
__global__ void __launch_bounds__(DecodeCfg<QX, LR>::THREADS)
    gemm_decode_kernel(const __grid_constant__ CUtensorMap tmap_w, const __grid_constant__ CUtensorMap tmap_x,
                       const __grid_constant__ CUtensorMap tmap_lb, const __grid_constant__ CUtensorMap tmap_thi,
                       const __grid_constant__ CUtensorMap tmap_tlo, int rank,
                       const uint8_t* __restrict__ sf_w, const uint8_t* __restrict__ sf_x,
                       const float* __restrict__ a_gs, const float* __restrict__ b_gs,
                       const uint16_t* __restrict__ xq, int64_t ld_x, const float* __restrict__ x_gs_in,
                       const uint32_t* __restrict__ x_amax, uint16_t* __restrict__ C, int M, int N, int K,
                       int64_t ldc, int max_seg, float* __restrict__ partial, uint32_t* __restrict__ counters,
                       uint32_t* __restrict__ status) {
  using Cfg = DecodeCfg<QX, LR>;
  constexpr int STAGES = Cfg::STAGES;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  // every 128-byte-swizzled tile (A, B, the low-rank operands) starts on a 1024-byte boundary
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * Cfg::A_BYTES;
  uint8_t* sLB = sB + STAGES * Cfg::B_BYTES;
  uint8_t* sTH = sLB + Cfg::LB_BYTES;
  uint8_t* sTL = sTH + Cfg::LT_BYTES;
  uint8_t* sSFA = sTL + Cfg::LT_BYTES;
  uint8_t* sSFB = sSFA + STAGES * Cfg::SFA_BYTES;
  ScaleTables* tab = reinterpret_cast<ScaleTables*>(sSFB + STAGES * Cfg::SFB_BYTES);
  uint64_t* full = reinterpret_cast<uint64_t*>(sSFB + STAGES * Cfg::SFB_BYTES + Cfg::TABLE_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* sf_ready = empty + STAGES;
  uint64_t* qdone = sf_ready + STAGES;     // [STAGES]: a quantizer group's scale words
  uint64_t* acc_full = qdone + STAGES;     // [2]
  uint64_t* acc_empty = acc_full + 2;      // [2]
  uint64_t* drain = acc_empty + 2;
  uint64_t* lora_full = drain + 1;         // LR: the low-rank operands of a tile landed
  uint64_t* lora_empty = lora_full + 1;    // LR: their MMAs completed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(lora_empty + 1);
  volatile uint32_t* abort_flag = tmem_slot + 1;
  volatile uint32_t* decision = tmem_slot + 2;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int k_atoms = (K + 63) / 64;
  const int64_t KT = (k_atoms + 3) / 4;
  const int64_t T = (N + Cfg::BM - 1) / Cfg::BM;
  const int64_t U = T * KT;
  const int64_t G = gridDim.x;
  const int64_t u0 = static_cast<int64_t>(blockIdx.x) * U / G;
  const int64_t u1 = (static_cast<int64_t>(blockIdx.x) + 1) * U / G;

  // A unit's loads: its weight part (the 128-row weight tile's K-tile and scale atoms,
  // plus the stage's byte count for the whole unit) and its activation part.
  auto issue_weight = [&](int s, int64_t u) {
    const int tile = static_cast<int>(u / KT), kt = static_cast<int>(u - tile * KT);
    // scale atoms of the K-tile: four of 64 values (NVFP4) or two of 128 values (MXFP4)
    constexpr int kAtoms = MX ? 2 : 4;
    const int sf_atoms = MX ? (K + 127) / 128 : k_atoms;
    const int ka0 = kt * kAtoms;
    const uint32_t sf_bytes = static_cast<uint32_t>(min(kAtoms, sf_atoms - ka0)) * Cfg::SF_ATOM;
    if constexpr (QX) {
      mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + sf_bytes);
    } else {
      mbar_arrive_expect_tx(&full[s], Cfg::A_BYTES + Cfg::B_BYTES + 2 * sf_bytes);
    }
    tma_load_2d(sA + s * Cfg::A_BYTES, &tmap_w, &full[s], kt * Cfg::KTILE_BYTES, tile * Cfg::BM);
    bulk_load(sSFA + s * Cfg::SFA_BYTES, sf_w + (static_cast<size_t>(tile) * sf_atoms + ka0) * Cfg::SF_ATOM, sf_bytes,
              &full[s]);
  };
  auto issue_act = [&](int s, int64_t u) {
    if constexpr (!QX) {
      const int kt = static_cast<int>(u % KT);
      constexpr int kAtoms = MX ? 2 : 4;
      const int sf_atoms = MX ? (K + 127) / 128 : k_atoms;
      const int ka0 = kt * kAtoms;
      const uint32_t sf_bytes = static_cast<uint32_t>(min(kAtoms, sf_atoms - ka0)) * Cfg::SF_ATOM;
      tma_load_2d(sB + s * Cfg::B_BYTES, &tmap_x, &full[s], kt * Cfg::KTILE_BYTES, 0);
      bulk_load(sSFB + s * Cfg::SFB_BYTES, sf_x + static_cast<size_t>(ka0) * Cfg::SF_ATOM, sf_bytes, &full[s]);
    }
  };
  // The producer thread initialises the barriers and, right away, requests the first
  // stages' weight parts (the weights do not come from the kernels this one is
  // launched behind), while the other warps allocate TMEM; the activation parts
  // follow after the dependency wait.
  int pre = 0;
  int64_t pre_u[STAGES];
  if (warp == 4 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
      mbar_init(&sf_ready[s], 4);  // lane 0 of each warp of the scale group
      mbar_init(&qdone[s], 4);
    }
    mbar_init(lora_full, 1);
    mbar_init(lora_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);  // lane 0 of each epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0u;
    fence_mbarrier_init();
    prefetch_tmap(&tmap_w);
    if (!QX) prefetch_tmap(&tmap_x);
    if (LR) {
      prefetch_tmap(&tmap_lb);
      prefetch_tmap(&tmap_thi);
      prefetch_tmap(&tmap_tlo);
    }
    int64_t s0, s1;
    for (int sg = 0; pre < STAGES && decode_segment(sg, u0, u1, KT, s0, s1); ++sg)
      for (int64_t u = s0; u < s1 && pre < STAGES; ++u, ++pre) {
        issue_weight(pre, u);
        pre_u[pre] = u;
      }
  }
  if (QX) {
    // activation rows past M are never written: their codes and scale words stay zero
    for (int i = threadIdx.x; i < STAGES * (Cfg::B_BYTES + Cfg::SFB_BYTES) / 16; i += blockDim.x) {
      const int off = i * 16;
      uint8_t* p = off < STAGES * Cfg::B_BYTES ? sB + off : sSFB + (off - STAGES * Cfg::B_BYTES);
      *reinterpret_cast<uint4*>(p) = make_uint4(0u, 0u, 0u, 0u);
    }
    fence_proxy_async_smem();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, Cfg::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;

  // set-up overlapped the previous kernel's tail; its outputs are visible from here
  // (the status word and tile counters were cleared by the memset launched before)
  grid_dependency_wait();

  if (warp == 4) {
    if (lane == 0) {
      // ---------------- producer ----------------
      int64_t issued_last[STAGES];
#pragma unroll
      for (int s = 0; s < STAGES; ++s) issued_last[s] = s < pre ? s : -1;
      int64_t i = 0, s0, s1;
      bool ok = true;
      int lora_uses = 0;
      for (int sg = 0; ok && decode_segment(sg, u0, u1, KT, s0, s1); ++sg) {
        if (LR && s0 % KT == 0) {
          // the segment that starts the tile's K loop also adds the low-rank term: B's rows
          // of this tile and t / alpha (hi, lo), values past the rank and rows past M as zeros
          if (!mbar_wait(lora_empty, (static_cast<uint32_t>(lora_uses) & 1u) ^ 1u, abort_flag, status,
                         kErrWaitEmpty + 3)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(lora_full, Cfg::LB_BYTES + 2 * Cfg::LT_BYTES);
          tma_load_2d(sLB, &tmap_lb, lora_full, 0, static_cast<int>(s0 / KT) * Cfg::BM);
          tma_load_2d(sTH, &tmap_thi, lora_full, 0, 0);
          tma_load_2d(sTL, &tmap_tlo, lora_full, 0, 0);
          ++lora_uses;
        }
        for (int64_t u = s0; u < s1; ++u, ++i) {
          const int s = static_cast<int>(i % STAGES);
          if (i >= pre) {  // (units below `pre` have their weight part in flight already)
            if (!mbar_wait(&empty[s], (static_cast<uint32_t>(i / STAGES) & 1u) ^ 1u, abort_flag, status,
                           kErrWaitEmpty)) {
              ok = false;
              break;
            }
            issue_weight(s, u);
          }
          issue_act(s, u);
          issued_last[s] = i;
        }
      }
      if (*abort_flag) {
        // a stage whose weight part went out before the wait completes only with its
        // activation part: send the ones the loop did not reach, then let every copy land
        for (int64_t j = i; j < pre; ++j) issue_act(static_cast<int>(j), pre_u[j]);
        for (int s = 0; s < STAGES; ++s)
          if (issued_last[s] >= 0)
            mbar_wait_drain(&full[s], static_cast<uint32_t>(issued_last[s] / STAGES) & 1u, status);
        if (LR && lora_uses > 0) mbar_wait_drain(lora_full, static_cast<uint32_t>(lora_uses - 1) & 1u, status);
      }
    }
  } else if (warp == 5) {
    if (lane == 0) {
      // ---------------- MMA issuer ----------------
      const uint32_t idesc = MX ? idesc_mxf4_e8m0(Cfg::BM, Cfg::BN) : idesc_mxf4nvf4(Cfg::BM, Cfg::BN);
      bool ok = true;
      int64_t i = 0, s0, s1;
      int lora_uses = 0;
      for (int q = 0; ok && decode_segment(q, u0, u1, KT, s0, s1); ++q) {
        const int buf = q & 1;
        if (q >= 2) {
          if (!mbar_wait(&acc_empty[buf], static_cast<uint32_t>((q >> 1) - 1) & 1u, abort_flag, status,
                         kErrWaitAccEmpty)) {
            ok = false;
            break;
          }
          tc_fence_after();
        }
        const uint32_t t_acc = tmem_base + Cfg::TMEM_ACC + buf * Cfg::BN;
        bool lora_in = false;
        if (LR && s0 % KT == 0) {
          // D^T += B_rows (t/alpha)^T in two parts, hi then lo: 128 x 32 x 16 BF16 MMAs over the rank
          if (!mbar_wait(lora_full, static_cast<uint32_t>(lora_uses) & 1u, abort_flag, status, kErrWaitFull + 8)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t idesc_lr = idesc_bf16(Cfg::BM, Cfg::BN);
          const uint32_t lb = smem_u32(sLB), th = smem_u32(sTH), tl = smem_u32(sTL);
          for (int kk = 0; kk < (rank + 15) / 16; ++kk)
            mma_bf16(t_acc, sdesc_kmajor_sw128(lb + 32 * kk), sdesc_kmajor_sw128(th + 32 * kk), idesc_lr,
                     kk != 0 ? 1u : 0u);
          for (int kk = 0; kk < (rank + 15) / 16; ++kk)
            mma_bf16(t_acc, sdesc_kmajor_sw128(lb + 32 * kk), sdesc_kmajor_sw128(tl + 32 * kk), idesc_lr, 1u);
          tc_commit(lora_empty);
          // MMAs of different shapes on one accumulator are not ordered by issue: the
          // 128 x 32 x 64 FP4 MMAs may start only once these K = 16 MMAs have completed
          if (!mbar_wait(lora_empty, static_cast<uint32_t>(lora_uses) & 1u, abort_flag, status, kErrWaitFull + 9)) {
            ok = false;
            break;
          }
          tc_fence_after();
          ++lora_uses;
          lora_in = true;
        }
        for (int64_t u = s0; u < s1; ++u, ++i) {
          const int kt = static_cast<int>(u % KT);
          const int s = static_cast<int>(i % STAGES);
          // the scale warps arrive only after the stage's bytes landed and its scales are in TMEM
          if (!mbar_wait(&sf_ready[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, status, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const int na = min(4, k_atoms - kt * 4);
          const uint32_t a_base = smem_u32(sA + s * Cfg::A_BYTES);
          const uint32_t b_base = smem_u32(sB + s * Cfg::B_BYTES);
          const uint32_t t_sf = tmem_base + Cfg::TMEM_SF + static_cast<uint32_t>(s) * 32;
          for (int j = 0; j < na; ++j) {
            if constexpr (MX)
              mma_mxf4_block32(t_acc, sdesc_kmajor_sw128(a_base + 32 * j), sdesc_kmajor_sw128(b_base + 32 * j), idesc,
                               t_sf + 4 * j, t_sf + 16 + 4 * j, (lora_in || u != s0 || j != 0) ? 1u : 0u);
            else
              mma_mxf4nvf4(t_acc, sdesc_kmajor_sw128(a_base + 32 * j), sdesc_kmajor_sw128(b_base + 32 * j), idesc,
                           t_sf + 4 * j, t_sf + 16 + 4 * j, (lora_in || u != s0 || j != 0) ? 1u : 0u);
          }
          tc_commit(&empty[s]);
        }
        if (!ok) break;
        tc_commit(&acc_full[buf]);
      }
      if (!ok) {
        tc_commit(drain);
        mbar_wait_drain(drain, 0u, status);
      }
    }
  } else if (warp >= Cfg::SF_WARP0) {
    // ---------------- scale warps: shared memory -> TMEM region of the stage ----------------
    // Each lane writes its 16-byte line of every atom to the four columns the MMA reads
    // for its 32-lane sub-partition (the 4-way replication of the scale layout).  The
    // region of stage s is free once the stage's bytes land again: the producer
    // reloads a stage only after the MMAs that read it have completed.
    const uint32_t quarter = static_cast<uint32_t>(warp & 3);
    const int group = (warp - Cfg::SF_WARP0) >> 2;
    float d6 = 0.0f;
    // QX work items of a unit for this warp: (row, block) = (it / 4, it % 4) of its
    // K-quarter, it = lane + 32 j over the M rows that exist (at most 4 per lane)
    const int items = QX ? M * 4 : 0;
    uint4 xv[4][2];  // the next unit's values: item j, 16 BF16 values as two 16-byte halves
    auto load_unit = [&](int64_t u) {
      const int kt = static_cast<int>(u % KT);
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int it = lane + 32 * j;
        const int row = it >> 2, blk = it & 3;
        const int k0 = kt * 256 + static_cast<int>(quarter) * 64 + blk * 16;
        if (it < items && k0 < K) {
          const uint4* p = reinterpret_cast<const uint4*>(xq + static_cast<int64_t>(row) * ld_x + k0);
          xv[j][0] = __ldcg(p);
          xv[j][1] = __ldcg(p + 1);
        } else {
          xv[j][0] = make_uint4(0u, 0u, 0u, 0u);
          xv[j][1] = make_uint4(0u, 0u, 0u, 0u);
        }
      }
    };
    int64_t i = 0, s0, s1, next_u = -1;
    if (QX) {
      // the first unit of this group
      int64_t a0, a1;
      for (int sg = 0, ii = 0; decode_segment(sg, u0, u1, KT, a0, a1); ++sg) {
        if (a1 - a0 + ii > group) {
          next_u = a0 + (group - ii);
          break;
        }
        ii += static_cast<int>(a1 - a0);
      }
      if (next_u >= 0) load_unit(next_u);
    }
    if constexpr (QX) {
      // the activation's per-tensor scale and the 127 decoded scales, as the quantizer builds them
      const float sg = decode_x_scale(x_gs_in, x_amax);
      d6 = __fmul_rn(6.0f, sg);
      const int t = threadIdx.x - Cfg::SF_WARP0 * 32;
      if (t < 128) {
        const float eff = __fmul_rn(e4m3_to_float(static_cast<uint32_t>(t)), sg);
        tab->eff[t] = eff;
        tab->rcp[t] = eff == 0.0f ? 0.0f : __frcp_rn(eff);
      }
      asm volatile("bar.sync 2, %0;" ::"n"(4 * Cfg::SF_GROUPS * 32) : "memory");  // the table is complete
    }
    bool ok = true;
    for (int sg = 0; ok && decode_segment(sg, u0, u1, KT, s0, s1); ++sg) {
      for (int64_t u = s0; u < s1; ++u, ++i) {
        if (static_cast<int>(i % Cfg::SF_GROUPS) != group) continue;
        const int s = static_cast<int>(i % STAGES);
        uint32_t v[32];
        if constexpr (QX) {
          uint4 cur[4][2];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            cur[j][0] = xv[j][0];
            cur[j][1] = xv[j][1];
          }
          // prefetch this group's next unit (the one SF_GROUPS units later in processing order)
          {
            int64_t nu = -1, ii = 0, a0, a1;
            for (int g2 = 0; decode_segment(g2, u0, u1, KT, a0, a1); ++g2) {
              const int64_t want = i + Cfg::SF_GROUPS;
              if (want < ii + (a1 - a0)) {
                if (want >= ii) nu = a0 + (want - ii);
                break;
              }
              ii += a1 - a0;
            }
            if (nu >= 0) load_unit(nu);
          }
          // the MMAs of unit i - STAGES are done, so the stage's B tile and TMEM region are
          // free: the activation is encoded while the unit's weights are still in flight
          if (!warp_wait(&empty[s], (static_cast<uint32_t>(i / STAGES) & 1u) ^ 1u, abort_flag, status,
                         kErrWaitFull + 9)) {
            ok = false;
            break;
          }
          uint32_t* words = reinterpret_cast<uint32_t*>(sSFB + s * Cfg::SFB_BYTES);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int it = lane + 32 * j;
            uint32_t sb = 0;
            if (32 * j < items) {  // warp-uniform: the warp has items in this round
              const uint32_t wd[8] = {cur[j][0].x, cur[j][0].y, cur[j][0].z, cur[j][0].w,
                                      cur[j][1].x, cur[j][1].y, cur[j][1].z, cur[j][1].w};
              uint64_t x2[8];
              uint32_t mb = 0;
#pragma unroll
              for (int k = 0; k < 8; ++k) {
                x2[k] = pack2(__uint_as_float(wd[k] << 16), __uint_as_float(wd[k] & 0xFFFF0000u));
                mb = __vmaxu2(mb, wd[k] & 0x7FFF7FFFu);
              }
              const float amax_b = bf16_bits_to_float(max(mb & 0xFFFFu, mb >> 16));
              sb = cvt_e4m3_satfinite(__fdiv_rn(amax_b, d6));
              uint32_t c0, c1;
              encode_codes(x2, tab->eff[sb], tab->rcp[sb], c0, c1);
              const int row = it >> 2, blk = it & 3;
              if (it < items) {
                // K bytes [32 quarter + 8 blk, +8) of row `row` in the K-major 128-byte-swizzled
                // B tile: 16-byte chunk 2 quarter + blk / 2, swizzled by the row
                const int chunk = (2 * static_cast<int>(quarter) + (blk >> 1)) ^ (row & 7);
                *reinterpret_cast<uint2*>(sB + s * Cfg::B_BYTES + row * 128 + chunk * 16 + (blk & 1) * 8) =
                    make_uint2(c0, c1);
              }
              // the row's four scale bytes of this K-quarter come from lanes 4r .. 4r+3
              const uint32_t b1 = __shfl_down_sync(0xFFFFFFFFu, sb, 1);
              const uint32_t b2 = __shfl_down_sync(0xFFFFFFFFu, sb, 2);
              const uint32_t b3 = __shfl_down_sync(0xFFFFFFFFu, sb, 3);
              if (it < items && blk == 0) words[quarter * 32 + row] = sb | (b1 << 8) | (b2 << 16) | (b3 << 24);
            }
          }
          fence_proxy_async_smem();  // the codes are read by the MMA (async proxy)
          __syncwarp();
          if (lane == 0) mbar_arrive(&qdone[s]);
          if (!warp_wait(&qdone[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, status, kErrWaitFull + 7)) {
            ok = false;
            break;
          }
          // the weight scales of the unit landed
          if (!warp_wait(&full[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, status, kErrWaitFull + 2)) {
            ok = false;
            break;
          }
          const uint8_t* fa = sSFA + s * Cfg::SFA_BYTES + lane * 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint4 a4 = *reinterpret_cast<const uint4*>(fa + j * Cfg::SF_ATOM);
            v[4 * j] = a4.x;
            v[4 * j + 1] = a4.y;
            v[4 * j + 2] = a4.z;
            v[4 * j + 3] = a4.w;
            // the atom line of lane L holds rows L, L+32, L+64, L+96: only row L exists
            v[16 + 4 * j] = words[j * 32 + lane];
            v[16 + 4 * j + 1] = 0u;
            v[16 + 4 * j + 2] = 0u;
            v[16 + 4 * j + 3] = 0u;
          }
        } else {
          if (!warp_wait(&full[s], static_cast<uint32_t>(i / STAGES) & 1u, abort_flag, status, kErrWaitFull + 2)) {
            ok = false;
            break;
          }
          const uint8_t* fa = sSFA + s * Cfg::SFA_BYTES + lane * 16;
          const uint8_t* fb = sSFB + s * Cfg::SFB_BYTES + lane * 16;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            // MXFP4: atom j / 2 serves MMAs j and j + 1; MMA j's two block-32 scale bytes
            // go to the low half of its words (scale-factor id 0)
            const int sh = MX ? 16 * (j & 1) : 0;
            const uint32_t keep = MX ? 0xFFFFu : 0xFFFFFFFFu;
            const uint4 a4 = *reinterpret_cast<const uint4*>(fa + (MX ? (j >> 1) : j) * Cfg::SF_ATOM);
            const uint4 b4 = *reinterpret_cast<const uint4*>(fb + (MX ? (j >> 1) : j) * Cfg::SF_ATOM);
            v[4 * j] = (a4.x >> sh) & keep;
            v[4 * j + 1] = (a4.y >> sh) & keep;
            v[4 * j + 2] = (a4.z >> sh) & keep;
            v[4 * j + 3] = (a4.w >> sh) & keep;
            v[16 + 4 * j] = (b4.x >> sh) & keep;
            v[16 + 4 * j + 1] = (b4.y >> sh) & keep;
            v[16 + 4 * j + 2] = (b4.z >> sh) & keep;
            v[16 + 4 * j + 3] = (b4.w >> sh) & keep;
          }
        }
        tc_fence_after();
        tmem_st_32x32b_x32(tmem_base + (quarter * 32u << 16) + Cfg::TMEM_SF + static_cast<uint32_t>(s) * 32, v);
        tmem_st_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(&sf_ready[s]);
      }
    }
  } else {
    // ---------------- epilogue (warps 0-3): lane = weight row n, 32 columns = activation rows m ----------------
    const float alpha = MX ? 1.0f  // MXFP4 has no per-tensor scales
                           : (QX ? __fmul_rn(decode_x_scale(x_gs_in, x_amax), *b_gs) : __fmul_rn(*a_gs, *b_gs));
    int64_t s0, s1;
    for (int q = 0; decode_segment(q, u0, u1, KT, s0, s1); ++q) {
      const int tile = static_cast<int>(s0 / KT);
      const int64_t tile_end = (static_cast<int64_t>(tile) + 1) * KT;
      const bool whole = (s0 == static_cast<int64_t>(tile) * KT) && s1 == tile_end;
      const int buf = q & 1;
      const bool got = warp_wait(&acc_full[buf], static_cast<uint32_t>(q >> 1) & 1u, abort_flag, status,
                                 kErrWaitAccFull);
      uint32_t v[32];
      if (got) {
        tc_fence_after();
        tmem_ld_32x32b_x32(tmem_base + (static_cast<uint32_t>(warp * 32) << 16) + Cfg::TMEM_ACC + buf * Cfg::BN, v);
        tmem_ld_wait();
        tc_fence_before();
      }
      __syncwarp();
      if (got && lane == 0) mbar_arrive(&acc_empty[buf]);
      // one decision for the four warps: go on only if none of them gave up
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (threadIdx.x == 0) *decision = *abort_flag ? 0u : 1u;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      const bool go = *decision == 1u;
      asm volatile("bar.sync 1, 128;" ::: "memory");
      if (!go) break;
      const int n = tile * Cfg::BM + warp * 32 + lane;
      if (whole) {
        if (n < N)
          for (int m = 0; m < M; ++m)
            C[static_cast<int64_t>(m) * ldc + n] =
                __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(__uint_as_float(v[m]), alpha)));
      } else {
        const int64_t c_first = decode_cta_of_unit(static_cast<int64_t>(tile) * KT, U, G);
        const int64_t c_last = decode_cta_of_unit(tile_end - 1, U, G);
        const int seg = static_cast<int>(blockIdx.x - c_first);
        const int nseg = static_cast<int>(c_last - c_first + 1);
        float* slot = partial + ((static_cast<int64_t>(tile) * max_seg + seg) * Cfg::BM + warp * 32 + lane) * Cfg::BN;
        float4* dst = reinterpret_cast<float4*>(slot);
        const int mq = (M + 3) / 4;  // only the activation rows that exist are kept
        for (int i = 0; i < mq; ++i)
          dst[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]), __uint_as_float(v[4 * i + 2]),
                               __uint_as_float(v[4 * i + 3]));
        // the four warps' partial rows are ordered before thread 0's release by the
        // barrier; the segment that arrives last acquires every other segment's rows
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (threadIdx.x == 0)
          *decision = (atom_add_acq_rel_gpu(&counters[tile], 1u) == static_cast<uint32_t>(nseg - 1)) ? 2u : 1u;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        const bool last = *decision == 2u;
        asm volatile("bar.sync 1, 128;" ::: "memory");
        if (last) {
          float acc[32];
#pragma unroll
          for (int m = 0; m < 32; ++m) acc[m] = 0.0f;
          for (int sg = 0; sg < nseg; ++sg) {
            const float4* src = reinterpret_cast<const float4*>(
                partial + ((static_cast<int64_t>(tile) * max_seg + sg) * Cfg::BM + warp * 32 + lane) * Cfg::BN);
            for (int i = 0; i < mq; ++i) {
              const float4 f = __ldcg(src + i);
              acc[4 * i] = __fadd_rn(acc[4 * i], f.x);
              acc[4 * i + 1] = __fadd_rn(acc[4 * i + 1], f.y);
              acc[4 * i + 2] = __fadd_rn(acc[4 * i + 2], f.z);
              acc[4 * i + 3] = __fadd_rn(acc[4 * i + 3], f.w);
            }
          }
          if (n < N)
            for (int m = 0; m < M; ++m)
              C[static_cast<int64_t>(m) * ldc + n] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__fmul_rn(acc[m], alpha)));
          if (threadIdx.x == 0) counters[tile] = 0u;  // ready for the next call
        }
      }
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tmem_base, Cfg::TMEM_COLS);
  }
}

// ---------------------------------------------------------------------------------------------
// host side
// ---------------------------------------------------------------------------------------------

// Programmatic dependent launch: the kernel may start (and run its set-up) while
// the previous kernel on the stream finishes; it calls grid_dependency_wait()
// before touching anything that kernel writes.  The quantizer does not signal
// early, so a dependent GEMM starts only as the quantizer's last CTAs exit and
// never holds SMs its predecessor still needs.
void set_programmatic(cudaLaunchAttribute& a) {
  a.id = cudaLaunchAttributeProgrammaticStreamSerialization;
  a.val.programmaticStreamSerializationAllowed = 1;
}

// Decode workspace after the 256-byte status block: one counter per 128-row
// weight tile (rounded up to 256 bytes), then the FP32 partial tiles.
size_t decode_counter_bytes(int64_t N) { return static_cast<size_t>(((N + 127) / 128 * 4 + 255) / 256 * 256); }

using EncodeTiledFn = CUresult (*)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                   const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                   CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      p = nullptr;
    return reinterpret_cast<EncodeTiledFn>(p);
  }();
  return fn;
}

// Row-major rows x (K/2) bytes of packed codes, box = box_rows x 128 bytes, 128-byte swizzle.
bool encode_codes_map(CUtensorMap* map, const uint8_t* codes, int64_t rows, int64_t K, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(K / 2), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(K / 2)};
  const cuuint32_t box[2] = {128u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<uint8_t*>(codes), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// Swizzled scale buffer of `rows` rows viewed as [row groups][K atoms][128 words]:
// box = 4 atoms (one K-tile) x `groups` row groups.  Out-of-range atoms/groups read 0.
bool encode_sf_map(CUtensorMap* map, const uint8_t* sf, int64_t rows, int64_t K, int groups, bool mx = false) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  // an atom holds 4 scales per row: 64 values of K (NVFP4) or 128 (MXFP4); a K-tile of
  // 256 values is 4 or 2 atoms
  const int64_t k_atoms = mx ? (K + 127) / 128 : (K + 63) / 64;
  const int64_t row_groups = (rows + 127) / 128;
  const cuuint64_t dims[3] = {128u, static_cast<cuuint64_t>(k_atoms), static_cast<cuuint64_t>(row_groups)};
  const cuuint64_t strides[2] = {512u, static_cast<cuuint64_t>(k_atoms * 512)};
  const cuuint32_t box[3] = {128u, mx ? 2u : 4u, static_cast<cuuint32_t>(groups)};
  const cuuint32_t estr[3] = {1u, 1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_UINT32, 3, const_cast<uint8_t*>(sf), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool LR, bool MX, bool SK = false>
int max_pair_clusters(int dev) {
  using Cfg = PairCfg<LR>;
  static std::once_flag once[64];
  static int clusters[64];
  std::call_once(once[dev & 63], [&] {
    int n = 0;
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(2 * 148);
    cfg.blockDim = dim3(Cfg::THREADS);
    cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 2;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    if (cudaFuncSetAttribute(gemm_pair_kernel<LR, MX, SK>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             Cfg::SMEM_BYTES) != cudaSuccess ||
        cudaOccupancyMaxActiveClusters(&n, gemm_pair_kernel<LR, MX, SK>, &cfg) != cudaSuccess) {
      cudaGetLastError();
      n = 0;
    }
    clusters[dev & 63] = n;
  });
  return clusters[dev & 63];
}

// BF16 output matrix, row stride ldc elements; box = 32 rows x 64 columns, 128-byte swizzle.
// BF16 M x N output (row stride ldc), box = 32 rows x box_cols (64: 128-byte swizzle,
// 32: 64-byte swizzle).
bool encode_c_map(CUtensorMap* map, uint16_t* c, int64_t M, int64_t N, int64_t ldc, int box_cols = 64) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(N), static_cast<cuuint64_t>(M)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(ldc * 2)};
  const cuuint32_t box[2] = {static_cast<cuuint32_t>(box_cols), 32u};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, c, dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
             box_cols == 64 ? CU_TENSOR_MAP_SWIZZLE_128B : CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_NONE, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// BF16 rows x R matrix (row stride R elements, R <= 64): box = box_rows x 64 values
// (one 128-byte row per box row), 128-byte swizzle; values past R and rows past the
// last read as zero.  The low-rank operands (B's rows, t / alpha).
bool encode_bf16_rows_map(CUtensorMap* map, const uint16_t* base, int64_t rows, int64_t R, int box_rows) {
  EncodeTiledFn enc = encode_fn();
  if (!enc) return false;
  const cuuint64_t dims[2] = {static_cast<cuuint64_t>(R), static_cast<cuuint64_t>(rows)};
  const cuuint64_t strides[1] = {static_cast<cuuint64_t>(R * 2)};
  const cuuint32_t box[2] = {64u, static_cast<cuuint32_t>(box_rows)};
  const cuuint32_t estr[2] = {1u, 1u};
  return enc(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<uint16_t*>(base), dims, strides, box, estr,
             CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
             CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <bool LR, bool MX>
cudaError_t launch_pair(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                        uint16_t* c, int64_t ldc, uint32_t* status, const uint16_t* lora_b, const uint16_t* thi,
                        const uint16_t* tlo, int64_t rank, cudaStream_t stream, uint8_t* scratch = nullptr) {
  using Cfg = PairCfg<LR>;
  CUtensorMap ta, tb, tsa, tsb, tc, tlb, tth, ttl;
  if (!encode_codes_map(&ta, a_codes, M, K, 128) || !encode_codes_map(&tb, b_codes, N, K, 128) ||
      !encode_sf_map(&tsa, a_sf, M, K, 1, MX) || !encode_sf_map(&tsb, b_sf, N, K, 2, MX) ||
      !encode_c_map(&tc, c, M, N, ldc, Cfg::C_BOX_COLS))
    return cudaErrorInvalidValue;
  if (LR) {
    if (!encode_bf16_rows_map(&tlb, lora_b, N, rank, 128) || !encode_bf16_rows_map(&tth, thi, M, rank, 128) ||
        !encode_bf16_rows_map(&ttl, tlo, M, rank, 128))
      return cudaErrorInvalidValue;
  } else {
    tlb = tth = ttl = tc;  // unused slots
  }
  int dev = 0;
  cudaGetDevice(&dev);
  const int max_clusters = max_pair_clusters<LR, MX>(dev);
  if (max_clusters <= 0) return cudaErrorLaunchOutOfResources;
  const int64_t tiles = ((M + 255) / 256) * ((N + 255) / 256);
  const int clusters = static_cast<int>(tiles < max_clusters ? tiles : max_clusters);
  // partial tiles (the instantiation with the stream-K part) when the schedule uses them;
  // they need the counters (cleared before the launch) and the partial-tile slots
  const int k_tiles = static_cast<int>(((K + 63) / 64 + 3) / 4);
  bool sk = false;
  if constexpr (!LR && !MX)
    sk = scratch != nullptr && clusters <= kMaxPairSlots &&
         pair_sk_tiles(clusters, static_cast<int>(tiles), k_tiles, true) > 0 && max_pair_clusters<LR, MX, true>(dev) > 0;
  uint32_t* piece_counters = sk ? reinterpret_cast<uint32_t*>(scratch) : nullptr;
  float* piece_partials = sk ? reinterpret_cast<float*>(scratch + pair_counter_bytes()) : nullptr;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  set_programmatic(attr[1]);
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  if constexpr (!LR && !MX) {
    if (sk)
      return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<LR, MX, true>, ta, tb, tsa, tsb, tc, tlb, tth, ttl,
                                static_cast<int>(rank), c, ldc, a_gs, b_gs, static_cast<int>(M), static_cast<int>(N),
                                static_cast<int>(K), status, piece_counters, piece_partials);
  }
  return cudaLaunchKernelEx(&cfg, gemm_pair_kernel<LR, MX>, ta, tb, tsa, tsb, tc, tlb, tth, ttl, static_cast<int>(rank), c,
                            ldc, a_gs, b_gs, static_cast<int>(M), static_cast<int>(N), static_cast<int>(K), status,
                            piece_counters, piece_partials);
}

// CTAs of the decode kernel: one per weight tile when the tiles number between 70 %
// and 100 % of the SMs (no partial tiles), otherwise one per SM (at most one per unit).
int64_t decode_grid(int64_t N, int64_t K, int sms) {
  const int64_t T = (N + DecodeCfg<false>::BM - 1) / DecodeCfg<false>::BM;
  const int64_t U = T * ((K + 255) / 256);
  if (T <= sms && 10 * T >= 7 * static_cast<int64_t>(sms)) return T;  // one whole tile per CTA
  return U < sms ? U : sms;
}

// Launch the decode kernel: QX = false reads the activation's codes and scales
// (tmap_x over a_codes, a_sf, a_gs); QX = true quantizes the BF16 activation x (row
// stride ld_x) itself, global scale from x_gs_in or the amax word x_amax.
template <bool QX, bool LR, bool MX = false>
cudaError_t launch_decode(const CUtensorMap& tw, const CUtensorMap& tx, const CUtensorMap& tlb, const CUtensorMap& tthi,
                          const CUtensorMap& ttlo, int rank, const uint8_t* a_sf, const float* a_gs,
                          const uint16_t* x, int64_t ld_x, const float* x_gs_in, const uint32_t* x_amax, int64_t M,
                          const uint8_t* b_sf,
                          const float* b_gs, int64_t N, int64_t K, uint16_t* c, int64_t ldc, uint32_t* status,
                          uint8_t* scratch, cudaStream_t stream) {
  using Cfg = DecodeCfg<QX, LR>;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  std::call_once(once[dev & 63], [&] {
    attr_err[dev & 63] = cudaFuncSetAttribute(gemm_decode_kernel<QX, LR, MX>,
                                              cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err[dev & 63] != cudaSuccess) return attr_err[dev & 63];
  const int64_t KT = (K + 255) / 256;
  const int64_t U = ((N + Cfg::BM - 1) / Cfg::BM) * KT;
  const int64_t G = decode_grid(N, K, sms > kMaxDecodeGrid ? kMaxDecodeGrid : sms);
  const int max_seg = static_cast<int>(decode_max_segments(KT, U, G));
  // the counters were cleared together with the status word (gemm_zero_bytes)
  uint32_t* counters = reinterpret_cast<uint32_t*>(scratch);
  float* partial = reinterpret_cast<float*>(scratch + decode_counter_bytes(N));
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(G));
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_programmatic(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_decode_kernel<QX, LR, MX>, tw, tx, tlb, tthi, ttlo, rank, b_sf, a_sf, a_gs, b_gs,
                            x, ld_x, x_gs_in, x_amax, c, static_cast<int>(M), static_cast<int>(N),
                            static_cast<int>(K), ldc, max_seg, partial, counters, status);
}

template <int BN>
cudaError_t launch_tile(const CUtensorMap& ta, const CUtensorMap& tb, const uint8_t* a_sf, const uint8_t* b_sf,
                        const float* a_gs, const float* b_gs, int64_t M, int64_t N, int64_t K, uint16_t* c,
                        int64_t ldc, uint32_t* status, cudaStream_t stream) {
  using Cfg = GemmCfg<BN>;
  static std::once_flag once[64];
  static cudaError_t attr_err[64];
  int dev = 0;
  cudaGetDevice(&dev);
  // the attribute is set once per device; its result is kept, so a failure is
  // reported on every call, not only the first
  std::call_once(once[dev & 63], [&] {
    attr_err[dev & 63] =
        cudaFuncSetAttribute(gemm_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize, Cfg::SMEM_BYTES);
  });
  if (attr_err[dev & 63] != cudaSuccess) return attr_err[dev & 63];
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t tiles = ((M + Cfg::BM - 1) / Cfg::BM) * ((N + BN - 1) / BN);
  const unsigned grid = static_cast<unsigned>(tiles < sms ? tiles : sms);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(Cfg::THREADS);
  cfg.dynamicSmemBytes = Cfg::SMEM_BYTES;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  set_programmatic(attr[0]);
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, gemm_kernel<BN>, ta, tb, a_sf, b_sf, a_gs, b_gs, c, static_cast<int>(M),
                            static_cast<int>(N), static_cast<int>(K), ldc, status);
}

}  // namespace

size_t gemm_scratch_bytes(int64_t M, int64_t N, int64_t K) {
  using Cfg = DecodeCfg<false>;
  if (M <= Cfg::BN) {
    // partial-tile slots for the largest grid the launcher uses (more CTAs, more segments)
    const int64_t KT = (K + 255) / 256;
    const int64_t T = (N + Cfg::BM - 1) / Cfg::BM;
    const int64_t G = decode_grid(N, K, kMaxDecodeGrid);
    const int64_t max_seg = decode_max_segments(KT, T * KT, G);
    return decode_counter_bytes(N) + static_cast<size_t>(T * max_seg) * Cfg::BM * Cfg::BN * 4;
  }
  if (uses_pair_kernel(M, N)) return pair_counter_bytes() + pair_partial_bytes();
  return 0;
}

size_t gemm_counter_bytes(int64_t M, int64_t N, int64_t) {
  if (M <= DecodeCfg<false>::BN) return decode_counter_bytes(N);
  if (uses_pair_kernel(M, N)) return pair_counter_bytes();
  return 0;
}

size_t gemm_zero_bytes(int64_t M, int64_t N, int64_t K) {
  // the status word of every kernel (a clear inside the kernel could erase the
  // timeout code of a CTA that started earlier), plus the counters at the start of the
  // scratch that follows it (decode tiles, or the pair kernel's shared tiles)
  const size_t counters = gemm_counter_bytes(M, N, K);
  return counters > 0 ? 256 + counters : sizeof(uint32_t);
}

cudaError_t launch_gemm(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                        const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                        uint16_t* c, int64_t ldc, uint32_t* status, cudaStream_t stream, uint8_t* scratch) {
  if (M <= DecodeCfg<false>::BN) {
    CUtensorMap tw, tx;
    if (!encode_codes_map(&tw, b_codes, N, K, 128) || !encode_codes_map(&tx, a_codes, M, K, DecodeCfg<false>::BN))
      return cudaErrorInvalidValue;
    if (scratch == nullptr) scratch = reinterpret_cast<uint8_t*>(status) + 256;
    return launch_decode<false, false>(tw, tx, tw, tw, tw, 0, a_sf, a_gs, nullptr, 0, nullptr, nullptr, M, b_sf, b_gs,
                                       N, K, c, ldc, status, scratch, stream);
  }
  if (uses_pair_kernel(M, N))
    return launch_pair<false, false>(a_codes, a_sf, a_gs, M, b_codes, b_sf, b_gs, N, K, c, ldc, status, nullptr, nullptr,
                                     nullptr, 0, stream, scratch ? scratch : reinterpret_cast<uint8_t*>(status) + 256);
  const int bn = N > 128 ? 256 : 128;
  CUtensorMap ta, tb;
  if (!encode_codes_map(&ta, a_codes, M, K, 128) || !encode_codes_map(&tb, b_codes, N, K, bn))
    return cudaErrorInvalidValue;
  if (bn == 256) return launch_tile<256>(ta, tb, a_sf, b_sf, a_gs, b_gs, M, N, K, c, ldc, status, stream);
  return launch_tile<128>(ta, tb, a_sf, b_sf, a_gs, b_gs, M, N, K, c, ldc, status, stream);
}

cudaError_t launch_decode_quantize_x(const uint16_t* x, int64_t M, int64_t K, int64_t ld_x, const float* x_gs_in,
                                     const uint32_t* x_amax, const uint8_t* b_codes, const uint8_t* b_sf,
                                     const float* b_gs, int64_t N, uint16_t* c, int64_t ldc, uint32_t* status,
                                     uint8_t* scratch, cudaStream_t stream) {
  CUtensorMap tw;
  if (!encode_codes_map(&tw, b_codes, N, K, 128)) return cudaErrorInvalidValue;
  // (the activation is read with plain loads; the unused tensor-map slots repeat tw)
  return launch_decode<true, false>(tw, tw, tw, tw, tw, 0, nullptr, nullptr, x, ld_x, x_gs_in, x_amax, M, b_sf, b_gs,
                                    N, K, c, ldc, status, scratch, stream);
}

cudaError_t launch_gemm_mx(const uint8_t* a_codes, const uint8_t* a_sf, int64_t M, const uint8_t* b_codes,
                           const uint8_t* b_sf, int64_t N, int64_t K, uint16_t* c, int64_t ldc, uint32_t* status,
                           cudaStream_t stream) {
  if (M <= DecodeCfg<false>::BN) {
    CUtensorMap tw, tx;
    if (!encode_codes_map(&tw, b_codes, N, K, 128) || !encode_codes_map(&tx, a_codes, M, K, DecodeCfg<false>::BN))
      return cudaErrorInvalidValue;
    return launch_decode<false, false, true>(tw, tx, tw, tw, tw, 0, a_sf, nullptr, nullptr, 0, nullptr, nullptr, M,
                                             b_sf, nullptr, N, K, c, ldc, status,
                                             reinterpret_cast<uint8_t*>(status) + 256, stream);
  }
  return launch_pair<false, true>(a_codes, a_sf, nullptr, M, b_codes, b_sf, nullptr, N, K, c, ldc, status, nullptr,
                                  nullptr, nullptr, 0, stream);
}

cudaError_t launch_gemm_lora(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                             const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                             uint16_t* c, int64_t ldc, uint32_t* status, const uint16_t* lora_b, const uint16_t* thi,
                             const uint16_t* tlo, int64_t R, cudaStream_t stream) {
  return launch_pair<true, false>(a_codes, a_sf, a_gs, M, b_codes, b_sf, b_gs, N, K, c, ldc, status, lora_b, thi, tlo, R,
                           stream);
}

cudaError_t launch_decode_lora(const uint8_t* a_codes, const uint8_t* a_sf, const float* a_gs, int64_t M,
                               const uint8_t* b_codes, const uint8_t* b_sf, const float* b_gs, int64_t N, int64_t K,
                               const uint16_t* lora_b, const uint16_t* thi, const uint16_t* tlo, int64_t R,
                               uint16_t* c, int64_t ldc, uint32_t* status, uint8_t* scratch, cudaStream_t stream) {
  using Cfg = DecodeCfg<false, true>;
  CUtensorMap tw, tx, tlb, tth, ttl;
  if (!encode_codes_map(&tw, b_codes, N, K, 128) || !encode_codes_map(&tx, a_codes, M, K, Cfg::BN) ||
      !encode_bf16_rows_map(&tlb, lora_b, N, R, 128) || !encode_bf16_rows_map(&tth, thi, M, R, Cfg::BN) ||
      !encode_bf16_rows_map(&ttl, tlo, M, R, Cfg::BN))
    return cudaErrorInvalidValue;
  return launch_decode<false, true>(tw, tx, tlb, tth, ttl, static_cast<int>(R), a_sf, a_gs, nullptr, 0, nullptr,
                                    nullptr, M, b_sf, b_gs, N, K, c, ldc, status, scratch, stream);
}

}  // namespace nvfp4
