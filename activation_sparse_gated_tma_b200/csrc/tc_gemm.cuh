// Persistent tcgen05 GEMM engine for sm_100a.
//
//   D[m][n] = sum_k A[m][k] * B[n][k]      (B K-major:  B stored [N][K] row-major)
//   D[m][n] = sum_k A[m][k] * B[k][n]      (B MN-major: B stored [K][N] row-major)
//
// A is always K-major ([M][K] row-major bf16).  DUAL runs a second B operand
// through the same A tile into a second accumulator (used for gate+up).
//
// One CTA per SM, 192 threads:
//   warp 0      TMA producer (one elected lane) filling a STAGES-deep smem ring
//   warp 1      TMEM allocator + single-thread tcgen05.mma issuer
//   warps 2..   epilogue (4 or 8 warps, Epi::kWarps): thread i of warp w owns
//               TMEM lane 32*(w%4)+i, i.e. one output row of the 128-row tile
//               (with 8 warps, two warps share a row and split its columns);
//               per tile it runs Epi::prepare (before the accumulator is
//               ready) and Epi::run.
// Accumulators are double-buffered in TMEM so the epilogue of tile i overlaps
// the MMAs of tile i+1.  Every wait is bounded (see mbar_wait).
#pragma once

#include <cuda.h>

#include "ptx.cuh"

namespace twell {

constexpr int kBM = 128;      // UMMA M (rows per tile, = TMEM lanes)
constexpr int kBK = 64;       // bf16 elements per 128-byte swizzle row
constexpr int kUmmaK = 16;    // K per tcgen05.mma kind::f16
// Threads of a CTA: warp 0 (TMA), warp 1 (TMEM + MMA) and the epilogue warps.
template <class Epi, int BN>
constexpr int gemm_threads() {
  return 64 + 32 * Epi::template kWarps<BN>;
}

struct GemmGeom {
  int M;                    // rows of A and D
  int N;                    // columns of D
  int K;                    // reduction length (multiple of kBK)
  const int* m_limit;       // optional: only rows < min(M, *m_limit) are computed
  int group_m;              // rasterisation: tiles walk group_m row blocks per column sweep
  int b_k_wrap;             // if > 0, B's k-block index is kb % b_k_wrap (A = [A0 | A1] against B twice)
  int k_splits;             // >= 1: the reduction is cut into k_splits slices, each its own tile;
                            // < 0: as many slices (at most -k_splits) as keep the live tiles
                            // (rows below *m_limit) within one pass of the grid
};

template <int BN, bool DUAL>
struct GemmSmem {
  static constexpr int kABytes = kBM * kBK * 2;
  static constexpr int kBBytes = BN * kBK * 2;
  static constexpr int kStageBytes = kABytes + kBBytes * (DUAL ? 2 : 1);
  static constexpr int kAccCols = BN * (DUAL ? 2 : 1);
  static constexpr int kTmemCols = (2 * kAccCols <= 32) ? 32 : (2 * kAccCols <= 64) ? 64 : (2 * kAccCols <= 128) ? 128 : (2 * kAccCols <= 256) ? 256 : 512;
  static_assert(2 * kAccCols <= 512, "two accumulators must fit in TMEM");
  static_assert(kStageBytes % 1024 == 0, "stages must keep 1024-byte swizzle-atom alignment");
};

// Shared memory of one CTA: the operand ring, the barriers, and EPI_SCRATCH
// bytes of private scratch for each of the EPI_WARPS epilogue warps.
template <int BN, bool DUAL, int STAGES, int EPI_SCRATCH, int EPI_WARPS>
constexpr size_t gemm_smem_bytes() {
  return 1024 /*alignment slack*/ + static_cast<size_t>(STAGES) * GemmSmem<BN, DUAL>::kStageBytes +
         (2 * STAGES + 4) * sizeof(uint64_t) + 16 + 128 + EPI_WARPS * static_cast<size_t>(EPI_SCRATCH);
}

__device__ __forceinline__ void tile_coords(int tile, int num_m, int num_n, int group_m, int& mb, int& nb) {
  const int per_group = group_m * num_n;
  const int grp = tile / per_group;
  const int first_m = grp * group_m;
  const int gm = min(group_m, num_m - first_m);
  const int r = tile - grp * per_group;
  mb = first_m + r % gm;
  nb = r / gm;
}

template <int BN, bool B_MN, bool DUAL, int STAGES, class Epi>
__global__ void __launch_bounds__(gemm_threads<Epi, BN>(), 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                   const __grid_constant__ CUtensorMap tmB2, const GemmGeom g, const typename Epi::Params ep,
                   int* ctrl) {
  using L = GemmSmem<BN, DUAL>;
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "UMMA N for M=128 must be a multiple of 16 up to 256");
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * L::kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  uint8_t* epi_scratch = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tmem_holder + 4) + 127) & ~uintptr_t(127));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], 32 * Epi::template kWarps<BN>);
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(tmem_holder, L::kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  // Everything above overlaps the tail of the previous kernel in the stream
  // (programmatic dependent launch); global memory is touched only below.
  griddep_launch_dependents();
  griddep_wait();

  int m_rows = g.M;
  if (g.m_limit) m_rows = min(m_rows, *g.m_limit);
  const int num_m = (m_rows + kBM - 1) / kBM;
  const int num_n = (g.N + BN - 1) / BN;
  const int num_mn = num_m * num_n;
  const int total_kb = g.K / kBK;
  int k_splits = g.k_splits > 1 ? g.k_splits : 1;
  if (g.k_splits < 0) {
    k_splits = num_mn > 0 ? static_cast<int>(gridDim.x) / num_mn : 1;
    k_splits = max(1, min(k_splits, -g.k_splits));
  }
  const int kb_per_split = (total_kb + k_splits - 1) / k_splits;
  k_splits = (total_kb + kb_per_split - 1) / kb_per_split;  // no empty slice
  const int num_tiles = num_mn * k_splits;

  if (warp == 0) {
    if (lane == 0 && num_tiles > blockIdx.x) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      if (DUAL) prefetch_tmap(&tmB2);
      int stage = 0;
      uint32_t phase = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x) {
        int mb, nb;
        tile_coords(tile % num_mn, num_m, num_n, g.group_m, mb, nb);
        const int kb0 = (tile / num_mn) * kb_per_split;
        const int kb1 = min(total_kb, kb0 + kb_per_split);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, ctrl)) { ok = false; break; }
          uint8_t* sa = smem + stage * L::kStageBytes;
          uint8_t* sb = sa + L::kABytes;
          mbar_arrive_expect_tx(&full[stage], L::kStageBytes);
          tma_load_2d(&tmA, &full[stage], sa, kb * kBK, mb * kBM);
          const int kbb = g.b_k_wrap > 0 ? kb % g.b_k_wrap : kb;
          if (!B_MN) {
            tma_load_2d(&tmB, &full[stage], sb, kbb * kBK, nb * BN);
            if (DUAL) tma_load_2d(&tmB2, &full[stage], sb + L::kBBytes, kbb * kBK, nb * BN);
          } else {
#pragma unroll
            for (int j = 0; j < BN / 64; ++j) {
              tma_load_2d(&tmB, &full[stage], sb + j * 8192, nb * BN + j * 64, kbb * kBK);
              if (DUAL) tma_load_2d(&tmB2, &full[stage], sb + L::kBBytes + j * 8192, nb * BN + j * 64, kbb * kBK);
            }
          }
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_bf16_f32(kBM, BN, false, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, ctrl)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * L::kAccCols;
        const int kb0 = (tile / num_mn) * kb_per_split;
        const int kb1 = min(total_kb, kb0 + kb_per_split);
        bool ok = true;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctrl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * L::kStageBytes);
          const uint32_t b_base = a_base + L::kABytes;
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k) {
            const uint64_t adesc = smem_desc_sw128(a_base + k * 32, 16, 1024);
            const uint64_t bdesc = B_MN ? smem_desc_sw128(b_base + k * 2048, 8192, 1024)
                                        : smem_desc_sw128(b_base + k * 32, 16, 1024);
            const uint32_t accum = (kb > kb0 || k > 0) ? 1u : 0u;
            umma_bf16(d, adesc, bdesc, idesc, accum);
            if (DUAL) {
              const uint32_t b2 = b_base + L::kBBytes;
              const uint64_t bdesc2 =
                  B_MN ? smem_desc_sw128(b2 + k * 2048, 8192, 1024) : smem_desc_sw128(b2 + k * 32, 16, 1024);
              umma_bf16(d + BN, adesc, bdesc2, idesc, accum);
            }
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&tfull[acc]);
      }
    }
  } else {
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    const int row_in_tile = q * 32 + lane;
    // With eight epilogue warps every quadrant has two; `part` says which half
    // of the tile's columns (as the epilogue divides them) this warp takes.
    constexpr int kParts = Epi::template kWarps<BN> / 4;
    const int part = (warp - 2) >> 2;
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      int mb, nb;
      tile_coords(tile % num_mn, num_m, num_n, g.group_m, mb, nb);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      // Loads that do not depend on the accumulator are issued while the MMAs run.
      typename Epi::template Pre<BN> pre;
      Epi::template prepare<BN>(ep, pre, mb * kBM + row_in_tile, m_rows, nb);
      if (!mbar_wait(&tfull[acc], acc_phase, ctrl)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * L::kAccCols;
      Epi::template run<BN>(ep, pre, taddr, mb * kBM + row_in_tile, m_rows, nb, lane, ctrl,
                            epi_scratch + (warp - 2) * Epi::kScratchBytes, part, kParts);
      tc_fence_before();
      mbar_arrive(&tempty[acc]);
    }
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, L::kTmemCols);
}

// ---------------------------------------------------------------------------
// Two-CTA variant for K-major A and B: a cluster of two CTAs (one per SM)
// computes each 256 x 256 tile with cta_group::2 UMMA (M = 256).  Rank r loads
// its own 128 rows of A and its own 128 columns of B (no multicast): the pair
// moves 2/3 of the operand bytes per FLOP of a one-CTA 128 x 256 tile, which
// matters because the one-CTA engine is bound by the L2 -> SM operand rate,
// not by the tensor pipe.  Both CTAs' loads complete on the leader's (rank 0)
// full barrier; the leader's single MMA thread issues the UMMAs and its
// commits reach the empty / accumulator-full barriers of both CTAs.  Each CTA's
// epilogue reads its own TMEM (its 128 rows, all 256 columns) and arrives on
// the leader's accumulator-empty barrier.
template <int STAGES, int EPI_SCRATCH, int EPI_WARPS>
constexpr size_t gemm_pair_smem_bytes() {
  return 1024 + static_cast<size_t>(STAGES) * 2 * kBM * kBK * 2 + (2 * STAGES + 4) * sizeof(uint64_t) + 16 + 128 +
         EPI_WARPS * static_cast<size_t>(EPI_SCRATCH);
}

template <int STAGES, class Epi>
__global__ void __launch_bounds__(gemm_threads<Epi, 256>(), 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                        const GemmGeom g, const typename Epi::Params ep, int* ctrl) {
  constexpr int BN = 256;                   // tile columns (both CTAs); each CTA holds BN / 2 of B
  constexpr int kABytes = kBM * kBK * 2;    // this CTA's 128 rows of A
  constexpr int kBBytes = kBM * kBK * 2;    // this CTA's 128 columns of B
  constexpr int kStageBytes = kABytes + kBBytes;
  constexpr uint32_t kAccCols = BN;
  constexpr uint32_t kTmemCols = 2 * kAccCols;
  constexpr int kEpiWarps = Epi::template kWarps<BN>;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + STAGES * kStageBytes);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint32_t* tmem_holder = reinterpret_cast<uint32_t*>(tempty + 2);
  uint8_t* epi_scratch = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tmem_holder + 4) + 127) & ~uintptr_t(127));

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;

  if (warp == 0 && lane == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);   // used in the leader: its producer's expect_tx + both CTAs' bytes
      mbar_init(&empty[s], 1);  // both CTAs: the leader's commit
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);                   // both CTAs: the leader's commit
      mbar_init(&tempty[a], 2 * 32 * kEpiWarps);  // used in the leader: both CTAs' epilogue threads
    }
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(tmem_holder, kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // the peer's barriers exist before any arrival reaches them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_holder;

  griddep_launch_dependents();
  griddep_wait();

  int m_rows = g.M;
  if (g.m_limit) m_rows = min(m_rows, *g.m_limit);
  const int num_m = (m_rows + 2 * kBM - 1) / (2 * kBM);
  const int num_n = (g.N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int total_kb = g.K / kBK;
  const int cluster = static_cast<int>(blockIdx.x >> 1);
  const int nclusters = static_cast<int>(gridDim.x >> 1);

  if (warp == 0) {
    if (lane == 0 && num_tiles > cluster) {
      prefetch_tmap(&tmA);
      prefetch_tmap(&tmB);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters) {
        int mb, nb;
        tile_coords(tile, num_m, num_n, g.group_m, mb, nb);
        for (int kb = 0; kb < total_kb; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1u, ctrl)) { ok = false; break; }
          if (leader) mbar_arrive_expect_tx(&full[stage], 2 * kStageBytes);
          const uint32_t bar = mapa_shared(&full[stage], 0);
          uint8_t* sa = smem + stage * kStageBytes;
          tma_load_2d_pair(&tmA, bar, sa, kb * kBK, mb * 2 * kBM + static_cast<int>(rank) * kBM);
          tma_load_2d_pair(&tmB, bar, sa + kABytes, kb * kBK, nb * BN + static_cast<int>(rank) * kBM);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && leader) {
      constexpr uint32_t idesc = idesc_bf16_f32(2 * kBM, BN, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int tile = cluster; tile < num_tiles && ok; tile += nclusters, ++it) {
        const int acc = it & 1;
        const uint32_t acc_phase = (it >> 1) & 1;
        if (!mbar_wait(&tempty[acc], acc_phase ^ 1u, ctrl)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * kAccCols;
        for (int kb = 0; kb < total_kb; ++kb) {
          if (!mbar_wait(&full[stage], phase, ctrl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(smem + stage * kStageBytes);
          const uint32_t b_base = a_base + kABytes;
#pragma unroll
          for (int k = 0; k < kBK / kUmmaK; ++k)
            umma_bf16_pair(d, smem_desc_sw128(a_base + k * 32, 16, 1024), smem_desc_sw128(b_base + k * 32, 16, 1024),
                           idesc, (kb > 0 || k > 0) ? 1u : 0u);
          umma_commit_pair(&empty[stage]);
          if (++stage == STAGES) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit_pair(&tfull[acc]);
      }
    }
  } else {
    const int q = warp & 3;
    const int row_in_tile = q * 32 + lane;
    constexpr int kParts = kEpiWarps / 4;
    const int part = (warp - 2) >> 2;
    const uint32_t tempty_leader0 = mapa_shared(&tempty[0], 0);
    const uint32_t tempty_leader1 = mapa_shared(&tempty[1], 0);
    int it = 0;
    for (int tile = cluster; tile < num_tiles; tile += nclusters, ++it) {
      int mb, nb;
      tile_coords(tile, num_m, num_n, g.group_m, mb, nb);
      const int acc = it & 1;
      const uint32_t acc_phase = (it >> 1) & 1;
      const int row = mb * 2 * kBM + static_cast<int>(rank) * kBM + row_in_tile;
      typename Epi::template Pre<BN> pre;
      Epi::template prepare<BN>(ep, pre, row, m_rows, nb);
      if (!mbar_wait(&tfull[acc], acc_phase, ctrl)) break;
      __syncwarp();
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * kAccCols;
      Epi::template run<BN>(ep, pre, taddr, row, m_rows, nb, lane, ctrl,
                            epi_scratch + (warp - 2) * Epi::kScratchBytes, part, kParts);
      tc_fence_before();
      mbar_arrive_cluster(acc ? tempty_leader1 : tempty_leader0);
    }
  }
  tc_fence_before();
  __syncthreads();
  cluster_sync();  // neither CTA leaves while its peer may still reach its shared memory
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, kTmemCols);
}

}  // namespace twell
