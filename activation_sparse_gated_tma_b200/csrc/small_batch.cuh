// Small-batch gate pass ("Sparser, Faster, Lighter Transformer Language
// Models", §3-4 steps 1-5 and §3-6, for batches of at most TWELL_SMALL_M rows).
//
// With few token rows the gate GEMM is a stream over W_g: every weight byte is
// used M times, so the pass is bound by reading W_g from HBM once.  The kernel
// below therefore puts W_g on the 128-row side of the tensor-core tile and the
// tokens on its narrow side:
//
//   D[n][m] = sum_k W_g^T[n][k] x[m][k]      (UMMA M = 128 hidden units, N = MP >= M tokens)
//
// and cuts the (128-unit tile, 64-wide k block) pairs into equal contiguous
// ranges, one per CTA (stream-K): every SM streams the same number of W_g
// bytes whatever N/128 is.  A CTA writes the partial sum of each tile piece it
// covers to a scratch slot; the last CTA to finish a TwELL tile (an atomic
// ticket, no waiting) adds the slots in a fixed order and packs the tile for
// all M rows, with the same records, order, counts and overflow routing as the
// gate GEMM's epilogue.
#pragma once

#include "epilogues.cuh"
#include "ptx.cuh"

namespace twell {

// ReLU + TwELL packing of one (row, TwELL tile) from its fp32 gate
// pre-activations, by one warp: lane l holds columns [l*T/32, +T/32) of the
// tile.  The packed entries keep ascending column order, the count is the
// true count, and an overflow tile takes a dense-row slot (bringing the row's
// x along when the slot is new) and stores ReLU(z) of all T columns there,
// exactly as EpiGateTwell does.  Returns the entries it listed in TwELL (0
// for an overflow tile), for the caller's count of kCtrlEntries.
template <int T>
__device__ __forceinline__ int pack_row_tile(const float (&v)[T / 32], const GateTwellParams& p, int row, int t,
                                             int lane, int* ctrl) {
  constexpr int V = T / 32;
  const int NT = p.N / T;
  // Column lane*V + j is active iff bit `lane` of act[j] is set.  Its rank
  // among the active columns: all active columns of lower lanes plus those of
  // this lane before j (independent ballots, no dependent shuffle chain).
  uint32_t act[V];
#pragma unroll
  for (int j = 0; j < V; ++j) act[j] = __ballot_sync(0xffffffffu, v[j] > 0.f);
  const uint32_t lower = (1u << lane) - 1u;
  int cnt = 0, off = 0;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    cnt += __popc(act[j]);
    off += __popc(act[j] & lower);
  }
  const int64_t rec = static_cast<int64_t>(row) * NT + t;
#pragma unroll
  for (int j = 0; j < V; ++j) {
    if (v[j] > 0.f) {
      if (off < p.C) {
        p.idx[rec * p.C + off] = static_cast<uint8_t>(lane * V + j);
        p.vals[rec * p.C + off] = v[j];
      }
      ++off;
    }
  }
  if (lane == 0) p.counts[rec] = static_cast<uint16_t>(cnt);
  if (cnt <= p.C) return cnt;
  int slot = -1;
  bool fresh = false;
  if (lane == 0) slot = acquire_row_slot(p.row_slot, p.slot_row, p.r_cap, row, ctrl, fresh);
  slot = __shfl_sync(0xffffffffu, slot, 0);
  fresh = __shfl_sync(0xffffffffu, fresh ? 1 : 0, 0) != 0;
  if (fresh) {
    const uint4* xs = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(row) * p.K);
    uint4* xd = reinterpret_cast<uint4*>(p.x_over + static_cast<int64_t>(slot) * p.K);
    for (int k = lane; k < p.K / 8; k += 32) xd[k] = xs[k];
  }
  if (slot >= 0) {
    float4* dst = reinterpret_cast<float4*>(p.dense_rows + static_cast<int64_t>(slot) * p.N + t * T + lane * V);
#pragma unroll
    for (int q = 0; q < V / 4; ++q)
      dst[q] = make_float4(relu_f(v[4 * q]), relu_f(v[4 * q + 1]), relu_f(v[4 * q + 2]), relu_f(v[4 * q + 3]));
  }
  return 0;
}

// pack_row_tile for up to R rows at once (rows[r] < 0: no row), written as
// straight-line code so that the rows' ballots, ranks and stores interleave;
// overflow tiles (rare) then take pack_row_tile's slot path one at a time.
template <int T, int R>
__device__ __forceinline__ int pack_rows(const float (&v)[R][T / 32], const int (&rows)[R], const GateTwellParams& p,
                                         int t, int lane, int* ctrl) {
  constexpr int V = T / 32;
  const int NT = p.N / T;
  const uint32_t lower = (1u << lane) - 1u;
  uint32_t act[R][V];
  int cnt[R], off[R];
#pragma unroll
  for (int r = 0; r < R; ++r)
#pragma unroll
    for (int j = 0; j < V; ++j) act[r][j] = __ballot_sync(0xffffffffu, rows[r] >= 0 && v[r][j] > 0.f);
#pragma unroll
  for (int r = 0; r < R; ++r) {
    cnt[r] = 0;
    off[r] = 0;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      cnt[r] += __popc(act[r][j]);
      off[r] += __popc(act[r][j] & lower);
    }
  }
  int listed = 0;
#pragma unroll
  for (int r = 0; r < R; ++r) {
    if (rows[r] < 0) continue;
    const int64_t rec = static_cast<int64_t>(rows[r]) * NT + t;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      if ((act[r][j] >> lane) & 1u) {
        if (off[r] < p.C) {
          p.idx[rec * p.C + off[r]] = static_cast<uint8_t>(lane * V + j);
          p.vals[rec * p.C + off[r]] = v[r][j];
        }
        ++off[r];
      }
    }
    if (lane == 0) p.counts[rec] = static_cast<uint16_t>(cnt[r]);
    if (cnt[r] <= p.C) listed += cnt[r];
  }
#pragma unroll
  for (int r = 0; r < R; ++r)
    if (rows[r] >= 0 && cnt[r] > p.C) pack_row_tile<T>(v[r], p, rows[r], t, lane, ctrl);  // slot path
  return listed;
}

// Scratch slots per 128-unit tile: the host sizes the CTA ranges (at least a
// third of a tile's k blocks each) so that no tile has more contributors.
constexpr int kStreamSlots = 4;

constexpr int kStreamMaxStages = 12;

struct GateStreamParams {
  GateTwellParams pk;  // TwELL outputs and the dense-row slot protocol
  float* part;         // [N/128][kStreamSlots][M][128] partial sums
  int* tickets;        // [N/T] tile pieces finished (the last one resets it to 0)
  int M, T;
  int kb;              // k blocks of 64 (K / 64)
  int64_t units;       // (N / 128) * kb
  int mp;              // token side of the tile (16, 32, 64 or 128; >= M)
  int stages;          // operand ring depth (2 .. kStreamMaxStages)
  int grid;            // CTAs that share the k blocks (the first `grid` of the launch)
};

// Control block at the start of the (1024-byte aligned) dynamic shared
// memory; the operand ring follows at kStreamCtrlBytes.
struct GateStreamShared {
  uint64_t full[kStreamMaxStages];
  uint64_t empty[kStreamMaxStages];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint32_t tmem;  // TMEM base address
  int last;       // this CTA finished a TwELL tile's last piece
  int fail;       // an epilogue wait gave up
  int sync_ok;    // (fused kernel) the grid barrier completed
};
constexpr int kStreamCtrlBytes = 1024;
static_assert(sizeof(GateStreamShared) <= kStreamCtrlBytes, "control block");

// Ring stage: 128 hidden units x 64 k of W_g^T, then mp tokens x 64 k of x.
__host__ __device__ constexpr int stream_stage_bytes(int mp) { return 128 * 64 * 2 + mp * 64 * 2; }
__host__ __device__ constexpr uint32_t stream_tmem_cols(int mp) { return 2 * mp < 32 ? 32u : 2u * mp; }
__host__ __device__ constexpr size_t stream_smem_bytes(int mp, int stages) {
  return 1024 /*alignment slack*/ + kStreamCtrlBytes + static_cast<size_t>(stages) * stream_stage_bytes(mp);
}

// First unit of CTA c's range, and the CTA whose range holds unit u (the
// largest c with stream_first(c) <= u).
__host__ __device__ __forceinline__ int64_t stream_first(int64_t c, int64_t units, int grid) {
  return c * units / grid;
}
__host__ __device__ __forceinline__ int stream_cta_of(int64_t u, int64_t units, int grid) {
  return static_cast<int>(((u + 1) * grid + units - 1) / units - 1);
}
// Number of CTAs whose ranges meet 128-unit tile b.
__host__ __device__ __forceinline__ int stream_contributors(int b, int kb, int64_t units, int grid) {
  const int64_t first = static_cast<int64_t>(b) * kb;
  return stream_cta_of(first + kb - 1, units, grid) - stream_cta_of(first, units, grid) + 1;
}

// Barrier initialisation and TMEM allocation (two accumulators of mp
// columns); every thread of the CTA calls it.
__device__ __forceinline__ void stream_setup(GateStreamShared* sh, const GateStreamParams& p) {
  const int warp = threadIdx.x >> 5;
  if (threadIdx.x == 0) {
    for (int s = 0; s < p.stages; ++s) {
      mbar_init(&sh->full[s], 1);
      mbar_init(&sh->empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&sh->tfull[a], 1);
      mbar_init(&sh->tempty[a], 128);
    }
    sh->last = 0;
    sh->fail = 0;
    sh->sync_ok = 0;
    fence_barrier_init();
  }
  if (warp == 1) {
    tmem_alloc(&sh->tmem, stream_tmem_cols(p.mp));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
}

// The gate pass proper, by role (192 threads): warp 0 TMA producer, warp 1
// MMA issuer, warps 2-5 epilogue (warp w reads TMEM lanes 32*(w%4) .. +31,
// i.e. hidden units) and packing.
__device__ __forceinline__ void stream_run(const CUtensorMap* tmW, const CUtensorMap* tmX, const GateStreamParams& p,
                                           int* ctrl, GateStreamShared* sh, uint8_t* ring) {
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int S = p.stages;
  const int MP = p.mp;
  const int stage_bytes = stream_stage_bytes(MP);
  const uint32_t tmem_base = sh->tmem;
  const int G = p.grid;
  const int64_t U = p.units;
  const int kb = p.kb;
  // CTAs past the first G take no part in the gate pass (empty range).
  const int64_t u0 = static_cast<int>(blockIdx.x) < G ? stream_first(blockIdx.x, U, G) : 0;
  const int64_t u1 = static_cast<int>(blockIdx.x) < G ? stream_first(static_cast<int64_t>(blockIdx.x) + 1, U, G) : 0;

  if (warp == 0) {
    if (lane == 0) {
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok;) {
        const int b = static_cast<int>(u / kb);
        const int k0 = static_cast<int>(u - static_cast<int64_t>(b) * kb);
        const int k1 = static_cast<int>(u1 - static_cast<int64_t>(b) * kb < kb ? u1 - static_cast<int64_t>(b) * kb : kb);
        for (int kk = k0; kk < k1; ++kk) {
          if (!mbar_wait(&sh->empty[stage], phase ^ 1u, ctrl)) { ok = false; break; }
          uint8_t* sa = ring + stage * stage_bytes;
          mbar_arrive_expect_tx(&sh->full[stage], stage_bytes);
          tma_load_2d(tmW, &sh->full[stage], sa, kk * 64, b * 128);
          tma_load_2d(tmX, &sh->full[stage], sa + 128 * 64 * 2, kk * 64, 0);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        u = static_cast<int64_t>(b) * kb + k1;
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      const uint32_t idesc = idesc_bf16_f32(128, MP, false, false);
      int stage = 0;
      uint32_t phase = 0;
      int it = 0;
      bool ok = true;
      for (int64_t u = u0; u < u1 && ok; ++it) {
        const int b = static_cast<int>(u / kb);
        const int k0 = static_cast<int>(u - static_cast<int64_t>(b) * kb);
        const int k1 = static_cast<int>(u1 - static_cast<int64_t>(b) * kb < kb ? u1 - static_cast<int64_t>(b) * kb : kb);
        const int acc = it & 1;
        if (!mbar_wait(&sh->tempty[acc], ((it >> 1) & 1) ^ 1u, ctrl)) break;
        tc_fence_after();
        const uint32_t d = tmem_base + acc * MP;
        for (int kk = k0; kk < k1; ++kk) {
          if (!mbar_wait(&sh->full[stage], phase, ctrl)) { ok = false; break; }
          tc_fence_after();
          const uint32_t a_base = smem_u32(ring + stage * stage_bytes);
          const uint32_t b_base = a_base + 128 * 64 * 2;
#pragma unroll
          for (int k = 0; k < 4; ++k)
            umma_bf16(d, smem_desc_sw128(a_base + k * 32, 16, 1024), smem_desc_sw128(b_base + k * 32, 16, 1024), idesc,
                      (kk > k0 || k > 0) ? 1u : 0u);
          umma_commit(&sh->empty[stage]);
          if (++stage == S) { stage = 0; phase ^= 1u; }
        }
        if (ok) umma_commit(&sh->tfull[acc]);
        u = static_cast<int64_t>(b) * kb + k1;
      }
    }
  } else {
    const int q = warp & 3;     // TMEM lane quadrant: hidden units 32q .. 32q + 31 of the tile
    const int ew = warp - 2;    // 0..3: rows ew, ew + 4, ... when packing
    const int nl = q * 32 + lane;
    const int T = p.T;
    const int sub = T / 128;    // 128-unit tiles per TwELL tile
    int it = 0;
    for (int64_t u = u0; u < u1; ++it) {
      const int b = static_cast<int>(u / kb);
      const int k1 = static_cast<int>(u1 - static_cast<int64_t>(b) * kb < kb ? u1 - static_cast<int64_t>(b) * kb : kb);
      u = static_cast<int64_t>(b) * kb + k1;
      const int acc = it & 1;
      // The four warps leave together if any wait gives up: they share named barriers below.
      if (!mbar_wait(&sh->tfull[acc], (it >> 1) & 1, ctrl) && lane == 0) sh->fail = 1;
      named_bar_sync(1, 128);
      if (sh->fail) break;
      tc_fence_after();
      const uint32_t taddr = tmem_base + (static_cast<uint32_t>(q * 32) << 16) + acc * MP;
      const int slot = static_cast<int>(blockIdx.x) - stream_cta_of(static_cast<int64_t>(b) * kb, U, G);
      float* dst = p.part + (static_cast<int64_t>(b) * kStreamSlots + slot) * p.M * 128 + nl;
#pragma unroll 1
      for (int c = 0; c < MP; c += 16) {
        uint32_t r[16];
        tmem_ld_32x32_x16(taddr + c, r);
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 16; ++i)
          if (c + i < p.M) dst[(c + i) * 128] = __uint_as_float(r[i]);
      }
      tc_fence_before();
      mbar_arrive(&sh->tempty[acc]);

      // Publish the piece; the last piece of the TwELL tile packs it.
      __threadfence();
      named_bar_sync(1, 128);
      const int t = b / sub;
      if (ew == 0 && lane == 0) {
        int need = 0;
        for (int h = 0; h < sub; ++h) need += stream_contributors(t * sub + h, kb, U, G);
        const int done = atomicAdd(p.tickets + t, 1);
        const bool last = done == need - 1;
        if (last) p.tickets[t] = 0;
        sh->last = last ? 1 : 0;
      }
      named_bar_sync(1, 128);
      if (sh->last) {
        fence_acq_rel_gpu();  // the other pieces' partial sums are visible
        // Rows ew, ew + 4, ... in groups of four, every slot's loads of a
        // group issued before any is used.
        int listed = 0;
        if (T == 128) {
          const int n_sl = stream_contributors(t, kb, U, G);
          const float* base = p.part + static_cast<int64_t>(t) * kStreamSlots * p.M * 128 + lane * 4;
#pragma unroll 1
          for (int m0 = ew; m0 < p.M; m0 += 16) {
            float4 a[4][kStreamSlots];
#pragma unroll
            for (int r = 0; r < 4; ++r)
#pragma unroll
              for (int j = 0; j < kStreamSlots; ++j) {
                const int m = m0 + 4 * r;
                a[r][j] = (j < n_sl && m < p.M)
                              ? __ldcg(reinterpret_cast<const float4*>(base + (static_cast<int64_t>(j) * p.M + m) * 128))
                              : make_float4(0.f, 0.f, 0.f, 0.f);
              }
            float v[4][4];
            int rows[4];
#pragma unroll
            for (int r = 0; r < 4; ++r) {
              rows[r] = m0 + 4 * r < p.M ? m0 + 4 * r : -1;
              v[r][0] = a[r][0].x; v[r][1] = a[r][0].y; v[r][2] = a[r][0].z; v[r][3] = a[r][0].w;
#pragma unroll
              for (int j = 1; j < kStreamSlots; ++j) {
                v[r][0] += a[r][j].x; v[r][1] += a[r][j].y; v[r][2] += a[r][j].z; v[r][3] += a[r][j].w;
              }
            }
            listed += pack_rows<128, 4>(v, rows, p.pk, t, lane, ctrl);
          }
        } else {
          // Lane l holds columns [8l, 8l + 8): 128-unit tile 2t + l / 16.
          const int bb = 2 * t + (lane >> 4);
          const int n_sl = stream_contributors(bb, kb, U, G);
          const float* base =
              p.part + static_cast<int64_t>(bb) * kStreamSlots * p.M * 128 + (lane & 15) * 8;
#pragma unroll 1
          for (int m0 = ew; m0 < p.M; m0 += 8) {
            float4 a[2][kStreamSlots][2];
#pragma unroll
            for (int r = 0; r < 2; ++r)
#pragma unroll
              for (int j = 0; j < kStreamSlots; ++j) {
                const int m = m0 + 4 * r;
                const bool use = j < n_sl && m < p.M;
                const float4* src = reinterpret_cast<const float4*>(base + (static_cast<int64_t>(j) * p.M + m) * 128);
                a[r][j][0] = use ? __ldcg(src) : make_float4(0.f, 0.f, 0.f, 0.f);
                a[r][j][1] = use ? __ldcg(src + 1) : make_float4(0.f, 0.f, 0.f, 0.f);
              }
            float v[2][8];
            int rows[2];
#pragma unroll
            for (int r = 0; r < 2; ++r) {
              rows[r] = m0 + 4 * r < p.M ? m0 + 4 * r : -1;
              v[r][0] = a[r][0][0].x; v[r][1] = a[r][0][0].y; v[r][2] = a[r][0][0].z; v[r][3] = a[r][0][0].w;
              v[r][4] = a[r][0][1].x; v[r][5] = a[r][0][1].y; v[r][6] = a[r][0][1].z; v[r][7] = a[r][0][1].w;
#pragma unroll
              for (int j = 1; j < kStreamSlots; ++j) {
                v[r][0] += a[r][j][0].x; v[r][1] += a[r][j][0].y; v[r][2] += a[r][j][0].z; v[r][3] += a[r][j][0].w;
                v[r][4] += a[r][j][1].x; v[r][5] += a[r][j][1].y; v[r][6] += a[r][j][1].z; v[r][7] += a[r][j][1].w;
              }
            }
            listed += pack_rows<256, 2>(v, rows, p.pk, t, lane, ctrl);
          }
        }
        if (lane == 0 && listed > 0) atomicAdd(ctrl + kCtrlEntries, listed);
      }
    }
  }
}

// Small-batch gate pass: set-up, the pass, TMEM released.
__global__ void __launch_bounds__(192, 1)
    gate_stream_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                       const GateStreamParams p, int* ctrl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GateStreamShared* sh = reinterpret_cast<GateStreamShared*>(base);
  if (threadIdx.x == 0) {
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  stream_setup(sh, p);
  griddep_launch_dependents();
  griddep_wait();
  stream_run(&tmW, &tmX, p, ctrl, sh, base + kStreamCtrlBytes);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if ((threadIdx.x >> 5) == 1) tmem_dealloc(sh->tmem, stream_tmem_cols(p.mp));
}

}  // namespace twell
