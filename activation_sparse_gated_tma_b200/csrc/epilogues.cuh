// Epilogues for the tcgen05 GEMM engine.  Each runs on the 128 epilogue
// threads; thread i owns accumulator row `row` (TMEM lane) of the current
// 128 x BN tile and reads its BN fp32 columns from TMEM in chunks of 32.
#pragma once

#include "ptx.cuh"

namespace twell {

// Row-slot protocol for the hybrid dense backup ("Sparser, Faster, Lighter
// Transformer Language Models", §3-6 and §4-3: rows over capacity go to a dense
// backup of bounded size).  row_slot[m] is -1 (free) until the first tile of
// row m overflows; that thread swaps in kSlotPending, takes the next slot from
// the n_over counter and publishes it.  Other tiles of the same row wait
// (bounded) for the publication.  Slots past R_cap publish kSlotNoCapacity.
constexpr int kSlotFree = -1;
constexpr int kSlotNoCapacity = -2;
constexpr int kSlotPending = -3;

__device__ __forceinline__ int acquire_row_slot(int* row_slot, int* slot_row, int r_cap, int row, int* ctrl,
                                                bool& fresh) {
  fresh = false;
  int s = atomicCAS(row_slot + row, kSlotFree, kSlotPending);
  if (s == kSlotFree) {
    const int ns = atomicAdd(ctrl + kCtrlNOver, 1);
    if (ns < r_cap) {
      slot_row[ns] = row;
      s = ns;
      fresh = true;
    } else {
      s = kSlotNoCapacity;
      set_flag(ctrl, kFlagNoCapacity);
    }
    atomicExch(row_slot + row, s);
    return s;
  }
  if (s != kSlotPending) return s;
  const unsigned long long t0 = global_ns();
  while (true) {
    s = atomicAdd(row_slot + row, 0);
    if (s != kSlotPending) return s;
    if (global_ns() - t0 > kWaitLimitNs) {
      set_flag(ctrl, kFlagWaitTimeout);
      return kSlotNoCapacity;
    }
  }
}

__device__ __forceinline__ float relu_f(float z) { return z > 0.f ? z : 0.f; }

// Epilogue interface (see tc_gemm.cuh): Pre<BN> holds what prepare() loads
// before the accumulator is ready; run() consumes it.  Most epilogues need none.
struct EpiNoPrepare {
  template <int BN>
  static constexpr int kWarps = 4;  // epilogue warps (4, or 8 to split the columns)
  template <int BN>
  struct Pre {};
  template <int BN, class Params>
  static __device__ __forceinline__ void prepare(const Params&, Pre<BN>&, int, int, int) {}
};

// ---------------------------------------------------------------------------
// Gate epilogue: ReLU + TwELL packing + overflow routing ("Sparser, Faster,
// Lighter Transformer Language Models", §3-4 steps 3-5 and §3-6).
// The CTA's output tile (BN columns) holds BN / T whole TwELL tiles, so every
// (row, tile) record is produced by one thread from its own TMEM lane: no
// cross-CTA or cross-thread step is needed to pack.
struct GateTwellParams {
  uint16_t* counts;    // [M][N/T]
  uint8_t* idx;        // [M][N/T][C]
  float* vals;         // [M][N/T][C]
  float* dense_rows;   // [R_cap][N]
  int* row_slot;       // [M]
  int* slot_row;       // [R_cap]
  const uint16_t* x;   // [M][K] gate input, copied to x_over for slotted rows
  uint16_t* x_over;    // [R_cap][K]
  int N, K, C, r_cap;
};

template <int T>
struct EpiGateTwell : EpiNoPrepare {
  using Params = GateTwellParams;
  // Per epilogue warp: one 32-column chunk of its 32 rows, laid out
  // [column][lane] so that every thread's dynamically indexed reads of its own
  // row hit distinct banks.
  static constexpr int kScratchBytes = 32 * 32 * 4;
  // Two TwELL tiles per CTA tile: eight warps, one TwELL tile each per row.
  template <int BN>
  static constexpr int kWarps = BN / T >= 2 ? 8 : 4;

  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>&, uint32_t taddr, int row, int m_rows,
                                             int nb, int lane, int* ctrl, void* scratch, int part, int nparts) {
    static_assert(BN % T == 0, "a CTA tile must hold whole TwELL tiles");
    float* stage = static_cast<float*>(scratch) + lane;
    const bool valid = row < m_rows;
    const int NT = p.N / T;
    constexpr int kSub = BN / T;  // TwELL tiles in the CTA tile
#pragma unroll 1
    for (int st = part * kSub / nparts; st < (part + 1) * kSub / nparts; ++st) {
      const int t = nb * (BN / T) + st;
      const uint32_t tcol = taddr + st * T;
      const int64_t rec = static_cast<int64_t>(row) * NT + t;
      uint8_t* idx_rec = p.idx + rec * p.C;
      float* val_rec = p.vals + rec * p.C;
      int cnt = 0;
#pragma unroll 1
      for (int c = 0; c < T / 32; ++c) {
        uint32_t r[32];
        tmem_ld_32x32(tcol + c * 32, r);
        tmem_wait_ld();
        // Bit j: column c*32+j is active (ReLU(z) > 0).
        uint32_t mask = 0;
#pragma unroll
        for (int j = 0; j < 32; ++j) mask |= (__uint_as_float(r[j]) > 0.f ? 1u : 0u) << j;
        if (!valid) mask = 0;
        if (mask != 0 && cnt < p.C) {
          // Stage the chunk, then pack only the set bits, in ascending column order.
#pragma unroll
          for (int j = 0; j < 32; ++j) stage[j * 32] = __uint_as_float(r[j]);
          while (mask != 0 && cnt < p.C) {
            const int j = __ffs(mask) - 1;
            mask &= mask - 1;
            idx_rec[cnt] = static_cast<uint8_t>(c * 32 + j);
            val_rec[cnt] = stage[j * 32];
            ++cnt;
          }
        }
        cnt += __popc(mask);
      }
      if (valid) p.counts[rec] = static_cast<uint16_t>(cnt);
      const bool ov = valid && cnt > p.C;
      // Entries the fused kernel will stream (it sizes its work units from the total).
      const int listed = warp_sum_int(ov ? 0 : cnt);
      if (lane == 0 && listed > 0) atomicAdd(ctrl + kCtrlEntries, listed);
      if (__any_sync(0xffffffffu, ov)) {
        int slot = -1;
        bool fresh = false;
        if (ov) slot = acquire_row_slot(p.row_slot, p.slot_row, p.r_cap, row, ctrl, fresh);
        // The lane that opened a slot brings its x row along (whole warp copies).
        uint32_t fresh_mask = __ballot_sync(0xffffffffu, fresh);
        while (fresh_mask) {
          const int src = __ffs(fresh_mask) - 1;
          fresh_mask &= fresh_mask - 1;
          const int r = __shfl_sync(0xffffffffu, row, src);
          const int sl = __shfl_sync(0xffffffffu, slot, src);
          const uint4* xs = reinterpret_cast<const uint4*>(p.x + static_cast<int64_t>(r) * p.K);
          uint4* xd = reinterpret_cast<uint4*>(p.x_over + static_cast<int64_t>(sl) * p.K);
          for (int v = lane; v < p.K / 8; v += 32) xd[v] = xs[v];
        }
        float* dst = slot >= 0 ? p.dense_rows + static_cast<int64_t>(slot) * p.N + t * T : nullptr;
#pragma unroll 1
        for (int c = 0; c < T / 32; ++c) {
          uint32_t r[32];
          tmem_ld_32x32(tcol + c * 32, r);
          tmem_wait_ld();
          if (dst) {
            float4* d4 = reinterpret_cast<float4*>(dst + c * 32);
#pragma unroll
            for (int v = 0; v < 8; ++v)
              d4[v] = make_float4(relu_f(__uint_as_float(r[4 * v + 0])), relu_f(__uint_as_float(r[4 * v + 1])),
                                  relu_f(__uint_as_float(r[4 * v + 2])), relu_f(__uint_as_float(r[4 * v + 3])));
          }
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// h as an unevaluated sum of two bf16 numbers: hi = bf16(h), lo = bf16(h - hi),
// so |h - hi - lo| <= 2^-9 |h - hi| <= 2^-18 |h| (about 16 significant bits)
// while the next GEMM still runs on bf16 tensor cores, once over hi and once
// over lo against the same weights.
__device__ __forceinline__ void split_bf16x8(const float (&h)[8], uint4& hi, uint4& lo) {
  uint32_t a[4], b[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    a[e] = pack_bf16x2(h[2 * e], h[2 * e + 1]);
    b[e] = pack_bf16x2(h[2 * e] - __uint_as_float(a[e] << 16), h[2 * e + 1] - __uint_as_float(a[e] & 0xFFFF0000u));
  }
  hi = make_uint4(a[0], a[1], a[2], a[3]);
  lo = make_uint4(b[0], b[1], b[2], b[3]);
}

// ---------------------------------------------------------------------------
// Dense FFN first stage: accumulator 0 = x W_g tile, accumulator 1 = x W_u
// tile (same columns).  Writes h = h_u * ReLU(h_g) ("Sparser, Faster, Lighter
// Transformer Language Models", §1-1) either as bf16 hi + lo parts (h [M][2N]:
// hi in columns [0, N), lo in [N, 2N)) or, with split == 0, rounded to one
// bf16 (h [M][N], as a plain bf16 dense FFN keeps it).
struct EpiGatedProduct : EpiNoPrepare {
  static constexpr int kScratchBytes = 0;
  struct Params {
    uint16_t* h;  // [M][2N] (split) or [M][N] bf16
    int N;
    int split;
  };
  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>&, uint32_t taddr, int row, int m_rows,
                                             int nb, int, int*, void*, int, int) {
    const bool valid = row < m_rows;
    const int64_t ld = p.split ? 2 * static_cast<int64_t>(p.N) : p.N;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t g[32], u[32];
      tmem_ld_32x32(taddr + c * 32, g);
      tmem_ld_32x32(taddr + BN + c * 32, u);
      tmem_wait_ld();
      if (valid) {
        uint4* dst = reinterpret_cast<uint4*>(p.h + static_cast<int64_t>(row) * ld + nb * BN + c * 32);
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float h[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) h[e] = __uint_as_float(u[8 * v + e]) * relu_f(__uint_as_float(g[8 * v + e]));
          uint4 hi, lo;
          split_bf16x8(h, hi, lo);
          dst[v] = hi;
          if (p.split) dst[v + p.N / 8] = lo;
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Plain fp32 store of the accumulator: y[row][col] = acc, col < ncols.
struct EpiStoreF32 : EpiNoPrepare {
  static constexpr int kScratchBytes = 0;
  struct Params {
    float* y;
    int ldy;
    int ncols;
    int accumulate;  // split-K: add into a zero-initialised y with vector atomics
  };
  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>&, uint32_t taddr, int row, int m_rows,
                                             int nb, int, int*, void*, int, int) {
    const bool valid = row < m_rows;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32(taddr + c * 32, r);
      tmem_wait_ld();
      const int col0 = nb * BN + c * 32;
      if (valid && col0 < p.ncols) {
        float* dst = p.y + static_cast<int64_t>(row) * p.ldy + col0;
        if (col0 + 32 <= p.ncols) {
#pragma unroll
          for (int v = 0; v < 8; ++v) {
            const float4 a = make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                         __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3]));
            if (p.accumulate)
              atomicAdd(reinterpret_cast<float4*>(dst) + v, a);
            else
              reinterpret_cast<float4*>(dst)[v] = a;
          }
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < p.ncols - col0) {
              if (p.accumulate)
                atomicAdd(dst + j, __uint_as_float(r[j]));
              else
                dst[j] = __uint_as_float(r[j]);
            }
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Overflow path, first stage: rows are dense-row slots r (< n_over).  The
// accumulator holds x_m W_u for m = slot_row[r]; the epilogue multiplies by
// the stored fp32 ReLU gate of that row where the tile overflowed and writes
// zero elsewhere (those tiles are served from TwELL).  h is written as an
// unevaluated sum of two bf16 numbers (hi + lo, |lo| <= 2^-9 |hi|) so that the
// second stage keeps ~16 bits of h while feeding bf16 tensor cores.
struct EpiOverflowProduct {
  static constexpr int kScratchBytes = 0;
  template <int BN>
  static constexpr int kWarps = 4;
  struct Params {
    const uint16_t* counts;   // [M][N/T]
    const float* dense_rows;  // [R_cap][N]
    const int* slot_row;      // [R_cap]
    uint16_t* h_over;         // [R_cap][2N]: bf16 hi part in columns [0, N), lo part in [N, 2N)
    int N, T, C;
  };
  template <int BN>
  struct Pre {
    float g[BN];  // the row's stored ReLU gate on the tile's columns (overflow tiles only)
    bool ov;      // the row's TwELL tile under these columns overflowed
  };
  template <int BN>
  static __device__ __forceinline__ void prepare(const Params& p, Pre<BN>& pre, int row, int m_rows, int nb) {
    const int m = row < m_rows ? p.slot_row[row] : -1;
    const int NT = p.N / p.T;
    const int t = (nb * BN) / p.T;
    pre.ov = m >= 0 && p.counts[static_cast<int64_t>(m) * NT + t] > p.C;
    if (pre.ov) {
      const float4* src = reinterpret_cast<const float4*>(p.dense_rows + static_cast<int64_t>(row) * p.N + nb * BN);
#pragma unroll
      for (int v = 0; v < BN / 4; ++v) {
        const float4 a = src[v];
        pre.g[4 * v + 0] = a.x;
        pre.g[4 * v + 1] = a.y;
        pre.g[4 * v + 2] = a.z;
        pre.g[4 * v + 3] = a.w;
      }
    }
  }
  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>& pre, uint32_t taddr, int row, int m_rows,
                                             int nb, int, int*, void*, int, int) {
    const bool valid = row < m_rows;
#pragma unroll
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t u[32];
      tmem_ld_32x32(taddr + c * 32, u);
      tmem_wait_ld();
      if (valid) {
        uint4* dst_hi = reinterpret_cast<uint4*>(p.h_over + static_cast<int64_t>(row) * 2 * p.N + nb * BN + c * 32);
        uint4* dst_lo = dst_hi + p.N / 8;
#pragma unroll
        for (int v = 0; v < 4; ++v) {
          float h[8];
#pragma unroll
          for (int e = 0; e < 8; ++e) h[e] = pre.ov ? __uint_as_float(u[8 * v + e]) * pre.g[c * 32 + 8 * v + e] : 0.f;
          split_bf16x8(h, dst_hi[v], dst_lo[v]);
        }
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Backward over the dense-row slots ("Sparser, Faster, Lighter Transformer
// Language Models", §3-6: the dense backup rows take the dense tensor-core
// path in training too).  The accumulator holds dh = dy_m W_d^T for slot r
// (m = slot_row[r]) on 128 hidden units.  On units of the row's overflow
// tiles with g = ReLU(z) > 0 (the stored gate) the epilogue forms, with u =
// x_m W_u^T (fp32, from the previous GEMM),
//   du = dh g,  dz = dh u,  h = u g
// (0 elsewhere: TwELL tiles are served by the gather passes), and writes each
// as bf16 hi + lo: du and dz row-major ([R][2N], hi in columns [0, N)) for the
// dx GEMMs, and h, du, dz transposed ([N][2 R_pad], hi in columns [0, R_pad))
// for the weight-gradient GEMMs, which reduce over the slots.
struct EpiBwdSlots : EpiNoPrepare {
  static constexpr int kScratchBytes = 0;
  struct Params {
    const float* u;           // [R][N] x_over W_u^T
    const float* dense_rows;  // [R_cap][N] stored ReLU gates
    const uint16_t* counts;   // [M][N/T]
    const int* slot_row;      // [R_cap]
    uint16_t* du_rows;        // [R][2N]
    uint16_t* dz_rows;        // [R][2N]
    uint16_t* h_t;            // [N][2 R_pad]
    uint16_t* du_t;           // [N][2 R_pad]
    uint16_t* dz_t;           // [N][2 R_pad]
    int N, T, C, r_pad;
  };
  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>&, uint32_t taddr, int row, int m_rows,
                                             int nb, int, int*, void*, int, int) {
    const bool valid = row < m_rows;
    const int m = valid ? p.slot_row[row] : -1;
    const int NT = p.N / p.T;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32(taddr + c * 32, r);
      tmem_wait_ld();
      const int n0 = nb * BN + c * 32;
      const bool ov = m >= 0 && p.counts[static_cast<int64_t>(m) * NT + n0 / p.T] > p.C;
      float du[32], dz[32], h[32];
      if (ov) {
        const float4* u4 = reinterpret_cast<const float4*>(p.u + static_cast<int64_t>(row) * p.N + n0);
        const float4* g4 = reinterpret_cast<const float4*>(p.dense_rows + static_cast<int64_t>(row) * p.N + n0);
#pragma unroll
        for (int v = 0; v < 8; ++v) {
          const float4 uu = u4[v], gg = g4[v];
          const float us[4] = {uu.x, uu.y, uu.z, uu.w}, gs[4] = {gg.x, gg.y, gg.z, gg.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            const float dh = __uint_as_float(r[4 * v + e]);
            const bool on = gs[e] > 0.f;
            du[4 * v + e] = on ? dh * gs[e] : 0.f;
            dz[4 * v + e] = on ? dh * us[e] : 0.f;
            h[4 * v + e] = on ? us[e] * gs[e] : 0.f;
          }
        }
      } else {
#pragma unroll
        for (int j = 0; j < 32; ++j) du[j] = dz[j] = h[j] = 0.f;
      }
      if (!valid) continue;
      uint4* dur = reinterpret_cast<uint4*>(p.du_rows + static_cast<int64_t>(row) * 2 * p.N + n0);
      uint4* dzr = reinterpret_cast<uint4*>(p.dz_rows + static_cast<int64_t>(row) * 2 * p.N + n0);
#pragma unroll
      for (int v = 0; v < 4; ++v) {
        float a[8], b[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          a[e] = du[8 * v + e];
          b[e] = dz[8 * v + e];
        }
        split_bf16x8(a, dur[v], dur[v + p.N / 8]);
        split_bf16x8(b, dzr[v], dzr[v + p.N / 8]);
      }
      // Transposed: for a fixed unit the warp's 32 rows are 32 consecutive slots.
      const int64_t ld = 2 * static_cast<int64_t>(p.r_pad);
#pragma unroll 4
      for (int j = 0; j < 32; ++j) {
        const int64_t o = static_cast<int64_t>(n0 + j) * ld + row;
        const uint16_t hh = float_to_bf16_bits(h[j]);
        const uint16_t uh = float_to_bf16_bits(du[j]);
        const uint16_t zh = float_to_bf16_bits(dz[j]);
        p.h_t[o] = hh;
        p.h_t[o + p.r_pad] = float_to_bf16_bits(h[j] - bf16_bits_to_float(hh));
        p.du_t[o] = uh;
        p.du_t[o + p.r_pad] = float_to_bf16_bits(du[j] - bf16_bits_to_float(uh));
        p.dz_t[o] = zh;
        p.dz_t[o + p.r_pad] = float_to_bf16_bits(dz[j] - bf16_bits_to_float(zh));
      }
    }
  }
};

// ---------------------------------------------------------------------------
// Overflow path, second stage: y[slot_row[r]][col] += acc (vector atomics, so
// split-K slices and the fused kernel's earlier partial sum combine).
struct EpiAccumulateRows : EpiNoPrepare {
  static constexpr int kScratchBytes = 0;
  struct Params {
    float* y;
    const int* slot_row;
    int ldy;
    int ncols;
  };
  template <int BN>
  static __device__ __forceinline__ void run(const Params& p, const Pre<BN>&, uint32_t taddr, int row, int m_rows,
                                             int nb, int, int*, void*, int, int) {
    const int m = row < m_rows ? p.slot_row[row] : -1;
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld_32x32(taddr + c * 32, r);
      tmem_wait_ld();
      const int col0 = nb * BN + c * 32;
      if (m >= 0 && col0 < p.ncols) {
        float* dst = p.y + static_cast<int64_t>(m) * p.ldy + col0;
        if (col0 + 32 <= p.ncols) {
#pragma unroll
          for (int v = 0; v < 8; ++v)
            atomicAdd(reinterpret_cast<float4*>(dst) + v,
                      make_float4(__uint_as_float(r[4 * v]), __uint_as_float(r[4 * v + 1]),
                                  __uint_as_float(r[4 * v + 2]), __uint_as_float(r[4 * v + 3])));
        } else {
#pragma unroll
          for (int j = 0; j < 32; ++j)
            if (j < p.ncols - col0) atomicAdd(dst + j, __uint_as_float(r[j]));
        }
      }
    }
  }
};

}  // namespace twell
