// Backward pass of the sparse gated FFN over its hybrid activations
// ("Sparser, Faster, Lighter Transformer Language Models", §3-6 and §3-7:
// training keeps the activations in the hybrid TwELL + dense-row form, and
// every backward product visits only the active units).
//
// Per token row x with upstream gradient dy, and every active unit n of the
// row (g = ReLU(z) > 0, taken from TwELL or, for overflow tiles, from the
// row's dense-row slot):
//
//   u = x . W_u^T[n],  dh = dy . W_d[n],  h = u g,  du = dh g,  dz = dh u
//   dx += du W_u^T[n] + dz W_g^T[n]
//   dW_d[n] += h dy,  dW_u^T[n] += du x,  dW_g^T[n] += dz x
//
// Passes:
//   1. count   : active entries per hidden unit (atomic counts);
//   2. scan    : exclusive prefix of the counts (one CTA) -> each unit's
//                segment of a unit-major entry list (the hybrid transpose);
//   3. rows    : static units: a row's TwELL entries cut into shares of at
//                most 32 entries (by tile ranges, from a per-row count and
//                a scan of the units per row), or, when the slotted rows'
//                entries go through the gather passes too, one 32-column
//                chunk of an overflow tile; the W_u^T, W_d and W_g^T rows of
//                every entry stream through a per-warp ring; the warp adds
//                du W_u^T + dz W_g^T into dx (vector atomics, dx cleared
//                first) and appends (row, h, du, dz) to the unit's segment;
//   4. units   : one warp per (piece of up to 64 of a unit's entries,
//                256-column chunk) reads the entries' x and dy chunks and
//                writes the chunk of the three weight-gradient rows (plain
//                stores for units of one piece, zero rows for units with no
//                entry; vector atomics into rows the row pass cleared for
//                units of several pieces).
#pragma once

#include "epilogues.cuh"
#include "sparse_updown.cuh"

namespace twell {

struct BwdEntry {
  int m;
  float h, du, dz;
};

struct BwdParams {
  const uint16_t* x;
  const uint16_t* wg_t;
  const uint16_t* wu_t;
  const uint16_t* wd;
  const float* dy;
  const uint16_t* counts;
  const uint8_t* idx;
  const float* vals;
  const int* row_slot;
  const float* dense_rows;
  int M, K, N, T, C;
  float* dx;
  float* dwg_t;
  float* dwu_t;
  float* dwd;
  int* cnt;            // [N] entries per unit (TwELL, then the overflow tiles' when gathered)
  int* over_total;     // [1] active entries in the slotted rows' overflow tiles
  int* off;            // [N + 1] start of each unit's segment
  int* fill;           // [N] entries written so far per unit
  BwdEntry* entries;   // unit-major entry list
  const int* slot_row; // [R_cap] row of each dense-row slot
  int r_cap;
  int gather_overflow; // 1: overflow tiles also go through the row and unit passes (else the dense-row GEMMs)
  int* row_entries;    // [M] TwELL entries per row
  int* row_units;      // [M + 1] first row-pass unit of each row (exclusive prefix)
  int* piece_off;      // [N + 1] first unit-pass piece of each hidden unit (exclusive prefix)
  int* piece_unit;     // [N + cap / 64] hidden unit of each unit-pass piece
  int stages, list_cap;
  int* ctrl;           // ctrl[kCtrlNOver]: slots in use
};

// ---------------------------------------------------------------- 1. count
// The positive gates of the slotted rows' overflow tiles, a warp per (slot,
// tile) and a lane per column: each adds 1 to its unit's cnt (when cnt is
// given).  Returns this lane's number of them.
__device__ __forceinline__ int bwd_overflow_gates(const BwdParams& p, int* cnt) {
  const int lane = threadIdx.x & 31;
  const int NT = p.N / p.T;
  const int n_over = min(ld_acquire(p.ctrl + kCtrlNOver), p.r_cap);
  const int64_t items = static_cast<int64_t>(n_over) * NT;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  int found = 0;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); i < items;
       i += stride) {
    const int slot = static_cast<int>(i / NT);
    const int t = static_cast<int>(i - static_cast<int64_t>(slot) * NT);
    const int row = p.slot_row[slot];
    if (row < 0 || row >= p.M || p.counts[static_cast<int64_t>(row) * NT + t] <= p.C) continue;
    const float4* g = reinterpret_cast<const float4*>(p.dense_rows + static_cast<int64_t>(slot) * p.N +
                                                      static_cast<int64_t>(t) * p.T);
    for (int j = lane; j < p.T / 4; j += 32) {
      const float4 v = g[j];
      const float e[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        if (e[i] > 0.f) {
          ++found;
          if (cnt != nullptr) atomicAdd(cnt + t * p.T + 4 * j + i, 1);
        }
      }
    }
  }
  return found;
}

__global__ void __launch_bounds__(256) twell_bwd_count_kernel(const BwdParams p) {
  griddep_launch_dependents();
  griddep_wait();
  const int NT = p.N / p.T;
  const int64_t records = static_cast<int64_t>(p.M) * NT;
  int over = 0;  // active entries of slotted rows' overflow tiles (their true counts)
  for (int64_t r = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; r < records;
       r += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int c = p.counts[r];
    if (c == 0) continue;
    const int m = static_cast<int>(r / NT);
    if (c > p.C) {
      if (p.row_slot[m] >= 0) over += c;
      continue;
    }
    const int t = static_cast<int>(r - static_cast<int64_t>(m) * NT);
    for (int s = 0; s < c; ++s) atomicAdd(p.cnt + t * p.T + p.idx[r * p.C + s], 1);
    atomicAdd(p.row_entries + m, c);
  }
  // The host picks the slotted rows' route from their number of entries.
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) over += __shfl_xor_sync(0xffffffffu, over, o);
  if ((threadIdx.x & 31) == 0 && over > 0) atomicAdd(p.over_total, over);
}

// When the slotted rows go through the gather passes: their overflow entries
// added to the units' counts.
__global__ void __launch_bounds__(256) twell_bwd_overflow_units_kernel(const BwdParams p) {
  griddep_launch_dependents();
  griddep_wait();
  bwd_overflow_gates(p, p.cnt);
}

// ---------------------------------------------------------------- 2. scan
// One CTA of 1024 threads, exclusive prefix of n values: thread i sums its
// run of consecutive values, the CTA scans the 1024 sums, and each thread
// writes its run's offsets; out[n] is the total.  mode 0: the values are
// in[i]; mode 1: the row-pass units of row i, ceil(in[i] / kBwdUnitEntries).
// With `pieces` given (mode 0 over the per-unit counts), the same pass also
// scans the unit-pass pieces of hidden unit i, max(1, ceil(in[i] /
// kBwdPieceEntries)), into pieces[], and writes i into owner[pieces[i] ..
// pieces[i + 1]).
constexpr int kBwdUnitEntries = 32;   // row-pass unit: at most this many TwELL entries
constexpr int kBwdPieceEntries = 64;  // unit-pass piece: at most this many entries of one hidden unit
constexpr int kBwdUnitBatch = 2;      // unit pass: entries whose loads are in flight together

__device__ __forceinline__ int bwd_pieces(int c) {
  return c > kBwdPieceEntries ? (c + kBwdPieceEntries - 1) / kBwdPieceEntries : 1;
}

__global__ void __launch_bounds__(1024) twell_bwd_scan_kernel(const int* __restrict__ in, int* __restrict__ out, int n,
                                                              int mode, int* __restrict__ pieces,
                                                              int* __restrict__ owner) {
  __shared__ int part[2][1024];
  griddep_launch_dependents();
  griddep_wait();
  const int t = threadIdx.x;
  const int per = (n + 1023) / 1024;
  const int a = t * per;
  const int b = a + per < n ? a + per : n;
  int s = 0, q = 0;
  for (int i = a; i < b; ++i) {
    const int v = in[i];
    s += mode == 0 ? v : (v + kBwdUnitEntries - 1) / kBwdUnitEntries;
    q += bwd_pieces(v);
  }
  part[0][t] = s;
  part[1][t] = q;
  __syncthreads();
  for (int o = 1; o < 1024; o <<= 1) {
    const int v0 = t >= o ? part[0][t - o] : 0;
    const int v1 = t >= o ? part[1][t - o] : 0;
    __syncthreads();
    part[0][t] += v0;
    part[1][t] += v1;
    __syncthreads();
  }
  int run = part[0][t] - s;   // exclusive start of this thread's run
  int prun = part[1][t] - q;  // and of its pieces
  for (int i = a; i < b; ++i) {
    const int v = in[i];
    out[i] = run;
    run += mode == 0 ? v : (v + kBwdUnitEntries - 1) / kBwdUnitEntries;
    if (pieces != nullptr) {
      pieces[i] = prun;
      const int w = bwd_pieces(v);
      for (int j = 0; j < w; ++j) owner[prun + j] = i;
      prun += w;
    }
  }
  if (t == 1023) {
    out[n] = part[0][1023];
    if (pieces != nullptr) pieces[n] = part[1][1023];
  }
}

// ---------------------------------------------------------------- 3. rows
// acc += the products of 8 fp32 values of a and the 8 bf16 values of b.
__device__ __forceinline__ void dot8_f32_bf16(const float (&a)[8], const uint4& b, float& s0, float& s1) {
  const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    s0 = fmaf(a[2 * e], __uint_as_float(bw[e] << 16), s0);
    s1 = fmaf(a[2 * e + 1], __uint_as_float(bw[e] & 0xFFFF0000u), s1);
  }
}

// Bytes of one warp's shared memory in the row pass: [ring: stages x (W_u^T row
// | W_d row | W_g^T row)][list n: int x cap][list g: float x cap][h, du, dz of
// the listed entries: 3 x float x cap].
__host__ __device__ constexpr size_t bwd_warp_bytes(int K, int stages, int list_cap) {
  return ((static_cast<size_t>(stages) * 6 * K + static_cast<size_t>(list_cap) * 20) + 127) / 128 * 128;
}

// Most warps per CTA of the row pass: eight while a lane's x, dy and dx
// pieces fit the registers of eight warps, else six.
template <int KV>
constexpr int bwd_max_warps() {
  return KV <= 8 ? 8 : 6;
}

template <int KV>
__device__ __forceinline__ void bwd_issue(const BwdParams& p, const WarpRing& w, int slot, int n, int lane) {
  uint4* dst = reinterpret_cast<uint4*>(w.ring + static_cast<size_t>(slot) * w.slot_bytes);
  const int kv = p.K / 8;
  const uint4* su = reinterpret_cast<const uint4*>(p.wu_t + static_cast<int64_t>(n) * p.K);
  const uint4* sd = reinterpret_cast<const uint4*>(p.wd + static_cast<int64_t>(n) * p.K);
  const uint4* sg = reinterpret_cast<const uint4*>(p.wg_t + static_cast<int64_t>(n) * p.K);
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    const int v = j * 32 + lane;
    if (v < kv) {
      cp_async16(dst + v, su + v, w.policy);
      cp_async16(dst + kv + v, sd + v, w.policy);
      cp_async16(dst + 2 * kv + v, sg + v, w.policy);
    }
  }
}

// The E listed entries of row m through the ring (one copy group per slot and
// lane, refilled `stages` entries ahead).
template <int KV>
__device__ __forceinline__ void bwd_stream(const BwdParams& p, const WarpRing& w, int E, int m, const uint4 (&xv)[KV],
                                           const float (&dyv)[KV][8], float (&acc)[KV][8], int lane) {
  const int S = w.stages;
  for (int e = 0; e < S; ++e) {
    if (e < E) bwd_issue<KV>(p, w, e, w.list_n[e], lane);
    cp_async_commit();
  }
  const int kv = p.K / 8;
  int slot = 0;
  for (int e = 0; e < E; ++e) {
    cp_async_wait_pending(S - 1);
    const uint4* ru = reinterpret_cast<const uint4*>(w.ring + static_cast<size_t>(slot) * w.slot_bytes);
    const uint4* rd = ru + kv;
    const uint4* rg = ru + 2 * kv;
    float qu[4] = {0.f, 0.f, 0.f, 0.f};
    float qd0 = 0.f, qd1 = 0.f;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      if (j * 32 + lane < kv) {
        dot8_acc4(xv[j], ru[j * 32 + lane], qu);
        dot8_f32_bf16(dyv[j], rd[j * 32 + lane], qd0, qd1);
      }
    }
    float u = (qu[0] + qu[1]) + (qu[2] + qu[3]);
    float dh = qd0 + qd1;
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      u += __shfl_xor_sync(0xffffffffu, u, o);
      dh += __shfl_xor_sync(0xffffffffu, dh, o);
    }
    const float g = w.list_g[e];
    const float du = dh * g;
    const float dz = dh * u;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      if (j * 32 + lane < kv) {
        axpy8_bf16(acc[j], du, ru[j * 32 + lane]);
        axpy8_bf16(acc[j], dz, rg[j * 32 + lane]);
      }
    }
    if (lane == 0) {
      float* keep = w.list_g + w.list_cap;  // h, du, dz of entry e, appended below
      keep[e] = u * g;
      keep[w.list_cap + e] = du;
      keep[2 * w.list_cap + e] = dz;
    }
    // This lane has read the slot: refill it with the entry S places ahead.
    if (e + S < E) bwd_issue<KV>(p, w, slot, w.list_n[e + S], lane);
    cp_async_commit();
    slot = slot + 1 == S ? 0 : slot + 1;
  }
  // Append the E entries to their units' segments: one atomic round trip for
  // up to 32 entries at a time instead of one per entry.
  __syncwarp();
  const float* keep = w.list_g + w.list_cap;
  for (int j = lane; j < E; j += 32) {
    const int n = w.list_n[j];
    BwdEntry en;
    en.m = m;
    en.h = keep[j];
    en.du = keep[w.list_cap + j];
    en.dz = keep[2 * w.list_cap + j];
    p.entries[p.off[n] + atomicAdd(p.fill + n, 1)] = en;
  }
  __syncwarp();
}

template <int KV>
__global__ void __launch_bounds__(32 * bwd_max_warps<KV>(), 1) twell_bwd_rows_kernel(const BwdParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int NT = p.N / p.T;
  WarpRing w;
  w.slot_bytes = 6u * p.K;
  w.stages = p.stages;
  w.ring = smem + static_cast<size_t>(warp) * bwd_warp_bytes(p.K, p.stages, p.list_cap);
  w.list_n = reinterpret_cast<int*>(w.ring + static_cast<size_t>(p.stages) * w.slot_bytes);
  w.list_g = reinterpret_cast<float*>(w.list_n + p.list_cap);
  w.list_cap = p.list_cap;
  w.policy = l2_evict_last_policy();
  griddep_launch_dependents();
  griddep_wait();

  // list_entries reads TwELL through the up/down kernel's parameter block.
  UpdownParams lp = {};
  lp.counts = p.counts;
  lp.idx = p.idx;
  lp.vals = p.vals;
  lp.N = p.N;
  lp.T = p.T;
  lp.C = p.C;

  // The weight-gradient rows of hidden units whose entries the unit pass cuts
  // into several pieces are added into with atomics there: clear them here.
  for (int n = blockIdx.x * (blockDim.x >> 5) + warp; n < p.N; n += gridDim.x * (blockDim.x >> 5)) {
    if (p.off[n + 1] - p.off[n] <= kBwdPieceEntries) continue;
    for (int k = lane * 4; k < p.K; k += 128) {
      const int64_t o = static_cast<int64_t>(n) * p.K + k;
      *reinterpret_cast<float4*>(p.dwd + o) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(p.dwu_t + o) = make_float4(0.f, 0.f, 0.f, 0.f);
      *reinterpret_cast<float4*>(p.dwg_t + o) = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  const int64_t n_twell = p.row_units[p.M];  // units over TwELL tiles (rows cut by entries)
  const int chunks = p.T / 32;
  const int n_over = p.gather_overflow ? min(ld_acquire(p.ctrl + kCtrlNOver), p.r_cap) : 0;
  const int64_t n_units = n_twell + static_cast<int64_t>(n_over) * NT * chunks;  // + overflow-tile chunks
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  uint4 xv[KV];
  float dyv[KV][8];
  float acc[KV][8];
  for (int64_t u = static_cast<int64_t>(warp) * gridDim.x + blockIdx.x; u < n_units; u += stride) {
    int row, t0 = 0, t1 = 0, slot = -1, ot = 0, oq = 0;
    if (u < n_twell) {
      // The row whose units hold u (largest row with row_units[row] <= u).
      int lo = 0, hi = p.M - 1;
      while (lo < hi) {
        const int mid = (lo + hi + 1) >> 1;
        if (p.row_units[mid] <= u) lo = mid; else hi = mid - 1;
      }
      row = lo;
      const int k = static_cast<int>(u - p.row_units[row]);
      const int nunits = p.row_units[row + 1] - p.row_units[row];
      // Inclusive per-tile prefix of the row's TwELL entries (list_n as scratch),
      // then this unit's tiles: equal shares of the row's entries.
      const uint16_t* crow = p.counts + static_cast<int64_t>(row) * NT;
      int total = 0;
      __syncwarp();
      for (int tb = 0; tb < NT; tb += 32) {
        const int t = tb + lane;
        const int c = t < NT ? static_cast<int>(crow[t]) : 0;
        const int incl = warp_inclusive_scan(c > 0 && c <= p.C ? c : 0, lane);
        if (t < NT) w.list_n[t] = total + incl;
        total += __shfl_sync(0xffffffffu, incl, 31);
      }
      __syncwarp();
      t0 = unit_cut(w.list_n, NT, total, nunits, k);
      t1 = unit_cut(w.list_n, NT, total, nunits, k + 1);
      if (t0 >= t1) continue;
    } else {
      const int64_t item = u - n_twell;
      slot = static_cast<int>(item / (NT * chunks));
      const int rem = static_cast<int>(item - static_cast<int64_t>(slot) * NT * chunks);
      ot = rem / chunks;
      oq = rem - ot * chunks;
      row = p.slot_row[slot];
      if (row < 0 || row >= p.M || p.counts[static_cast<int64_t>(row) * NT + ot] <= p.C) continue;
    }
    const uint16_t* xr = p.x + static_cast<int64_t>(row) * p.K;
    const float* dyr = p.dy + static_cast<int64_t>(row) * p.K;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      const int k0 = (j * 32 + lane) * 8;
      const bool in = k0 < p.K;
      xv[j] = in ? *reinterpret_cast<const uint4*>(xr + k0) : make_uint4(0, 0, 0, 0);
      const float4 a = in ? *reinterpret_cast<const float4*>(dyr + k0) : make_float4(0.f, 0.f, 0.f, 0.f);
      const float4 b = in ? *reinterpret_cast<const float4*>(dyr + k0 + 4) : make_float4(0.f, 0.f, 0.f, 0.f);
      dyv[j][0] = a.x; dyv[j][1] = a.y; dyv[j][2] = a.z; dyv[j][3] = a.w;
      dyv[j][4] = b.x; dyv[j][5] = b.y; dyv[j][6] = b.z; dyv[j][7] = b.w;
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    }
    if (slot < 0) {
      int cursor = t0;
      while (cursor < t1) {
        const int E = list_entries(lp, w, row, cursor, t1, lane);
        if (E > 0) bwd_stream<KV>(p, w, E, row, xv, dyv, acc, lane);
      }
    } else {
      // Every positive gate of 32 columns of the overflow tile, in column order.
      const int col = ot * p.T + oq * 32 + lane;
      const float gv = p.dense_rows[static_cast<int64_t>(slot) * p.N + col];
      const uint32_t bal = __ballot_sync(0xffffffffu, gv > 0.f);
      __syncwarp();
      if (gv > 0.f) {
        const int pos = __popc(bal & ((1u << lane) - 1u));
        w.list_n[pos] = col;
        w.list_g[pos] = gv;
      }
      __syncwarp();
      if (bal == 0) continue;
      bwd_stream<KV>(p, w, __popc(bal), row, xv, dyv, acc, lane);
    }
    float* dxr = p.dx + static_cast<int64_t>(row) * p.K;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      const int k0 = (j * 32 + lane) * 8;
      if (k0 < p.K) {
        atomicAdd(reinterpret_cast<float4*>(dxr + k0), make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]));
        atomicAdd(reinterpret_cast<float4*>(dxr + k0 + 4), make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]));
      }
    }
  }
}

// ---------------------------------------------------------------- 5. dense-row slots
// Operands of the slots' backward GEMMs: for slot r < R, dy of its row split
// into bf16 hi + lo ([R_pad][2K] and the halves [R_pad][K] apart) and its x
// row ([R_pad][K]); rows R .. R_pad - 1 are zero, so the GEMMs that reduce
// over slots may run over R_pad.
__global__ void __launch_bounds__(256) twell_bwd_slot_operands_kernel(const float* __restrict__ dy,
                                                                       const uint16_t* __restrict__ x_over,
                                                                       const int* __restrict__ slot_row, int R,
                                                                       int r_pad, int K, uint16_t* dy_cat,
                                                                       uint16_t* dy_hi, uint16_t* dy_lo,
                                                                       uint16_t* x_pad) {
  griddep_launch_dependents();
  griddep_wait();
  const int per_row = K / 8;
  const int64_t items = static_cast<int64_t>(r_pad) * per_row;
  for (int64_t i = blockIdx.x * static_cast<int64_t>(blockDim.x) + threadIdx.x; i < items;
       i += static_cast<int64_t>(gridDim.x) * blockDim.x) {
    const int r = static_cast<int>(i / per_row);
    const int k = static_cast<int>(i - static_cast<int64_t>(r) * per_row) * 8;
    uint4 hi = make_uint4(0, 0, 0, 0), lo = hi, xv = hi;
    if (r < R) {
      const int m = slot_row[r];
      const float4 a = *reinterpret_cast<const float4*>(dy + static_cast<int64_t>(m) * K + k);
      const float4 b = *reinterpret_cast<const float4*>(dy + static_cast<int64_t>(m) * K + k + 4);
      const float v[8] = {a.x, a.y, a.z, a.w, b.x, b.y, b.z, b.w};
      split_bf16x8(v, hi, lo);
      xv = *reinterpret_cast<const uint4*>(x_over + static_cast<int64_t>(r) * K + k);
    }
    *reinterpret_cast<uint4*>(dy_cat + static_cast<int64_t>(r) * 2 * K + k) = hi;
    *reinterpret_cast<uint4*>(dy_cat + static_cast<int64_t>(r) * 2 * K + K + k) = lo;
    *reinterpret_cast<uint4*>(dy_hi + static_cast<int64_t>(r) * K + k) = hi;
    *reinterpret_cast<uint4*>(dy_lo + static_cast<int64_t>(r) * K + k) = lo;
    *reinterpret_cast<uint4*>(x_pad + static_cast<int64_t>(r) * K + k) = xv;
  }
}

// ---------------------------------------------------------------- 4. units
// Warp item = (piece, chunk c of 256 columns); a piece is up to 64 entries of
// one hidden unit n, and lane l holds columns c*256 + 8l .. +8 of the three
// gradient rows.  A unit with one piece stores its rows; the pieces of a unit
// with more entries add into rows the row pass cleared.
__global__ void __launch_bounds__(256) twell_bwd_units_kernel(const BwdParams p) {
  griddep_launch_dependents();
  griddep_wait();
  const int lane = threadIdx.x & 31;
  const int chunks = (p.K + 255) / 256;
  const int64_t items = static_cast<int64_t>(p.piece_off[p.N]) * chunks;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5);
  for (int64_t it = static_cast<int64_t>(blockIdx.x) * (blockDim.x >> 5) + (threadIdx.x >> 5); it < items;
       it += stride) {
    const int piece = static_cast<int>(it / chunks);
    const int k0 = static_cast<int>(it - static_cast<int64_t>(piece) * chunks) * 256 + lane * 8;
    const int n = p.piece_unit[piece];
    const int r = piece - p.piece_off[n];
    const bool split = p.piece_off[n + 1] - p.piece_off[n] > 1;
    const bool in = k0 < p.K;
    float ad[8], au[8], ag[8];
#pragma unroll
    for (int e = 0; e < 8; ++e) ad[e] = au[e] = ag[e] = 0.f;
    const int e0 = p.off[n] + r * kBwdPieceEntries;
    const int e1 = min(p.off[n + 1], e0 + kBwdPieceEntries);
    for (int b = e0; b < e1; b += 32) {
      // Lane j holds entry b + j; the warp then walks them in order.
      BwdEntry mine = {0, 0.f, 0.f, 0.f};
      if (b + lane < e1) mine = p.entries[b + lane];
      const int cntb = e1 - b < 32 ? e1 - b : 32;
      // kBwdUnitBatch entries per step, their x and dy loads issued before any is
      // used.  Past the last entry a step loads the row of lane (j & 31)'s
      // entry (row 0 for lanes past e1) and skips its arithmetic.
      for (int j0 = 0; j0 < cntb; j0 += kBwdUnitBatch) {
        int m[kBwdUnitBatch];
        float h[kBwdUnitBatch], du[kBwdUnitBatch], dz[kBwdUnitBatch];
#pragma unroll
        for (int q = 0; q < kBwdUnitBatch; ++q) {
          const int j = (j0 + q) & 31;
          const bool ok = j0 + q < cntb;
          m[q] = __shfl_sync(0xffffffffu, mine.m, j);
          const float hq = __shfl_sync(0xffffffffu, mine.h, j);
          const float uq = __shfl_sync(0xffffffffu, mine.du, j);
          const float zq = __shfl_sync(0xffffffffu, mine.dz, j);
          h[q] = ok ? hq : 0.f;
          du[q] = ok ? uq : 0.f;
          dz[q] = ok ? zq : 0.f;
        }
        if (in) {
          uint4 xq[kBwdUnitBatch];
          float4 d0[kBwdUnitBatch], d1[kBwdUnitBatch];
#pragma unroll
          for (int q = 0; q < kBwdUnitBatch; ++q) {
            const int64_t row = static_cast<int64_t>(m[q]) * p.K + k0;
            xq[q] = *reinterpret_cast<const uint4*>(p.x + row);
            d0[q] = *reinterpret_cast<const float4*>(p.dy + row);
            d1[q] = *reinterpret_cast<const float4*>(p.dy + row + 4);
          }
#pragma unroll
          for (int q = 0; q < kBwdUnitBatch; ++q) {
            if (j0 + q >= cntb) break;  // the same for the whole warp
            const float dv[8] = {d0[q].x, d0[q].y, d0[q].z, d0[q].w, d1[q].x, d1[q].y, d1[q].z, d1[q].w};
            const uint32_t xw[4] = {xq[q].x, xq[q].y, xq[q].z, xq[q].w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const float xlo = __uint_as_float(xw[e] << 16);
              const float xhi = __uint_as_float(xw[e] & 0xFFFF0000u);
              au[2 * e] = fmaf(du[q], xlo, au[2 * e]);
              au[2 * e + 1] = fmaf(du[q], xhi, au[2 * e + 1]);
              ag[2 * e] = fmaf(dz[q], xlo, ag[2 * e]);
              ag[2 * e + 1] = fmaf(dz[q], xhi, ag[2 * e + 1]);
            }
#pragma unroll
            for (int e = 0; e < 8; ++e) ad[e] = fmaf(h[q], dv[e], ad[e]);
          }
        }
      }
    }
    if (in) {
      const int64_t o = static_cast<int64_t>(n) * p.K + k0;
      float4* dd = reinterpret_cast<float4*>(p.dwd + o);
      float4* du4 = reinterpret_cast<float4*>(p.dwu_t + o);
      float4* dg4 = reinterpret_cast<float4*>(p.dwg_t + o);
      const float4 a0 = make_float4(ad[0], ad[1], ad[2], ad[3]), a1 = make_float4(ad[4], ad[5], ad[6], ad[7]);
      const float4 u0 = make_float4(au[0], au[1], au[2], au[3]), u1 = make_float4(au[4], au[5], au[6], au[7]);
      const float4 g0 = make_float4(ag[0], ag[1], ag[2], ag[3]), g1 = make_float4(ag[4], ag[5], ag[6], ag[7]);
      if (split) {
        atomicAdd(dd, a0); atomicAdd(dd + 1, a1);
        atomicAdd(du4, u0); atomicAdd(du4 + 1, u1);
        atomicAdd(dg4, g0); atomicAdd(dg4 + 1, g1);
      } else {
        dd[0] = a0; dd[1] = a1;
        du4[0] = u0; du4[1] = u1;
        dg4[0] = g0; dg4[1] = g1;
      }
    }
  }
}

}  // namespace twell
