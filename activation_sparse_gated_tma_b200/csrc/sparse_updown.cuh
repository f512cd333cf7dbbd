// Fused sparse up + down projection over TwELL ("Sparser, Faster, Lighter
// Transformer Language Models", §3-5):
//
//   y_m = sum_{n in A_m} g_{m,n} * (x_m . W_u[:, n]) * W_d[n, :]
//
// Work distribution (persistent grid, one CTA per SM, warps independent):
//   * A warp takes the next token row from a queue.  It scans the row's TwELL
//     counts; if the row holds more than unit_cap entries it cuts the row's
//     tile range into units of about unit_cap entries, keeps the first unit
//     and publishes the others on a second queue.  Rows are 100x apart in
//     active count (the pages report a row maximum above 10x the mean), so a
//     heavy row is shared by several warps instead of stalling one.
//   * When the row queue is empty, warps take published units.
//   * A row that is not split is stored by its warp.  A split row is cleared
//     by the warp that splits it before its units are published; every unit
//     (the first one too) then adds its partial y_m with vector atomics, so no
//     warp ever waits for another.
// Inside a unit:
//   * x_m (bf16, read with an L2 evict-first hint) and the fp32 partial of y_m
//     stay in registers, spread over the lanes in 16-byte pieces: lane l holds
//     elements [(j*32 + l)*8, +8).
//   * The warp lists the unit's active entries (n, g) from the TwELL records of
//     its non-overflow tiles into shared memory.
//   * The rows W_u^T[n] and W_d[n] of upcoming entries stream into the warp's
//     shared-memory ring, several entries ahead, as 16-byte cp.async copies
//     that every lane issues for itself: lane l copies, and later reads, only
//     the pieces l, l + 32, ... of each row, so completion is tracked per lane
//     with commit/wait groups (one group per ring slot) and no barrier or
//     mbarrier is needed.
//   * Per entry: u = x_m . W_u^T[n] (warp shuffle reduce), h = u * g,
//     partial += h * W_d[n].
// Overflow tiles (count > C) are skipped here; the dense-row path adds them.
#pragma once

#include "ptx.cuh"

namespace twell {

constexpr int kUpdownListCap = 256;  // largest list of a warp (entries per segment; also the N/T limit)
constexpr int kUnitCap = 32;         // largest target entries per unit of a split row

struct UpdownParams {
  const uint16_t* x;
  const uint16_t* wu_t;
  const uint16_t* wd;
  const uint16_t* counts;
  const uint8_t* idx;
  const float* vals;
  int M, K, N, T, C;
  float* y;
  int* ctrl;
  int4* units;     // [M * N/T] published units {row, tile begin, tile end, unused}
  int stages;
  int list_cap;    // list entries per warp: >= N/T and >= C
  int scan_target;                   // rows the split-off units wait for (M; M + 1 only under fault injection)
  unsigned long long wait_limit_ns;  // limit of that wait
  // Small-batch kernel only (twell_updown_small_kernel):
  const int* row_slot;      // [M] dense-row slot of each row (< 0: none)
  const float* dense_rows;  // [R_cap][N] ReLU gates of overflow tiles
  int tiles_per_unit;       // TwELL tiles per static work unit (1..32)
};

// Most warps per CTA: twelve for K <= 2048 (a warp's state then fits the 168
// registers that twelve warps leave each thread without spilling), else eight.
template <int KV>
constexpr int updown_max_warps() {
  return KV <= 8 ? 12 : 8;
}

// acc += h * d for 8 bf16 elements of d, as four packed fp32x2 FMAs (each lane
// of a pair rounds exactly as a scalar fp32 FMA would).
__device__ __forceinline__ void axpy8_bf16(float (&acc)[8], float h, const uint4& d) {
  const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float lo = __uint_as_float(dw[e] << 16);
    const float hi = __uint_as_float(dw[e] & 0xFFFF0000u);
    asm("{\n\t.reg .b64 pa, pb, pc;\n\t"
        "mov.b64 pa, {%2, %3};\n\t"
        "mov.b64 pb, {%4, %4};\n\t"
        "mov.b64 pc, {%0, %1};\n\t"
        "fma.rn.f32x2 pc, pa, pb, pc;\n\t"
        "mov.b64 {%0, %1}, pc;\n\t}"
        : "+f"(acc[2 * e]), "+f"(acc[2 * e + 1]) : "f"(lo), "f"(hi), "f"(h));
  }
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 16-byte asynchronous copy global -> shared (bypassing L1), with an L2
// cache-policy hint.  Completion is tracked per thread with commit/wait groups.
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc, uint64_t policy) {
  asm volatile("cp.async.cg.shared.global.L2::cache_hint [%0], [%1], 16, %2;" ::"r"(smem_u32(smem_dst)), "l"(gsrc),
               "l"(policy)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}
// Wait until at most n of this thread's committed groups are still pending.
__device__ __forceinline__ void cp_async_wait_pending(int n) {
  switch (n) {
    case 0: cp_async_wait<0>(); break;
    case 1: cp_async_wait<1>(); break;
    case 2: cp_async_wait<2>(); break;
    case 3: cp_async_wait<3>(); break;
    case 4: cp_async_wait<4>(); break;
    case 5: cp_async_wait<5>(); break;
    default: cp_async_wait<6>(); break;
  }
}

__device__ __forceinline__ int ld_acquire(const int* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.b32 %0, [%1];" : "=r"(v) : "l"(p) : "memory");
  return v;
}

__device__ __forceinline__ int warp_inclusive_scan(int v, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xffffffffu, v, o);
    if (lane >= o) v += t;
  }
  return v;
}

// Shared memory of one warp: [ring: stages x (2K bf16 W_u row | 2K bf16 W_d row)]
// [list n: int x cap][list g: float x cap].
__host__ __device__ constexpr size_t updown_warp_bytes(int K, int stages, int list_cap) {
  return ((static_cast<size_t>(stages) * 4 * K + static_cast<size_t>(list_cap) * 8) + 127) / 128 * 128;
}

// Per-warp streaming state.  The ring is lane-private in effect: lane l
// copies, and later reads, only the 16-byte pieces l, l + 32, l + 64, ... of
// every row it holds, so no lane ever waits for another lane's copies.
struct WarpRing {
  uint8_t* ring;
  int* list_n;
  float* list_g;
  int list_cap;
  uint32_t slot_bytes;
  int stages;  // >= 2
  uint64_t policy;
};

// Lists the entries (n, g) of the non-overflow tiles [cursor, te) of `row`
// into the warp's list, advancing `cursor`; stops before the list would pass
// its capacity.  Returns the number listed.
__device__ __forceinline__ int list_entries(const UpdownParams& p, const WarpRing& w, int row, int& cursor, int te,
                                            int lane) {
  const int NT = p.N / p.T;
  const uint16_t* crow = p.counts + static_cast<int64_t>(row) * NT;
  int E = 0;
  __syncwarp();  // every lane is done reading the previous list
  while (cursor < te) {
    const int t = cursor + lane;
    const int c = t < te ? static_cast<int>(crow[t]) : 0;
    const int ce = (c > 0 && c <= p.C) ? c : 0;
    const int incl = warp_inclusive_scan(ce, lane);
    const uint32_t fit = __ballot_sync(0xffffffffu, E + incl <= w.list_cap);
    const int k = __popc(fit);  // fitting lanes form a prefix: incl is non-decreasing
    if (lane < k && ce > 0) {
      const int64_t rec = (static_cast<int64_t>(row) * NT + t) * p.C;
      const int off = E + incl - ce;
      const int nbase = t * p.T;
      if ((p.C & 7) == 0) {
        // Eight slots per step: one 8-byte and two 16-byte loads, all issued
        // before the first store (records are 8-slot aligned when C % 8 == 0).
#pragma unroll 1
        for (int s0 = 0; s0 < ce; s0 += 8) {
          const uint2 iv = *reinterpret_cast<const uint2*>(p.idx + rec + s0);
          const float4 v0 = *reinterpret_cast<const float4*>(p.vals + rec + s0);
          const float4 v1 = *reinterpret_cast<const float4*>(p.vals + rec + s0 + 4);
          const float g[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
#pragma unroll
          for (int s = 0; s < 8; ++s) {
            if (s0 + s < ce) {
              const uint32_t word = s < 4 ? iv.x : iv.y;
              w.list_n[off + s0 + s] = nbase + static_cast<int>((word >> (8 * (s & 3))) & 0xFFu);
              w.list_g[off + s0 + s] = g[s];
            }
          }
        }
      } else {
        for (int s = 0; s < ce; ++s) {
          w.list_n[off + s] = nbase + p.idx[rec + s];
          w.list_g[off + s] = p.vals[rec + s];
        }
      }
    }
    if (k > 0) E += __shfl_sync(0xffffffffu, incl, k - 1);
    cursor += k;
    if (k < 32) break;
  }
  if (cursor > te) cursor = te;
  __syncwarp();
  return E;
}

// This lane's pieces of W_u^T[n] and W_d[n] into ring slot `slot`.
template <int KV>
__device__ __forceinline__ void issue_entry(const UpdownParams& p, const WarpRing& w, int slot, int n, int lane) {
  uint4* dst = reinterpret_cast<uint4*>(w.ring + static_cast<size_t>(slot) * w.slot_bytes);
  const uint4* su = reinterpret_cast<const uint4*>(p.wu_t + static_cast<int64_t>(n) * p.K);
  const uint4* sd = reinterpret_cast<const uint4*>(p.wd + static_cast<int64_t>(n) * p.K);
  const int kv = p.K / 8;
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    const int v = j * 32 + lane;
    if (v < kv) {
      cp_async16(dst + v, su + v, w.policy);
      cp_async16(dst + kv + v, sd + v, w.policy);
    }
  }
}

// s[e] += the products of the e-th bf16 pair of a and b: four independent
// accumulation chains per entry instead of one.  The mixed-precision FMA takes
// the bf16 halves as they are (the product of two bf16 numbers is exact in
// fp32), so no unpacking is needed; the result equals fp32 FMAs on the
// widened values.
__device__ __forceinline__ void dot8_acc4(const uint4& a, const uint4& b, float (&s)[4]) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    asm("{\n\t.reg .b16 al, ah, bl, bh;\n\t"
        "mov.b32 {al, ah}, %1;\n\t"
        "mov.b32 {bl, bh}, %2;\n\t"
        "fma.rn.f32.bf16 %0, al, bl, %0;\n\t"
        "fma.rn.f32.bf16 %0, ah, bh, %0;\n\t}"
        : "+f"(s[e]) : "r"(aw[e]), "r"(bw[e]));
  }
}

// Streams the E listed entries through the ring and accumulates them.  Every
// ring slot is one copy group per lane: the first `stages` entries are put in
// flight, and each consumed slot is refilled with the entry `stages` places
// ahead (an empty group past the end keeps the group count uniform).  Entries
// are taken two at a time: the two dot products (four partial sums each), their
// shuffle reductions and the two accumulations are independent, so each warp
// keeps several short dependency chains in flight instead of one long one.
template <int KV>
__device__ __forceinline__ void stream_entries(const UpdownParams& p, const WarpRing& w, int E, const uint4 (&xv)[KV],
                                               float (&acc)[KV][8], int lane) {
  const int S = w.stages;
  for (int e = 0; e < S; ++e) {
    if (e < E) issue_entry<KV>(p, w, e, w.list_n[e], lane);
    cp_async_commit();
  }
  auto slot = [&](int s) { return reinterpret_cast<const uint4*>(w.ring + static_cast<size_t>(s) * w.slot_bytes); };
  int sa = 0;
  for (int e = 0; e < E; e += 2) {
    const bool two = e + 1 < E;
    const int sb = sa + 1 == S ? 0 : sa + 1;
    cp_async_wait_pending(S - 2);  // this lane's pieces of entries e and e + 1 have landed
    const uint4* ua = slot(sa);
    const uint4* ub = slot(sb);
    float qa[4] = {0.f, 0.f, 0.f, 0.f}, qb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      if ((j * 32 + lane) * 8 < p.K) {
        dot8_acc4(xv[j], ua[j * 32 + lane], qa);
        if (two) dot8_acc4(xv[j], ub[j * 32 + lane], qb);
      }
    }
    float part_a = (qa[0] + qa[1]) + (qa[2] + qa[3]);
    float part_b = (qb[0] + qb[1]) + (qb[2] + qb[3]);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      part_a += __shfl_xor_sync(0xffffffffu, part_a, o);
      part_b += __shfl_xor_sync(0xffffffffu, part_b, o);
    }
    const float ha = part_a * w.list_g[e];
    const float hb = two ? part_b * w.list_g[e + 1] : 0.f;
    const uint4* da = ua + p.K / 8;  // the W_d row starts 2K bytes into the slot
    const uint4* db = ub + p.K / 8;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      if ((j * 32 + lane) * 8 < p.K) {
        axpy8_bf16(acc[j], ha, da[j * 32 + lane]);
        if (two) axpy8_bf16(acc[j], hb, db[j * 32 + lane]);
      }
    }
    // The two slots were read (by this lane) above; refill them.
    if (e + S < E) issue_entry<KV>(p, w, sa, w.list_n[e + S], lane);
    cp_async_commit();
    if (e + 1 + S < E) issue_entry<KV>(p, w, sb, w.list_n[e + 1 + S], lane);
    cp_async_commit();
    sa = sb + 1 == S ? 0 : sb + 1;
  }
}

// 16-byte read-only load with an L2 evict-first hint: x rows are read once per
// row or unit, while the gathered weight rows (evict-last) are reused across
// rows and should keep their place in L2.
__device__ __forceinline__ uint4 ldg_evict_first(const uint4* src) {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(pol));
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.L2::cache_hint.v4.u32 {%0, %1, %2, %3}, [%4], %5;"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(src), "l"(pol));
  return v;
}

template <int KV>
__device__ __forceinline__ void load_x(const UpdownParams& p, int row, uint4 (&xv)[KV], float (&acc)[KV][8],
                                       int lane) {
  const uint16_t* xr = p.x + static_cast<int64_t>(row) * p.K;
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    const int k0 = (j * 32 + lane) * 8;
    xv[j] = k0 < p.K ? ldg_evict_first(reinterpret_cast<const uint4*>(xr + k0)) : make_uint4(0, 0, 0, 0);
#pragma unroll
    for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
  }
}

template <int KV>
__device__ __forceinline__ void zero_y(const UpdownParams& p, int row, int lane) {
  float* yr = p.y + static_cast<int64_t>(row) * p.K;
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    const int k0 = (j * 32 + lane) * 8;
    if (k0 < p.K) {
      float4* dst = reinterpret_cast<float4*>(yr + k0);
      dst[0] = make_float4(0.f, 0.f, 0.f, 0.f);
      dst[1] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
}

template <int KV>
__device__ __forceinline__ void write_y(const UpdownParams& p, int row, const float (&acc)[KV][8], bool add,
                                        int lane) {
  float* yr = p.y + static_cast<int64_t>(row) * p.K;
#pragma unroll
  for (int j = 0; j < KV; ++j) {
    const int k0 = (j * 32 + lane) * 8;
    if (k0 < p.K) {
      float4* dst = reinterpret_cast<float4*>(yr + k0);
      const float4 a = make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]);
      const float4 b = make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]);
      if (add) {
        atomicAdd(dst, a);
        atomicAdd(dst + 1, b);
      } else {
        __stcs(dst, a);
        __stcs(dst + 1, b);
      }
    }
  }
}

// Unit k of a row covers tiles [cut(k), cut(k+1)); cut(k) is one past the first
// tile whose inclusive entry prefix reaches ceil(k * total / nunits).
__device__ __forceinline__ int unit_cut(const int* prefix, int NT, int total, int nunits, int k) {
  if (k <= 0) return 0;
  if (k >= nunits) return NT;
  const int target = static_cast<int>((static_cast<int64_t>(k) * total + nunits - 1) / nunits);
  int lo = 0, hi = NT - 1;
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (prefix[mid] >= target)
      hi = mid;
    else
      lo = mid + 1;
  }
  return lo + 1;
}

template <int KV>
__global__ void __launch_bounds__(32 * updown_max_warps<KV>(), 1) twell_updown_kernel(const UpdownParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int NT = p.N / p.T;
  int* ctrl = p.ctrl;

  WarpRing w;
  w.slot_bytes = 4u * p.K;
  w.stages = p.stages;
  w.ring = smem + static_cast<size_t>(warp) * updown_warp_bytes(p.K, p.stages, p.list_cap);
  w.list_n = reinterpret_cast<int*>(w.ring + static_cast<size_t>(p.stages) * w.slot_bytes);
  w.list_g = reinterpret_cast<float*>(w.list_n + p.list_cap);
  w.list_cap = p.list_cap;
  w.policy = l2_evict_last_policy();
  // Set-up above overlaps the previous kernel (programmatic dependent launch).
  griddep_launch_dependents();
  griddep_wait();

  // Units of about two thirds of (total entries / warps) entries, between 2
  // and kUnitCap: larger units when every warp has many entries (fewer fixed
  // per-unit costs), smaller ones when it has few (no warp is left with a
  // long last unit); measured best at 16 for 24 entries per warp and at 32
  // for 130-380.
  const int per_warp = ld_acquire(ctrl + kCtrlEntries) / static_cast<int>(gridDim.x * (blockDim.x >> 5));
  int unit_cap = 2 * per_warp / 3;
  unit_cap = unit_cap < 2 ? 2 : (unit_cap > kUnitCap ? kUnitCap : unit_cap);

  uint4 xv[KV];
  float acc[KV][8];
  bool ok = true;

  // ---------------------------------------------------------------- rows
  while (ok) {
    int row = 0;
    if (lane == 0) row = atomicAdd(ctrl + kCtrlQueue, 1);
    row = __shfl_sync(0xffffffffu, row, 0);
    if (row >= p.M) break;
    load_x<KV>(p, row, xv, acc, lane);

    // Inclusive per-tile prefix of the row's listed entries (list_n as scratch).
    const uint16_t* crow = p.counts + static_cast<int64_t>(row) * NT;
    int total = 0;
    for (int tb = 0; tb < NT; tb += 32) {
      const int t = tb + lane;
      const int c = t < NT ? static_cast<int>(crow[t]) : 0;
      const int ce = (c > 0 && c <= p.C) ? c : 0;
      const int incl = warp_inclusive_scan(ce, lane);
      if (t < NT) w.list_n[t] = total + incl;
      total += __shfl_sync(0xffffffffu, incl, 31);
    }
    __syncwarp();
    int nunits = (total + unit_cap - 1) / unit_cap;
    if (nunits > NT) nunits = NT;
    if (nunits < 1) nunits = 1;
    const int own_end = unit_cut(w.list_n, NT, total, nunits, 1);
    if (nunits > 1) {
      int base = 0;
      if (lane == 0) base = atomicAdd(ctrl + kCtrlUnitTail, nunits - 1);
      base = __shfl_sync(0xffffffffu, base, 0);
      for (int k = 1 + lane; k < nunits; k += 32)
        p.units[base + k - 1] = make_int4(row, unit_cut(w.list_n, NT, total, nunits, k),
                                          unit_cut(w.list_n, NT, total, nunits, k + 1), 0);
      // Every unit of a split row adds into y_m: clear it before any unit is taken.
      zero_y<KV>(p, row, lane);
      __threadfence();
    }
    __syncwarp();
    if (lane == 0) atomicAdd(ctrl + kCtrlScanned, 1);

    int cursor = 0;
    while (ok && cursor < own_end) {
      const int E = list_entries(p, w, row, cursor, own_end, lane);
      if (E > 0) stream_entries<KV>(p, w, E, xv, acc, lane);
    }
    if (!ok) break;
    write_y<KV>(p, row, acc, nunits > 1, lane);
  }

  // ---------------------------------------------------------------- split-off units
  // Units are taken only once every row has been scanned, so every reserved
  // unit record has been written (its writer fenced before counting the row).
  if (ok) {
    int ready = 1;
    if (lane == 0) {
      const unsigned long long t0 = global_ns();
      while (ld_acquire(ctrl + kCtrlScanned) < p.scan_target) {
        if (global_ns() - t0 > p.wait_limit_ns) {
          set_flag(ctrl, kFlagWaitTimeout);
          ready = 0;
          break;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ready, 0) != 0;
  }
  const int n_units = ok ? ld_acquire(ctrl + kCtrlUnitTail) : 0;
  // Every unit is published by now: warp g takes unit g directly, later units
  // come from the queue (numbered from the warp count on), so that the warps
  // arriving together do not all contend for one counter.
  const int n_warps = static_cast<int>(gridDim.x * (blockDim.x >> 5));
  const int gw = static_cast<int>(blockIdx.x * (blockDim.x >> 5)) + warp;
  bool first_unit = true;
  while (ok) {
    int ux = 0, uy = 0, uz = 0;
    int have = 0;
    if (lane == 0) {
      const int h = first_unit ? gw : n_warps + atomicAdd(ctrl + kCtrlUnitHead, 1);
      if (h < n_units) {
        const int4 u = p.units[h];
        ux = u.x;
        uy = u.y;
        uz = u.z;
        have = 1;
      }
    }
    have = __shfl_sync(0xffffffffu, have, 0);
    // No direct unit means fewer units than warps, so the queue is empty too.
    if (!have) break;
    first_unit = false;
    const int row = __shfl_sync(0xffffffffu, ux, 0);
    const int tb = __shfl_sync(0xffffffffu, uy, 0);
    const int te = __shfl_sync(0xffffffffu, uz, 0);
    if (tb >= te) continue;
    load_x<KV>(p, row, xv, acc, lane);
    int cursor = tb;
    int listed = 0;
    while (ok && cursor < te) {
      const int E = list_entries(p, w, row, cursor, te, lane);
      listed += E;
      if (E > 0) stream_entries<KV>(p, w, E, xv, acc, lane);
    }
    if (!ok) break;
    if (listed > 0) write_y<KV>(p, row, acc, true, lane);
  }

  // The last warp out rewinds the queues for the next launch.
  if (lane == 0) {
    __threadfence();
    const int total = gridDim.x * (blockDim.x >> 5);
    if (atomicAdd(ctrl + kCtrlDone, 1) == total - 1) {
      ctrl[kCtrlQueue] = 0;
      ctrl[kCtrlUnitHead] = 0;
      ctrl[kCtrlUnitTail] = 0;
      ctrl[kCtrlScanned] = 0;
      __threadfence();
      ctrl[kCtrlDone] = 0;
    }
  }
}

// ---------------------------------------------------------------------------
// Small batches (at most TWELL_SMALL_M rows).  With few rows the queue-based
// kernel above leaves most warps idle or waiting on the row scan; here the
// work is cut statically instead: unit u is row u / G of the tile group
// u % G (tiles_per_unit consecutive TwELL tiles), and the warps take units
// in turn (numbered warp-major across the CTAs).  A unit holds at most tiles_per_unit * C TwELL entries, so
// every warp's chain is short, and no warp ever waits for another.  Overflow
// tiles are served here too, from the row's dense-row slot (every positive
// gate of the tile, in ascending order): small batches run no dense-row
// GEMMs.  Every unit adds its partial y_m with vector atomics into y, which
// the host clears first.  Weight rows used by several tokens of the batch are
// read from HBM once and then from L2 (evict-last).
// One warp's share of the small-batch units: units first, first + stride, ...
template <int KV>
__device__ __forceinline__ void run_small_units(const UpdownParams& p, const WarpRing& w, int64_t first, int64_t stride,
                                                int lane) {
  const int NT = p.N / p.T;
  const int tpu = p.tiles_per_unit;
  const int groups = (NT + tpu - 1) / tpu;
  const int64_t n_units = static_cast<int64_t>(p.M) * groups;
  uint4 xv[KV];
  float acc[KV][8];
  for (int64_t u = first; u < n_units; u += stride) {
    const int row = static_cast<int>(u / groups);
    const int t0 = static_cast<int>(u - static_cast<int64_t>(row) * groups) * tpu;
    const int t1 = t0 + tpu < NT ? t0 + tpu : NT;
    const int c = t0 + lane < t1 ? static_cast<int>(p.counts[static_cast<int64_t>(row) * NT + t0 + lane]) : 0;
    if (__ballot_sync(0xffffffffu, c > 0) == 0) continue;
    const uint32_t ov = __ballot_sync(0xffffffffu, c > p.C);
    load_x<KV>(p, row, xv, acc, lane);
    int cursor = t0;
    while (cursor < t1) {
      const int E = list_entries(p, w, row, cursor, t1, lane);
      if (E > 0) stream_entries<KV>(p, w, E, xv, acc, lane);
    }
    const int slot = ov ? p.row_slot[row] : -1;
    if (slot >= 0) {
      uint32_t rest = ov;
      int E = 0;
      __syncwarp();
      while (rest) {
        const int t = t0 + __ffs(rest) - 1;
        rest &= rest - 1;
        if (E + p.T > w.list_cap) {
          __syncwarp();
          stream_entries<KV>(p, w, E, xv, acc, lane);
          E = 0;
          __syncwarp();
        }
        const float* src = p.dense_rows + static_cast<int64_t>(slot) * p.N + static_cast<int64_t>(t) * p.T;
        for (int j0 = 0; j0 < p.T; j0 += 32) {
          const float gv = src[j0 + lane];
          const uint32_t bal = __ballot_sync(0xffffffffu, gv > 0.f);
          if (gv > 0.f) {
            const int pos = E + __popc(bal & ((1u << lane) - 1u));
            w.list_n[pos] = t * p.T + j0 + lane;
            w.list_g[pos] = gv;
          }
          E += __popc(bal);
        }
      }
      __syncwarp();
      if (E > 0) stream_entries<KV>(p, w, E, xv, acc, lane);
    }
    write_y<KV>(p, row, acc, true, lane);
  }
}

template <int KV>
__global__ void __launch_bounds__(32 * updown_max_warps<KV>(), 1) twell_updown_small_kernel(const UpdownParams p) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  WarpRing w;
  w.slot_bytes = 4u * p.K;
  w.stages = p.stages;
  w.ring = smem + static_cast<size_t>(warp) * updown_warp_bytes(p.K, p.stages, p.list_cap);
  w.list_n = reinterpret_cast<int*>(w.ring + static_cast<size_t>(p.stages) * w.slot_bytes);
  w.list_g = reinterpret_cast<float*>(w.list_n + p.list_cap);
  w.list_cap = p.list_cap;
  w.policy = l2_evict_last_policy();
  griddep_launch_dependents();
  griddep_wait();
  // Consecutive units go to different SMs (warp-major numbering), so that a
  // batch with fewer units than warps still spreads over every SM.
  run_small_units<KV>(p, w, static_cast<int64_t>(warp) * gridDim.x + blockIdx.x,
                      static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5), lane);
}

}  // namespace twell
