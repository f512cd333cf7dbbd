// Fused sparse up + down projection over TwELL ("Sparser, Faster, Lighter
// Transformer Language Models", §3-5):
//
//   y_m = sum_{n in A_m} g_{m,n} * (x_m . W_u[:, n]) * W_d[n, :]
//
// Each warp owns one token row at a time; rows come from a dynamic queue so
// that rows with 10x more active units do not stall a static partition.
//   * x_m (bf16) and the fp32 accumulator of y_m stay in registers, spread over
//     the lanes in 16-byte pieces: lane l holds elements [(j*32 + l)*8, +8).
//   * The warp first lists the row's active units (n, g) from the TwELL
//     records of its non-overflow tiles into shared memory.
//   * Lane 0 streams the rows W_u^T[n] and W_d[n] of upcoming list entries
//     into a private shared-memory ring with 1-D bulk copies (cp.async.bulk,
//     completion on one mbarrier per slot), several entries ahead, so many
//     gathers are in flight per SM without holding them in registers.
//   * For each entry the warp forms u = x_m . W_u^T[n] (warp shuffle reduce),
//     h = u * g, and accumulates h * W_d[n] into y_m.
// Overflow tiles (count > C) are skipped here; the dense-row path adds them.
#pragma once

#include "ptx.cuh"

namespace twell {

constexpr int kUpdownListCap = 256;  // list entries per warp and segment

__device__ __forceinline__ float dot8_bf16(const uint4& a, const uint4& b) {
  const uint32_t aw[4] = {a.x, a.y, a.z, a.w};
  const uint32_t bw[4] = {b.x, b.y, b.z, b.w};
  float s = 0.f;
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    s = fmaf(__uint_as_float(aw[e] << 16), __uint_as_float(bw[e] << 16), s);
    s = fmaf(__uint_as_float(aw[e] & 0xFFFF0000u), __uint_as_float(bw[e] & 0xFFFF0000u), s);
  }
  return s;
}

__device__ __forceinline__ void axpy8_bf16(float (&acc)[8], float h, const uint4& d) {
  const uint32_t dw[4] = {d.x, d.y, d.z, d.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    acc[2 * e] = fmaf(h, __uint_as_float(dw[e] << 16), acc[2 * e]);
    acc[2 * e + 1] = fmaf(h, __uint_as_float(dw[e] & 0xFFFF0000u), acc[2 * e + 1]);
  }
}

__device__ __forceinline__ uint64_t l2_evict_last_policy() {
  uint64_t pol;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(pol));
  return pol;
}

// 1-D bulk copy global -> shared (no multicast), completion on an mbarrier.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar,
                                          uint64_t policy) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1], %2, [%3], %4;" ::"r"(
          smem_u32(smem_dst)),
      "l"(gsrc), "r"(bytes), "r"(smem_u32(bar)), "l"(policy)
      : "memory");
}

__device__ __forceinline__ void fence_proxy_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
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
// [list n: int x cap][list g: float x cap][mbarriers: stages].
__host__ __device__ constexpr size_t updown_warp_bytes(int K, int stages) {
  return ((static_cast<size_t>(stages) * 4 * K + kUpdownListCap * 8 + stages * 8) + 127) / 128 * 128;
}

template <int KV>
__global__ void __launch_bounds__(256, 1)
    twell_updown_kernel(const uint16_t* __restrict__ x, const uint16_t* __restrict__ wu_t,
                        const uint16_t* __restrict__ wd, const uint16_t* __restrict__ counts,
                        const uint8_t* __restrict__ idx, const float* __restrict__ vals, int M, int K, int N,
                        int T, int C, float* __restrict__ y, int* ctrl, int stages) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31;
  const int warp = threadIdx.x >> 5;
  const int NT = N / T;
  const uint32_t slot_bytes = 4u * K;
  uint8_t* base = smem + static_cast<size_t>(warp) * updown_warp_bytes(K, stages);
  uint8_t* ring = base;
  int* list_n = reinterpret_cast<int*>(ring + static_cast<size_t>(stages) * slot_bytes);
  float* list_g = reinterpret_cast<float*>(list_n + kUpdownListCap);
  uint64_t* bars = reinterpret_cast<uint64_t*>(list_g + kUpdownListCap);
  if (lane == 0) {
    for (int s = 0; s < stages; ++s) mbar_init(&bars[s], 1);
    fence_barrier_init();
  }
  __syncwarp();
  const uint64_t policy = l2_evict_last_policy();

  int* queue = ctrl + kCtrlQueue;
  int* done = ctrl + kCtrlQueue + 1;
  int head = 0;            // ring slot of the next list entry
  uint32_t head_phase = 0;  // parity that slot's mbarrier completes next
  bool ok = true;

  while (ok) {
    int row = 0;
    if (lane == 0) row = atomicAdd(queue, 1);
    row = __shfl_sync(0xffffffffu, row, 0);
    if (row >= M) break;

    uint4 xv[KV];
    float acc[KV][8];
    const uint16_t* xr = x + static_cast<int64_t>(row) * K;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      const int k0 = (j * 32 + lane) * 8;
      xv[j] = k0 < K ? *reinterpret_cast<const uint4*>(xr + k0) : make_uint4(0, 0, 0, 0);
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[j][e] = 0.f;
    }

    const uint16_t* crow = counts + static_cast<int64_t>(row) * NT;
    int tile_cursor = 0;
    while (ok && tile_cursor < NT) {
      // ---- list the active units of the next tiles (at most kUpdownListCap entries)
      int E = 0;
      while (tile_cursor < NT) {
        const int t = tile_cursor + lane;
        const int c = t < NT ? static_cast<int>(crow[t]) : 0;
        const int ce = (c > 0 && c <= C) ? c : 0;
        const int incl = warp_inclusive_scan(ce, lane);
        const uint32_t fit = __ballot_sync(0xffffffffu, E + incl <= kUpdownListCap);
        const int k = __popc(fit);  // fitting lanes form a prefix (incl is non-decreasing)
        if (lane < k && ce > 0) {
          const int64_t rec = (static_cast<int64_t>(row) * NT + t) * C;
          const int off = E + incl - ce;
          for (int s = 0; s < ce; ++s) {
            list_n[off + s] = t * T + idx[rec + s];
            list_g[off + s] = vals[rec + s];
          }
        }
        if (k > 0) E += __shfl_sync(0xffffffffu, incl, k - 1);
        tile_cursor += min(k, 32);
        if (k < 32) break;
      }
      __syncwarp();
      if (E == 0) continue;

      // ---- stream the listed rows through the ring
      const int pre = min(stages, E);
      if (lane == 0) {
        int s = head;
        for (int e = 0; e < pre; ++e) {
          const int n = list_n[e];
          uint8_t* dst = ring + static_cast<size_t>(s) * slot_bytes;
          mbar_arrive_expect_tx(&bars[s], slot_bytes);
          bulk_load(dst, wu_t + static_cast<int64_t>(n) * K, slot_bytes / 2, &bars[s], policy);
          bulk_load(dst + slot_bytes / 2, wd + static_cast<int64_t>(n) * K, slot_bytes / 2, &bars[s], policy);
          if (++s == stages) s = 0;
        }
      }
      int consumed = 0;
      for (int e = 0; e < E; ++e) {
        const int s = head;
        if (!mbar_wait(&bars[s], head_phase, ctrl)) { ok = false; break; }
        const uint4* su = reinterpret_cast<const uint4*>(ring + static_cast<size_t>(s) * slot_bytes);
        const uint4* sd = su + K / 8;  // W_d row starts 2K bytes into the slot
        const float g = list_g[e];
        float part = 0.f;
#pragma unroll
        for (int j = 0; j < KV; ++j)
          if ((j * 32 + lane) * 8 < K) part += dot8_bf16(xv[j], su[j * 32 + lane]);
        const float h = warp_sum(part) * g;
#pragma unroll
        for (int j = 0; j < KV; ++j)
          if ((j * 32 + lane) * 8 < K) axpy8_bf16(acc[j], h, sd[j * 32 + lane]);
        __syncwarp();
        ++consumed;
        if (lane == 0 && e + stages < E) {
          // All lanes finished reading slot s; refill it with entry e + stages.
          fence_proxy_async_smem();
          const int n = list_n[e + stages];
          uint8_t* dst = ring + static_cast<size_t>(s) * slot_bytes;
          mbar_arrive_expect_tx(&bars[s], slot_bytes);
          bulk_load(dst, wu_t + static_cast<int64_t>(n) * K, slot_bytes / 2, &bars[s], policy);
          bulk_load(dst + slot_bytes / 2, wd + static_cast<int64_t>(n) * K, slot_bytes / 2, &bars[s], policy);
        }
        if (++head == stages) { head = 0; head_phase ^= 1u; }
      }
      if (!ok) {
        // Let copies already in flight land before the CTA can exit (bounded).
        int s = head;
        uint32_t ph = head_phase;
        for (int e = consumed; e < min(E, consumed + stages); ++e) {
          mbar_wait(&bars[s], ph, ctrl);
          if (++s == stages) { s = 0; ph ^= 1u; }
        }
      }
      __syncwarp();
    }
    if (!ok) break;

    float* yr = y + static_cast<int64_t>(row) * K;
#pragma unroll
    for (int j = 0; j < KV; ++j) {
      const int k0 = (j * 32 + lane) * 8;
      if (k0 < K) {
        __stcs(reinterpret_cast<float4*>(yr + k0), make_float4(acc[j][0], acc[j][1], acc[j][2], acc[j][3]));
        __stcs(reinterpret_cast<float4*>(yr + k0) + 1, make_float4(acc[j][4], acc[j][5], acc[j][6], acc[j][7]));
      }
    }
  }
  // The last warp out rewinds the queue so the next launch starts from row 0.
  if (lane == 0) {
    const int total = gridDim.x * (blockDim.x >> 5);
    if (atomicAdd(done, 1) == total - 1) {
      atomicExch(queue, 0);
      atomicExch(done, 0);
    }
  }
}

}  // namespace twell
