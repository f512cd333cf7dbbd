// Small-batch forward in one persistent kernel ("Sparser, Faster, Lighter
// Transformer Language Models", §3-4 and §3-5, one pass from gate to y):
//
//   phase 1  the stream-K gate pass of small_batch.cuh: W_g streams through
//            the tensor cores, the last CTA of every TwELL tile packs it
//            (records, counts, dense-row slots); every CTA also clears its
//            slice of y;
//   phase 2  a grid barrier (one counter; each CTA adds itself and waits,
//            bounded, for all; a wait that gives up raises kFlagWaitTimeout
//            and the CTA returns, so the host sees TWELL_ERR_DEVICE_CHECK);
//   phase 3  the small-batch up/down units of sparse_updown.cuh on all warps
//            of the CTA, with the operand ring's shared memory reused as the
//            warps' weight-row rings.
//
// The grid is at most one CTA per SM (its shared memory allows no second
// one), so every CTA of the grid is resident and the barrier completes.
#pragma once

#include "small_batch.cuh"
#include "sparse_updown.cuh"

namespace twell {

template <int KV>
__global__ void __launch_bounds__(192, 1)
    twell_fused_small_kernel(const __grid_constant__ CUtensorMap tmW, const __grid_constant__ CUtensorMap tmX,
                             const GateStreamParams gp, const UpdownParams up, int* ctrl) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* base = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~uintptr_t(1023));
  GateStreamShared* sh = reinterpret_cast<GateStreamShared*>(base);
  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {  // kernel parameters: safe to touch before the dependency resolves
    prefetch_tmap(&tmW);
    prefetch_tmap(&tmX);
  }
  stream_setup(sh, gp);
  griddep_launch_dependents();
  griddep_wait();

  // y is the sum of the units' partials: every CTA clears its slice first.
  {
    const int64_t n4 = static_cast<int64_t>(up.M) * up.K / 4;
    const int64_t a = static_cast<int64_t>(blockIdx.x) * n4 / gridDim.x;
    const int64_t b = (static_cast<int64_t>(blockIdx.x) + 1) * n4 / gridDim.x;
    float4* y4 = reinterpret_cast<float4*>(up.y);
    for (int64_t i = a + threadIdx.x; i < b; i += blockDim.x) y4[i] = make_float4(0.f, 0.f, 0.f, 0.f);
  }

  stream_run(&tmW, &tmX, gp, ctrl, sh, base + kStreamCtrlBytes);
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(sh->tmem, stream_tmem_cols(gp.mp));

  // Grid barrier: TwELL, the dense-row slots and the cleared y are complete.
  if (threadIdx.x == 0) {
    __threadfence();
    atomicAdd(ctrl + kCtrlGridSync, 1);
    int ok = 1;
    const unsigned long long t0 = global_ns();
    while (ld_acquire(ctrl + kCtrlGridSync) < up.scan_target) {
      if (global_ns() - t0 > up.wait_limit_ns) {
        set_flag(ctrl, kFlagWaitTimeout);
        ok = 0;
        break;
      }
    }
    sh->sync_ok = ok;
  }
  __syncthreads();
  if (!sh->sync_ok) return;
  fence_acq_rel_gpu();
  fence_proxy_async_smem();  // the ring's bytes were last touched by TMA and the tensor cores

  WarpRing w;
  w.slot_bytes = 4u * up.K;
  w.stages = up.stages;
  w.ring = base + kStreamCtrlBytes + static_cast<size_t>(warp) * updown_warp_bytes(up.K, up.stages, up.list_cap);
  w.list_n = reinterpret_cast<int*>(w.ring + static_cast<size_t>(up.stages) * w.slot_bytes);
  w.list_g = reinterpret_cast<float*>(w.list_n + up.list_cap);
  w.list_cap = up.list_cap;
  w.policy = l2_evict_last_policy();
  run_small_units<KV>(up, w, static_cast<int64_t>(warp) * gridDim.x + blockIdx.x,
                      static_cast<int64_t>(gridDim.x) * (blockDim.x >> 5), lane);
}

}  // namespace twell
