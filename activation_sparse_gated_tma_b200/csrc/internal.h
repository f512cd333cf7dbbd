// Internal launch interface between the C ABI (twell_api.cu) and the kernel
// translation units.  Not part of the public ABI.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stdint.h>

#include <utility>

#include "epilogues.cuh"
#include "tc_gemm.cuh"

namespace twell {

// Gate GEMM with the ReLU + TwELL epilogue.  TwELL tile width T in {128, 256};
// CTA tile width bn in {128, 256}, a multiple of T.
cudaError_t launch_gate_twell(int T, int bn, const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const GemmGeom& g,
                              const GateTwellParams& p, int* ctrl, int grid, cudaStream_t s);
// Gate GEMM on CTA pairs (cta_group::2, 256 x 256 tiles; see tc_gemm_pair_kernel):
// tm_wg's box is 128 rows (each CTA's half of a tile's columns).  grid is even.
cudaError_t launch_gate_twell_pair(int T, const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const GemmGeom& g,
                                   const GateTwellParams& p, int* ctrl, int grid, cudaStream_t s);
// D = A B^T (both K-major), fp32 store (or vector-atomic add), BN = 128.
cudaError_t launch_store_f32_kmajor(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmGeom& g,
                                   const EpiStoreF32::Params& p, int* ctrl, int grid, cudaStream_t s);
// Backward, dense-row slots: dh = [dy_hi | dy_lo] W_d^T with the du/dz/h epilogue, BN = 128.
cudaError_t launch_bwd_slots(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmGeom& g,
                             const EpiBwdSlots::Params& p, int* ctrl, int grid, cudaStream_t s);
// h = (x W_u) * ReLU(x W_g), bf16, BN = 128.
cudaError_t launch_gated_product(const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const CUtensorMap& tm_wu,
                                 const GemmGeom& g, const EpiGatedProduct::Params& p, int* ctrl, int grid,
                                 cudaStream_t s);
// y = h W_d (W_d stored [N][K], read MN-major), fp32 store, BN = 256.
cudaError_t launch_down_store(const CUtensorMap& tm_h, const CUtensorMap& tm_wd, const GemmGeom& g,
                              const EpiStoreF32::Params& p, int* ctrl, int grid, cudaStream_t s);
// Overflow rows: h_over = (x_over W_u) * dense_rows on overflow tiles, BN in {64, 128}.
cudaError_t launch_overflow_product(int bn, const CUtensorMap& tm_xo, const CUtensorMap& tm_wu, const GemmGeom& g,
                                    const EpiOverflowProduct::Params& p, int* ctrl, int grid, cudaStream_t s);
// Overflow rows: y[slot_row[r]] += h_over[r] W_d, BN = 256.
cudaError_t launch_overflow_down(const CUtensorMap& tm_ho, const CUtensorMap& tm_wd, const GemmGeom& g,
                                 const EpiAccumulateRows::Params& p, int* ctrl, int grid, cudaStream_t s);

constexpr int kGateGroupM = 16;

// Launch with programmatic stream serialisation: the kernel may be scheduled
// while the previous kernel in the stream is still running.  Every kernel of
// this library issues griddepcontrol.wait before its first global memory
// access, so ordering is kept; only the launch and set-up overlap.
template <class... KArgs, class... Args>
cudaError_t launch_pdl(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t s, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

// launch_pdl for clusters of two CTAs.
template <class... KArgs, class... Args>
cudaError_t launch_pdl_pair(void (*kern)(KArgs...), int grid, int block, size_t smem, cudaStream_t s,
                            Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(static_cast<unsigned>(grid));
  cfg.blockDim = dim3(static_cast<unsigned>(block));
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = 2;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
}

}  // namespace twell
