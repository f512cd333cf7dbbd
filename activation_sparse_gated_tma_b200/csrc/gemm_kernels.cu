// Instantiations of the tcgen05 GEMM engine for the gate, dense-FFN and
// overflow stages.
#include "internal.h"

namespace twell {

namespace {

template <int BN, bool B_MN, bool DUAL, int STAGES, class Epi>
cudaError_t launch(const CUtensorMap& a, const CUtensorMap& b, const CUtensorMap& b2, const GemmGeom& g,
                   const typename Epi::Params& ep, int* ctrl, int grid, cudaStream_t s) {
  constexpr int warps = Epi::template kWarps<BN>;
  constexpr size_t smem = gemm_smem_bytes<BN, DUAL, STAGES, Epi::kScratchBytes, warps>();
  static_assert(smem <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
  auto kern = tc_gemm_kernel<BN, B_MN, DUAL, STAGES, Epi>;
  // The attribute is per device; setting it is cheap and idempotent.
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  return launch_pdl(kern, grid, gemm_threads<Epi, BN>(), smem, s, a, b, b2, g, ep, ctrl);
}

}  // namespace

cudaError_t launch_gate_twell(int T, int bn, const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const GemmGeom& g,
                              const GateTwellParams& p, int* ctrl, int grid, cudaStream_t s) {
  if (T == 128 && bn == 128) return launch<128, false, false, 6, EpiGateTwell<128>>(tm_x, tm_wg, tm_wg, g, p, ctrl, grid, s);
  if (T == 128 && bn == 256) return launch<256, false, false, 4, EpiGateTwell<128>>(tm_x, tm_wg, tm_wg, g, p, ctrl, grid, s);
  if (T == 256 && bn == 256) return launch<256, false, false, 4, EpiGateTwell<256>>(tm_x, tm_wg, tm_wg, g, p, ctrl, grid, s);
  return cudaErrorInvalidValue;
}

namespace {
template <int T>
cudaError_t launch_pair_t(const CUtensorMap& a, const CUtensorMap& b, const GemmGeom& g, const GateTwellParams& p,
                          int* ctrl, int grid, cudaStream_t s) {
  using Epi = EpiGateTwell<T>;
  constexpr int warps = Epi::template kWarps<256>;
  constexpr int kStages = gemm_pair_smem_bytes<6, Epi::kScratchBytes, warps>() <= 232448 ? 6 : 5;
  constexpr size_t smem = gemm_pair_smem_bytes<kStages, Epi::kScratchBytes, warps>();
  static_assert(smem <= 232448, "exceeds the 227 KB per-CTA shared memory limit");
  auto kern = tc_gemm_pair_kernel<kStages, Epi>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  if (grid <= 0) return cudaSuccess;
  return launch_pdl_pair(kern, grid, gemm_threads<Epi, 256>(), smem, s, a, b, g, p, ctrl);
}
}  // namespace

cudaError_t launch_gate_twell_pair(int T, const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const GemmGeom& g,
                                   const GateTwellParams& p, int* ctrl, int grid, cudaStream_t s) {
  if (grid % 2) return cudaErrorInvalidValue;
  if (T == 128) return launch_pair_t<128>(tm_x, tm_wg, g, p, ctrl, grid, s);
  if (T == 256) return launch_pair_t<256>(tm_x, tm_wg, g, p, ctrl, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_store_f32_kmajor(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmGeom& g,
                                   const EpiStoreF32::Params& p, int* ctrl, int grid, cudaStream_t s) {
  return launch<128, false, false, 6, EpiStoreF32>(tm_a, tm_b, tm_b, g, p, ctrl, grid, s);
}

cudaError_t launch_bwd_slots(const CUtensorMap& tm_a, const CUtensorMap& tm_b, const GemmGeom& g,
                             const EpiBwdSlots::Params& p, int* ctrl, int grid, cudaStream_t s) {
  return launch<128, false, false, 6, EpiBwdSlots>(tm_a, tm_b, tm_b, g, p, ctrl, grid, s);
}

cudaError_t launch_gated_product(const CUtensorMap& tm_x, const CUtensorMap& tm_wg, const CUtensorMap& tm_wu,
                                 const GemmGeom& g, const EpiGatedProduct::Params& p, int* ctrl, int grid,
                                 cudaStream_t s) {
  return launch<128, false, true, 4, EpiGatedProduct>(tm_x, tm_wg, tm_wu, g, p, ctrl, grid, s);
}

cudaError_t launch_down_store(const CUtensorMap& tm_h, const CUtensorMap& tm_wd, const GemmGeom& g,
                              const EpiStoreF32::Params& p, int* ctrl, int grid, cudaStream_t s) {
  return launch<256, true, false, 4, EpiStoreF32>(tm_h, tm_wd, tm_wd, g, p, ctrl, grid, s);
}

cudaError_t launch_overflow_product(int bn, const CUtensorMap& tm_xo, const CUtensorMap& tm_wu, const GemmGeom& g,
                                    const EpiOverflowProduct::Params& p, int* ctrl, int grid, cudaStream_t s) {
  if (bn == 64) return launch<64, false, false, 8, EpiOverflowProduct>(tm_xo, tm_wu, tm_wu, g, p, ctrl, grid, s);
  if (bn == 128) return launch<128, false, false, 6, EpiOverflowProduct>(tm_xo, tm_wu, tm_wu, g, p, ctrl, grid, s);
  return cudaErrorInvalidValue;
}

cudaError_t launch_overflow_down(const CUtensorMap& tm_ho, const CUtensorMap& tm_wd, const GemmGeom& g,
                                 const EpiAccumulateRows::Params& p, int* ctrl, int grid, cudaStream_t s) {
  return launch<256, true, false, 4, EpiAccumulateRows>(tm_ho, tm_wd, tm_wd, g, p, ctrl, grid, s);
}

}  // namespace twell
