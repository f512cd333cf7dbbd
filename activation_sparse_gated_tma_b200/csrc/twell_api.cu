// C ABI of the sparse gated FFN forward path (declared in include/twell.h).
// Host side only does validation, TMA descriptor encoding and launches;
// every arithmetic step runs in the kernels.
#include <cudaTypedefs.h>

#include <cstdarg>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <tuple>

#include "../../include/twell.h"
#include "internal.h"
#include "fused_small.cuh"
#include "sparse_backward.cuh"

namespace twell {
namespace {

// Batches up to this many rows take the static-unit up/down kernel (no work
// queues, overflow tiles gathered from the dense-row slots): with few rows
// the queue-based kernel's row scan and unit hand-off are a long serial
// chain, and the dense-row GEMMs run near-empty.  (Measured at 99% and 99.9%
// sparsity, K=2048, N=8192: M=256 60 -> 57 us and 43 -> 30 us; at M=1024 the
// queue-based kernel is faster.)
constexpr int kStaticUpdownMaxM = 256;

thread_local char g_err[512] = "";
thread_local int g_launches = 0;
// One-shot fault injection (twell_test_expire_wait): the wait limit, in ns, of
// the next fused-kernel launch on this thread, whose wait target is then made
// unreachable; 0 = none.
thread_local long long g_expire_wait_ns = 0;
// Route of the slotted rows in twell_ffn_bwd on this thread
// (twell_bwd_slot_route): 0 by cost, 1 the dense-slot GEMMs, 2 the gather passes.
thread_local int g_bwd_slot_route = 0;

// Optional launch tracing: events[2i] / events[2i+1] bracket the i-th kernel.
struct Trace {
  cudaEvent_t* events = nullptr;
  int capacity = 0;
  int count = 0;
  const char* names[256];
};
thread_local Trace g_trace;

cudaError_t trace_begin(cudaStream_t s) {
  if (g_trace.events && g_trace.count < g_trace.capacity) return cudaEventRecord(g_trace.events[2 * g_trace.count], s);
  return cudaSuccess;
}
cudaError_t trace_end(cudaStream_t s, const char* name) {
  ++g_launches;
  if (g_trace.events && g_trace.count < g_trace.capacity) {
    cudaError_t e = cudaEventRecord(g_trace.events[2 * g_trace.count + 1], s);
    if (e != cudaSuccess) return e;
    if (g_trace.count < 256) g_trace.names[g_trace.count] = name;
    ++g_trace.count;
  }
  return cudaSuccess;
}

twell_status fail(twell_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof g_err, fmt, ap);
  va_end(ap);
  return st;
}

#define TW_CUDA(expr)                                                                              \
  do {                                                                                             \
    cudaError_t e_ = (expr);                                                                       \
    if (e_ != cudaSuccess) return fail(TWELL_ERR_CUDA, "%s: %s", #expr, cudaGetErrorString(e_)); \
  } while (0)

bool aligned16(const void* p) { return p && (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ---------------------------------------------------------------- device info
struct DeviceInfo {
  int sms = 0;
  int cc_major = 0;
};

twell_status device_info(DeviceInfo& info) {
  int dev = 0;
  TW_CUDA(cudaGetDevice(&dev));
  static std::mutex mu;
  static std::map<int, DeviceInfo> cache;
  std::lock_guard<std::mutex> lock(mu);
  auto it = cache.find(dev);
  if (it == cache.end()) {
    DeviceInfo d;
    TW_CUDA(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
    TW_CUDA(cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev));
    it = cache.emplace(dev, d).first;
  }
  info = it->second;
  if (info.cc_major != 10) return fail(TWELL_ERR_UNSUPPORTED, "needs an sm_100 device (found cc %d.x)", info.cc_major);
  return TWELL_OK;
}

// ---------------------------------------------------------------- TMA descriptors
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// bf16 row-major [outer][inner] matrix, box [box_outer][64], 128-byte swizzle,
// zero fill out of bounds.  Cached by (device, pointer, shape, box).
twell_status tmap_bf16(const void* ptr, uint64_t inner, uint64_t outer, uint32_t box_outer, CUtensorMap& out) {
  using Key = std::tuple<int, uintptr_t, uint64_t, uint64_t, uint32_t>;
  static std::mutex mu;
  static std::map<Key, CUtensorMap> cache;
  int dev = 0;
  TW_CUDA(cudaGetDevice(&dev));
  const Key key{dev, reinterpret_cast<uintptr_t>(ptr), inner, outer, box_outer};
  {
    std::lock_guard<std::mutex> lock(mu);
    auto it = cache.find(key);
    if (it != cache.end()) {
      out = it->second;
      return TWELL_OK;
    }
  }
  auto enc = encode_fn();
  if (!enc) return fail(TWELL_ERR_CUDA, "cuTensorMapEncodeTiled is not available from the driver");
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {inner * 2};
  cuuint32_t box[2] = {64, box_outer};
  cuuint32_t estr[2] = {1, 1};
  CUresult r = enc(&out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), dims, strides, box, estr,
                   CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                   CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) return fail(TWELL_ERR_CUDA, "cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
  std::lock_guard<std::mutex> lock(mu);
  if (cache.size() > 4096) cache.clear();
  cache.emplace(key, out);
  return TWELL_OK;
}

// ---------------------------------------------------------------- buffer layout
size_t align256(size_t v) { return (v + 255) & ~size_t(255); }

struct Layout {
  size_t ctrl, counts, idx, vals, row_slot, slot_row, dense_rows, x_over, h_over, units, z, total;
};

bool shape_ok(int M, int K, int N, int T, int C, int R_cap) {
  return M >= 1 && K >= 64 && K <= 4096 && K % 64 == 0 && (T == 128 || T == 256) && N >= T && N % T == 0 &&
         N / T <= kUpdownListCap &&
         C >= 1 && C <= T && C <= 255 && R_cap >= 1 && static_cast<int64_t>(M) * N < (int64_t(1) << 40);
}

Layout layout(int M, int K, int N, int T, int C, int R_cap) {
  const size_t NT = static_cast<size_t>(N / T);
  Layout L;
  size_t o = 0;
  L.ctrl = o; o = align256(o + kCtrlWords * sizeof(int));
  L.counts = o; o = align256(o + size_t(M) * NT * 2);
  L.idx = o; o = align256(o + size_t(M) * NT * C);
  L.vals = o; o = align256(o + size_t(M) * NT * C * 4);
  L.row_slot = o; o = align256(o + size_t(M) * 4);
  L.slot_row = o; o = align256(o + size_t(R_cap) * 4);
  L.dense_rows = o; o = align256(o + size_t(R_cap) * N * 4);
  L.x_over = o; o = align256(o + size_t(R_cap) * K * 2);
  L.h_over = o; o = align256(o + size_t(R_cap) * N * 4);
  L.units = o; o = align256(o + size_t(M) * NT * 16);
  // Small batches: partial gate sums [N/128][kStreamSlots][M][128] fp32, then one ticket per TwELL tile.
  L.z = o; o = align256(o + (M <= TWELL_SMALL_M ? size_t(kStreamSlots) * M * N * 4 + NT * 4 : 0));
  L.total = o;
  return L;
}

twell_status check_buf(const twell_buf* tw) {
  if (!tw) return fail(TWELL_ERR_INVALID, "twell_buf is NULL");
  if (!shape_ok(tw->M, tw->K, tw->N, tw->T, tw->C, tw->R_cap)) return fail(TWELL_ERR_INVALID, "twell_buf has invalid sizes");
  if (!tw->counts || !tw->idx || !tw->vals || !tw->dense_rows || !tw->row_slot || !tw->slot_row || !tw->ctrl ||
      !tw->x_over || !tw->h_over || !tw->units || (tw->M <= TWELL_SMALL_M && !tw->z))
    return fail(TWELL_ERR_INVALID, "twell_buf is not initialised");
  return TWELL_OK;
}

// ---------------------------------------------------------------- small kernels
// Start of a gate pass: no row holds a dense-row slot, control words at zero.
// The small-batch path also clears its n_tickets tile tickets.
__global__ void twell_reset_kernel(int* __restrict__ row_slot, int M, int* __restrict__ ctrl, int* __restrict__ tickets,
                                   int n_tickets) {
  griddep_launch_dependents();
  griddep_wait();
  const int i = blockIdx.x * blockDim.x + threadIdx.x;
  if (i < kCtrlWords) ctrl[i] = 0;
  for (int r = i; r < M; r += gridDim.x * blockDim.x) row_slot[r] = kSlotFree;
  for (int k = i; k < n_tickets; k += gridDim.x * blockDim.x) tickets[k] = 0;
}

// Tickets of the small-batch gate pass (after the partial sums in z).
int* small_tickets(const twell_buf* tw) {
  return reinterpret_cast<int*>(tw->z + static_cast<size_t>(kStreamSlots) * tw->M * tw->N);
}

// Operand ring depth of the small-batch gate pass in `budget` bytes of
// shared memory (at most kStreamMaxStages).
int stream_stages(int mp, size_t budget) {
  const size_t fixed = 1024 + kStreamCtrlBytes;
  const int st = budget > fixed ? static_cast<int>((budget - fixed) / stream_stage_bytes(mp)) : 0;
  return st > kStreamMaxStages ? kStreamMaxStages : st;
}

// Small-batch gate pass (gp.mp, gp.stages set by the caller).
cudaError_t launch_gate_stream(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const GateStreamParams& gp, int* ctrl,
                               int grid, cudaStream_t s) {
  const size_t smem = stream_smem_bytes(gp.mp, gp.stages);
  if (gp.stages < 2 || smem > 232448) return cudaErrorInvalidValue;
  cudaError_t e = cudaFuncSetAttribute(gate_stream_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(gate_stream_kernel, grid, 192, smem, s, tm_w, tm_x, gp, ctrl);
}

// Start of a gate pass (both paths): control words, row slots and, for small
// batches, the tile tickets.
cudaError_t launch_reset(const twell_buf* tw, cudaStream_t s) {
  const bool small = tw->z != nullptr;
  const int n_tickets = small ? tw->N / tw->T : 0;
  const int rwork = tw->M > n_tickets ? tw->M : n_tickets;
  const int rgrid = (rwork + 255) / 256 < 1024 ? (rwork + 255) / 256 : 1024;
  return launch_pdl(twell_reset_kernel, rgrid > 0 ? rgrid : 1, 256, 0, s, tw->row_slot, tw->M, tw->ctrl,
                    small ? small_tickets(tw) : nullptr, n_tickets);
}

GateTwellParams gate_twell_params(const uint16_t* x, const twell_buf* tw) {
  GateTwellParams p;
  p.counts = tw->counts; p.idx = tw->idx; p.vals = tw->vals; p.dense_rows = tw->dense_rows;
  p.row_slot = tw->row_slot; p.slot_row = tw->slot_row; p.x = x; p.x_over = tw->x_over;
  p.N = tw->N; p.K = tw->K; p.C = tw->C; p.r_cap = tw->R_cap;
  return p;
}

// Tensor maps, parameters and grid of the small-batch gate pass: stream-K over
// W_g with the tokens on the narrow side of the tile, ranges of at least a
// third of a tile's k blocks (so at most kStreamSlots CTAs meet a tile), at
// most one CTA per SM.
twell_status small_gate_plan(const uint16_t* x, const uint16_t* wg_t, const twell_buf* tw, int sms, size_t smem_budget,
                             CUtensorMap& tm_w, CUtensorMap& tm_x, GateStreamParams& gp, int& grid) {
  const int M = tw->M, K = tw->K, N = tw->N;
  const int mp = M <= 16 ? 16 : M <= 32 ? 32 : M <= 64 ? 64 : 128;
  twell_status st;
  if ((st = tmap_bf16(wg_t, K, N, 128, tm_w)) != TWELL_OK) return st;
  if ((st = tmap_bf16(x, K, M, mp, tm_x)) != TWELL_OK) return st;
  gp.pk = gate_twell_params(x, tw);
  gp.part = tw->z;
  gp.tickets = small_tickets(tw);
  gp.M = M;
  gp.T = tw->T;
  gp.kb = K / kBK;
  gp.units = static_cast<int64_t>(N / 128) * gp.kb;
  gp.mp = mp;
  gp.stages = stream_stages(mp, smem_budget);
  const int64_t pmin = (gp.kb + 2) / 3;
  const int64_t by_len = gp.units / pmin;
  grid = static_cast<int>(by_len < sms ? (by_len > 0 ? by_len : 1) : sms);
  gp.grid = grid;
  return TWELL_OK;
}

// Small-batch up/down parameters for `warps_total` warps (each with `stages`
// ring stages and the full entry list).
UpdownParams small_updown_params(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw,
                                 float* y, int stages, int64_t warps_total) {
  UpdownParams p = {};
  p.x = x; p.wu_t = wu_t; p.wd = wd;
  p.counts = tw->counts; p.idx = tw->idx; p.vals = tw->vals;
  p.M = tw->M; p.K = tw->K; p.N = tw->N; p.T = tw->T; p.C = tw->C;
  p.y = y; p.ctrl = tw->ctrl;
  p.stages = stages;
  p.list_cap = kUpdownListCap;
  p.row_slot = tw->row_slot;
  p.dense_rows = tw->dense_rows;
  p.scan_target = 0;
  p.wait_limit_ns = kWaitLimitNs;
  // About one unit per warp, each within the list (tiles * C <= list) and one ballot (<= 32 tiles).
  const int NT = tw->N / tw->T;
  const int64_t records = static_cast<int64_t>(tw->M) * NT;
  int tpu = static_cast<int>((records + warps_total - 1) / warps_total);
  const int tpu_max = kUpdownListCap / tw->C < 32 ? kUpdownListCap / tw->C : 32;
  p.tiles_per_unit = tpu < 1 ? 1 : (tpu > tpu_max ? tpu_max : tpu);
  return p;
}

template <int KV>
cudaError_t launch_fused_small_kv(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const GateStreamParams& gp,
                                  const UpdownParams& up, int* ctrl, int grid, size_t smem, cudaStream_t s) {
  cudaError_t e = cudaFuncSetAttribute(twell_fused_small_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(twell_fused_small_kernel<KV>, grid, 192, smem, s, tm_w, tm_x, gp, up, ctrl);
}

cudaError_t launch_fused_small(const CUtensorMap& tm_w, const CUtensorMap& tm_x, const GateStreamParams& gp,
                               const UpdownParams& up, int* ctrl, int grid, size_t smem, cudaStream_t s) {
  switch ((up.K + 255) / 256) {
#define TW_KV(n) \
  case n:        \
    return launch_fused_small_kv<n>(tm_w, tm_x, gp, up, ctrl, grid, smem, s);
    TW_KV(1) TW_KV(2) TW_KV(3) TW_KV(4) TW_KV(5) TW_KV(6) TW_KV(7) TW_KV(8)
    TW_KV(9) TW_KV(10) TW_KV(11) TW_KV(12) TW_KV(13) TW_KV(14) TW_KV(15) TW_KV(16)
#undef TW_KV
    default:
      return cudaErrorInvalidValue;
  }
}

// ---------------------------------------------------------------- backward
constexpr int kBwdMaxK = 2560;      // the row pass keeps x, dy and dx pieces of a row in registers
constexpr int kBwdGatherSlots = 8;  // up to this many slotted rows always go through the gather passes

// Whether the slotted rows' backward goes through the eight dense-slot GEMMs
// rather than the gather passes, given R slotted rows holding `entries`
// active entries.  Measured on one B200 (whole backward): the GEMMs cost
// about 30 us + 26 ps per weight element N*K (launch- and tail-bound at these
// row counts: M=2048 K=1536 N=4096 0.21 ms, M=8192 K=2048 N=5632 0.40 ms,
// M=16384 K=2560 N=10240 0.70 ms), an entry in the gather passes about
// 1.6 ps per K column.  The cut-over is taken a little short of the break-even
// count, at 14 N + 12e6 / K entries.
bool bwd_dense_slots(int R, long long entries, int N, int K) {
  if (g_bwd_slot_route == 1) return R > 0;
  if (g_bwd_slot_route == 2 || R <= kBwdGatherSlots) return false;
  return entries > 14LL * N + 12000000LL / K;
}

struct BwdLayout {
  size_t cnt, fill, row_entries, over_total, off, row_units, piece_off, piece_unit, entries;
  // dense-row slots (R_pad = R_cap rounded up to 64)
  size_t dy_cat, dy_hi, dy_lo, x_pad, u, du_rows, dz_rows, h_t, du_t, dz_t;
  size_t total;
  int64_t cap;
  int r_pad_max;
};

BwdLayout bwd_layout(int M, int K, int N, int T, int C, int R_cap) {
  BwdLayout L;
  L.cap = static_cast<int64_t>(M) * (N / T) * C + static_cast<int64_t>(R_cap) * N;
  L.r_pad_max = (R_cap + 63) / 64 * 64;
  const size_t rp = static_cast<size_t>(L.r_pad_max);
  size_t o = 0;
  L.cnt = o; o = align256(o + size_t(N) * 4);
  L.fill = o; o = align256(o + size_t(N) * 4);
  L.row_entries = o; o = align256(o + size_t(M) * 4);
  L.over_total = o; o = align256(o + 4);
  L.off = o; o = align256(o + size_t(N + 1) * 4);
  L.row_units = o; o = align256(o + size_t(M + 1) * 4);
  L.piece_off = o; o = align256(o + size_t(N + 1) * 4);
  // pieces = sum over units of max(1, ceil(cnt / 64)) <= N + cap / 64
  L.piece_unit = o; o = align256(o + (size_t(N) + size_t(L.cap / 64) + 1) * 4);
  L.entries = o; o = align256(o + size_t(L.cap) * sizeof(BwdEntry));
  L.dy_cat = o; o = align256(o + rp * 2 * K * 2);
  L.dy_hi = o; o = align256(o + rp * K * 2);
  L.dy_lo = o; o = align256(o + rp * K * 2);
  L.x_pad = o; o = align256(o + rp * K * 2);
  L.u = o; o = align256(o + rp * N * 4);
  L.du_rows = o; o = align256(o + rp * 2 * N * 2);
  L.dz_rows = o; o = align256(o + rp * 2 * N * 2);
  L.h_t = o; o = align256(o + size_t(N) * 2 * rp * 2);
  L.du_t = o; o = align256(o + size_t(N) * 2 * rp * 2);
  L.dz_t = o; o = align256(o + size_t(N) * 2 * rp * 2);
  L.total = o;
  return L;
}

template <int KV>
cudaError_t launch_bwd_rows_kv(BwdParams p, int sms, cudaStream_t s) {
  constexpr size_t kBudget = 232448;
  const size_t list = static_cast<size_t>(kUpdownListCap) * 20 + 128;  // n, g, h, du, dz per listed entry
  int warps = bwd_max_warps<KV>(), stages = 0;
  for (; warps >= 2; --warps) {
    const size_t per_warp = kBudget / warps;
    stages = per_warp > list ? static_cast<int>((per_warp - list) / (6 * static_cast<size_t>(p.K))) : 0;
    if (stages >= 2) break;
  }
  if (stages < 2) return cudaErrorInvalidValue;
  if (stages > 4) stages = 4;
  p.stages = stages;
  p.list_cap = kUpdownListCap;
  const size_t smem = static_cast<size_t>(warps) * bwd_warp_bytes(p.K, stages, kUpdownListCap);
  cudaError_t e = cudaFuncSetAttribute(twell_bwd_rows_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  return launch_pdl(twell_bwd_rows_kernel<KV>, sms, 32 * warps, smem, s, p);
}

cudaError_t launch_bwd_rows(const BwdParams& p, int sms, cudaStream_t s) {
  switch ((p.K + 255) / 256) {
#define TW_KV(n) \
  case n:        \
    return launch_bwd_rows_kv<n>(p, sms, s);
    TW_KV(1) TW_KV(2) TW_KV(3) TW_KV(4) TW_KV(5) TW_KV(6) TW_KV(7) TW_KV(8) TW_KV(9) TW_KV(10)
#undef TW_KV
    default:
      return cudaErrorInvalidValue;
  }
}

// Launch shape of the fused kernel.
struct UpdownShape {
  int warps, stages, list_cap;
};

// Twelve warps (K <= 2048) with a list just large enough (>= N/T,
// >= C, >= 96 entries) when each warp still gets enough ring stages (three up
// to K = 1536, two above); else eight warps with the full list when each gets
// two; else four.
UpdownShape updown_shape(int K, int NT, int C, int max_warps) {
  constexpr size_t kBudget = 232448;  // 227 KB of dynamic shared memory per CTA
  const size_t slot = 4 * static_cast<size_t>(K);
  UpdownShape u{0, 0, 0};
  if (max_warps > 8) {
    int cap = NT > C ? NT : C;
    if (cap < 96) cap = 96;
    cap = (cap + 31) / 32 * 32;
    const size_t per_warp = kBudget / max_warps;
    const size_t fixed = static_cast<size_t>(cap) * 8 + 128;
    const int st = per_warp > fixed ? static_cast<int>((per_warp - fixed) / slot) : 0;
    if (st >= (K <= 1536 ? 3 : 2)) return {max_warps, st > 8 ? 8 : st, cap};
  }
  for (int warps = 8; warps >= 4; warps /= 2) {
    const size_t per_warp = kBudget / warps;
    const size_t fixed = static_cast<size_t>(kUpdownListCap) * 8 + 128;
    int st = per_warp > fixed ? static_cast<int>((per_warp - fixed) / slot) : 0;
    if (st > 8) st = 8;
    u = {warps, st, kUpdownListCap};
    if (st >= 2) return u;
  }
  return u;
}

template <int KV>
cudaError_t launch_updown_kv(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw,
                             float* y, int sms, cudaStream_t s) {
  const UpdownShape u = updown_shape(tw->K, tw->N / tw->T, tw->C, updown_max_warps<KV>());
  if (u.stages < 2) return cudaErrorInvalidValue;
  const size_t smem = static_cast<size_t>(u.warps) * updown_warp_bytes(tw->K, u.stages, u.list_cap);
  cudaError_t e = cudaFuncSetAttribute(twell_updown_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  UpdownParams p = {};
  p.x = x; p.wu_t = wu_t; p.wd = wd;
  p.counts = tw->counts; p.idx = tw->idx; p.vals = tw->vals;
  p.M = tw->M; p.K = tw->K; p.N = tw->N; p.T = tw->T; p.C = tw->C;
  p.y = y; p.ctrl = tw->ctrl; p.units = reinterpret_cast<int4*>(tw->units);
  p.stages = u.stages;
  p.list_cap = u.list_cap;
  p.scan_target = tw->M;
  p.wait_limit_ns = kWaitLimitNs;
  if (g_expire_wait_ns > 0) {
    p.scan_target = tw->M + 1;
    p.wait_limit_ns = static_cast<unsigned long long>(g_expire_wait_ns);
    g_expire_wait_ns = 0;
  }
  return launch_pdl(twell_updown_kernel<KV>, sms, 32 * u.warps, smem, s, p);
}

// Small batches: the static-unit kernel with the full entry list (it must
// hold one overflow tile, T entries) and two to four ring stages per warp.
template <int KV>
cudaError_t launch_updown_small_kv(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw,
                                   float* y, int sms, cudaStream_t s) {
  constexpr size_t kBudget = 232448;
  const size_t slot = 4 * static_cast<size_t>(tw->K);
  const size_t fixed = static_cast<size_t>(kUpdownListCap) * 8 + 128;
  int warps = updown_max_warps<KV>(), stages = 0;
  for (; warps >= 4; warps = warps > 8 ? 8 : warps / 2) {
    const size_t per_warp = kBudget / warps;
    stages = per_warp > fixed ? static_cast<int>((per_warp - fixed) / slot) : 0;
    if (stages >= 2) break;
  }
  if (stages < 2) return cudaErrorInvalidValue;
  if (stages > 4) stages = 4;
  const size_t smem = static_cast<size_t>(warps) * updown_warp_bytes(tw->K, stages, kUpdownListCap);
  cudaError_t e = cudaFuncSetAttribute(twell_updown_small_kernel<KV>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       static_cast<int>(smem));
  if (e != cudaSuccess) return e;
  const UpdownParams p = small_updown_params(x, wu_t, wd, tw, y, stages, static_cast<int64_t>(sms) * warps);
  return launch_pdl(twell_updown_small_kernel<KV>, sms, 32 * warps, smem, s, p);
}

cudaError_t launch_updown_small(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw,
                                float* y, int sms, cudaStream_t s) {
  switch ((tw->K + 255) / 256) {
#define TW_KV(n) \
  case n:        \
    return launch_updown_small_kv<n>(x, wu_t, wd, tw, y, sms, s);
    TW_KV(1) TW_KV(2) TW_KV(3) TW_KV(4) TW_KV(5) TW_KV(6) TW_KV(7) TW_KV(8)
    TW_KV(9) TW_KV(10) TW_KV(11) TW_KV(12) TW_KV(13) TW_KV(14) TW_KV(15) TW_KV(16)
#undef TW_KV
    default:
      return cudaErrorInvalidValue;
  }
}

cudaError_t launch_updown(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw, float* y,
                          int sms, cudaStream_t s) {
  switch ((tw->K + 255) / 256) {
#define TW_KV(n) \
  case n:        \
    return launch_updown_kv<n>(x, wu_t, wd, tw, y, sms, s);
    TW_KV(1) TW_KV(2) TW_KV(3) TW_KV(4) TW_KV(5) TW_KV(6) TW_KV(7) TW_KV(8)
    TW_KV(9) TW_KV(10) TW_KV(11) TW_KV(12) TW_KV(13) TW_KV(14) TW_KV(15) TW_KV(16)
#undef TW_KV
    default:
      return cudaErrorInvalidValue;
  }
}

int gemm_grid(int rows, int cols, int bn, int sms, int k_splits = 1) {
  const long tiles = static_cast<long>((rows + kBM - 1) / kBM) * ((cols + bn - 1) / bn) * k_splits;
  return static_cast<int>(tiles < sms ? tiles : sms);
}

// Reduction slices for a GEMM with few output tiles: as many as keep all
// tiles in one wave on the SMs, every slice at least 8 k-blocks long and none
// empty.
int choose_k_splits(int rows, int cols, int bn, int K, int sms) {
  const int tiles = ((rows + kBM - 1) / kBM) * ((cols + bn - 1) / bn);
  const int kb = K / kBK;
  int splits = sms / tiles;
  if (splits > kb / 8) splits = kb / 8;
  if (splits < 1) return 1;
  const int per = (kb + splits - 1) / splits;
  return (kb + per - 1) / per;
}

// Dense FFN ("Sparser, Faster, Lighter Transformer Language Models", §1-1
// computed in full, §2-2 dense pipeline).  GEMM 1 puts x W_g and x W_u of the
// same column tile into two TMEM accumulators and writes h; GEMM 2 computes
// y = h W_d.  With `split`, h is stored as bf16 hi + lo halves (h [M][2N]) and
// GEMM 2 reduces over [h_hi | h_lo] against W_d twice (b_k_wrap), so h keeps
// about 16 significant bits; without it h is one bf16 (h [M][N]).
twell_status dense_ffn_impl(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd, int M,
                            int K, int N, uint16_t* h_scratch, float* y, bool split, cudaStream_t stream) {
  g_launches = 0;
  if (M < 1 || K < 64 || K % 64 != 0 || N < 128 || N % 128 != 0)
    return fail(TWELL_ERR_INVALID, "invalid sizes M=%d K=%d N=%d (need K %% 64 == 0, N %% 128 == 0)", M, K, N);
  if (!aligned16(x) || !aligned16(wg_t) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(h_scratch) || !aligned16(y))
    return fail(TWELL_ERR_INVALID, "all pointers must be non-NULL and 16-byte aligned");
  twell_status st;
  DeviceInfo dev;
  if ((st = device_info(dev)) != TWELL_OK) return st;
  const int hcols = split ? 2 * N : N;
  CUtensorMap tm_x, tm_wg, tm_wu, tm_h, tm_wd;
  if ((st = tmap_bf16(x, K, M, kBM, tm_x)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wg_t, K, N, 128, tm_wg)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wu_t, K, N, 128, tm_wu)) != TWELL_OK) return st;
  if ((st = tmap_bf16(h_scratch, hcols, M, kBM, tm_h)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wd, K, N, 64, tm_wd)) != TWELL_OK) return st;

  EpiGatedProduct::Params p1{h_scratch, N, split ? 1 : 0};
  GemmGeom g1{M, N, K, nullptr, kGateGroupM, 0, 1};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_gated_product(tm_x, tm_wg, tm_wu, g1, p1, nullptr, gemm_grid(M, N, 128, dev.sms), stream));
  TW_CUDA(trace_end(stream, "dense_gate_up_gemm"));
  const int ks2 = choose_k_splits(M, K, 256, hcols, dev.sms);
  if (ks2 > 1) TW_CUDA(cudaMemsetAsync(y, 0, static_cast<size_t>(M) * K * sizeof(float), stream));
  EpiStoreF32::Params p2{y, K, K, ks2 > 1 ? 1 : 0};
  GemmGeom g2{M, K, hcols, nullptr, kGateGroupM, split ? N / kBK : 0, ks2};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_down_store(tm_h, tm_wd, g2, p2, nullptr, gemm_grid(M, K, 256, dev.sms, ks2), stream));
  TW_CUDA(trace_end(stream, "dense_down_gemm"));
  return TWELL_OK;
}

}  // namespace
}  // namespace twell

using namespace twell;

extern "C" {

const char* twell_status_str(twell_status st) {
  switch (st) {
    case TWELL_OK: return "ok";
    case TWELL_ERR_INVALID: return "invalid argument";
    case TWELL_ERR_CAPACITY: return "dense-row capacity exceeded";
    case TWELL_ERR_CUDA: return "CUDA error";
    case TWELL_ERR_DEVICE_CHECK: return "device status flag raised";
    case TWELL_ERR_UNSUPPORTED: return "unsupported device or shape";
  }
  return "unknown status";
}

const char* twell_last_error(void) { return g_err; }

int twell_last_launch_count(void) { return g_launches; }

twell_status twell_test_expire_wait(long long limit_ns) {
  if (limit_ns != 0 && (limit_ns < 1000 || limit_ns > 1000000000))
    return fail(TWELL_ERR_INVALID, "limit_ns must be 0 or in [1000, 1000000000], got %lld", limit_ns);
  g_expire_wait_ns = limit_ns;
  return TWELL_OK;
}

twell_status twell_bwd_slot_route(int route) {
  if (route < 0 || route > 2) return fail(TWELL_ERR_INVALID, "route must be 0, 1 or 2, got %d", route);
  g_bwd_slot_route = route;
  return TWELL_OK;
}

twell_status twell_trace_events(cudaEvent_t* events, int capacity) {
  if (events && capacity < 1) return fail(TWELL_ERR_INVALID, "capacity must be >= 1");
  g_trace.events = events;
  g_trace.capacity = events ? capacity : 0;
  g_trace.count = 0;
  return TWELL_OK;
}

int twell_trace_count(void) { return g_trace.count; }

const char* twell_trace_name(int i) {
  return (i >= 0 && i < g_trace.count && i < 256) ? g_trace.names[i] : nullptr;
}

size_t twell_buf_bytes(int M, int K, int N, int T, int C, int R_cap) {
  if (!shape_ok(M, K, N, T, C, R_cap)) return 0;
  return layout(M, K, N, T, C, R_cap).total;
}

twell_status twell_buf_init(twell_buf* tw, void* base, size_t bytes, int M, int K, int N, int T, int C, int R_cap) {
  g_launches = 0;
  if (!tw) return fail(TWELL_ERR_INVALID, "twell_buf is NULL");
  if (!shape_ok(M, K, N, T, C, R_cap))
    return fail(TWELL_ERR_INVALID, "invalid sizes M=%d K=%d N=%d T=%d C=%d R_cap=%d", M, K, N, T, C, R_cap);
  if (!base || (reinterpret_cast<uintptr_t>(base) & 255u)) return fail(TWELL_ERR_INVALID, "base must be 256-byte aligned");
  const Layout L = layout(M, K, N, T, C, R_cap);
  if (bytes < L.total) return fail(TWELL_ERR_INVALID, "buffer too small: %zu < %zu bytes", bytes, L.total);
  uint8_t* b = static_cast<uint8_t*>(base);
  tw->ctrl = reinterpret_cast<int32_t*>(b + L.ctrl);
  tw->counts = reinterpret_cast<uint16_t*>(b + L.counts);
  tw->idx = b + L.idx;
  tw->vals = reinterpret_cast<float*>(b + L.vals);
  tw->row_slot = reinterpret_cast<int32_t*>(b + L.row_slot);
  tw->slot_row = reinterpret_cast<int32_t*>(b + L.slot_row);
  tw->dense_rows = reinterpret_cast<float*>(b + L.dense_rows);
  tw->x_over = reinterpret_cast<uint16_t*>(b + L.x_over);
  tw->h_over = reinterpret_cast<uint16_t*>(b + L.h_over);
  tw->units = b + L.units;
  tw->z = M <= TWELL_SMALL_M ? reinterpret_cast<float*>(b + L.z) : nullptr;
  tw->M = M; tw->K = K; tw->N = N; tw->T = T; tw->C = C; tw->R_cap = R_cap;
  return TWELL_OK;
}

twell_status twell_gate_pack(const uint16_t* x, const uint16_t* wg_t, int M, int K, int N, twell_buf* tw,
                             int* n_over_host, cudaStream_t stream) {
  g_launches = 0;
  twell_status st = check_buf(tw);
  if (st != TWELL_OK) return st;
  if (M != tw->M || K != tw->K || N != tw->N)
    return fail(TWELL_ERR_INVALID, "shape (%d,%d,%d) does not match the buffer (%d,%d,%d)", M, K, N, tw->M, tw->K, tw->N);
  if (!aligned16(x) || !aligned16(wg_t)) return fail(TWELL_ERR_INVALID, "x and wg_t must be non-NULL and 16-byte aligned");
  DeviceInfo dev;
  if ((st = device_info(dev)) != TWELL_OK) return st;

  const bool small = tw->z != nullptr;
  // 256-wide CTA tiles halve the operand traffic per FLOP of the one-CTA engine.
  const int bn = (N % 256 == 0 && (M > 256 || tw->T == 256)) ? 256 : 128;
  CUtensorMap tm_x, tm_wg;
  if (!small) {
    if ((st = tmap_bf16(x, K, M, kBM, tm_x)) != TWELL_OK) return st;
    if ((st = tmap_bf16(wg_t, K, N, bn, tm_wg)) != TWELL_OK) return st;
  }
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_reset(tw, stream));
  TW_CUDA(trace_end(stream, "twell_reset"));

  const GateTwellParams p = gate_twell_params(x, tw);
  if (small) {
    CUtensorMap tm_w128, tm_xs;
    GateStreamParams gp;
    int grid = 0;
    if ((st = small_gate_plan(x, wg_t, tw, dev.sms, 232448, tm_w128, tm_xs, gp, grid)) != TWELL_OK) return st;
    TW_CUDA(trace_begin(stream));
    TW_CUDA(launch_gate_stream(tm_w128, tm_xs, gp, tw->ctrl, grid, stream));
    TW_CUDA(trace_end(stream, "gate_stream_pack"));
  } else if (M > 256 && N % 256 == 0 && dev.sms >= 2) {
    // CTA pairs on 256 x 256 tiles: each CTA moves 2/3 of the operand bytes per FLOP.
    CUtensorMap tm_wg128;
    if ((st = tmap_bf16(wg_t, K, N, 128, tm_wg128)) != TWELL_OK) return st;
    const long tiles = static_cast<long>((M + 255) / 256) * (N / 256);
    const int pairs = static_cast<int>(tiles < dev.sms / 2 ? tiles : dev.sms / 2);
    GemmGeom g{M, N, K, nullptr, kGateGroupM / 2, 0, 1};
    TW_CUDA(trace_begin(stream));
    TW_CUDA(launch_gate_twell_pair(tw->T, tm_x, tm_wg128, g, p, tw->ctrl, 2 * pairs, stream));
    TW_CUDA(trace_end(stream, "gate_twell_gemm"));
  } else {
    GemmGeom g{M, N, K, nullptr, kGateGroupM, 0, 1};
    TW_CUDA(trace_begin(stream));
    TW_CUDA(launch_gate_twell(tw->T, bn, tm_x, tm_wg, g, p, tw->ctrl, gemm_grid(M, N, bn, dev.sms), stream));
    TW_CUDA(trace_end(stream, "gate_twell_gemm"));
  }

  if (n_over_host) {
    int n_over = 0;
    int flags = 0;
    if ((st = twell_read_status(tw, &n_over, &flags, stream)) == TWELL_ERR_DEVICE_CHECK) return st;
    *n_over_host = n_over;
    if (n_over > tw->R_cap)
      return fail(TWELL_ERR_CAPACITY, "%d rows overflowed, dense-row capacity is %d", n_over, tw->R_cap);
  }
  return TWELL_OK;
}

twell_status twell_read_status(const twell_buf* tw, int* n_over_host, int* device_flags, cudaStream_t stream) {
  twell_status st = check_buf(tw);
  if (st != TWELL_OK) return st;
  int words[2] = {0, 0};
  TW_CUDA(cudaMemcpyAsync(words, tw->ctrl, sizeof words, cudaMemcpyDeviceToHost, stream));
  TW_CUDA(cudaStreamSynchronize(stream));
  if (n_over_host) *n_over_host = words[kCtrlNOver];
  if (device_flags) *device_flags = words[kCtrlFlags];
  if (words[kCtrlFlags] & ~kFlagNoCapacity)
    return fail(TWELL_ERR_DEVICE_CHECK, "device status flags 0x%x", words[kCtrlFlags]);
  if (words[kCtrlNOver] > tw->R_cap)
    return fail(TWELL_ERR_CAPACITY, "%d rows overflowed, dense-row capacity is %d", words[kCtrlNOver], tw->R_cap);
  return TWELL_OK;
}

twell_status twell_ffn_fwd(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw, int K,
                           float* y, cudaStream_t stream) {
  g_launches = 0;
  twell_status st = check_buf(tw);
  if (st != TWELL_OK) return st;
  if (K != tw->K) return fail(TWELL_ERR_INVALID, "K=%d does not match the buffer's K=%d", K, tw->K);
  if (!aligned16(x) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y))
    return fail(TWELL_ERR_INVALID, "x, wu_t, wd and y must be non-NULL and 16-byte aligned");
  DeviceInfo dev;
  if ((st = device_info(dev)) != TWELL_OK) return st;
  const int N = tw->N;

  if (tw->M <= kStaticUpdownMaxM) {
    // Small batch: y cleared, then one kernel for TwELL and overflow tiles alike.
    TW_CUDA(trace_begin(stream));
    TW_CUDA(cudaMemsetAsync(y, 0, static_cast<size_t>(tw->M) * K * sizeof(float), stream));
    TW_CUDA(launch_updown_small(x, wu_t, wd, tw, y, dev.sms, stream));
    TW_CUDA(trace_end(stream, "twell_updown_small"));
    return TWELL_OK;
  }

  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_updown(x, wu_t, wd, tw, y, dev.sms, stream));
  TW_CUDA(trace_end(stream, "twell_updown"));

  // Dense-row path for overflow tiles; rows beyond the device-side n_over are skipped.
  CUtensorMap tm_xo, tm_wu, tm_ho, tm_wd;
  if ((st = tmap_bf16(tw->x_over, K, tw->R_cap, kBM, tm_xo)) != TWELL_OK) return st;
  // Narrow tiles when the slotted rows are too few to occupy the SMs with 128-wide ones.
  const int bn1 = static_cast<long>((tw->R_cap + kBM - 1) / kBM) * (N / 128) * 2 <= dev.sms ? 64 : 128;
  if ((st = tmap_bf16(wu_t, K, N, bn1, tm_wu)) != TWELL_OK) return st;
  if ((st = tmap_bf16(tw->h_over, 2 * N, tw->R_cap, kBM, tm_ho)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wd, K, N, 64, tm_wd)) != TWELL_OK) return st;

  EpiOverflowProduct::Params p1;
  p1.counts = tw->counts; p1.dense_rows = tw->dense_rows; p1.slot_row = tw->slot_row; p1.h_over = tw->h_over;
  p1.N = N; p1.T = tw->T; p1.C = tw->C;
  GemmGeom g1{tw->R_cap, N, K, tw->ctrl + kCtrlNOver, kGateGroupM, 0, 1};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_overflow_product(bn1, tm_xo, tm_wu, g1, p1, tw->ctrl, gemm_grid(tw->R_cap, N, bn1, dev.sms), stream));
  TW_CUDA(trace_end(stream, "overflow_up_gemm"));

  EpiAccumulateRows::Params p2;
  p2.y = y; p2.slot_row = tw->slot_row; p2.ldy = K; p2.ncols = K;
  // The live rows (n_over) are known only on the device: the kernel picks the
  // number of reduction slices (each at least 8 k-blocks) from them.
  const int ks2_max = (2 * N / kBK) / 8 > 1 ? (2 * N / kBK) / 8 : 1;
  GemmGeom g2{tw->R_cap, K, 2 * N, tw->ctrl + kCtrlNOver, kGateGroupM, N / kBK, -ks2_max};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_overflow_down(tm_ho, tm_wd, g2, p2, tw->ctrl, gemm_grid(tw->R_cap, K, 256, dev.sms, ks2_max),
                               stream));
  TW_CUDA(trace_end(stream, "overflow_down_gemm"));
  return TWELL_OK;
}

twell_status twell_ffn_fused(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd, int M,
                             int K, int N, twell_buf* tw, float* y, int* n_over_host, cudaStream_t stream) {
  g_launches = 0;
  twell_status st = check_buf(tw);
  if (st != TWELL_OK) return st;
  if (M != tw->M || K != tw->K || N != tw->N)
    return fail(TWELL_ERR_INVALID, "shape (%d,%d,%d) does not match the buffer (%d,%d,%d)", M, K, N, tw->M, tw->K, tw->N);
  if (!aligned16(x) || !aligned16(wg_t) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(y))
    return fail(TWELL_ERR_INVALID, "x, wg_t, wu_t, wd and y must be non-NULL and 16-byte aligned");
  DeviceInfo dev;
  if ((st = device_info(dev)) != TWELL_OK) return st;

  if (!tw->z) {
    // Larger batches: the gate GEMM with its packing epilogue, then the fused up/down kernel.
    if ((st = twell_gate_pack(x, wg_t, M, K, N, tw, n_over_host, stream)) != TWELL_OK) return st;
    const int gate_launches = g_launches;
    if ((st = twell_ffn_fwd(x, wu_t, wd, tw, K, y, stream)) != TWELL_OK) return st;
    g_launches += gate_launches;
    return TWELL_OK;
  }

  // Small batches: one persistent kernel after the reset.
  constexpr size_t kBudget = 232448;
  CUtensorMap tm_w, tm_x;
  GateStreamParams gp;
  int grid = 0;
  if ((st = small_gate_plan(x, wg_t, tw, dev.sms, kBudget, tm_w, tm_x, gp, grid)) != TWELL_OK) return st;
  constexpr int kWarps = 6;
  const size_t fixed = 1024 + kStreamCtrlBytes;
  const size_t list_bytes = static_cast<size_t>(kUpdownListCap) * 8 + 128;
  int stages = static_cast<int>(((kBudget - fixed) / kWarps - list_bytes) / (4 * static_cast<size_t>(K)));
  if (stages > 4) stages = 4;
  if (stages < 2 || gp.stages < 2) return fail(TWELL_ERR_INVALID, "K=%d leaves too little shared memory", K);
  // Every SM takes part in the up/down phase; the first gp.grid CTAs also in the gate pass.
  grid = dev.sms;
  UpdownParams up = small_updown_params(x, wu_t, wd, tw, y, stages, static_cast<int64_t>(grid) * kWarps);
  up.scan_target = grid;
  if (g_expire_wait_ns > 0) {
    up.scan_target = grid + 1;
    up.wait_limit_ns = static_cast<unsigned long long>(g_expire_wait_ns);
    g_expire_wait_ns = 0;
  }
  const size_t ring = fixed + kWarps * updown_warp_bytes(K, stages, kUpdownListCap);
  const size_t gate = stream_smem_bytes(gp.mp, gp.stages);
  const size_t smem = ring > gate ? ring : gate;
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_reset(tw, stream));
  TW_CUDA(trace_end(stream, "twell_reset"));
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_fused_small(tm_w, tm_x, gp, up, tw->ctrl, grid, smem, stream));
  TW_CUDA(trace_end(stream, "twell_fused_small"));

  if (n_over_host) {
    int n_over = 0;
    if ((st = twell_read_status(tw, &n_over, nullptr, stream)) == TWELL_ERR_DEVICE_CHECK) return st;
    *n_over_host = n_over;
    if (n_over > tw->R_cap)
      return fail(TWELL_ERR_CAPACITY, "%d rows overflowed, dense-row capacity is %d", n_over, tw->R_cap);
  }
  return TWELL_OK;
}

size_t twell_bwd_scratch_bytes(int M, int K, int N, int T, int C, int R_cap) {
  if (!shape_ok(M, K, N, T, C, R_cap)) return 0;
  return bwd_layout(M, K, N, T, C, R_cap).total;
}

twell_status twell_ffn_bwd(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                           const twell_buf* tw, const float* dy, int K, float* dx, float* dwg_t, float* dwu_t,
                           float* dwd, void* scratch, size_t scratch_bytes, cudaStream_t stream) {
  g_launches = 0;
  twell_status st = check_buf(tw);
  if (st != TWELL_OK) return st;
  if (K != tw->K) return fail(TWELL_ERR_INVALID, "K=%d does not match the buffer's K=%d", K, tw->K);
  if (K > kBwdMaxK) return fail(TWELL_ERR_INVALID, "twell_ffn_bwd supports K <= %d (got %d)", kBwdMaxK, K);
  if (!aligned16(x) || !aligned16(wg_t) || !aligned16(wu_t) || !aligned16(wd) || !aligned16(dy) || !aligned16(dx) ||
      !aligned16(dwg_t) || !aligned16(dwu_t) || !aligned16(dwd))
    return fail(TWELL_ERR_INVALID, "every array must be non-NULL and 16-byte aligned");
  const int M = tw->M, N = tw->N;
  const BwdLayout L = bwd_layout(M, K, N, tw->T, tw->C, tw->R_cap);
  if (!scratch || (reinterpret_cast<uintptr_t>(scratch) & 255u))
    return fail(TWELL_ERR_INVALID, "scratch must be non-NULL and 256-byte aligned");
  if (scratch_bytes < L.total) return fail(TWELL_ERR_INVALID, "scratch too small: %zu < %zu bytes", scratch_bytes, L.total);
  DeviceInfo dev;
  if ((st = device_info(dev)) != TWELL_OK) return st;

  uint8_t* sb = static_cast<uint8_t*>(scratch);
  BwdParams p = {};
  p.x = x; p.wg_t = wg_t; p.wu_t = wu_t; p.wd = wd; p.dy = dy;
  p.counts = tw->counts; p.idx = tw->idx; p.vals = tw->vals; p.row_slot = tw->row_slot; p.dense_rows = tw->dense_rows;
  p.M = M; p.K = K; p.N = N; p.T = tw->T; p.C = tw->C;
  p.dx = dx; p.dwg_t = dwg_t; p.dwu_t = dwu_t; p.dwd = dwd;
  p.cnt = reinterpret_cast<int*>(sb + L.cnt);
  p.fill = reinterpret_cast<int*>(sb + L.fill);
  p.row_entries = reinterpret_cast<int*>(sb + L.row_entries);
  p.over_total = reinterpret_cast<int*>(sb + L.over_total);
  p.off = reinterpret_cast<int*>(sb + L.off);
  p.row_units = reinterpret_cast<int*>(sb + L.row_units);
  p.piece_off = reinterpret_cast<int*>(sb + L.piece_off);
  p.piece_unit = reinterpret_cast<int*>(sb + L.piece_unit);
  p.entries = reinterpret_cast<BwdEntry*>(sb + L.entries);
  p.slot_row = tw->slot_row;
  p.r_cap = tw->R_cap;
  p.ctrl = tw->ctrl;

  TW_CUDA(cudaMemsetAsync(sb, 0, L.off, stream));  // unit counts, fill, row entries, overflow total
  TW_CUDA(cudaMemsetAsync(dx, 0, static_cast<size_t>(M) * K * sizeof(float), stream));
  const int64_t records = static_cast<int64_t>(M) * (N / tw->T);
  const int64_t cgrid = (records + 255) / 256;
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_pdl(twell_bwd_count_kernel, static_cast<int>(cgrid < 4 * dev.sms ? cgrid : 4 * dev.sms), 256, 0,
                     stream, p));
  TW_CUDA(trace_end(stream, "bwd_count"));
  // The number of slotted rows and of their overflow entries choose the
  // slotted rows' route: read both once.
  int n_over = 0, n_over_entries = 0;
  TW_CUDA(cudaMemcpyAsync(&n_over, tw->ctrl + kCtrlNOver, sizeof n_over, cudaMemcpyDeviceToHost, stream));
  TW_CUDA(cudaMemcpyAsync(&n_over_entries, p.over_total, sizeof n_over_entries, cudaMemcpyDeviceToHost, stream));
  TW_CUDA(cudaStreamSynchronize(stream));
  const int R = n_over < tw->R_cap ? n_over : tw->R_cap;
  const bool dense_slots = bwd_dense_slots(R, n_over_entries, N, K);
  p.gather_overflow = dense_slots ? 0 : 1;
  if (!dense_slots && n_over_entries > 0) {
    TW_CUDA(trace_begin(stream));
    TW_CUDA(launch_pdl(twell_bwd_overflow_units_kernel, static_cast<int>(cgrid < 4 * dev.sms ? cgrid : 4 * dev.sms),
                       256, 0, stream, p));
    TW_CUDA(trace_end(stream, "bwd_overflow_units"));
  }

  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_pdl(twell_bwd_scan_kernel, 1, 1024, 0, stream, static_cast<const int*>(p.cnt), p.off, N, 0,
                     p.piece_off, p.piece_unit));
  TW_CUDA(launch_pdl(twell_bwd_scan_kernel, 1, 1024, 0, stream, static_cast<const int*>(p.row_entries), p.row_units,
                     M, 1, static_cast<int*>(nullptr), static_cast<int*>(nullptr)));
  TW_CUDA(trace_end(stream, "bwd_scan"));
  ++g_launches;  // the bracket holds two scans
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_bwd_rows(p, dev.sms, stream));
  TW_CUDA(trace_end(stream, "bwd_rows"));
  // Items: (piece, 256-column chunk); at least one piece per hidden unit, and
  // about entries / 64 more.  The grid covers the SMs; warps stride.
  const int64_t items = static_cast<int64_t>(N) * ((K + 255) / 256);
  const int64_t ugrid = (items + 7) / 8;
  // A plain launch: launched early (programmatic serialisation) the unit
  // pass's CTAs are placed while the row pass runs, and the whole backward was
  // slower (M=16384 K=2560 N=10240: 2.93 ms against 2.66 ms; M=8192 K=2048
  // N=5632: 1.20 against 1.19 ms).  griddepcontrol.wait in the kernel is then
  // a no-op.
  TW_CUDA(trace_begin(stream));
  twell_bwd_units_kernel<<<static_cast<int>(ugrid < 8 * dev.sms ? ugrid : 8 * dev.sms), 256, 0, stream>>>(p);
  TW_CUDA(cudaGetLastError());
  TW_CUDA(trace_end(stream, "bwd_units"));
  if (!dense_slots) return TWELL_OK;

  // ---- dense-row slots on the tensor cores (after the unit pass: the weight
  // gradients are added into the rows it wrote).
  const int r_pad = (R + 63) / 64 * 64;
  uint16_t* dy_cat = reinterpret_cast<uint16_t*>(sb + L.dy_cat);
  uint16_t* dy_hi = reinterpret_cast<uint16_t*>(sb + L.dy_hi);
  uint16_t* dy_lo = reinterpret_cast<uint16_t*>(sb + L.dy_lo);
  uint16_t* x_pad = reinterpret_cast<uint16_t*>(sb + L.x_pad);
  float* u = reinterpret_cast<float*>(sb + L.u);
  uint16_t* du_rows = reinterpret_cast<uint16_t*>(sb + L.du_rows);
  uint16_t* dz_rows = reinterpret_cast<uint16_t*>(sb + L.dz_rows);
  uint16_t* h_t = reinterpret_cast<uint16_t*>(sb + L.h_t);
  uint16_t* du_t = reinterpret_cast<uint16_t*>(sb + L.du_t);
  uint16_t* dz_t = reinterpret_cast<uint16_t*>(sb + L.dz_t);
  const size_t t_bytes = static_cast<size_t>(N) * 2 * r_pad * 2;
  TW_CUDA(cudaMemsetAsync(h_t, 0, t_bytes, stream));
  TW_CUDA(cudaMemsetAsync(du_t, 0, t_bytes, stream));
  TW_CUDA(cudaMemsetAsync(dz_t, 0, t_bytes, stream));
  const int64_t oitems = static_cast<int64_t>(r_pad) * (K / 8);
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_pdl(twell_bwd_slot_operands_kernel, static_cast<int>((oitems + 255) / 256), 256, 0, stream, dy,
                     tw->x_over, tw->slot_row, R, r_pad, K, dy_cat, dy_hi, dy_lo, x_pad));
  TW_CUDA(trace_end(stream, "bwd_slot_operands"));

  CUtensorMap tm_xpad, tm_wu_k, tm_dycat, tm_wd_k, tm_du_rows, tm_dz_rows, tm_wu_mn, tm_wg_mn, tm_du_t, tm_dz_t,
      tm_h_t, tm_xpad_mn, tm_dyhi_mn, tm_dylo_mn;
  if ((st = tmap_bf16(x_pad, K, r_pad, kBM, tm_xpad)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wu_t, K, N, 128, tm_wu_k)) != TWELL_OK) return st;
  if ((st = tmap_bf16(dy_cat, 2 * K, r_pad, kBM, tm_dycat)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wd, K, N, 128, tm_wd_k)) != TWELL_OK) return st;
  if ((st = tmap_bf16(du_rows, 2 * N, r_pad, kBM, tm_du_rows)) != TWELL_OK) return st;
  if ((st = tmap_bf16(dz_rows, 2 * N, r_pad, kBM, tm_dz_rows)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wu_t, K, N, 64, tm_wu_mn)) != TWELL_OK) return st;
  if ((st = tmap_bf16(wg_t, K, N, 64, tm_wg_mn)) != TWELL_OK) return st;
  if ((st = tmap_bf16(du_t, 2 * r_pad, N, kBM, tm_du_t)) != TWELL_OK) return st;
  if ((st = tmap_bf16(dz_t, 2 * r_pad, N, kBM, tm_dz_t)) != TWELL_OK) return st;
  if ((st = tmap_bf16(h_t, 2 * r_pad, N, kBM, tm_h_t)) != TWELL_OK) return st;
  if ((st = tmap_bf16(x_pad, K, r_pad, 64, tm_xpad_mn)) != TWELL_OK) return st;
  if ((st = tmap_bf16(dy_hi, K, r_pad, 64, tm_dyhi_mn)) != TWELL_OK) return st;
  if ((st = tmap_bf16(dy_lo, K, r_pad, 64, tm_dylo_mn)) != TWELL_OK) return st;

  // u = x_slot W_u^T  [R][N] fp32
  EpiStoreF32::Params pu{u, N, N, 0};
  GemmGeom gu{R, N, K, nullptr, kGateGroupM, 0, 1};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_store_f32_kmajor(tm_xpad, tm_wu_k, gu, pu, tw->ctrl, gemm_grid(R, N, 128, dev.sms), stream));
  TW_CUDA(trace_end(stream, "bwd_slot_u"));
  // dh = [dy_hi | dy_lo] W_d^T, epilogue: du, dz, h on the overflow tiles
  EpiBwdSlots::Params ps;
  ps.u = u; ps.dense_rows = tw->dense_rows; ps.counts = tw->counts; ps.slot_row = tw->slot_row;
  ps.du_rows = du_rows; ps.dz_rows = dz_rows; ps.h_t = h_t; ps.du_t = du_t; ps.dz_t = dz_t;
  ps.N = N; ps.T = tw->T; ps.C = tw->C; ps.r_pad = r_pad;
  GemmGeom gh{R, N, 2 * K, nullptr, kGateGroupM, K / kBK, 1};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_bwd_slots(tm_dycat, tm_wd_k, gh, ps, tw->ctrl, gemm_grid(R, N, 128, dev.sms), stream));
  TW_CUDA(trace_end(stream, "bwd_slot_dh"));
  // dx[slot rows] += [du_hi | du_lo] W_u^T... as rows of W_u^T: sum_n du_n wu_t[n]; likewise dz with W_g^T
  const int ksx = choose_k_splits(R, K, 256, 2 * N, dev.sms);
  EpiAccumulateRows::Params px{dx, tw->slot_row, K, K};
  GemmGeom gx{R, K, 2 * N, nullptr, kGateGroupM, N / kBK, ksx};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_overflow_down(tm_du_rows, tm_wu_mn, gx, px, tw->ctrl, gemm_grid(R, K, 256, dev.sms, ksx), stream));
  TW_CUDA(launch_overflow_down(tm_dz_rows, tm_wg_mn, gx, px, tw->ctrl, gemm_grid(R, K, 256, dev.sms, ksx), stream));
  TW_CUDA(trace_end(stream, "bwd_slot_dx"));
  // dW += (per-slot factor)^T (slot rows): reductions over the R_pad slots
  const int ksw = choose_k_splits(N, K, 256, 2 * r_pad, dev.sms);
  GemmGeom gw{N, K, 2 * r_pad, nullptr, kGateGroupM, r_pad / kBK, ksw};
  const int wgrid = gemm_grid(N, K, 256, dev.sms, ksw);
  EpiStoreF32::Params pwu{dwu_t, K, K, 1}, pwg{dwg_t, K, K, 1}, pwd{dwd, K, K, 1};
  TW_CUDA(trace_begin(stream));
  TW_CUDA(launch_down_store(tm_du_t, tm_xpad_mn, gw, pwu, tw->ctrl, wgrid, stream));
  TW_CUDA(launch_down_store(tm_dz_t, tm_xpad_mn, gw, pwg, tw->ctrl, wgrid, stream));
  TW_CUDA(launch_down_store(tm_h_t, tm_dyhi_mn, gw, pwd, tw->ctrl, wgrid, stream));
  TW_CUDA(launch_down_store(tm_h_t, tm_dylo_mn, gw, pwd, tw->ctrl, wgrid, stream));
  TW_CUDA(trace_end(stream, "bwd_slot_dw"));
  g_launches += 4;  // the brackets above hold two dx and four weight-gradient launches
  return TWELL_OK;
}

twell_status dense_ffn_fwd(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd, int M,
                           int K, int N, uint16_t* h_scratch, float* y, cudaStream_t stream) {
  return dense_ffn_impl(x, wg_t, wu_t, wd, M, K, N, h_scratch, y, true, stream);
}

twell_status dense_ffn_fwd_bf16h(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                                 int M, int K, int N, uint16_t* h_scratch, float* y, cudaStream_t stream) {
  return dense_ffn_impl(x, wg_t, wu_t, wd, M, K, N, h_scratch, y, false, stream);
}

}  // extern "C"

// ---------------------------------------------------------------------------
// Dense FFN for callers that cannot allocate device memory at call time: a
// runtime that has handed all device memory to its own pool, or an embedding
// that forbids allocation while it executes.  The hidden activations h (bf16
// hi + lo halves, [M][2N]), which dense_ffn_fwd takes as a caller buffer, live
// here in a fixed array that is part of the library's device image; every
// device that loads the library keeps it (32 MiB) until the process exits.
namespace twell {
namespace {

constexpr size_t kNoAllocHiddenElems = size_t(16) << 20;  // 16 Mi bf16 values = 32 MiB
__device__ __align__(256) uint16_t g_noalloc_hidden[kNoAllocHiddenElems];

// Id of the calling thread's current CUDA context (false if none is current
// or the driver lacks the query).  Ids are never reused within a process, so
// a context re-created after cudaDeviceReset gets a new one.
bool current_context_id(unsigned long long* id) {
  static PFN_cuCtxGetCurrent_v4000 get_current = nullptr;
  static PFN_cuCtxGetId_v12000 get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<PFN_cuCtxGetCurrent_v4000>(p);
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<PFN_cuCtxGetId_v12000>(p);
  });
  CUcontext ctx = nullptr;
  if (!get_current || !get_id || get_current(&ctx) != CUDA_SUCCESS || !ctx) return false;
  return get_id(ctx, id) == CUDA_SUCCESS;
}

// Device address of the fixed array in the current context.  In host code the
// array's name is only a host-side handle, so the address is looked up with
// cudaGetSymbolAddress (with the device current) and cached per context: a
// context torn down by cudaDeviceReset and created again gets a new id, so the
// address is looked up again rather than reused.
twell_status noalloc_hidden_ptr(uint16_t** out) {
  static std::mutex mu;
  static std::map<unsigned long long, uint16_t*> addr;
  unsigned long long ctx = 0;
  bool have_ctx = current_context_id(&ctx);
  std::lock_guard<std::mutex> lock(mu);
  if (have_ctx) {
    auto it = addr.find(ctx);
    if (it != addr.end()) {
      *out = it->second;
      return TWELL_OK;
    }
  }
  void* p = nullptr;
  TW_CUDA(cudaGetSymbolAddress(&p, g_noalloc_hidden));  // also makes the primary context current
  if (!have_ctx) have_ctx = current_context_id(&ctx);
  if (have_ctx) addr[ctx] = static_cast<uint16_t*>(p);
  *out = static_cast<uint16_t*>(p);
  return TWELL_OK;
}

}  // namespace
}  // namespace twell

extern "C" twell_status dense_ffn_fwd_noalloc(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t,
                                              const uint16_t* wd, int M, int K, int N, float* y,
                                              cudaStream_t stream) {
  g_launches = 0;
  if (M < 1 || N < 1 || 2 * static_cast<size_t>(M) * static_cast<size_t>(N) > kNoAllocHiddenElems)
    return fail(TWELL_ERR_INVALID,
                "dense_ffn_fwd_noalloc: h needs M*2N = %lld bf16 values, more than the built-in scratch of %zu "
                "(32 MiB)",
                2 * static_cast<long long>(M) * N, kNoAllocHiddenElems);
  uint16_t* h = nullptr;
  twell_status st = noalloc_hidden_ptr(&h);
  if (st != TWELL_OK) return st;
  return dense_ffn_fwd(x, wg_t, wu_t, wd, M, K, N, h, y, stream);
}
