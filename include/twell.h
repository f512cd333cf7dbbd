/*
 * twell.h - C ABI of the B200 (sm_100a) ReLU-gated sparse FFN forward path.
 *
 * The operation ("Sparser, Faster, Lighter Transformer Language Models",
 * review page dimensionstp.github.io, §1-1 problem definition):
 *
 *     h_u = x W_u,   h_g = ReLU(x W_g),   h = h_u (.) h_g,   y = h W_d
 *
 * with x [M x K] tokens, W_g and W_u mapping K -> N, W_d mapping N -> K.
 * The sparse path computes it in two steps (§2-2, §3-4, §3-5):
 *   twell_gate_pack : gate GEMM on tensor cores whose epilogue applies ReLU and
 *                     packs every row's non-zeros tile-locally into TwELL
 *                     (Tile-wise ELLPACK), never writing the dense gate;
 *   twell_ffn_fwd   : fused up + down projection that visits only the active
 *                     hidden units: y_m = sum_{n in A_m} g_{m,n} (x_m W_u[:,n]) W_d[n,:].
 * twell_ffn_fused runs both steps in one call; for small batches in one
 * persistent kernel (the one-pass inference kernel of the summary page
 * alanhou.org, "Inference Kernels").
 * Tiles whose active count exceeds the capacity C are routed to a dense-row
 * backup (§3-6 hybrid format; §4-3 static capacity of at most M/8 rows,
 * overflow reported to the host, which retries with larger storage).
 * dense_ffn_fwd computes the same y with dense tensor-core GEMMs.
 *
 * Conventions for every entry point:
 *   - bf16 tensors are passed as uint16_t bit patterns; all matrices are
 *     row-major and contiguous; every pointer must be 16-byte aligned.
 *   - All device pointers are owned by the caller.  The library allocates no
 *     device memory and keeps no state except cached TMA descriptors (keyed by
 *     pointer and shape) and per-device kernel attributes.
 *   - Work is enqueued on `stream` and is asynchronous unless stated.
 *   - Invalid arguments return TWELL_ERR_INVALID before anything is launched.
 *   - A failing CUDA call returns TWELL_ERR_CUDA (message: twell_last_error()).
 *
 * Weight layouts (N rows of K, so each hidden unit n is one contiguous row):
 *   wg_t[n][k] = W_g[k][n],  wu_t[n][k] = W_u[k][n],  wd[n][k] = W_d[n][k].
 * The gate bias, if any, rides in the GEMM (x[:,K-1] = 1, wg_t[:,K-1] = -b).
 */
#ifndef TWELL_H_
#define TWELL_H_

#include <stddef.h>
#include <stdint.h>

#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TWELL_OK = 0,
  TWELL_ERR_INVALID = 1,      /* bad shape, pointer, alignment or buffer; nothing launched */
  TWELL_ERR_CAPACITY = 2,     /* more rows overflowed than the dense-row buffer holds */
  TWELL_ERR_CUDA = 3,         /* a CUDA runtime/driver call failed */
  TWELL_ERR_DEVICE_CHECK = 4, /* a kernel raised a device status flag (bounded wait expired) */
  TWELL_ERR_UNSUPPORTED = 5   /* no sm_100 device, or a shape outside the kernels' limits */
} twell_status;

/*
 * TwELL activations plus the hybrid dense-row backup, all in one caller-owned
 * device block carved by twell_buf_init.  Sizes: NT = N / T.
 *
 *   counts     uint16 [M][NT]     true number of active units (z > 0) of row m
 *                                 in column tile t; a count > C marks the tile
 *                                 as overflow (its slots are then not used)
 *   idx        uint8  [M][NT][C]  local index n - t*T of the first min(count, C)
 *                                 active units, ascending; later slots undefined
 *   vals       fp32   [M][NT][C]  ReLU(z) of those units (the fp32 GEMM result)
 *   dense_rows fp32   [R_cap][N]  ReLU(z) of the overflow tiles of the row that
 *                                 owns the slot; other tiles of the slot undefined
 *   row_slot   int32  [M]         dense-row slot of row m; -1 = none;
 *                                 -2 = needed but R_cap was exhausted
 *   slot_row   int32  [R_cap]     row that owns each slot (valid for slots < n_over)
 *   ctrl       int32  [64]        device control words: [0] n_over (rows that
 *                                 asked for a slot), [1] status flags, [2..6]
 *                                 work-queue counters of the fused kernel, [7]
 *                                 entries of the non-overflow tiles, [8] grid
 *                                 barrier of twell_ffn_fused's small-batch kernel
 *   x_over     bf16   [R_cap][K]  scratch: gathered x rows of slotted rows
 *   h_over     bf16   [R_cap][2N] scratch: overflow-tile hidden activations as
 *                                 bf16 hi (columns < N) + lo (columns >= N) parts
 *   units      int32  [M*NT][4]   scratch: work units of rows split across warps
 *   z          fp32   [4][M][N] + int32 [NT]
 *                                 scratch, only for M <= TWELL_SMALL_M (else NULL):
 *                                 partial gate sums of the small-batch gate pass
 *                                 (up to four CTAs per 128-unit tile), then one
 *                                 ticket per TwELL tile
 */
typedef struct twell_buf {
  uint16_t* counts;
  uint8_t* idx;
  float* vals;
  float* dense_rows;
  int32_t* row_slot;
  int32_t* slot_row;
  int32_t* ctrl;
  uint16_t* x_over;
  uint16_t* h_over;
  void* units;
  float* z;
  int M, K, N, T, C, R_cap;
} twell_buf;

/* Batches of at most this many rows take the small-batch gate pass: it
 * streams W_g through the tensor cores with the tokens on the narrow side of
 * the tile (128 hidden units x up to 128 tokens), cut into equal contiguous
 * k ranges per SM; the last CTA to finish a TwELL tile packs it.  (Batches of
 * up to 256 rows also take the static-unit up/down pass of twell_ffn_fwd.) */
#define TWELL_SMALL_M 128

/* Bytes of device memory twell_buf_init needs for these sizes (0 if invalid). */
size_t twell_buf_bytes(int M, int K, int N, int T, int C, int R_cap);

/*
 * Carve `base` (device pointer, >= twell_buf_bytes(...) bytes, 256-byte
 * aligned) into the arrays of `tw`.  Host-side pointer arithmetic only; the
 * contents are initialised by twell_gate_pack.  Limits: M >= 1, K % 64 == 0,
 * 64 <= K <= 4096, T in {128, 256}, N % T == 0, N / T <= 256,
 * 1 <= C <= min(T, 255), 1 <= R_cap.
 */
twell_status twell_buf_init(twell_buf* tw, void* base, size_t bytes, int M, int K, int N, int T, int C,
                            int R_cap);

/*
 * Gate GEMM + ReLU + TwELL pack + overflow routing ("Sparser, Faster, Lighter
 * Transformer Language Models", §3-4 steps 1-5, §3-6, §4-3).  x [M][K], wg_t
 * [N][K] device bf16.  M, K, N must equal the buffer's.  Fills every array of
 * `tw` described above.  Launches: a small reset kernel, then one gate GEMM
 * whose epilogue packs TwELL; for M <= TWELL_SMALL_M instead the small-batch
 * gate pass described at TWELL_SMALL_M (the same records, order, counts and
 * overflow routing).
 *
 * n_over_host: if NULL the call is fully asynchronous; the overflow count stays
 * on the device (ctrl[0]) and twell_read_status reports it later.  If not NULL
 * the call synchronises `stream`, stores the number of rows that asked for a
 * dense-row slot and returns TWELL_ERR_CAPACITY when it exceeds R_cap; the
 * caller then re-initialises a buffer with R_cap >= *n_over_host and calls
 * again (the pages' CPU-side flag and retry).
 */
twell_status twell_gate_pack(const uint16_t* x, const uint16_t* wg_t, int M, int K, int N, twell_buf* tw,
                             int* n_over_host, cudaStream_t stream);

/*
 * Fused sparse up + down projection over `tw` ("Sparser, Faster, Lighter
 * Transformer Language Models", §3-5; filled by twell_gate_pack on the same
 * stream), then the dense-row path for overflow tiles (§3-6, §4-3).  wu_t, wd [N][K]
 * device bf16; y [M][K] device fp32, fully overwritten.  K must equal tw->K.
 * For M <= 256: y is cleared (a memset on `stream`) and one static-unit
 * kernel serves TwELL and overflow tiles (no dense-row GEMMs).  Asynchronous.
 * If the gate pass ran out of dense-row slots, the rows marked -2 in row_slot
 * miss their overflow tiles and twell_read_status returns TWELL_ERR_CAPACITY.
 */
twell_status twell_ffn_fwd(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd, const twell_buf* tw,
                           int K, float* y, cudaStream_t stream);

/*
 * The whole sparse forward in one call: x [M][K], wg_t, wu_t, wd [N][K] device
 * bf16, y [M][K] device fp32 (overwritten); M, K, N must equal the buffer's.
 * For M <= TWELL_SMALL_M it launches the reset kernel and then one persistent
 * kernel (one CTA per SM at most, 192 threads) that runs the small-batch gate
 * pass, waits at a grid barrier (bounded: a wait that gives up raises a device
 * flag and the CTA returns, so twell_read_status then reports
 * TWELL_ERR_DEVICE_CHECK), and runs the small-batch up/down units; `tw` holds
 * the TwELL records afterwards as after twell_gate_pack.  For larger M it is
 * twell_gate_pack followed by twell_ffn_fwd.  n_over_host as for
 * twell_gate_pack, except that on small batches the capacity check runs after
 * the forward (a TWELL_ERR_CAPACITY result leaves y incomplete; retry with a
 * larger R_cap).
 */
twell_status twell_ffn_fused(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd, int M,
                             int K, int N, twell_buf* tw, float* y, int* n_over_host, cudaStream_t stream);

/*
 * Backward pass over the hybrid activations (training; "Sparser, Faster,
 * Lighter Transformer Language Models", §3-6 and §3-7: every product visits
 * only the active units).  Given the TwELL + dense-row buffer `tw` of the
 * forward (twell_gate_pack on the same x, wg_t) and the upstream gradient
 * dy [M][K] (device fp32), writes, all device fp32 and fully overwritten:
 *   dx    [M][K]  = sum_n du_n W_u^T[n] + dz_n W_g^T[n]
 *   dwg_t [N][K]  = sum_m dz_{m,n} x_m,   dwu_t [N][K] = sum_m du_{m,n} x_m,
 *   dwd   [N][K]  = sum_m h_{m,n} dy_m      (rows of inactive units are 0)
 * with, per active (m, n): u = x_m W_u^T[n], dh = dy_m . W_d[n], h = u g,
 * du = dh g, dz = dh u (g = ReLU(z) from TwELL or the row's dense-row slot).
 * scratch: device, 256-byte aligned, >= twell_bwd_scratch_bytes(...) bytes
 * (per-unit counts and offsets, the pieces of heavy units, a unit-major list
 * of 16-byte entries (row, h, du, dz): the hybrid activations transposed, and
 * the operands of the dense-slot GEMMs).  Limits: those of twell_buf_init and
 * K <= 2560.
 * Host side: the call queues two memsets (counters, dx) and the count
 * kernel, which also counts the active entries of the slotted rows' overflow
 * tiles; it reads that count and the number of slotted rows R (two 4-byte
 * device-to-host copies and a synchronize of `stream`), then queues the rest
 * without waiting: four kernels (two scans, row pass, unit pass), and before
 * them, when the slotted rows go through the gather passes, one kernel that
 * adds their entries to the per-unit counts.  The
 * slotted rows take one of two routes (twell_bwd_slot_route):
 * their entries join the row and unit passes, or three memsets, an operand
 * kernel and eight tensor-core GEMMs cover them.  By default the GEMMs are
 * taken when R > 8 and the rows hold more than 14 N + 12e6 / K entries (the
 * measured break-even on one B200, a little short of it).  The sums over rows
 * and units are taken in an order that atomics decide, so repeated calls
 * agree to rounding, not bit for bit.
 */
size_t twell_bwd_scratch_bytes(int M, int K, int N, int T, int C, int R_cap);

/*
 * Route of the slotted rows in the following twell_ffn_bwd calls on the
 * calling thread: 0 by the entry count above (the default), 1 always the
 * dense-slot GEMMs (when any row is slotted), 2 always the gather passes.
 * Both routes compute the same gradients (to rounding).  Returns
 * TWELL_ERR_INVALID for any other value.
 */
twell_status twell_bwd_slot_route(int route);
twell_status twell_ffn_bwd(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                           const twell_buf* tw, const float* dy, int K, float* dx, float* dwg_t, float* dwu_t,
                           float* dwd, void* scratch, size_t scratch_bytes, cudaStream_t stream);

/*
 * Synchronises `stream` and reads the buffer's device control words.
 * Returns TWELL_ERR_DEVICE_CHECK if a device status flag other than the
 * capacity flag is set, else TWELL_ERR_CAPACITY if n_over > R_cap, else
 * TWELL_OK.  Either output pointer may be NULL.
 */
twell_status twell_read_status(const twell_buf* tw, int* n_over_host, int* device_flags, cudaStream_t stream);

/*
 * Dense comparison FFN (§1-1 computed in full, §2-2 "dense pipeline"):
 * GEMM 1 computes x W_g and x W_u for the same column tile into two TMEM
 * accumulators and writes h = (x W_u) * ReLU(x W_g) into h_scratch as two
 * bf16 halves, hi = bf16(h) in columns [0, N) and lo = bf16(h - hi) in
 * columns [N, 2N) of h_scratch [M][2N] (device, caller-owned); GEMM 2 writes
 * y = h_hi W_d + h_lo W_d, fp32 [M][K].  h keeps about 16 significant bits, so
 * y meets the same accuracy bound as the sparse path (a single bf16 h leaves
 * an error of 2^-9 of each row's own scale, which heavy-tailed rows carry far
 * above the global rms of y).  Limits: K % 64 == 0, N % 128 == 0.
 * Asynchronous.
 */
twell_status dense_ffn_fwd(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                           int M, int K, int N, uint16_t* h_scratch, float* y, cudaStream_t stream);

/*
 * The same dense FFN with h rounded to a single bf16 (h_scratch [M][N]), as a
 * plain bf16 dense FFN keeps it.  Faster than dense_ffn_fwd (GEMM 2 reduces
 * over N, not 2N) but less accurate: reported next to it as a second dense
 * comparison point, not held to the sparse path's accuracy bound.
 */
twell_status dense_ffn_fwd_bf16h(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                                 int M, int K, int N, uint16_t* h_scratch, float* y, cudaStream_t stream);

/*
 * dense_ffn_fwd without a caller-provided hidden buffer, for callers that
 * cannot allocate device memory when they call (a runtime that has handed all
 * device memory to its own pool, or an embedding that forbids allocation while
 * it executes).  The pages describe no such variant; it is an interface
 * convenience of this library.
 *
 * The hidden activations (bf16 hi + lo, M x 2N values) use a fixed 32 MiB
 * array inside the library's device image (every device that loads the
 * library holds it until the process exits), so M * 2N must not exceed
 * 16,777,216 (M * N <= 8,388,608); larger problems return TWELL_ERR_INVALID
 * with a message and launch nothing.  No device memory is allocated or freed
 * by this call.  The array's device address is looked up with
 * cudaGetSymbolAddress on the first call in each CUDA context (with that
 * context's device current) and cached per context id, so a context that
 * cudaDeviceReset tore down and the runtime created again is looked up anew;
 * make the first call in a context before any stream capture.  All calls share
 * the one array and it keeps the last call's contents, so calls that overlap
 * on the GPU (other streams, other host threads) race on it; serialise them.
 * Otherwise identical to dense_ffn_fwd: y [M][K] fp32 is overwritten,
 * asynchronous on `stream`.
 */
twell_status dense_ffn_fwd_noalloc(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t, const uint16_t* wd,
                                   int M, int K, int N, float* y, cudaStream_t stream);

/*
 * Host-side fault injection for tests of the device status path.  Arms a
 * one-shot for the next twell_ffn_fwd on this thread: its fused kernel waits
 * for one more scanned token row than exist, a condition nothing makes true,
 * with a wait limit of limit_ns nanoseconds instead of the usual 2 s.  The
 * wait expires, the kernel raises its timeout flag and returns (the rows of
 * split work units are then left incomplete), and twell_read_status reports
 * TWELL_ERR_DEVICE_CHECK.  On a small batch the one-shot is taken instead by
 * the next twell_ffn_fused, whose grid barrier then waits for one CTA more
 * than the grid holds (y is left unwritten past the barrier).  The
 * small-batch twell_ffn_fwd has no such wait and leaves the one-shot armed.  The next twell_gate_pack clears the flag.  No
 * memory access changes.  limit_ns must lie in [1000, 1000000000]; 0 disarms.
 */
twell_status twell_test_expire_wait(long long limit_ns);

/* Static description of a status code. */
const char* twell_status_str(twell_status status);

/* Message of the last TWELL_ERR_CUDA / TWELL_ERR_INVALID on this thread. */
const char* twell_last_error(void);

/* Number of kernels the last call on this thread enqueued (for launch accounting). */
int twell_last_launch_count(void);

/*
 * Per-kernel timing hook.  After twell_trace_events(events, capacity) with an
 * array of 2*capacity caller-created CUDA events, each kernel that later
 * calls on this thread enqueue is bracketed by cudaEventRecord(events[2i]) and
 * cudaEventRecord(events[2i+1]) on the call's stream, for the first `capacity`
 * kernels.  twell_trace_count() returns how many were recorded and
 * twell_trace_name(i) the kernel's name (static string).  Passing NULL turns
 * tracing off.  Tracing adds event records only; the work is unchanged.
 */
twell_status twell_trace_events(cudaEvent_t* events, int capacity);
int twell_trace_count(void);
const char* twell_trace_name(int i);

#ifdef __cplusplus
}
#endif

#endif /* TWELL_H_ */
