/*
 * CPU oracle for the ReLU-gated sparse FFN forward pass.  TEST INFRASTRUCTURE
 * ONLY: the tests, the package's smoke check and the benchmark's CPU-baseline
 * leg call it; the CUDA library never does, and nothing here is shared with it.
 *
 * Source: "Sparser, Faster, Lighter Transformer Language Models" (review page,
 * dimensionstp.github.io):
 *   §1-1 problem definition:  h_u = x W_u,  h_g = ReLU(x W_g),  h = h_u * h_g,
 *                             y = h W_d      (W_g, W_u: K -> N; W_d: N -> K)
 *   §1-1 skip rule:           h_g[m,n] = 0  =>  W_u column n and W_d row n are
 *                             not needed for token m
 *   §3-4 TwELL:               columns cut into tiles of width T; per (row, tile)
 *                             a non-zero count plus packed values and indices
 *   §3-5 sparse rewrite:      y_m = sum_{n in A_m} (h_g)_{m,n} (x_m W_u[:,n]) W_d[n,:]
 *   §3-6 hybrid format:       entries that do not fit the compact capacity are
 *                             kept in a dense backup row instead
 *
 * Everything is computed in double precision from the exact bf16 inputs.
 * Loops are the definitions written out; threads only split the list of rows.
 *
 * Weight layouts (row-major, bf16 bit patterns):
 *   wg_t[n][k] = W_g[k][n],  wu_t[n][k] = W_u[k][n],  wd[n][k] = W_d[n][k].
 */
#include <math.h>
#include <pthread.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

/* bf16 -> double: a bf16 is the top 16 bits of an IEEE binary32. */
static double bf16_to_double(uint16_t b) {
    uint32_t u = ((uint32_t)b) << 16;
    float f;
    memcpy(&f, &u, sizeof f);
    return (double)f;
}

void oracle_bf16_to_f64(const uint16_t* src, int64_t n, double* dst) {
    for (int64_t i = 0; i < n; ++i) dst[i] = bf16_to_double(src[i]);
}

/* ------------------------------------------------------------------------ */
/* Row-parallel driver: work(ctx, r) for r in [0, nrows), split over threads. */
typedef void (*row_fn)(void* ctx, int64_t r);
typedef struct { row_fn fn; void* ctx; int64_t begin, end; } span_t;

static void* run_span(void* p) {
    span_t* s = (span_t*)p;
    for (int64_t r = s->begin; r < s->end; ++r) s->fn(s->ctx, r);
    return NULL;
}

static void for_rows(int64_t nrows, int nthreads, row_fn fn, void* ctx) {
    if (nthreads < 1) nthreads = 1;
    if (nthreads > 256) nthreads = 256;
    if (nthreads > nrows) nthreads = (int)(nrows > 0 ? nrows : 1);
    if (nthreads == 1) {
        for (int64_t r = 0; r < nrows; ++r) fn(ctx, r);
        return;
    }
    pthread_t th[256];
    span_t sp[256];
    for (int i = 0; i < nthreads; ++i) {
        sp[i].fn = fn;
        sp[i].ctx = ctx;
        sp[i].begin = nrows * i / nthreads;
        sp[i].end = nrows * (i + 1) / nthreads;
        pthread_create(&th[i], NULL, run_span, &sp[i]);
    }
    for (int i = 0; i < nthreads; ++i) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------ */
/* Gate pre-activation  z[r][n] = sum_k x[rows[r]][k] * W_g[k][n]  (§1-1). */
typedef struct {
    const uint16_t* x; const uint16_t* wg_t; int K, N;
    const int64_t* rows; double* z;
} gate_ctx;

static void gate_row(void* p, int64_t r) {
    gate_ctx* c = (gate_ctx*)p;
    const uint16_t* xr = c->x + c->rows[r] * (int64_t)c->K;
    double* zr = c->z + r * (int64_t)c->N;
    for (int n = 0; n < c->N; ++n) {
        const uint16_t* w = c->wg_t + (int64_t)n * c->K;
        double acc = 0.0;
        for (int k = 0; k < c->K; ++k) acc += bf16_to_double(xr[k]) * bf16_to_double(w[k]);
        zr[n] = acc;
    }
}

void oracle_gate(const uint16_t* x, const uint16_t* wg_t, int K, int N,
                 const int64_t* rows, int64_t nrows, double* z, int nthreads) {
    gate_ctx c = {x, wg_t, K, N, rows, z};
    for_rows(nrows, nthreads, gate_row, &c);
}

/* ------------------------------------------------------------------------ */
/* TwELL packing of gate pre-activations (§3-4), with the hybrid dense backup
 * for tiles whose non-zero count exceeds the capacity (§3-6).
 *
 *   active(m, n)  <=>  z[m][n] > 0          (ReLU gives an exact zero otherwise)
 *   counts[r][t]  = number of active n in tile t (the true count, even if > C)
 *   if counts <= C: idx/vals[r][t][0..cnt-1] = (n - t*T, ReLU(z)) in ascending n,
 *                   remaining slots idx = 0, vals = 0
 *   if counts >  C: the tile overflows: overflow[r][t] = 1, its slots are left
 *                   zero and dense[r][t*T + j] = ReLU(z[r][t*T + j]) for all j.
 *   dense[r][n] = 0 in every tile that does not overflow.
 */
void oracle_twell_pack(const double* z, int64_t nrows, int N, int T, int C,
                       int32_t* counts, int32_t* idx, double* vals,
                       uint8_t* overflow, double* dense) {
    const int NT = N / T;
    for (int64_t r = 0; r < nrows; ++r) {
        const double* zr = z + r * (int64_t)N;
        for (int t = 0; t < NT; ++t) {
            int cnt = 0;
            for (int j = 0; j < T; ++j)
                if (zr[t * T + j] > 0.0) ++cnt;
            int64_t rec = r * NT + t;
            counts[rec] = cnt;
            for (int s = 0; s < C; ++s) { idx[rec * C + s] = 0; vals[rec * C + s] = 0.0; }
            for (int j = 0; j < T; ++j) dense[r * (int64_t)N + t * T + j] = 0.0;
            if (cnt <= C) {
                overflow[rec] = 0;
                int s = 0;
                for (int j = 0; j < T; ++j) {
                    double v = zr[t * T + j];
                    if (v > 0.0) { idx[rec * C + s] = j; vals[rec * C + s] = v; ++s; }
                }
            } else {
                overflow[rec] = 1;
                for (int j = 0; j < T; ++j) {
                    double v = zr[t * T + j];
                    dense[r * (int64_t)N + t * T + j] = v > 0.0 ? v : 0.0;
                }
            }
        }
    }
}

/* ------------------------------------------------------------------------ */
/* Sparse output by the §3-5 rewrite, reading the active set from TwELL:
 *   y_m = sum over active n of g_{m,n} * (x_m . W_u[:,n]) * W_d[n,:]
 * where (n, g) come from the packed slots of non-overflow tiles and from the
 * non-zero entries of the dense backup row for overflow tiles. */
typedef struct {
    const uint16_t* x; const uint16_t* wu_t; const uint16_t* wd; int K, N, T, C;
    const int64_t* rows; const int32_t* counts; const int32_t* idx; const double* vals;
    const uint8_t* overflow; const double* dense; double* y;
} twell_y_ctx;

static void add_neuron(const twell_y_ctx* c, const uint16_t* xr, double* yr, int n, double g) {
    const uint16_t* u_row = c->wu_t + (int64_t)n * c->K;
    double u = 0.0;
    for (int k = 0; k < c->K; ++k) u += bf16_to_double(xr[k]) * bf16_to_double(u_row[k]);
    const double h = g * u;
    const uint16_t* d_row = c->wd + (int64_t)n * c->K;
    for (int k = 0; k < c->K; ++k) yr[k] += h * bf16_to_double(d_row[k]);
}

static void twell_y_row(void* p, int64_t r) {
    const twell_y_ctx* c = (const twell_y_ctx*)p;
    const uint16_t* xr = c->x + c->rows[r] * (int64_t)c->K;
    double* yr = c->y + r * (int64_t)c->K;
    for (int k = 0; k < c->K; ++k) yr[k] = 0.0;
    const int NT = c->N / c->T;
    for (int t = 0; t < NT; ++t) {
        int64_t rec = r * NT + t;
        if (!c->overflow[rec]) {
            for (int s = 0; s < c->counts[rec]; ++s)
                add_neuron(c, xr, yr, t * c->T + c->idx[rec * c->C + s], c->vals[rec * c->C + s]);
        } else {
            for (int j = 0; j < c->T; ++j) {
                double g = c->dense[r * (int64_t)c->N + t * c->T + j];
                if (g != 0.0) add_neuron(c, xr, yr, t * c->T + j, g);
            }
        }
    }
}

void oracle_ffn_twell(const uint16_t* x, const uint16_t* wu_t, const uint16_t* wd,
                      int K, int N, int T, int C, const int64_t* rows, int64_t nrows,
                      const int32_t* counts, const int32_t* idx, const double* vals,
                      const uint8_t* overflow, const double* dense, double* y, int nthreads) {
    twell_y_ctx c = {x, wu_t, wd, K, N, T, C, rows, counts, idx, vals, overflow, dense, y};
    for_rows(nrows, nthreads, twell_y_row, &c);
}

/* ------------------------------------------------------------------------ */
/* Dense output by the §1-1 definition, computing every hidden unit:
 *   h_u = x W_u,  h_g = ReLU(x W_g),  h = h_u * h_g,  y = h W_d. */
typedef struct {
    const uint16_t* x; const uint16_t* wg_t; const uint16_t* wu_t; const uint16_t* wd;
    int K, N; const int64_t* rows; double* y; double* scratch; /* [nrows][N] */
} dense_ctx;

static void dense_row(void* p, int64_t r) {
    const dense_ctx* c = (const dense_ctx*)p;
    const uint16_t* xr = c->x + c->rows[r] * (int64_t)c->K;
    double* h = c->scratch + r * (int64_t)c->N;
    for (int n = 0; n < c->N; ++n) {
        double hg = 0.0, hu = 0.0;
        for (int k = 0; k < c->K; ++k) {
            double xv = bf16_to_double(xr[k]);
            hg += xv * bf16_to_double(c->wg_t[(int64_t)n * c->K + k]);
            hu += xv * bf16_to_double(c->wu_t[(int64_t)n * c->K + k]);
        }
        if (hg < 0.0) hg = 0.0;
        h[n] = hu * hg;
    }
    double* yr = c->y + r * (int64_t)c->K;
    for (int k = 0; k < c->K; ++k) {
        double acc = 0.0;
        for (int n = 0; n < c->N; ++n) acc += h[n] * bf16_to_double(c->wd[(int64_t)n * c->K + k]);
        yr[k] = acc;
    }
}

void oracle_ffn_dense(const uint16_t* x, const uint16_t* wg_t, const uint16_t* wu_t,
                      const uint16_t* wd, int K, int N, const int64_t* rows, int64_t nrows,
                      double* y, int nthreads) {
    double* scratch = (double*)malloc(sizeof(double) * (size_t)(nrows > 0 ? nrows : 1) * (size_t)N);
    if (!scratch) return;
    dense_ctx c = {x, wg_t, wu_t, wd, K, N, rows, y, scratch};
    for_rows(nrows, nthreads, dense_row, &c);
    free(scratch);
}
