/*
 * nf4_oracle.c -- CPU oracle for the host-streamed NF4 LoRA hot path.
 *
 * TEST INFRASTRUCTURE ONLY (see nf4_oracle.h): loaded by the tests, the
 * smoke check and the benchmark's CPU-baseline leg, never by the product.
 * Plain C11, libm and pthreads; no BLAS, no blocking, no reordering of any
 * sum: every output element is one loop in index order, accumulated in
 * double and rounded once.  Threads only split the set of output elements.
 */
#include "nf4_oracle.h"

#include <math.h>
#include <pthread.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

/* ------------------------------------------------------------------------ */
/* allocation                                                               */
/* ------------------------------------------------------------------------ */
/* A checker must fail loudly: an allocation the oracle cannot make ends the
 * process with a message rather than leaving outputs unwritten. */

static void *xmalloc(size_t n) {
  void *p = malloc(n ? n : 1);
  if (!p) {
    fprintf(stderr, "nf4 oracle: out of memory allocating %zu bytes\n", n);
    abort();
  }
  return p;
}

static void *xcalloc(size_t n, size_t size) {
  void *p = calloc(n ? n : 1, size ? size : 1);
  if (!p) {
    fprintf(stderr, "nf4 oracle: out of memory allocating %zu x %zu bytes\n", n, size);
    abort();
  }
  return p;
}

/* ------------------------------------------------------------------------ */
/* bf16 <-> fp32                                                            */
/* ------------------------------------------------------------------------ */

float orc_bf16_to_f32(uint16_t h) {
  uint32_t u = (uint32_t)h << 16;
  float f;
  memcpy(&f, &u, sizeof f);
  return f;
}

/* Round to nearest, ties to even.  NaN becomes a quiet NaN. */
uint16_t orc_f32_to_bf16(float f) {
  uint32_t u;
  memcpy(&u, &f, sizeof u);
  if ((u & 0x7fffffffu) > 0x7f800000u) return (uint16_t)((u >> 16) | 0x0040u);
  uint32_t lsb = (u >> 16) & 1u;
  u += 0x7fffu + lsb;
  return (uint16_t)(u >> 16);
}

/* ------------------------------------------------------------------------ */
/* NormalFloat-4 codebook                                                   */
/* ------------------------------------------------------------------------ */
/* The pages name the data type (4-bit NF4, Poros API reference,
 * PorosTrainer.from_pretrained "quantization") but print no values.  NF4 is
 * a fixed published data type: QLoRA (Dettmers et al. 2023), Appendix E
 * "NormalFloat 4-bit data type", prints its 16 values, and those exact
 * float32 numbers are what this oracle uses.
 *
 * Where they come from (section "4-bit NormalFloat Quantization" of the same
 * paper): standard-normal quantiles at probabilities spaced evenly from
 * delta = 1 - (1/32 + 1/30)/2 down to 1/2 -- eight on the positive side and
 * seven mirrored on the negative side, the 1/2 end excluded -- plus an exact
 * zero, all divided by the largest magnitude so that the ends are -1 and +1.
 * The printed values carry that construction with the probabilities and the
 * final division in single precision, so they sit a few float32 ulps away
 * from the same construction in exact arithmetic; orc_normal_quantile below
 * lets the tests check that distance. */

static const float kNf4Published[16] = {
    -1.0f,
    -0.6961928009986877f,
    -0.5250730514526367f,
    -0.39491748809814453f,
    -0.28444138169288635f,
    -0.18477343022823334f,
    -0.09105003625154495f,
    0.0f,
    0.07958029955625534f,
    0.16093020141124725f,
    0.24611230194568634f,
    0.33791524171829224f,
    0.44070982933044434f,
    0.5626170039176941f,
    0.7229568362236023f,
    1.0f,
};

static double normal_cdf(double x) { return 0.5 * erfc(-x / sqrt(2.0)); }

/* Inverse standard-normal CDF by bisection on erfc (used only by the tests'
 * check of the construction above). */
double orc_normal_quantile(double p) {
  double lo = -40.0, hi = 40.0;
  for (int it = 0; it < 4000; ++it) {
    double mid = 0.5 * (lo + hi);
    if (mid <= lo || mid >= hi) break;
    if (normal_cdf(mid) < p)
      lo = mid;
    else
      hi = mid;
  }
  return 0.5 * (lo + hi);
}

void orc_nf4_codebook(float out[16]) {
  for (int i = 0; i < 16; ++i) out[i] = kNf4Published[i];
}

/* Nearest codebook entry by a linear scan of fp32 distances |x - c_i|.
 * Reading: the pages fix no tie rule; a strict '<' keeps the lower index. */
static int nearest_code(const float cb[16], float x) {
  int best = 0;
  float bd = fabsf(x - cb[0]);
  for (int i = 1; i < 16; ++i) {
    float d = fabsf(x - cb[i]);
    if (d < bd) {
      bd = d;
      best = i;
    }
  }
  return best;
}

int orc_nf4_nearest(float x) {
  float cb[16];
  orc_nf4_codebook(cb);
  return nearest_code(cb, x);
}

/* ------------------------------------------------------------------------ */
/* NF4 storage format                                                       */
/* ------------------------------------------------------------------------ */
/* Format reading: row-major W[n_out, k_in], flat index e = n*k_in + k,
 * 64-element blocks along e (so a block never crosses a row when
 * k_in % 64 == 0), one fp32 absmax per block, 4-bit codes two per byte with
 * the even element in the high nibble.  0.5 + 4/64 = 0.5625 byte/param,
 * which is what reproduces the ~4/~18/~40 GB host footprints quoted for the
 * NF4 base ("Poros on consumer GPUs", "What you need besides VRAM"). */

int64_t orc_nf4_storage_bytes(int64_t n_out, int64_t k_in) {
  int64_t p = n_out * k_in;
  return p / 2 + 4 * (p / 64);
}

static int shape_ok(int64_t n_out, int64_t k_in) {
  return n_out > 0 && k_in > 0 && (k_in % 64) == 0;
}

int orc_nf4_quantize(const uint16_t *w, int64_t n_out, int64_t k_in,
                     uint8_t *codes, float *absmax) {
  if (!shape_ok(n_out, k_in)) return -1;
  float cb[16];
  orc_nf4_codebook(cb);
  const int64_t nblk = n_out * k_in / 64;
  for (int64_t b = 0; b < nblk; ++b) {
    const uint16_t *blk = w + b * 64;
    float a = 0.0f;
    for (int i = 0; i < 64; ++i) {
      float v = fabsf(orc_bf16_to_f32(blk[i]));
      if (v > a) a = v;
    }
    absmax[b] = a;
    for (int i = 0; i < 64; ++i) {
      int code;
      if (a == 0.0f) {
        code = 7; /* all-zero block: the exact-zero entry */
      } else {
        float x = orc_bf16_to_f32(blk[i]) / a; /* IEEE fp32 division */
        code = nearest_code(cb, x);
      }
      int64_t e = b * 64 + i;
      if ((e & 1) == 0)
        codes[e >> 1] = (uint8_t)(code << 4);
      else
        codes[e >> 1] = (uint8_t)(codes[e >> 1] | code);
    }
  }
  return 0;
}

static int code_at(const uint8_t *codes, int64_t e) {
  uint8_t byte = codes[e >> 1];
  return (e & 1) ? (byte & 0x0f) : (byte >> 4);
}

int orc_nf4_dequant(const uint8_t *codes, const float *absmax, int64_t n_out,
                    int64_t k_in, uint16_t *out) {
  if (!shape_ok(n_out, k_in)) return -1;
  float cb[16];
  orc_nf4_codebook(cb);
  const int64_t total = n_out * k_in;
  for (int64_t e = 0; e < total; ++e) {
    float v = cb[code_at(codes, e)] * absmax[e / 64]; /* fp32 product */
    out[e] = orc_f32_to_bf16(v);
  }
  return 0;
}

/* ------------------------------------------------------------------------ */
/* a minimal parallel-for over an index range                               */
/* ------------------------------------------------------------------------ */

typedef void (*range_fn)(void *ctx, int64_t lo, int64_t hi);

typedef struct {
  range_fn fn;
  void *ctx;
  int64_t lo, hi;
} range_job;

static void *range_thread(void *p) {
  range_job *j = (range_job *)p;
  j->fn(j->ctx, j->lo, j->hi);
  return NULL;
}

static void parallel_for(int64_t n, int n_threads, range_fn fn, void *ctx) {
  if (n_threads < 1) n_threads = 1;
  if (n_threads > 256) n_threads = 256;
  if ((int64_t)n_threads > n) n_threads = (int)(n > 0 ? n : 1);
  if (n_threads == 1) {
    fn(ctx, 0, n);
    return;
  }
  pthread_t th[256];
  range_job jobs[256];
  int started[256];
  for (int i = 0; i < n_threads; ++i) {
    jobs[i].fn = fn;
    jobs[i].ctx = ctx;
    jobs[i].lo = n * i / n_threads;
    jobs[i].hi = n * (i + 1) / n_threads;
    started[i] = pthread_create(&th[i], NULL, range_thread, &jobs[i]) == 0;
    if (!started[i]) fn(ctx, jobs[i].lo, jobs[i].hi);
  }
  for (int i = 0; i < n_threads; ++i)
    if (started[i]) pthread_join(th[i], NULL);
}

/* ------------------------------------------------------------------------ */
/* LoRA linear                                                              */
/* ------------------------------------------------------------------------ */
/* The layer computed for every projection (q/k/v/o/gate/up/down) with the
 * frozen base W and the trainable rank-r adapter (A [r,K], B [N,r]),
 * Poros API reference, PorosTrainer.from_pretrained (lora_rank, lora_alpha;
 * dropout 0 here):
 *   forward   Y  = X W^T + (alpha/r) (X A^T) B^T
 *   backward  dX = dY W + (alpha/r) (dY B) A
 *             dB = (alpha/r) dY^T (X A^T)
 *             dA = (alpha/r) (dY B)^T X
 * W is frozen -- read, never written (HN comment on host-RAM streaming). */

/* A source of rows of W, as doubles, for columns [k0, k1). */
typedef struct {
  const double *dense;   /* [N,K] or NULL */
  const uint16_t *wbf16; /* [N,K] bf16 bit patterns or NULL */
  const uint8_t *codes;
  const float *absmax;
  float cb[16];
  int64_t K;
} wsrc;

static void w_row(const wsrc *w, int64_t n, int64_t k0, int64_t k1,
                  double *out) {
  if (w->dense) {
    for (int64_t k = k0; k < k1; ++k) out[k - k0] = w->dense[n * w->K + k];
    return;
  }
  if (w->wbf16) {
    for (int64_t k = k0; k < k1; ++k)
      out[k - k0] = (double)orc_bf16_to_f32(w->wbf16[n * w->K + k]);
    return;
  }
  for (int64_t k = k0; k < k1; ++k) {
    int64_t e = n * w->K + k;
    float v = w->cb[code_at(w->codes, e)] * w->absmax[e / 64];
    out[k - k0] = (double)orc_bf16_to_f32(orc_f32_to_bf16(v));
  }
}

/* ---- forward: parallel over output columns n ---- */
typedef struct {
  const wsrc *w;
  const double *X; /* [n_rows, K] token rows to compute */
  const double *t; /* [n_rows, r] */
  const double *B; /* [N, r] */
  int64_t n_rows, N, K;
  int r;
  double s;
  double *Y; /* [n_rows, N] */
} fwd_ctx;

static void fwd_cols(void *p, int64_t lo, int64_t hi) {
  fwd_ctx *c = (fwd_ctx *)p;
  double *row = (double *)xmalloc(sizeof(double) * (size_t)c->K);
  if (!row) return;
  for (int64_t n = lo; n < hi; ++n) {
    w_row(c->w, n, 0, c->K, row);
    for (int64_t i = 0; i < c->n_rows; ++i) {
      const double *x = c->X + i * c->K;
      double acc = 0.0;
      for (int64_t k = 0; k < c->K; ++k) acc += x[k] * row[k];
      double lora = 0.0;
      for (int j = 0; j < c->r; ++j) lora += c->t[i * c->r + j] * c->B[n * c->r + j];
      c->Y[i * c->N + n] = acc + c->s * lora;
    }
  }
  free(row);
}

/* t = X A^T for the given rows (cheap; single thread) */
static void lora_down(const double *X, const double *A, int64_t rows,
                      int64_t K, int r, double *t) {
  for (int64_t i = 0; i < rows; ++i)
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t k = 0; k < K; ++k) acc += X[i * K + k] * A[j * K + k];
      t[i * r + j] = acc;
    }
}

/* ---- dX: parallel over output columns k (contraction over n in order) ---- */
typedef struct {
  const wsrc *w;
  const double *dY; /* [n_rows, N] */
  const double *u;  /* [n_rows, r] */
  const double *A;  /* [r, K] */
  int64_t n_rows, N, K;
  int r;
  double s;
  double *dX; /* [n_rows, K] */
  const double *g; /* [n_rows, K] multiplier of the LoRA term (dropout), or NULL */
} dx_ctx;

static void dx_cols(void *p, int64_t lo, int64_t hi) {
  dx_ctx *c = (dx_ctx *)p;
  int64_t width = hi - lo;
  if (width <= 0) return;
  double *row = (double *)xmalloc(sizeof(double) * (size_t)width);
  double *acc = (double *)xcalloc((size_t)(c->n_rows * width), sizeof(double));
  if (!row || !acc) {
    free(row);
    free(acc);
    return;
  }
  for (int64_t n = 0; n < c->N; ++n) {
    w_row(c->w, n, lo, hi, row);
    for (int64_t i = 0; i < c->n_rows; ++i) {
      double g = c->dY[i * c->N + n];
      double *a = acc + i * width;
      for (int64_t k = 0; k < width; ++k) a[k] += g * row[k];
    }
  }
  for (int64_t i = 0; i < c->n_rows; ++i)
    for (int64_t k = lo; k < hi; ++k) {
      double lora = 0.0;
      for (int j = 0; j < c->r; ++j) lora += c->u[i * c->r + j] * c->A[j * c->K + k];
      if (c->g) lora *= c->g[i * c->K + k];
      c->dX[i * c->K + k] = acc[i * width + (k - lo)] + c->s * lora;
    }
  free(row);
  free(acc);
}

/* dB[n, j] = s sum_i dY[i, n] t[i, j];  dA[j, k] = s sum_i u[i, j] X[i, k] */
static void lora_grads(const double *X, const double *dY, const double *t,
                       const double *u, int64_t T, int64_t N, int64_t K, int r,
                       double s, double *dA, double *dB) {
  for (int64_t n = 0; n < N; ++n)
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t i = 0; i < T; ++i) acc += dY[i * N + n] * t[i * r + j];
      dB[n * r + j] = s * acc;
    }
  for (int j = 0; j < r; ++j)
    for (int64_t k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int64_t i = 0; i < T; ++i) acc += u[i * r + j] * X[i * K + k];
      dA[j * K + k] = s * acc;
    }
}

/* u = dY B  ([T,N] x [N,r]) */
static void lora_up_t(const double *dY, const double *B, int64_t T, int64_t N,
                      int r, double *u) {
  for (int64_t i = 0; i < T; ++i)
    for (int j = 0; j < r; ++j) {
      double acc = 0.0;
      for (int64_t n = 0; n < N; ++n) acc += dY[i * N + n] * B[n * r + j];
      u[i * r + j] = acc;
    }
}

void orc_lora_fwd_f64(const double *W, const double *X, const double *A,
                      const double *B, int64_t T, int64_t N, int64_t K, int r,
                      double s, double *Y, double *t) {
  orc_lora_fwd_f64m(W, X, X, A, B, T, N, K, r, s, Y, t);
}

void orc_lora_fwd_f64m(const double *W, const double *X, const double *Xl,
                       const double *A, const double *B, int64_t T, int64_t N,
                       int64_t K, int r, double s, double *Y, double *t) {
  wsrc w;
  memset(&w, 0, sizeof w);
  w.dense = W;
  w.K = K;
  lora_down(Xl, A, T, K, r, t);
  fwd_ctx c = {&w, X, t, B, T, N, K, r, s, Y};
  fwd_cols(&c, 0, N);
}

void orc_lora_bwd_f64(const double *W, const double *X, const double *A,
                      const double *B, const double *dY, int64_t T, int64_t N,
                      int64_t K, int r, double s, double *dX, double *dA,
                      double *dB) {
  orc_lora_bwd_f64m(W, X, NULL, A, B, dY, T, N, K, r, s, dX, dA, dB);
}

void orc_lora_bwd_f64m(const double *W, const double *Xl, const double *g,
                       const double *A, const double *B, const double *dY,
                       int64_t T, int64_t N, int64_t K, int r, double s,
                       double *dX, double *dA, double *dB) {
  const double *X = Xl;
  wsrc w;
  memset(&w, 0, sizeof w);
  w.dense = W;
  w.K = K;
  double *t = (double *)xmalloc(sizeof(double) * (size_t)(T * r));
  double *u = (double *)xmalloc(sizeof(double) * (size_t)(T * r));
  if (!t || !u) {
    free(t);
    free(u);
    return;
  }
  lora_down(X, A, T, K, r, t);
  lora_up_t(dY, B, T, N, r, u);
  dx_ctx c = {&w, dY, u, A, T, N, K, r, s, dX, g};
  dx_cols(&c, 0, K);
  lora_grads(X, dY, t, u, T, N, K, r, s, dA, dB);
  free(t);
  free(u);
}

/* ---- counter-based RNG: Philox4x32-10 (Salmon, Moraes, Dror, Shaw,
 * "Parallel Random Numbers: As Easy as 1, 2, 3", SC 2011), from its
 * published definition: a 4 x 32-bit counter and a 2 x 32-bit key; each of
 * 10 rounds multiplies counter words 0 and 2 by the two round multipliers
 * (full 64-bit products split into high and low halves) and mixes the high
 * halves with the other two words and the key; between rounds the key is
 * bumped by the two Weyl constants. ---- */

void orc_philox4x32_10(const uint32_t ctr_in[4], const uint32_t key_in[2],
                       uint32_t out[4]) {
  uint32_t c0 = ctr_in[0], c1 = ctr_in[1], c2 = ctr_in[2], c3 = ctr_in[3];
  uint32_t k0 = key_in[0], k1 = key_in[1];
  for (int round = 0; round < 10; ++round) {
    if (round > 0) {
      k0 += 0x9E3779B9u;
      k1 += 0xBB67AE85u;
    }
    const uint64_t p0 = (uint64_t)0xD2511F53u * c0;
    const uint64_t p1 = (uint64_t)0xCD9E8D57u * c2;
    const uint32_t hi0 = (uint32_t)(p0 >> 32), lo0 = (uint32_t)p0;
    const uint32_t hi1 = (uint32_t)(p1 >> 32), lo1 = (uint32_t)p1;
    const uint32_t n0 = hi1 ^ c1 ^ k0, n2 = hi0 ^ c3 ^ k1;
    c0 = n0;
    c1 = lo1;
    c2 = n2;
    c3 = lo0;
  }
  out[0] = c0;
  out[1] = c1;
  out[2] = c2;
  out[3] = c3;
}

/* ---- LoRA dropout (Poros API reference: lora_dropout, default 0.05; the
 * dropout sits on the adapter branch's input).  The mask of element e of a
 * row-major [T,K] input (e = t*K + k) under (seed, offset):
 *   q = e / 4;  w = Philox4x32-10(ctr = {lo(q), hi(q), lo(offset), hi(offset)},
 *                                 key = {lo(seed), hi(seed)})[e % 4]
 *   keep  <=>  (w >> 8) >= floor(p * 2^24)   (p * 2^24 formed in fp32)
 * and the kept value is bf16_rne(fp32(x) * scale), scale = fp32(1 / fp32(1 - p)).
 * The caller picks the offset per (step, layer, projection) so that the
 * backward (and any recompute) draws the same mask. ---- */

static uint32_t drop_threshold(float p) { return (uint32_t)(p * 16777216.0f); }

static float drop_scale(float p) {
  volatile float one_minus = 1.0f - p; /* fp32 rounding of each step */
  return 1.0f / one_minus;
}

int orc_dropout_keep(uint64_t seed, uint64_t offset, float p, int64_t T, int64_t K,
                     uint8_t *keep) {
  if (T < 0 || K < 0 || !(p >= 0.0f && p < 1.0f)) return -1;
  const uint32_t thr = drop_threshold(p);
  const uint32_t key[2] = {(uint32_t)seed, (uint32_t)(seed >> 32)};
  const int64_t n = T * K;
  for (int64_t e = 0; e < n; ++e) {
    const uint64_t q = (uint64_t)e >> 2;
    const uint32_t ctr[4] = {(uint32_t)q, (uint32_t)(q >> 32), (uint32_t)offset,
                             (uint32_t)(offset >> 32)};
    uint32_t w[4];
    orc_philox4x32_10(ctr, key, w);
    keep[e] = (w[e & 3] >> 8) >= thr ? 1 : 0;
  }
  return 0;
}

int orc_dropout_apply(const uint16_t *X, int64_t T, int64_t K, uint64_t seed,
                      uint64_t offset, float p, uint16_t *out) {
  uint8_t *keep = (uint8_t *)xmalloc((size_t)(T * K > 0 ? T * K : 1));
  if (!keep) return -1;
  if (orc_dropout_keep(seed, offset, p, T, K, keep) != 0) {
    free(keep);
    return -1;
  }
  const float scale = drop_scale(p);
  for (int64_t e = 0; e < T * K; ++e) {
    volatile float v = orc_bf16_to_f32(X[e]) * scale;
    out[e] = keep[e] ? orc_f32_to_bf16(v) : 0;
  }
  free(keep);
  return 0;
}

/* dropout of one problem: NULL = none */
typedef struct {
  float p;
  uint64_t seed, offset;
} drop_cfg;

/* the adapter branch's input (bf16 X_d, widened) and the dX multiplier
 * keep * scale, or NULLs when there is no dropout */
static int drop_inputs(const drop_cfg *d, const uint16_t *X, int64_t T, int64_t K,
                       double **Xl, double **g) {
  *Xl = NULL;
  *g = NULL;
  if (!d) return 0;
  uint16_t *xd = (uint16_t *)xmalloc(sizeof(uint16_t) * (size_t)(T * K > 0 ? T * K : 1));
  uint8_t *keep = (uint8_t *)xmalloc((size_t)(T * K > 0 ? T * K : 1));
  *Xl = (double *)xmalloc(sizeof(double) * (size_t)(T * K > 0 ? T * K : 1));
  *g = (double *)xmalloc(sizeof(double) * (size_t)(T * K > 0 ? T * K : 1));
  int rc = -1;
  if (xd && keep && *Xl && *g && orc_dropout_apply(X, T, K, d->seed, d->offset, d->p, xd) == 0 &&
      orc_dropout_keep(d->seed, d->offset, d->p, T, K, keep) == 0) {
    const double scale = (double)drop_scale(d->p);
    for (int64_t e = 0; e < T * K; ++e) {
      (*Xl)[e] = (double)orc_bf16_to_f32(xd[e]);
      (*g)[e] = keep[e] ? scale : 0.0;
    }
    rc = 0;
  }
  free(xd);
  free(keep);
  if (rc) {
    free(*Xl);
    free(*g);
    *Xl = *g = NULL;
  }
  return rc;
}

/* ---- the method's data types ---- */

static double *widen_bf16(const uint16_t *src, int64_t n) {
  double *d = (double *)xmalloc(sizeof(double) * (size_t)(n > 0 ? n : 1));
  if (!d) return NULL;
  for (int64_t i = 0; i < n; ++i) d[i] = (double)orc_bf16_to_f32(src[i]);
  return d;
}

static double *gather_rows(const double *M, int64_t cols, const int64_t *rows,
                           int64_t n_rows) {
  double *d = (double *)xmalloc(sizeof(double) * (size_t)(n_rows * cols > 0 ? n_rows * cols : 1));
  if (!d) return NULL;
  for (int64_t i = 0; i < n_rows; ++i)
    memcpy(d + i * cols, M + rows[i] * cols, sizeof(double) * (size_t)cols);
  return d;
}

static int lora_args_ok(int64_t N, int64_t K, int64_t T, int r,
                        const int64_t *rows, int64_t n_rows) {
  if (!shape_ok(N, K) || T <= 0 || r <= 0) return 0;
  if (rows) {
    for (int64_t i = 0; i < n_rows; ++i)
      if (rows[i] < 0 || rows[i] >= T) return 0;
  }
  return 1;
}

static int lora_fwd_src(const wsrc *wp, const drop_cfg *drop, int64_t N, int64_t K,
                        const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                        int r, float alpha, const int64_t *rows, int64_t n_rows, float *Y,
                        float *t_out, int n_threads) {
  if (!lora_args_ok(N, K, T, r, rows, n_rows)) return -1;
  if (!rows) n_rows = T;
  const double s = (double)alpha / (double)r;
  const wsrc w = *wp;
  double *Xl = NULL, *g = NULL; /* adapter-branch input after dropout */
  if (drop_inputs(drop, X, T, K, &Xl, &g) != 0) return -1;

  double *Xd = widen_bf16(X, T * K);
  double *Ad = widen_bf16(A, (int64_t)r * K);
  double *Bd = widen_bf16(B, N * r);
  double *t = (double *)xmalloc(sizeof(double) * (size_t)(T * r));
  double *Yd = (double *)xmalloc(sizeof(double) * (size_t)(n_rows * N > 0 ? n_rows * N : 1));
  double *Xs = NULL, *ts = NULL;
  int rc = -1;
  if (!Xd || !Ad || !Bd || !t || !Yd) goto done;
  lora_down(Xl ? Xl : Xd, Ad, T, K, r, t);
  if (rows) {
    Xs = gather_rows(Xd, K, rows, n_rows);
    ts = gather_rows(t, r, rows, n_rows);
    if (!Xs || !ts) goto done;
  }
  {
    fwd_ctx c = {&w, rows ? Xs : Xd, rows ? ts : t, Bd, n_rows, N, K, r, s, Yd};
    parallel_for(N, n_threads, fwd_cols, &c);
  }
  for (int64_t i = 0; i < n_rows * N; ++i) Y[i] = (float)Yd[i];
  if (t_out)
    for (int64_t i = 0; i < T * r; ++i) t_out[i] = (float)t[i];
  rc = 0;
done:
  free(Xl);
  free(g);
  free(Xd);
  free(Ad);
  free(Bd);
  free(t);
  free(Yd);
  free(Xs);
  free(ts);
  return rc;
}

static int lora_bwd_src(const wsrc *wp, const drop_cfg *drop, int64_t N, int64_t K,
                        const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                        int r, float alpha, const uint16_t *dY, const int64_t *rows,
                        int64_t n_rows, float *dX, float *dA, float *dB,
                        int n_threads) {
  if (!lora_args_ok(N, K, T, r, rows, n_rows)) return -1;
  if (!rows) n_rows = T;
  const double s = (double)alpha / (double)r;
  const wsrc w = *wp;
  double *Xl = NULL, *g = NULL, *gs = NULL; /* adapter-branch input, dX multiplier */
  if (drop_inputs(drop, X, T, K, &Xl, &g) != 0) return -1;

  double *Xd = widen_bf16(X, T * K);
  double *Ad = widen_bf16(A, (int64_t)r * K);
  double *Bd = widen_bf16(B, N * r);
  double *dYd = widen_bf16(dY, T * N);
  double *t = (double *)xmalloc(sizeof(double) * (size_t)(T * r));
  double *u = (double *)xmalloc(sizeof(double) * (size_t)(T * r));
  double *dXd = (double *)xmalloc(sizeof(double) * (size_t)(n_rows * K > 0 ? n_rows * K : 1));
  double *dAd = (double *)xmalloc(sizeof(double) * (size_t)(r * K));
  double *dBd = (double *)xmalloc(sizeof(double) * (size_t)(N * r));
  double *dYs = NULL, *us = NULL;
  int rc = -1;
  if (!Xd || !Ad || !Bd || !dYd || !t || !u || !dXd || !dAd || !dBd) goto done;
  lora_down(Xl ? Xl : Xd, Ad, T, K, r, t);
  lora_up_t(dYd, Bd, T, N, r, u);
  if (rows) {
    dYs = gather_rows(dYd, N, rows, n_rows);
    us = gather_rows(u, r, rows, n_rows);
    if (!dYs || !us) goto done;
    if (g && !(gs = gather_rows(g, K, rows, n_rows))) goto done;
  }
  {
    dx_ctx c = {&w, rows ? dYs : dYd, rows ? us : u, Ad, n_rows, N, K, r, s, dXd,
                rows ? gs : g};
    parallel_for(K, n_threads, dx_cols, &c);
  }
  lora_grads(Xl ? Xl : Xd, dYd, t, u, T, N, K, r, s, dAd, dBd);
  for (int64_t i = 0; i < n_rows * K; ++i) dX[i] = (float)dXd[i];
  for (int64_t i = 0; i < (int64_t)r * K; ++i) dA[i] = (float)dAd[i];
  for (int64_t i = 0; i < N * r; ++i) dB[i] = (float)dBd[i];
  rc = 0;
done:
  free(Xl);
  free(g);
  free(gs);
  free(Xd);
  free(Ad);
  free(Bd);
  free(dYd);
  free(t);
  free(u);
  free(dXd);
  free(dAd);
  free(dBd);
  free(dYs);
  free(us);
  return rc;
}

static wsrc nf4_src(const uint8_t *codes, const float *absmax, int64_t K) {
  wsrc w;
  memset(&w, 0, sizeof w);
  w.codes = codes;
  w.absmax = absmax;
  w.K = K;
  orc_nf4_codebook(w.cb);
  return w;
}

static wsrc bf16_src(const uint16_t *W, int64_t K) {
  wsrc w;
  memset(&w, 0, sizeof w);
  w.wbf16 = W;
  w.K = K;
  return w;
}

int orc_lora_fwd(const uint8_t *codes, const float *absmax, int64_t N,
                 int64_t K, const uint16_t *X, int64_t T, const uint16_t *A,
                 const uint16_t *B, int r, float alpha, const int64_t *rows,
                 int64_t n_rows, float *Y, float *t_out, int n_threads) {
  const wsrc w = nf4_src(codes, absmax, K);
  return lora_fwd_src(&w, NULL, N, K, X, T, A, B, r, alpha, rows, n_rows, Y, t_out, n_threads);
}

int orc_lora_bwd(const uint8_t *codes, const float *absmax, int64_t N,
                 int64_t K, const uint16_t *X, int64_t T, const uint16_t *A,
                 const uint16_t *B, int r, float alpha, const uint16_t *dY,
                 const int64_t *rows, int64_t n_rows, float *dX, float *dA,
                 float *dB, int n_threads) {
  const wsrc w = nf4_src(codes, absmax, K);
  return lora_bwd_src(&w, NULL, N, K, X, T, A, B, r, alpha, dY, rows, n_rows, dX, dA, dB,
                      n_threads);
}

int orc_lora_fwd_bf16w(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X,
                       int64_t T, const uint16_t *A, const uint16_t *B, int r,
                       float alpha, const int64_t *rows, int64_t n_rows, float *Y,
                       float *t_out, int n_threads) {
  const wsrc w = bf16_src(W, K);
  return lora_fwd_src(&w, NULL, N, K, X, T, A, B, r, alpha, rows, n_rows, Y, t_out, n_threads);
}

int orc_lora_bwd_bf16w(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X,
                       int64_t T, const uint16_t *A, const uint16_t *B, int r,
                       float alpha, const uint16_t *dY, const int64_t *rows,
                       int64_t n_rows, float *dX, float *dA, float *dB, int n_threads) {
  const wsrc w = bf16_src(W, K);
  return lora_bwd_src(&w, NULL, N, K, X, T, A, B, r, alpha, dY, rows, n_rows, dX, dA, dB,
                      n_threads);
}

/* ---- merge_and_unload (Poros API reference, PorosModel.merge_and_unload):
 * the adapter folded into the base, W' = deq(W) + (alpha/r) B A, in the
 * compute dtype bf16.  Each element: the exact bf16 value of the base plus
 * the rank-r sum accumulated in double, rounded ONCE to bf16 (nearest,
 * ties to even). ---- */

/* double -> bf16, one rounding (nearest, ties to even).  A double that is
 * not a float first goes to the float of the same sign nearer to zero
 * (truncation), with the discarded part recorded as a sticky bit in the
 * float's last place, so that the float -> bf16 rounding below sees a tie
 * only for values exactly halfway between two bf16 numbers. */
static uint16_t bf16_from_double(double v) {
  if (v != v) return 0x7FC0u;
  float f = (float)v;
  if ((double)f != v && isfinite(f)) {
    /* truncate toward zero, then set the sticky bit */
    if (fabs((double)f) > fabs(v)) f = nextafterf(f, 0.0f);
    uint32_t b;
    memcpy(&b, &f, sizeof b);
    b |= 1u;
    memcpy(&f, &b, sizeof b);
  }
  return orc_f32_to_bf16(f);
}

int orc_lora_merge(const uint8_t *codes, const float *absmax, const uint16_t *Wbf16,
                   int64_t N, int64_t K, const uint16_t *A, const uint16_t *B, int r,
                   float alpha, uint16_t *out) {
  if (!shape_ok(N, K) || r <= 0 || (!Wbf16 && (!codes || !absmax))) return -1;
  const double s = (double)alpha / (double)r;
  wsrc w = Wbf16 ? bf16_src(Wbf16, K) : nf4_src(codes, absmax, K);
  double *row = (double *)xmalloc(sizeof(double) * (size_t)K);
  if (!row) return -1;
  for (int64_t n = 0; n < N; ++n) {
    w_row(&w, n, 0, K, row);
    for (int64_t k = 0; k < K; ++k) {
      double acc = 0.0;
      for (int j = 0; j < r; ++j)
        acc += (double)orc_bf16_to_f32(B[n * r + j]) * (double)orc_bf16_to_f32(A[(int64_t)j * K + k]);
      out[n * K + k] = bf16_from_double(row[k] + s * acc);
    }
  }
  free(row);
  return 0;
}

/* The NF4 LoRA linear with dropout p (seed, offset) on the adapter branch:
 *   X_d = dropout(X);  t = X_d A^T;  Y = X W^T + s t B^T
 *   u = dY B;  dX = dY W + (s u A) * keep * scale;  dB = s dY^T t;  dA = s u^T X_d
 * p = 0 gives exactly orc_lora_fwd / orc_lora_bwd. */
int orc_lora_fwd_drop(const uint8_t *codes, const float *absmax, int64_t N, int64_t K,
                      const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                      int r, float alpha, float p, uint64_t seed, uint64_t offset,
                      const int64_t *rows, int64_t n_rows, float *Y, float *t_out,
                      int n_threads) {
  const wsrc w = nf4_src(codes, absmax, K);
  const drop_cfg d = {p, seed, offset};
  return lora_fwd_src(&w, &d, N, K, X, T, A, B, r, alpha, rows, n_rows, Y, t_out, n_threads);
}

int orc_lora_bwd_drop(const uint8_t *codes, const float *absmax, int64_t N, int64_t K,
                      const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                      int r, float alpha, float p, uint64_t seed, uint64_t offset,
                      const uint16_t *dY, const int64_t *rows, int64_t n_rows, float *dX,
                      float *dA, float *dB, int n_threads) {
  const wsrc w = nf4_src(codes, absmax, K);
  const drop_cfg d = {p, seed, offset};
  return lora_bwd_src(&w, &d, N, K, X, T, A, B, r, alpha, dY, rows, n_rows, dX, dA, dB,
                      n_threads);
}

/* ======================================================================
 * Decoder-layer glue around the seven projections (the pages train LoRA
 * on Qwen2.5 / Llama-3.1 decoder layers and rematerialize each block in
 * the backward -- Poros on consumer GPUs, "OOM playbook": activation
 * memory at the rematerialization boundary).  Plain double arithmetic,
 * row-major tensors; these are the textbook definitions.
 * ====================================================================== */

/* RMSNorm: y[t,i] = x[t,i] * g[i] / sqrt(mean_i x[t,i]^2 + eps) */
void orc_rmsnorm_fwd(const double *x, const double *g, int64_t T, int64_t n, double eps,
                     double *y) {
  for (int64_t t = 0; t < T; ++t) {
    double ss = 0.0;
    for (int64_t i = 0; i < n; ++i) ss += x[t * n + i] * x[t * n + i];
    const double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int64_t i = 0; i < n; ++i) y[t * n + i] = x[t * n + i] * r * g[i];
  }
}

/* dx of RMSNorm (g frozen): with r = (mean x^2 + eps)^-1/2 and w = g * dy,
 * dx_i = r w_i - r^3 x_i (sum_j w_j x_j) / n */
void orc_rmsnorm_bwd(const double *x, const double *g, const double *dy, int64_t T,
                     int64_t n, double eps, double *dx) {
  for (int64_t t = 0; t < T; ++t) {
    double ss = 0.0, wx = 0.0;
    for (int64_t i = 0; i < n; ++i) {
      ss += x[t * n + i] * x[t * n + i];
      wx += g[i] * dy[t * n + i] * x[t * n + i];
    }
    const double r = 1.0 / sqrt(ss / (double)n + eps);
    for (int64_t i = 0; i < n; ++i)
      dx[t * n + i] = r * g[i] * dy[t * n + i] - r * r * r * x[t * n + i] * wx / (double)n;
  }
}

/* SwiGLU gate: m = silu(a) * b, silu(a) = a / (1 + e^-a) */
static double silu_d(double a) { return a / (1.0 + exp(-a)); }

void orc_silu_mul_fwd(const double *a, const double *b, int64_t n, double *m) {
  for (int64_t i = 0; i < n; ++i) m[i] = silu_d(a[i]) * b[i];
}

/* da = dm * b * silu'(a), silu'(a) = s (1 + a (1 - s)), s = 1/(1+e^-a); db = dm * silu(a) */
void orc_silu_mul_bwd(const double *a, const double *b, const double *dm, int64_t n,
                      double *da, double *db) {
  for (int64_t i = 0; i < n; ++i) {
    const double s = 1.0 / (1.0 + exp(-a[i]));
    da[i] = dm[i] * b[i] * s * (1.0 + a[i] * (1.0 - s));
    db[i] = dm[i] * a[i] * s;
  }
}

/* Causal scaled dot-product attention with grouped KV heads.
 * q [T, H*d], k and v [T, KV*d] (head h reads KV head h / (H/KV));
 * o [T, H*d]; lse [H, T] = log sum_j exp(scale q_i . k_j) over j <= i. */
void orc_attention_fwd(const double *q, const double *k, const double *v, int64_t T, int H,
                       int KV, int d, double scale, double *o, double *lse) {
  const int grp = H / KV;
  double *p = (double *)xmalloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  if (!p) return;
  for (int h = 0; h < H; ++h) {
    const int kh = h / grp;
    for (int64_t i = 0; i < T; ++i) {
      double mx = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        double s = 0.0;
        for (int c = 0; c < d; ++c)
          s += q[i * H * d + h * d + c] * k[j * KV * d + kh * d + c];
        p[j] = s * scale;
        if (p[j] > mx) mx = p[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        p[j] = exp(p[j] - mx);
        sum += p[j];
      }
      lse[(int64_t)h * T + i] = mx + log(sum);
      for (int c = 0; c < d; ++c) {
        double acc = 0.0;
        for (int64_t j = 0; j <= i; ++j) acc += p[j] * v[j * KV * d + kh * d + c];
        o[i * H * d + h * d + c] = acc / sum;
      }
    }
  }
  free(p);
}

/* Its gradients: with P the attention probabilities,
 *   dV = P^T dO, dP = dO V^T, dS = P * (dP - rowsum(P * dP)),
 *   dQ = scale dS K, dK = scale dS^T Q, summed over the query heads that
 * share a KV head. */
void orc_attention_bwd(const double *q, const double *k, const double *v, const double *dout,
                       int64_t T, int H, int KV, int d, double scale, double *dq, double *dk,
                       double *dv) {
  const int grp = H / KV;
  double *p = (double *)xmalloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  double *dp = (double *)xmalloc(sizeof(double) * (size_t)(T > 0 ? T : 1));
  if (!p || !dp) {
    free(p);
    free(dp);
    return;
  }
  memset(dq, 0, sizeof(double) * (size_t)(T * H * d));
  memset(dk, 0, sizeof(double) * (size_t)(T * KV * d));
  memset(dv, 0, sizeof(double) * (size_t)(T * KV * d));
  for (int h = 0; h < H; ++h) {
    const int kh = h / grp;
    for (int64_t i = 0; i < T; ++i) {
      double mx = -INFINITY;
      for (int64_t j = 0; j <= i; ++j) {
        double s = 0.0;
        for (int c = 0; c < d; ++c)
          s += q[i * H * d + h * d + c] * k[j * KV * d + kh * d + c];
        p[j] = s * scale;
        if (p[j] > mx) mx = p[j];
      }
      double sum = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        p[j] = exp(p[j] - mx);
        sum += p[j];
      }
      double pdp = 0.0;
      for (int64_t j = 0; j <= i; ++j) {
        p[j] /= sum;
        double s = 0.0;
        for (int c = 0; c < d; ++c)
          s += dout[i * H * d + h * d + c] * v[j * KV * d + kh * d + c];
        dp[j] = s;
        pdp += p[j] * s;
      }
      for (int64_t j = 0; j <= i; ++j) {
        const double ds = p[j] * (dp[j] - pdp);
        for (int c = 0; c < d; ++c) {
          dv[j * KV * d + kh * d + c] += p[j] * dout[i * H * d + h * d + c];
          dq[i * H * d + h * d + c] += scale * ds * k[j * KV * d + kh * d + c];
          dk[j * KV * d + kh * d + c] += scale * ds * q[i * H * d + h * d + c];
        }
      }
    }
  }
  free(p);
  free(dp);
}
