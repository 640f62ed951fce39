/*
 * nf4_oracle.h -- CPU oracle for the host-streamed NF4 LoRA hot path.
 *
 * TEST INFRASTRUCTURE ONLY.  This is the plain, slow, obviously correct
 * reference that the CUDA path is checked against.  Only the test suite,
 * the smoke check and the benchmark's CPU-baseline leg may load it.  It
 * shares no code, header, table or constant generator with the CUDA
 * library, and it never calls it.
 *
 * Sources (the web pages this method is documented on):
 *   [P1] "Poros on consumer GPUs", section "What you need besides VRAM":
 *        the frozen base is stored NF4 and lives in host RAM; its size is
 *        fixed by the NF4 storage format (~4 / ~18 / ~40 GB at 7B/32B/72B).
 *   [P2] Poros API reference, PorosTrainer.from_pretrained: quantization
 *        "nf4" = 4-bit NF4 QLoRA; lora_rank 16, lora_alpha 32.
 *   [P3] HN comment (host-RAM base, prefetch-one-ahead ring): the base is
 *        frozen, read and never written, and must only arrive before the
 *        matmul that uses it.
 * The pages give no codebook, block length or formula.  The readings used
 * here (NormalFloat construction, 64-element blocks with an fp32 absmax,
 * nibble order, tie-break, LoRA formulas) are stated next to each function.
 *
 * Parity pins: every function below is pinned by tests that do not re-type
 * its formula (closed forms, exact round trips, brute-force nearest search,
 * permutation/selection closed forms, finite differences).
 */
#ifndef NF4_ORACLE_H
#define NF4_ORACLE_H

#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* NormalFloat-4 codebook: the 16 ascending fp32 values QLoRA (Dettmers et
 * al. 2023) prints in its Appendix E. */
void orc_nf4_codebook(float out[16]);

/* Standard normal quantile by bisection on erfc (double).  Exposed so the
 * tests can compare it to an independent inverse-CDF algorithm and check the
 * published codebook against the construction it comes from. */
double orc_normal_quantile(double p);

/* Index of the codebook entry nearest to x (fp32 distances, ties -> lower). */
int orc_nf4_nearest(float x);

/* Host bytes of one [n_out, k_in] NF4 weight: codes (2 per byte) + fp32
 * absmax per 64-element block. */
int64_t orc_nf4_storage_bytes(int64_t n_out, int64_t k_in);

/* Quantize a row-major bf16 weight [n_out, k_in] (bit patterns).
 * codes: n_out*k_in/2 bytes, element e in byte e/2, even e in the HIGH nibble.
 * absmax: n_out*k_in/64 floats.  Returns 0, or -1 if sizes are invalid. */
int orc_nf4_quantize(const uint16_t *w, int64_t n_out, int64_t k_in,
                     uint8_t *codes, float *absmax);

/* Dequantize to bf16 bit patterns: bf16_rne(fp32(c[code] * absmax)). */
int orc_nf4_dequant(const uint8_t *codes, const float *absmax, int64_t n_out,
                    int64_t k_in, uint16_t *out);

/* float <-> bf16 (round to nearest even), exposed for tests. */
uint16_t orc_f32_to_bf16(float f);
float orc_bf16_to_f32(uint16_t h);

/* ---- LoRA linear, double core (used directly by the finite-difference
 * tests; inputs are dense doubles, W is the dense [N,K] base matrix). ----
 *   t = X A^T                     [T,r]
 *   Y = X W^T + s t B^T           [T,N]
 *   u = dY B                      [T,r]
 *   dX = dY W + s u A             [T,K]
 *   dB = s dY^T t                 [N,r]
 *   dA = s u^T X                  [r,K]
 */
void orc_lora_fwd_f64(const double *W, const double *X, const double *A,
                      const double *B, int64_t T, int64_t N, int64_t K, int r,
                      double s, double *Y, double *t);
void orc_lora_bwd_f64(const double *W, const double *X, const double *A,
                      const double *B, const double *dY, int64_t T, int64_t N,
                      int64_t K, int r, double s, double *dX, double *dA,
                      double *dB);

/* Masked variants of the double core (dropout on the adapter branch):
 * fwd: t = Xl A^T with Xl the adapter branch's input, Y = X W^T + s t B^T;
 * bwd: t = Xl A^T, u = dY B, dX = dY W + (s u A) * g (elementwise; g NULL
 * = 1), dB = s dY^T t, dA = s u^T Xl.  The unmasked functions above are
 * these with Xl = X and g = NULL. */
void orc_lora_fwd_f64m(const double *W, const double *X, const double *Xl,
                       const double *A, const double *B, int64_t T, int64_t N,
                       int64_t K, int r, double s, double *Y, double *t);
void orc_lora_bwd_f64m(const double *W, const double *Xl, const double *g,
                       const double *A, const double *B, const double *dY,
                       int64_t T, int64_t N, int64_t K, int r, double s,
                       double *dX, double *dA, double *dB);

/* ---- counter-based RNG and LoRA dropout ----
 * Philox4x32-10 as published (Salmon et al., SC 2011): out = the 10-round
 * bijection of the 128-bit counter under the 64-bit key. */
void orc_philox4x32_10(const uint32_t ctr[4], const uint32_t key[2], uint32_t out[4]);

/* Dropout mask of a row-major [T,K] input: keep[e] for e = t*K + k, from
 * word e%4 of Philox(ctr = {lo(e/4), hi(e/4), lo(offset), hi(offset)},
 * key = {lo(seed), hi(seed)}): keep <=> (word >> 8) >= floor(p * 2^24).
 * 0 <= p < 1.  Returns 0 or -1. */
int orc_dropout_keep(uint64_t seed, uint64_t offset, float p, int64_t T, int64_t K,
                     uint8_t *keep);

/* X_d = keep ? bf16_rne(fp32(x) * scale) : +0,  scale = fp32(1 / fp32(1 - p)). */
int orc_dropout_apply(const uint16_t *X, int64_t T, int64_t K, uint64_t seed,
                      uint64_t offset, float p, uint16_t *out);

/* ---- LoRA linear on the method's data types ----
 * W given as NF4 codes + absmax; X, A, B, dY as bf16 bit patterns; every
 * input is widened exactly, every sum is accumulated in double and rounded
 * once to fp32.  s = alpha / r.
 * rows/n_rows: the token rows of Y (fwd) or dX (bwd) to compute (NULL = all
 * T rows, in order); outputs are packed [n_rows, N] / [n_rows, K].
 * t_out [T,r], dA [r,K] and dB [N,r] always cover every token.
 * n_threads: worker threads over output rows; results do not depend on it.
 * Returns 0, or -1 on invalid sizes. */
int orc_lora_fwd(const uint8_t *codes, const float *absmax, int64_t N,
                 int64_t K, const uint16_t *X, int64_t T, const uint16_t *A,
                 const uint16_t *B, int r, float alpha, const int64_t *rows,
                 int64_t n_rows, float *Y, float *t_out, int n_threads);
int orc_lora_bwd(const uint8_t *codes, const float *absmax, int64_t N,
                 int64_t K, const uint16_t *X, int64_t T, const uint16_t *A,
                 const uint16_t *B, int r, float alpha, const uint16_t *dY,
                 const int64_t *rows, int64_t n_rows, float *dX, float *dA,
                 float *dB, int n_threads);

/* The NF4 LoRA linear with dropout p under (seed, offset) on the adapter
 * branch (Poros API reference, lora_dropout):
 *   X_d = dropout(X);  t = X_d A^T;  Y = X deq(W)^T + s t B^T;
 *   u = dY B;  dX = dY deq(W) + (s u A) * keep * scale;
 *   dB = s dY^T t;  dA = s u^T X_d.
 * Conventions as orc_lora_fwd / orc_lora_bwd (which are p = 0). */
int orc_lora_fwd_drop(const uint8_t *codes, const float *absmax, int64_t N, int64_t K,
                      const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                      int r, float alpha, float p, uint64_t seed, uint64_t offset,
                      const int64_t *rows, int64_t n_rows, float *Y, float *t_out,
                      int n_threads);
int orc_lora_bwd_drop(const uint8_t *codes, const float *absmax, int64_t N, int64_t K,
                      const uint16_t *X, int64_t T, const uint16_t *A, const uint16_t *B,
                      int r, float alpha, float p, uint64_t seed, uint64_t offset,
                      const uint16_t *dY, const int64_t *rows, int64_t n_rows, float *dX,
                      float *dA, float *dB, int n_threads);

/* The same forward / backward with a dense bf16 base W [N,K] (bf16 bit
 * patterns) in place of NF4 -- the quantization="bf16_bitwise" base of the
 * Poros API reference.  Same conventions and returns as above. */
int orc_lora_fwd_bf16w(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X,
                       int64_t T, const uint16_t *A, const uint16_t *B, int r,
                       float alpha, const int64_t *rows, int64_t n_rows, float *Y,
                       float *t_out, int n_threads);
int orc_lora_bwd_bf16w(const uint16_t *W, int64_t N, int64_t K, const uint16_t *X,
                       int64_t T, const uint16_t *A, const uint16_t *B, int r,
                       float alpha, const uint16_t *dY, const int64_t *rows,
                       int64_t n_rows, float *dX, float *dA, float *dB, int n_threads);

/* merge_and_unload: out[n,k] = bf16_rne(deq(W)[n,k] + (alpha/r) sum_j B[n,j]
 * A[j,k]), the sum in double, ONE rounding to bf16.  The base is NF4
 * (codes, absmax; Wbf16 NULL) or dense bf16 (Wbf16 [N,K]; codes, absmax
 * ignored).  A bf16 [r,K], B bf16 [N,r], out bf16 [N,K].  0 or -1. */
int orc_lora_merge(const uint8_t *codes, const float *absmax, const uint16_t *Wbf16,
                   int64_t N, int64_t K, const uint16_t *A, const uint16_t *B, int r,
                   float alpha, uint16_t *out);

/* ---- decoder-layer glue (double, row-major; textbook definitions) ---- */
/* RMSNorm y = x g / sqrt(mean x^2 + eps) over rows of n; and its dx (g frozen). */
void orc_rmsnorm_fwd(const double *x, const double *g, int64_t T, int64_t n, double eps,
                     double *y);
void orc_rmsnorm_bwd(const double *x, const double *g, const double *dy, int64_t T,
                     int64_t n, double eps, double *dx);
/* SwiGLU gate m = silu(a) b, and its gradients. */
void orc_silu_mul_fwd(const double *a, const double *b, int64_t n, double *m);
void orc_silu_mul_bwd(const double *a, const double *b, const double *dm, int64_t n,
                      double *da, double *db);
/* Causal SDPA, H query heads sharing KV heads in groups of H/KV: q [T,H*d],
 * k, v [T,KV*d], o [T,H*d], lse [H,T]; and its gradients. */
void orc_attention_fwd(const double *q, const double *k, const double *v, int64_t T, int H,
                       int KV, int d, double scale, double *o, double *lse);
void orc_attention_bwd(const double *q, const double *k, const double *v, const double *dout,
                       int64_t T, int H, int KV, int d, double scale, double *dq, double *dk,
                       double *dv);

#ifdef __cplusplus
}
#endif
#endif
