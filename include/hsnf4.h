/*
 * hsnf4.h -- C ABI of libhsnf4.so: host-streamed NF4 LoRA layers for B200
 * (sm_100a).
 *
 * The method (from the Poros documentation pages and an HN comment by the
 * author of a similar trainer):
 *   - LoRA fine-tuning keeps the base weights frozen: they are read, never
 *     written, so they need not live in VRAM; they only have to arrive
 *     before the matmul that uses them (HN comment, "host-RAM base,
 *     prefetch-one-ahead ring").
 *   - The base is stored as 4-bit NF4 (Poros API reference,
 *     PorosTrainer.from_pretrained, quantization="nf4") in pinned host RAM
 *     ("Poros on consumer GPUs", "What you need besides VRAM") and streams
 *     into a small pool of pre-allocated VRAM buffers, block_size decoder
 *     layers at a time, one block ahead, on a dedicated copy stream
 *     (HN comment; Poros API reference, block_size / enable_prefetch).
 *   - Every targeted projection is a LoRA linear (rank r, alpha; Poros API
 *     reference, lora_rank / lora_alpha):
 *        Y  = X deq(W)^T + (alpha/r) (X A^T) B^T
 *        dX = dY deq(W) + (alpha/r) (dY B) A
 *        dB = (alpha/r) dY^T (X A^T),   dA = (alpha/r) (dY B)^T X
 *
 * Conventions for every entry point:
 *   - All tensors are row-major and contiguous.  bf16 tensors are passed as
 *     raw 16-bit storage (void*).  Pointers are DEVICE pointers unless a
 *     parameter says "host".  Device pointers must be 16-byte aligned.
 *   - `stream` is a cudaStream_t passed as void*; NULL means the legacy
 *     default stream.  Work is enqueued asynchronously on it; results are
 *     valid once the stream has reached that point.
 *   - The caller owns every buffer (weights, activations, workspace, the
 *     pinned slab, the ring).  The library allocates no device memory on
 *     any call; it owns only CUDA events and the streamer's host state.
 *   - Calls never throw.  They return an hsnf4_status; on failure a
 *     human-readable detail (with the offending sizes) is kept per thread
 *     and read with hsnf4_last_error().  Arguments are validated before
 *     anything is enqueued, so a rejected call has no device side effect.
 *   - Kernels never spin without bound: every pipeline wait gives up after
 *     a time limit, records a flag on the device and returns.  Read and
 *     clear those flags with hsnf4_device_status().
 *   - Results are deterministic: no floating-point atomics, fixed
 *     reduction orders, no dependence on buffer addresses.
 *
 * NF4 storage format (the reading fixed once for this library; the pages
 * name the type but print no layout):
 *   - W is [n_out, k_in] row-major; flat index e = n*k_in + k.
 *   - 64-element blocks along e, one fp32 absmax per block:
 *     absmax[n_out*k_in/64].  k_in must be a multiple of 64, so a block
 *     never crosses a row.
 *   - 4-bit codes, two per byte: codes[n_out*k_in/2]; element e is in byte
 *     e/2, even e in the HIGH nibble.
 *   - code i means the i-th entry of the 16-value NormalFloat codebook
 *     (nf4_codebook()); value = bf16_rne(fp32(codebook[i] * absmax)).
 *   - 0.5625 byte/param, which reproduces the host footprints of
 *     "What you need besides VRAM" (~4 / ~18 / ~40 GB at 7B / 32B / 72B).
 */
#ifndef HSNF4_H
#define HSNF4_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  HSNF4_OK = 0,
  HSNF4_ERR_INVALID = 1, /* bad argument (size, pointer, alignment, rank) */
  HSNF4_ERR_OOM = 2,     /* a caller-provided buffer is too small */
  HSNF4_ERR_CUDA = 3,    /* a CUDA runtime call failed (detail names it) */
  HSNF4_ERR_TIMEOUT = 4, /* a bounded host wait ran out */
  HSNF4_ERR_STATE = 5,   /* streamer protocol misuse */
  HSNF4_ERR_DEVICE = 6   /* a kernel recorded a failed (timed-out) wait */
} hsnf4_status;

/* Formats of the frozen base weight (Poros API reference, the
 * `quantization` knob: "nf4", the default, and "bf16_bitwise", the dense
 * 16-bit base that still streams and keeps bitwise resident parity). */
#define HSNF4_BASE_NF4 0  /* codes + absmax, 0.5625 bytes per weight */
#define HSNF4_BASE_BF16 1 /* dense bf16, 2 bytes per weight */

/* One frozen base weight as the kernels consume it (device pointers).
 * format HSNF4_BASE_NF4 (0, what a zero-initialised struct holds): codes
 * and absmax as below.  format HSNF4_BASE_BF16: codes points to the dense
 * bf16 [n_out, k_in] row-major weight and absmax must be NULL.  Every LoRA
 * entry point takes either format; a group call takes one format for all
 * its problems. */
typedef struct {
  const void *codes;    /* NF4: uint8 [n_out*k_in/2]; BF16: bf16 [n_out, k_in] */
  const float *absmax;  /* NF4: fp32 [n_out*k_in/64]; BF16: NULL */
  int64_t n_out, k_in;
  int32_t format;       /* HSNF4_BASE_NF4 or HSNF4_BASE_BF16 */
  int32_t reserved;     /* 0 */
} hsnf4_nf4_weight;

/* ----------------------------------------------------------------------- */
/* errors and diagnostics                                                  */
/* ----------------------------------------------------------------------- */

/* Static string for a status code. */
const char *hsnf4_status_string(int status);

/* Copy this thread's last error detail into buf (NUL-terminated, truncated
 * to n bytes).  Returns the status of that last failed call (0 if none). */
int hsnf4_last_error(char *buf, size_t n);

/* Synchronize `stream`, then read and clear the device-side failure flags
 * that bounded waits in the kernels record (bit set = a wait gave up; in
 * the fused GEMM, 0x80 = a K-split arrival count that did not settle, which
 * leaves that tile's output unwritten).  *flags (host) receives the flags;
 * returns HSNF4_ERR_DEVICE if any was set. */
int hsnf4_device_status(void *stream, uint32_t *flags);

/* Self-test of the kernels' bounded waits: launches one CTA whose thread
 * waits on a shared-memory barrier that nothing arrives at, through the same
 * bounded wait the pipeline kernels use.  The wait gives up after its time
 * limit (about 2 s), records flag 0x40 and the kernel returns; the context
 * stays usable.  Read the flag with hsnf4_device_status(). */
int hsnf4_selftest_stall(void *stream);

/* Kernel timing for roofline reports.  While enabled, the library brackets
 * every launch of the enabled kernel kinds with CUDA events on the launch
 * stream, and accumulates per kind: launches, device time and algorithmic
 * work (FLOPs for the fused GEMM; bytes read + written for the dequant and
 * the merge; distinct activation bytes read for the rank-r projection and
 * gradient kernels).  Kinds, by bit: 0 lora_gemm_fwd, 1 lora_gemm_dx,
 * 2 nf4_dequant, 3 lora_merge, 4 lora_project, 5 lora_grad.
 * hsnf4_profile(1) starts (and clears) timing of every kind,
 * hsnf4_profile_kinds(mask) of the kinds whose bits are set (events between
 * launches delay the next launch, so timing fewer kinds disturbs a run
 * less), hsnf4_profile(0) stops.  hsnf4_profile_read synchronizes on the
 * recorded events and fills out[0..n) (host), returning the number of
 * entries (<= max_out) or a negative status. */
typedef struct {
  char name[32];        /* the kind's name, as listed above */
  uint64_t launches;
  double total_ms;      /* sum of per-launch event durations */
  double work;          /* total algorithmic FLOPs or bytes */
} hsnf4_kernel_time;

int hsnf4_profile(int enable);
int hsnf4_profile_kinds(unsigned int kinds);
int hsnf4_profile_read(hsnf4_kernel_time *out, int max_out);

/* Number of kernels this library has launched in this process (every
 * entry point counts each launch it makes, on any device or stream).  Read
 * it before and after a region to count the region's launches.  The method
 * has no counterpart to it; it is a measurement aid. */
uint64_t hsnf4_kernel_launches(void);

/* Host-side fault injection for failure-path tests: the next call that
 * reaches `site` fails with HSNF4_ERR_CUDA without calling CUDA.  Sites:
 * "copy_enqueue" (the streamer's H2D copy), "event_record" (streamer event
 * records).  NULL or "" clears.  Nothing is injected on the device. */
int hsnf4_inject_fault(const char *site);

/* ----------------------------------------------------------------------- */
/* NF4 quantize / dequantize                                               */
/* ----------------------------------------------------------------------- */

/* The 16 fp32 codebook values the kernels use, ascending (host out[16]):
 * the NormalFloat-4 data type exactly as QLoRA (Dettmers et al. 2023)
 * prints it in Appendix E -- standard-normal quantiles at probabilities
 * evenly spaced from 1 - (1/32 + 1/30)/2 down to 1/2 (8 positive, 7
 * negative, plus 0), divided by the largest.  Codes and dequantized values
 * are therefore those of any NF4 implementation that uses the published
 * table.  Errors: INVALID if out is NULL. */
int nf4_codebook(float *out);

/* Quantize + pack a bf16 weight (Poros API reference: quantization="nf4").
 * w_bf16 [n_out, k_in] -> codes [n_out*k_in/2], absmax [n_out*k_in/64].
 * Per block: absmax = max|w| (exact), x = w / absmax (IEEE fp32 division),
 * code = nearest codebook entry by fp32 |x - c_i| (ties -> lower index);
 * an all-zero block gets absmax 0 and code 7 (the 0.0 entry).
 * Errors: INVALID if n_out < 1, k_in < 1, k_in % 64, null or misaligned
 * pointers.  Non-finite inputs give unspecified codes. */
int nf4_quantize_pack(const void *w_bf16, int64_t n_out, int64_t k_in,
                      void *codes, float *absmax, void *stream);

/* Dequantize NF4 to bf16: out[e] = bf16_rne(fp32(codebook[code[e]] *
 * absmax[e/64])), bit-exact by construction.  Same errors as above. */
int nf4_dequant(const void *codes, const float *absmax, int64_t n_out,
                int64_t k_in, void *w_bf16_out, void *stream);

/* Merge the adapter into the base (Poros API reference,
 * PorosModel.merge_and_unload): W' = deq(W) + s B A, s = alpha / r, each
 * element computed in fp32 (the rank-r sum on the tensor cores, then
 * scaled, added to the bf16 value of deq(W)) and rounded once to bf16.
 * W: NF4 or BF16 base [n_out, k_in]; A bf16 [r, k_in]; B bf16 [n_out, r];
 * W_out bf16 [n_out, k_in] (may not alias the inputs).  Rank limits as for
 * the LoRA linear below.  Errors: INVALID (sizes, rank, pointers). */
int lora_merge(const hsnf4_nf4_weight *W, const void *A, const void *B, int r,
               float alpha, void *W_out, void *stream);

/* ----------------------------------------------------------------------- */
/* LoRA linear forward / backward (north of the ring: weights may live in  */
/* a ring slot or in a resident buffer -- the result is bitwise the same)  */
/* ----------------------------------------------------------------------- */

/* Limits: 8 <= r <= 64 and r % 8 == 0; 1 <= T <= 32768; n_out, k_in
 * multiples of 64.  alpha is any finite float; the scale is s = alpha / r
 * (fp32).  Workspace needs depend on the shapes and the device's SM count. */

/* Workspace bytes lora_linear_fwd needs for these sizes. */
size_t lora_linear_fwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r);

/* Forward of one LoRA linear (fused NF4 dequant + tcgen05 GEMM, the rank-r
 * term added as an extra K-slice of the same tensor-core accumulation):
 *   t = X A^T (fp32, written to t_save if not NULL)
 *   Y = X deq(W)^T + s t B^T   (fp32 accumulate, bf16 out)
 * W: NF4 weight [n_out, k_in];  X bf16 [T, k_in];  A bf16 [r, k_in];
 * B bf16 [n_out, r];  Y bf16 [T, n_out];  t_save fp32 [T, r] or NULL.
 * workspace: device scratch of >= lora_linear_fwd_workspace() bytes,
 * 256-byte aligned, free after the stream passes the call; its contents on
 * entry do not matter (the only words read before this call writes them
 * are the K-split arrival counters, which each launch tags with a fresh
 * 56-bit value, so a never-written word counts as empty, and which a
 * completed launch leaves at 0, so a replayed graph finds them empty too;
 * after a device-side wait timeout, capture such a graph again).  Errors: INVALID (sizes, rank, pointers), OOM
 * (workspace too small; detail gives needed vs given). */
int lora_linear_fwd(const hsnf4_nf4_weight *W, const void *X, int64_t T,
                    const void *A, const void *B, int r, float alpha, void *Y,
                    float *t_save, void *workspace, size_t ws_bytes,
                    void *stream);

/* The same forward for callers that cannot allocate device memory (a
 * runtime that reserves its whole device-memory budget at start-up and
 * forbids later allocations, a plugin or callback that may not call the
 * allocator): no workspace argument; the scratch is a 64 MiB array compiled
 * into the library, which every GPU that loads the library holds until the
 * process exits.  The method has no counterpart to this entry point; it
 * is a convenience of this library.
 *   - Sizes whose scratch need (lora_linear_fwd_workspace) exceeds 64 MiB
 *     are rejected with HSNF4_ERR_INVALID before anything touches the GPU.
 *   - It allocates nothing: no cudaMalloc, no cudaFree, no allocating
 *     library routine.  The first call on each device looks up the array's
 *     device address (cudaGetSymbolAddress, with that device current) and
 *     caches it for the device's current context; make that first call
 *     before any stream capture.  A later context on the device (after
 *     cudaDeviceReset, for one) looks the address up again on its first
 *     call, which then likewise belongs before any capture.
 *   - All calls share the one array, which keeps the last call's contents.
 *     Nothing in it needs clearing (as for lora_linear_fwd's workspace).
 *     Calls whose GPU work overlaps -- other streams, other host threads --
 *     race on it; serialize them.
 * Arguments, results and errors are otherwise those of lora_linear_fwd. */
int lora_linear_fwd_noalloc(const hsnf4_nf4_weight *W, const void *X, int64_t T,
                            const void *A, const void *B, int r, float alpha, void *Y,
                            float *t_save, void *stream);

/* Workspace bytes lora_linear_bwd needs for these sizes. */
size_t lora_linear_bwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r);

/* Backward of one LoRA linear; W is only read:
 *   u  = dY B                         (fp32)
 *   dX = dY deq(W) + s u A            (bf16 out, fp32 accumulate)
 *   dB = s dY^T t,   dA = s u^T X     (fp32 out, overwritten)
 * t_save: fp32 [T, r] from lora_linear_fwd (t = X A^T).  dY bf16 [T, n_out],
 * dX bf16 [T, k_in], dA fp32 [r, k_in], dB fp32 [n_out, r].
 * Errors as for lora_linear_fwd. */
int lora_linear_bwd(const hsnf4_nf4_weight *W, const void *X,
                    const float *t_save, int64_t T, const void *A,
                    const void *B, int r, float alpha, const void *dY,
                    void *dX, float *dA, float *dB, void *workspace,
                    size_t ws_bytes, void *stream);

/* Grouped forms: n (1..8) independent LoRA linears that share T, r and
 * alpha, run as ONE rank-r projection pass, ONE persistent fused-GEMM
 * launch whose CTAs take the group's tiles longest-first (with a K split,
 * reduced in fixed order, for problems whose tiles are few and long), and
 * in the backward ONE adapter-gradient launch.  A problem's K split (and so
 * its fp32 summation order) depends on the whole group's shapes and the
 * device's SM count, so its result can differ from the single-problem call
 * in the last bits; it never depends on timing or on buffer addresses.  Per
 * problem the arguments mean exactly what they mean for lora_linear_fwd /
 * lora_linear_bwd. */
typedef struct {
  hsnf4_nf4_weight W;
  const void *X;   /* bf16 [T, k_in] */
  const void *A;   /* bf16 [r, k_in] */
  const void *B;   /* bf16 [n_out, r] */
  void *Y;         /* bf16 [T, n_out] */
  float *t_save;   /* fp32 [T, r] or NULL */
  /* LoRA dropout on the adapter branch (Poros API reference, lora_dropout):
   * t = dropout(X) A^T.  p in [0, 1), 0 = none (a zero-initialised struct
   * has none).  The mask of X[t, k] comes from Philox4x32-10 keyed by
   * dropout_seed at counter {(t*k_in + k)/4, dropout_offset}: word
   * (t*k_in + k) % 4 kept iff its top 24 bits >= floor(p * 2^24); kept
   * values are bf16_rne(x * fp32(1 / (1 - p))).  The backward of the same
   * step must pass the same seed and offset (it recomputes the mask). */
  float dropout_p;
  uint32_t reserved;
  uint64_t dropout_seed;
  uint64_t dropout_offset;
} hsnf4_lora_fwd_args;

typedef struct {
  hsnf4_nf4_weight W;
  const void *X;        /* bf16 [T, k_in] */
  const float *t_save;  /* fp32 [T, r] */
  const void *A;        /* bf16 [r, k_in] */
  const void *B;        /* bf16 [n_out, r] */
  const void *dY;       /* bf16 [T, n_out] */
  void *dX;             /* bf16 [T, k_in] */
  float *dA;            /* fp32 [r, k_in] */
  float *dB;            /* fp32 [n_out, r] */
  /* dropout as in the forward (same p, seed, offset): dA = s u^T dropout(X)
   * and dX's adapter term is (s u A) * keep / (1 - p), added in fp32 to the
   * bf16 dY deq(W) and rounded again (two roundings of dX when p > 0). */
  float dropout_p;
  uint32_t reserved;
  uint64_t dropout_seed;
  uint64_t dropout_offset;
} hsnf4_lora_bwd_args;

/* The dropout of the adapter branch on its own: X_d = dropout(X) as defined
 * at hsnf4_lora_fwd_args (X, X_d bf16 [T, k_in], k_in a multiple of 64,
 * 0 <= p < 1).  The grouped calls apply it internally; this entry point
 * exposes the mask for checking and reuse.  Errors: INVALID. */
int lora_dropout_apply(const void *X, int64_t T, int64_t k_in, float p, uint64_t seed,
                       uint64_t offset, void *X_d, void *stream);

/* Workspace bytes of a grouped call (depends on the shapes, on which
 * problems use dropout and on the current device's SM count). */
size_t lora_group_fwd_workspace(const hsnf4_lora_fwd_args *probs, int n, int64_t T, int r);
size_t lora_group_bwd_workspace(const hsnf4_lora_bwd_args *probs, int n, int64_t T, int r);

int lora_group_fwd(const hsnf4_lora_fwd_args *probs, int n, int64_t T, int r, float alpha,
                   void *workspace, size_t ws_bytes, void *stream);

/* The fused GEMM's work plan for a group, built exactly as a launch builds
 * it, from the shapes alone (host only; no device memory, no GPU needed):
 * n problems of n_out[i] x k_in[i] weights at T tokens and rank r, mode 0
 * (forward; contraction k_in) or 1 (dX; contraction n_out).  A plan cuts the
 * 256-row x up-to-512-token tiles' K ranges (64-step units) into pieces
 * spread over CTA pairs: longest-first over uniform splits, or stream-K
 * (equal shares of all K steps per pair).  `covered` is 1 when every tile's
 * K range is covered once by pieces in order.  A split tile's pieces are
 * added in split order either by the last of them to finish, inside the
 * kernel (when every piece has later work in its pair to overlap with:
 * `fixup_tiles`), or by a reduce pass after it.  Errors: INVALID. */
typedef struct {
  int32_t stream_k;        /* 1: stream-K plan; 0: longest-first over uniform K splits */
  int32_t pairs;           /* CTA pairs given work */
  int32_t units;           /* work units (K pieces) */
  int32_t split_tiles;     /* tiles cut into several pieces (each piece writes a partial) */
  int64_t total_steps;     /* 64-wide K steps over all units */
  int64_t max_pair_steps;  /* the most K steps any pair runs */
  int64_t min_pair_steps;
  int32_t covered;
  int32_t fixup_tiles;     /* split tiles whose pieces are added inside the kernel */
} hsnf4_gemm_plan_info;

int hsnf4_gemm_plan(int mode, const int64_t *n_out, const int64_t *k_in, int n, int64_t T,
                    int r, hsnf4_gemm_plan_info *out);
int lora_group_bwd(const hsnf4_lora_bwd_args *probs, int n, int64_t T, int r, float alpha,
                   void *workspace, size_t ws_bytes, void *stream);

/* ----------------------------------------------------------------------- */
/* Decoder-layer glue around the projections                               */
/* ----------------------------------------------------------------------- */
/* The pages train LoRA on Qwen2.5 / Llama-3.1 decoder layers and recompute
 * each block's forward inside its backward (Poros on consumer GPUs, "OOM
 * playbook": activation memory at the rematerialization boundary; Poros API
 * reference, patch_hf_model).  These are the layer's other pieces: pre-norm
 * RMSNorm, causal grouped-query SDPA (head_dim 128, no rotary embedding),
 * the SwiGLU gate and the residual adds.  Tensors are row-major bf16 [T, n]
 * device arrays, 16-byte aligned, n a multiple of 8; every output is rounded
 * once to bf16 from fp32 arithmetic; results do not depend on timing.
 * Errors: INVALID (sizes, pointers), CUDA. */

/* y = x g / sqrt(mean x^2 + eps) per row, x = xa, or x = bf16(xa + xb)
 * (written to h_out) when xb is not NULL -- the residual add fused in front
 * of the norm.  g bf16 [n]. */
int decoder_rmsnorm_fwd(const void *xa, const void *xb, const void *g, void *h_out, void *y,
                        int64_t T, int64_t n, float eps, void *stream);

/* dx = bf16(dres + dRMSNorm/dx . (dy1 + dy2 + dy3)) with x the norm's input
 * (g frozen: no dg); dy2, dy3, dres may be NULL.  The branch gradients are
 * summed in fp32. */
int decoder_rmsnorm_bwd(const void *x, const void *g, const void *dy1, const void *dy2,
                        const void *dy3, const void *dres, void *dx, int64_t T, int64_t n,
                        float eps, void *stream);

/* m = silu(a) b (n elements); da = dm b silu'(a), db = dm silu(a). */
int decoder_swiglu_fwd(const void *a, const void *b, void *m, int64_t n, void *stream);
int decoder_swiglu_bwd(const void *a, const void *b, const void *dm, void *da, void *db,
                       int64_t n, void *stream);

/* out = x + y (n elements; out may alias x or y). */
int decoder_add(const void *x, const void *y, void *out, int64_t n, void *stream);

/* Causal SDPA with H query heads over KV heads (H % KV == 0; head h reads
 * KV head h / (H / KV)), head_dim 128, scale 1/sqrt(128):  q, o [T, H*128],
 * k, v [T, KV*128]; lse fp32 [H, T] (log-sum-exp of the scaled scores, kept
 * for the backward). */
int decoder_attention_fwd(const void *q, const void *k, const void *v, void *o, float *lse,
                          int64_t T, int H, int KV, void *stream);

/* Its gradients from the forward's o and lse:  dq [T, H*128], dk, dv
 * [T, KV*128] (overwritten); scratch: caller-owned device memory of
 * decoder_attention_scratch_bytes(T, H) bytes (the row dots and per-head
 * fp32 partials of dk and dv, added over each KV group in head order). */
size_t decoder_attention_scratch_bytes(int64_t T, int H);
int decoder_attention_bwd(const void *q, const void *k, const void *v, const void *o,
                          const float *lse, const void *dout, void *dq, void *dk, void *dv,
                          float *scratch, int64_t T, int H, int KV, void *stream);

/* ----------------------------------------------------------------------- */
/* Host-pinned NF4 base -> VRAM ring streamer                              */
/* ----------------------------------------------------------------------- */
/* HN comment: the base sits in host RAM and streams into a small pool of
 * pre-allocated VRAM buffers, prefetched one ahead on a dedicated CUDA
 * stream.  Poros API reference: block_size (layers per block, default 4;
 * larger = fewer transfers, more VRAM; never affects parity),
 * enable_prefetch, and the block manager's cross-stream lifetime safety.
 *
 * Layout: a stack is n_layers layers; layer l has n_proj projections.  The
 * pinned slab holds the layers back to back; inside a layer, projection p's
 * codes then its absmax (or its dense bf16 weight), each starting on a
 * 1 KiB boundary (stream_layer_offsets).  A block is block_size consecutive layers (the
 * last block may be shorter) and is one contiguous byte range of the slab.
 * The ring holds n_slots (default 2) block slots in caller-provided device
 * memory.
 *
 * Protocol for block b (prefetch one ahead):
 *   acquire(b) -> prefetch(next) -> compute on b -> release(b)
 * prefetch(b) enqueues the H2D copy of block b on the copy stream after
 * the target slot's previous block was released (the copy stream waits on
 * that release event -- the lifetime fence); acquire(b) makes the compute
 * stream wait for the copy.  A block still resident in a slot is reused
 * without a copy (the turn-around between forward and backward passes)
 * unless reuse is disabled. */

#define HSNF4_MAX_PROJ 8
#define HSNF4_MAX_SLOTS 8

typedef struct {
  int n_proj;
  int64_t n_out[HSNF4_MAX_PROJ];
  int64_t k_in[HSNF4_MAX_PROJ];
  int base_format;  /* HSNF4_BASE_NF4 (0) or HSNF4_BASE_BF16, for every
                       projection of the layer: with BF16 a projection's
                       slab range is its bf16 [n_out, k_in] weight (1 KiB
                       aligned) and acquire returns it with format BF16 */
} hsnf4_layer_desc;

/* Sharded streaming across the GPUs of one node (data-parallel ranks that
 * stream the same stack).  No counterpart in the pages, which describe one
 * GPU: each of `world` ranks copies 1/world of every block over its own
 * PCIe link, then a gather enqueued on the copy stream rebuilds the whole
 * block in every rank's slot over NVLink, so per-GPU PCIe bytes fall
 * world-fold.  Block b of B bytes is cut into world shards of
 * S = round_up(ceil(B / world), 1 KiB) bytes (the last ones shorter or
 * empty); rank j's shard is bytes [j*S, min((j+1)*S, B)) and lands at the
 * same offset of the slot.  The gather callback (block = the block being
 * fetched, for the caller's bookkeeping) is called, with the
 * streamer's lock held, right after this rank's shard copy is enqueued on
 * copy_stream; it must enqueue on copy_stream the in-place all-gather that
 * makes slot[j*S, (j+1)*S) hold rank j's shard for every j (for example
 * NCCL all-gather with sendbuff = slot + rank*S, recvbuff = slot, count S),
 * and return 0, or nonzero on failure (prefetch then fails with
 * HSNF4_ERR_CUDA).  Every rank must make the same prefetch calls in the
 * same order, since each one issues a collective. */
typedef int (*hsnf4_gather_fn)(void *slot, size_t shard_bytes, int world, int block,
                               void *copy_stream, void *user);

typedef struct {
  int block_size;      /* layers per block, >= 1 */
  int enable_prefetch; /* 0: acquire() issues the copy itself (no overlap) */
  int reuse_resident;  /* 1: a prefetch of a block still resident in a slot
                          (in use or released) is satisfied without a copy;
                          0: only a copy not yet acquired satisfies it, so
                          every pass re-streams its blocks */
  int poison_on_release; /* debug: fill a released slot with 0xFF bytes */
  int n_slots;         /* block slots in the ring: 0 (= 2, prefetch one
                          ahead) or 2..HSNF4_MAX_SLOTS; more slots reuse
                          more blocks at each forward/backward turn-around */
  int shard_world;     /* ranks sharing the stream: 0 or 1 = not sharded
                          (unless gather is set: then 1 rank, one shard) */
  int shard_rank;      /* this rank, in [0, shard_world) */
  hsnf4_gather_fn gather; /* required when shard_world >= 2; NULL otherwise */
  void *gather_user;   /* passed to gather */
  int shard_slab;      /* sharded streams only.  0: pinned_slab holds the
                          whole stack; 1: it holds only this rank's shards,
                          block after block, laid out as
                          stream_shard_slab_layout gives -- about 1/world of
                          the stack, so that the node's ranks together pin
                          one copy of the base */
} hsnf4_stream_config;

typedef struct {
  uint64_t h2d_bytes;  /* bytes copied host -> device */
  uint64_t copies;     /* H2D copies issued */
  uint64_t reuses;     /* prefetches satisfied by a resident block */
  uint64_t acquires, releases;
  uint64_t gathers;    /* gather callbacks made (sharded streams) */
} hsnf4_stream_stats;

typedef struct hsnf4_streamer hsnf4_streamer;

/* Bytes of one layer in the slab (multiple of 1 KiB). */
int stream_layer_bytes(const hsnf4_layer_desc *layer, size_t *out_bytes);

/* Byte offsets of projection p's codes and absmax inside its layer (for a
 * BF16 layer: the weight's offset, twice). */
int stream_layer_offsets(const hsnf4_layer_desc *layer, int proj,
                         size_t *codes_off, size_t *absmax_off);

/* Total slab bytes for n_layers layers (host out). */
int stream_slab_bytes(const hsnf4_layer_desc *layers, int n_layers,
                      size_t *out_bytes);

/* Device bytes the default 2-slot ring needs for this stack and block_size. */
int stream_ring_bytes(const hsnf4_layer_desc *layers, int n_layers,
                      int block_size, size_t *out_bytes);

/* Bytes of one block slot (the largest block); a ring of n_slots needs
 * n_slots times this. */
int stream_slot_bytes(const hsnf4_layer_desc *layers, int n_layers,
                      int block_size, size_t *out_bytes);

/* This rank's shard of a block of block_bytes bytes shared by world ranks:
 * *shard_bytes = S (the stride), *off and *len the rank's byte range
 * (len may be 0).  Pure host arithmetic. */
int stream_shard_range(size_t block_bytes, int world, int rank, size_t *shard_bytes,
                       size_t *off, size_t *len);

/* Layout of a shard slab (hsnf4_stream_config.shard_slab): rank `rank`'s
 * shards of every block (stream_shard_range of the block's bytes), packed
 * block after block in block order.  For block >= 0, *block_off and *len
 * (either may be NULL) receive where that block's shard starts in the shard
 * slab and its length; *total_bytes (may be NULL) the size of the whole
 * shard slab.  block = -1 asks for the total only.  Pure host arithmetic.
 * Errors: INVALID (layers, sizes, rank or block out of range). */
int stream_shard_slab_layout(const hsnf4_layer_desc *layers, int n_layers, int block_size,
                             int world, int rank, int block, size_t *block_off, size_t *len,
                             size_t *total_bytes);

/* Bytes of one block slot of a stream sharded over `world` ranks (the
 * largest block rounded up to world * S); a ring of n_slots needs n_slots
 * times this.  world 1 gives stream_slot_bytes rounded up to 1 KiB. */
int stream_slot_bytes_sharded(const hsnf4_layer_desc *layers, int n_layers, int block_size,
                              int world, size_t *out_bytes);

/* Create a streamer.  pinned_slab: HOST pointer to page-locked memory of
 * slab_bytes holding the stack (or, with cfg->shard_slab, this rank's
 * shards of it); ring_dev: device memory of ring_bytes
 * (>= stream_ring_bytes(), 1 KiB aligned); copy_stream: the dedicated H2D
 * stream.  The caller keeps all three alive until stream_destroy.  Errors:
 * INVALID, OOM (ring or slab too small: needed vs given), CUDA. */
int stream_create(const void *pinned_slab, size_t slab_bytes,
                  const hsnf4_layer_desc *layers, int n_layers,
                  const hsnf4_stream_config *cfg, void *ring_dev,
                  size_t ring_bytes, void *copy_stream,
                  hsnf4_streamer **out);

/* Number of blocks (ceil(n_layers / block_size)). */
int stream_num_blocks(const hsnf4_streamer *s);

/* Enqueue block b's H2D copy into a free slot (asynchronous).  STATE if the
 * only candidate slot holds a block that was acquired and not released. */
int stream_block_prefetch(hsnf4_streamer *s, int block);

/* Prefetch along the upcoming visit order (upcoming[0] first): blocks
 * already copied (or, with reuse_resident, in use or still resident) are
 * kept, and the next blocks that are not resident are copied into free
 * slots, evicting the released block needed furthest in the future, until
 * every slot holds a block that is copied, kept or in use.  *issued
 * (optional) receives the number of copies enqueued.  With 2 slots this is
 * prefetch-one-ahead. */
int stream_prefetch_ahead(hsnf4_streamer *s, const int *upcoming, int n, int *issued);

/* Make `compute_stream` wait for block b and return its weights:
 * out[i*n_proj + p] for layer (first layer of b) + i, projection p;
 * max_out must be >= layers_in_block * n_proj.  With enable_prefetch = 0
 * the copy is issued here.  STATE if b is not prefetched. */
int stream_block_acquire(hsnf4_streamer *s, int block, void *compute_stream,
                         hsnf4_nf4_weight *out, int max_out);

/* Host-side bounded wait until block b's copy has landed (polls the ready
 * event); TIMEOUT after timeout_ms.  STATE if b is not prefetched. */
int stream_block_acquire_host(hsnf4_streamer *s, int block, int timeout_ms);

/* Record that compute on block b (enqueued so far on compute_stream) is
 * done with its slot; the slot can be overwritten after that point. */
int stream_block_release(hsnf4_streamer *s, int block, void *compute_stream);

int stream_stats(const hsnf4_streamer *s, hsnf4_stream_stats *out);

/* Destroy (synchronizes the copy stream; events are released). */
int stream_destroy(hsnf4_streamer *s);

#ifdef __cplusplus
}
#endif
#endif
