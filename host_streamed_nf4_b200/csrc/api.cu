// api.cu -- the C ABI of libhsnf4.so: argument validation, error reporting,
// the NF4 codebook, and the launch sequences of the LoRA linear.
#include <math.h>
#include <stdarg.h>
#include <stdio.h>
#include <string.h>

#include <atomic>
#include <mutex>

#include "internal.h"

namespace hsnf4 {

// ---------------------------------------------------------------- errors

static thread_local char t_detail[512] = "";
static thread_local int t_status = HSNF4_OK;

int fail(int status, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(t_detail, sizeof t_detail, fmt, ap);
  va_end(ap);
  t_status = status;
  return status;
}

int cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return HSNF4_OK;
  return fail(HSNF4_ERR_CUDA, "%s: %s (%s)", what, cudaGetErrorName(e), cudaGetErrorString(e));
}

static std::atomic<int> g_fault{kFaultNone};

bool take_fault(FaultSite site) {
  int expected = site;
  return g_fault.compare_exchange_strong(expected, kFaultNone);
}

// ---------------------------------------------------------------- codebook
// NormalFloat-4, the "nf4" type of the Poros API reference: the 16 float32
// values of the data type as QLoRA (Dettmers et al. 2023) prints them in its
// Appendix E, as IEEE-754 bit patterns, code 0 (-1) up to code 15 (+1).  They
// are standard-normal quantiles at evenly spaced probabilities plus an exact
// zero, normalised to [-1, 1] (the paper's "4-bit NormalFloat Quantization").

static const uint32_t kNf4Bits[16] = {
    0xbf800000u, 0xbf3239b1u, 0xbf066b30u, 0xbeca32a0u, 0xbe91a24du, 0xbe3d353fu,
    0xbdba7871u, 0x00000000u, 0x3da2faffu, 0x3e24cae3u, 0x3e7c04ddu, 0x3ead033au,
    0x3ee1a4b8u, 0x3f1007abu, 0x3f3913b3u, 0x3f800000u,
};

const Nf4Codebook& codebook() {
  static const Nf4Codebook cb = [] {
    Nf4Codebook c;
    memcpy(c.v, kNf4Bits, sizeof c.v);
    return c;
  }();
  return cb;
}

}  // namespace hsnf4

using namespace hsnf4;

// ---------------------------------------------------------------- C ABI

extern "C" {

const char* hsnf4_status_string(int status) {
  switch (status) {
    case HSNF4_OK: return "ok";
    case HSNF4_ERR_INVALID: return "invalid argument";
    case HSNF4_ERR_OOM: return "buffer too small";
    case HSNF4_ERR_CUDA: return "CUDA error";
    case HSNF4_ERR_TIMEOUT: return "timed out";
    case HSNF4_ERR_STATE: return "protocol misuse";
    case HSNF4_ERR_DEVICE: return "device wait gave up";
    default: return "unknown status";
  }
}

int hsnf4_last_error(char* buf, size_t n) {
  if (buf && n) {
    strncpy(buf, t_detail, n - 1);
    buf[n - 1] = 0;
  }
  return t_status;
}

int hsnf4_device_status(void* stream, uint32_t* flags) {
  if (!flags) return fail(HSNF4_ERR_INVALID, "hsnf4_device_status: flags is NULL");
  int rc = cuda_status(cudaStreamSynchronize(static_cast<cudaStream_t>(stream)),
                       "hsnf4_device_status: cudaStreamSynchronize");
  if (rc) return rc;
  uint32_t f = 0, fr = 0, fm = 0;
  rc = cuda_status(read_gemm_flags(&f), "hsnf4_device_status: read flags");
  if (!rc) rc = cuda_status(read_rank_flags(&fr), "hsnf4_device_status: read flags");
  if (!rc) rc = cuda_status(read_merge_flags(&fm), "hsnf4_device_status: read flags");
  if (rc) return rc;
  f |= fr | fm;
  *flags = f;
  if (f) return fail(HSNF4_ERR_DEVICE, "a kernel wait gave up (flags 0x%x)", f);
  return HSNF4_OK;
}

int hsnf4_selftest_stall(void* stream) {
  return cuda_status(launch_selftest_stall(static_cast<cudaStream_t>(stream)),
                     "hsnf4_selftest_stall launch");
}

int hsnf4_inject_fault(const char* site) {
  if (!site || !*site) {
    g_fault.store(kFaultNone);
    return HSNF4_OK;
  }
  if (!strcmp(site, "copy_enqueue")) {
    g_fault.store(kFaultCopyEnqueue);
    return HSNF4_OK;
  }
  if (!strcmp(site, "event_record")) {
    g_fault.store(kFaultEventRecord);
    return HSNF4_OK;
  }
  return fail(HSNF4_ERR_INVALID, "hsnf4_inject_fault: unknown site '%s'", site);
}

int nf4_codebook(float* out) {
  if (!out) return fail(HSNF4_ERR_INVALID, "nf4_codebook: out is NULL");
  memcpy(out, codebook().v, sizeof(float) * 16);
  return HSNF4_OK;
}

static int check_nf4_shape(const char* fn, int64_t n_out, int64_t k_in) {
  if (n_out < 1 || k_in < 1 || k_in % 64 != 0)
    return fail(HSNF4_ERR_INVALID,
                "%s: need n_out >= 1 and k_in a positive multiple of 64 (got n_out=%lld, "
                "k_in=%lld)",
                fn, (long long)n_out, (long long)k_in);
  if (n_out > (int64_t(1) << 31) || k_in > (int64_t(1) << 31))
    return fail(HSNF4_ERR_INVALID, "%s: dimension too large", fn);
  return HSNF4_OK;
}

static int check_ptrs(const char* fn, std::initializer_list<std::pair<const void*, const char*>> ps) {
  for (auto& p : ps) {
    if (!p.first) return fail(HSNF4_ERR_INVALID, "%s: %s is NULL", fn, p.second);
    if (!aligned16(p.first))
      return fail(HSNF4_ERR_INVALID, "%s: %s is not 16-byte aligned", fn, p.second);
  }
  return HSNF4_OK;
}

int nf4_quantize_pack(const void* w_bf16, int64_t n_out, int64_t k_in, void* codes,
                      float* absmax, void* stream) {
  int rc = check_nf4_shape("nf4_quantize_pack", n_out, k_in);
  if (rc) return rc;
  rc = check_ptrs("nf4_quantize_pack", {{w_bf16, "w_bf16"}, {codes, "codes"}, {absmax, "absmax"}});
  if (rc) return rc;
  return cuda_status(launch_nf4_quantize(w_bf16, n_out, k_in, codes, absmax,
                                         static_cast<cudaStream_t>(stream)),
                     "nf4_quantize_pack launch");
}

int nf4_dequant(const void* codes, const float* absmax, int64_t n_out, int64_t k_in,
                void* w_bf16_out, void* stream) {
  int rc = check_nf4_shape("nf4_dequant", n_out, k_in);
  if (rc) return rc;
  rc = check_ptrs("nf4_dequant", {{codes, "codes"}, {absmax, "absmax"}, {w_bf16_out, "w_bf16_out"}});
  if (rc) return rc;
  return cuda_status(launch_nf4_dequant(codes, absmax, n_out, k_in, w_bf16_out,
                                        static_cast<cudaStream_t>(stream)),
                     "nf4_dequant launch");
}

// ---------------------------------------------------------------- LoRA linear

static int r_padded(int r) { return (r + 15) / 16 * 16; }

static int check_weight(const char* fn, int i, const hsnf4_nf4_weight& W) {
  if (W.n_out < 64 || W.n_out % 64 || W.k_in < 64 || W.k_in % 64)
    return fail(HSNF4_ERR_INVALID,
                "%s: problem %d: n_out and k_in must be positive multiples of 64 (got %lld x %lld)",
                fn, i, (long long)W.n_out, (long long)W.k_in);
  if (W.n_out > (1 << 30) || W.k_in > (1 << 30))
    return fail(HSNF4_ERR_INVALID, "%s: problem %d: weight dimension too large", fn, i);
  if (W.format == HSNF4_BASE_NF4)
    return check_ptrs(fn, {{W.codes, "W.codes"}, {W.absmax, "W.absmax"}});
  if (W.format == HSNF4_BASE_BF16) {
    if (W.absmax)
      return fail(HSNF4_ERR_INVALID, "%s: problem %d: a BF16 base weight takes absmax = NULL",
                  fn, i);
    return check_ptrs(fn, {{W.codes, "W.codes (bf16 weight)"}});
  }
  return fail(HSNF4_ERR_INVALID, "%s: problem %d: unknown base format %d", fn, i, W.format);
}

// one base format per group (the fused GEMM reads all its problems one way)
static int check_one_format(const char* fn, int n, const int32_t* formats) {
  for (int i = 1; i < n; ++i)
    if (formats[i] != formats[0])
      return fail(HSNF4_ERR_INVALID, "%s: problem %d has base format %d, problem 0 has %d; a "
                  "group takes one format", fn, i, formats[i], formats[0]);
  return HSNF4_OK;
}

static int check_dropout(const char* fn, int i, float p) {
  if (!(p >= 0.0f && p < 1.0f))
    return fail(HSNF4_ERR_INVALID, "%s: problem %d: dropout_p must be in [0, 1) (got %g)", fn, i,
                static_cast<double>(p));
  return HSNF4_OK;
}

static int check_group(const char* fn, int n, int64_t T, int r, float alpha) {
  if (n < 1 || n > 8)
    return fail(HSNF4_ERR_INVALID, "%s: 1..8 problems per call (got %d)", fn, n);
  if (T < 1 || T > 32768)
    return fail(HSNF4_ERR_INVALID, "%s: T must be in [1, 32768] (got %lld)", fn, (long long)T);
  if (r < 8 || r > 64 || r % 8)
    return fail(HSNF4_ERR_INVALID, "%s: rank must be a multiple of 8 in [8, 64] (got %d)", fn, r);
  if (!isfinite(alpha)) return fail(HSNF4_ERR_INVALID, "%s: alpha is not finite", fn);
  return HSNF4_OK;
}

// Workspace layout of a forward group:
//   [s*t bf16 [T, r_pad] per problem][t fp32 [T, r] per problem without t_save]
//   [X_d bf16 [T, k_in] per problem with dropout]
//   [projection partials][GEMM split-K partial tiles]
// Nothing in it needs clearing between calls: every byte a call reads was
// written earlier in the same call, except the GEMM's K-split arrival words,
// which each launch tags with a fresh 56-bit value (a word holding any other
// value counts as no arrivals).
struct FwdLayout {
  size_t zs[8], tscratch[8], xd[8], prj, gemm, total;
};

static void fwd_layout(const hsnf4_lora_fwd_args* p, int n, int64_t T, int r, FwdLayout* L) {
  const int rp = r_padded(r);
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    L->zs[i] = off;
    off += round_up(static_cast<size_t>(T) * rp * 2, 256);
  }
  for (int i = 0; i < n; ++i) {
    L->tscratch[i] = off;
    if (!p[i].t_save) off += round_up(static_cast<size_t>(T) * r * 4, 256);
  }
  for (int i = 0; i < n; ++i) {
    L->xd[i] = off;
    if (p[i].dropout_p > 0.0f) off += round_up(static_cast<size_t>(T) * p[i].W.k_in * 2, 256);
  }
  ProjectDesc pd[8];
  GemmProblemDesc gd[8];
  for (int i = 0; i < n; ++i) {
    // with dropout the projection reads this problem's own X_d: a distinct
    // input, as the launch will see it (only equality of inputs matters here)
    const void* z = p[i].dropout_p > 0.0f ? reinterpret_cast<const void*>(uintptr_t(16) * (i + 1))
                                          : p[i].X;
    pd[i] = {z, p[i].W.k_in, p[i].A, true, nullptr, nullptr};
    gd[i] = {p[i].W.codes, p[i].W.absmax, p[i].W.n_out, p[i].W.k_in, p[i].X, p[i].B, nullptr,
             p[i].Y, p[i].W.format == HSNF4_BASE_BF16};
  }
  L->prj = off;
  off += project_workspace_bytes(pd, n, T, r);
  L->gemm = off;
  off += gemm_workspace_bytes(kGemmFwd, gd, n, T, r);
  L->total = off;
}

// Workspace layout of a backward group:
//   [s*u bf16 [T, r_pad] per problem][u fp32 [T, r] per problem]
//   [u and t as two bf16 parts each, 4 x [T, r_pad] per problem: the
//    adapter-gradient operands]
//   [X_d bf16 [T, k_in] and its keep-mask bytes [T, k_in / 8] per problem
//    with dropout]
//   [projection partials][GEMM split-K partial tiles]
// As for the forward, nothing in it needs clearing between calls.
struct BwdLayout {
  size_t su[8], u[8], parts[8], xd[8], bits[8], prj, gemm, total;
};

static void bwd_layout(const hsnf4_lora_bwd_args* p, int n, int64_t T, int r, BwdLayout* L) {
  const int rp = r_padded(r);
  size_t off = 0;
  for (int i = 0; i < n; ++i) {
    L->su[i] = off;
    off += round_up(static_cast<size_t>(T) * rp * 2, 256);
  }
  for (int i = 0; i < n; ++i) {
    L->u[i] = off;
    off += round_up(static_cast<size_t>(T) * r * 4, 256);
  }
  for (int i = 0; i < n; ++i) {
    L->parts[i] = off;
    off += 4 * round_up(static_cast<size_t>(T) * rp * 2, 256);
  }
  for (int i = 0; i < n; ++i) {
    L->xd[i] = off;
    if (p[i].dropout_p > 0.0f) off += round_up(static_cast<size_t>(T) * p[i].W.k_in * 2, 256);
    L->bits[i] = off;
    if (p[i].dropout_p > 0.0f) off += round_up(static_cast<size_t>(T) * p[i].W.k_in / 8, 256);
  }
  ProjectDesc pd[8];
  GemmProblemDesc gd[8];
  for (int i = 0; i < n; ++i) {
    pd[i] = {p[i].dY, p[i].W.n_out, p[i].B, false, nullptr, nullptr};
    gd[i] = {p[i].W.codes, p[i].W.absmax, p[i].W.n_out, p[i].W.k_in, p[i].dY, p[i].A, nullptr,
             p[i].dX, p[i].W.format == HSNF4_BASE_BF16};
  }
  L->prj = off;
  off += project_workspace_bytes(pd, n, T, r);
  L->gemm = off;
  off += gemm_workspace_bytes(kGemmDx, gd, n, T, r);
  L->total = off;
}

size_t lora_group_fwd_workspace(const hsnf4_lora_fwd_args* probs, int n, int64_t T, int r) {
  if (!probs || n < 1 || n > 8 || T < 1 || r < 1) return 0;
  FwdLayout L;
  fwd_layout(probs, n, T, r, &L);
  return L.total;
}

int hsnf4_gemm_plan(int mode, const int64_t* n_out, const int64_t* k_in, int n, int64_t T,
                    int r, hsnf4_gemm_plan_info* out) {
  if (!n_out || !k_in || !out)
    return fail(HSNF4_ERR_INVALID, "hsnf4_gemm_plan: NULL argument");
  if (mode != 0 && mode != 1)
    return fail(HSNF4_ERR_INVALID, "hsnf4_gemm_plan: mode %d (0 forward, 1 dX)", mode);
  if (n < 1 || n > 8 || T < 1 || r < 1 || r > 64)
    return fail(HSNF4_ERR_INVALID, "hsnf4_gemm_plan: n=%d T=%lld r=%d", n, (long long)T, r);
  GemmProblemDesc d[8] = {};
  for (int i = 0; i < n; ++i) {
    if (n_out[i] < 64 || k_in[i] < 64 || n_out[i] % 64 || k_in[i] % 64)
      return fail(HSNF4_ERR_INVALID, "hsnf4_gemm_plan: problem %d: %lld x %lld", i,
                  (long long)n_out[i], (long long)k_in[i]);
    d[i].n_out = n_out[i];
    d[i].k_in = k_in[i];
  }
  const int rc = check_gemm_tokens(mode == 0 ? kGemmFwd : kGemmDx, T, r);
  if (rc) return rc;
  return gemm_plan_info(mode == 0 ? kGemmFwd : kGemmDx, d, n, T, r, out);
}

size_t lora_group_bwd_workspace(const hsnf4_lora_bwd_args* probs, int n, int64_t T, int r) {
  if (!probs || n < 1 || n > 8 || T < 1 || r < 1) return 0;
  BwdLayout L;
  bwd_layout(probs, n, T, r, &L);
  return L.total;
}

static int check_workspace(const char* fn, void* ws, size_t have, size_t need) {
  if (have < need)
    return fail(HSNF4_ERR_OOM, "%s: workspace too small: need %zu bytes, given %zu", fn, need,
                have);
  if (need && !ws) return fail(HSNF4_ERR_INVALID, "%s: workspace is NULL", fn);
  if ((reinterpret_cast<uintptr_t>(ws) & 255u) != 0)
    return fail(HSNF4_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
  return HSNF4_OK;
}

int lora_group_fwd(const hsnf4_lora_fwd_args* probs, int n, int64_t T, int r, float alpha,
                   void* workspace, size_t ws_bytes, void* stream) {
  static const char* fn = "lora_group_fwd";
  if (!probs) return fail(HSNF4_ERR_INVALID, "%s: probs is NULL", fn);
  int rc = check_group(fn, n, T, r, alpha);
  if (!rc) rc = check_gemm_tokens(kGemmFwd, T, r);
  if (rc) return rc;
  for (int i = 0; i < n; ++i) {
    const hsnf4_lora_fwd_args& p = probs[i];
    rc = check_weight(fn, i, p.W);
    if (!rc) rc = check_ptrs(fn, {{p.X, "X"}, {p.A, "A"}, {p.B, "B"}, {p.Y, "Y"}});
    if (!rc && p.t_save && !aligned16(p.t_save))
      rc = fail(HSNF4_ERR_INVALID, "%s: problem %d: t_save misaligned", fn, i);
    if (!rc) rc = check_dropout(fn, i, p.dropout_p);
    if (rc) return rc;
  }
  {
    int32_t formats[8];
    for (int i = 0; i < n; ++i) formats[i] = probs[i].W.format;
    rc = check_one_format(fn, n, formats);
    if (rc) return rc;
  }
  FwdLayout L;
  fwd_layout(probs, n, T, r, &L);
  rc = check_workspace(fn, workspace, ws_bytes, L.total);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(r);
  ProjectDesc pd[8];
  GemmProblemDesc gd[8];
  DropDesc dd[8];
  int nd = 0;
  for (int i = 0; i < n; ++i) {
    const hsnf4_lora_fwd_args& p = probs[i];
    float* t_out = p.t_save ? p.t_save : reinterpret_cast<float*>(ws + L.tscratch[i]);
    // with dropout the adapter branch reads X_d = dropout(X); the base reads X
    const void* xl = p.X;
    if (p.dropout_p > 0.0f) {
      xl = ws + L.xd[i];
      dd[nd++] = {p.X, ws + L.xd[i], nullptr, nullptr, p.W.k_in, p.dropout_p, p.dropout_seed,
                  p.dropout_offset};
    }
    pd[i] = {xl, p.W.k_in, p.A, true, t_out, ws + L.zs[i]};
    gd[i] = {p.W.codes, p.W.absmax, p.W.n_out, p.W.k_in, p.X, p.B, ws + L.zs[i], p.Y,
             p.W.format == HSNF4_BASE_BF16};
  }
  if (nd) {
    rc = cuda_status(launch_dropout_apply(dd, nd, T, st), "lora_group_fwd: dropout launch");
    if (rc) return rc;
  }
  rc = cuda_status(launch_lora_project_group(pd, n, T, r, s, ws + L.prj, st),
                   "lora_group_fwd: projection launch");
  if (rc) return rc;
  return launch_lora_gemm_group(kGemmFwd, gd, n, T, r, ws + L.gemm, L.total - L.gemm, st);
}

int lora_group_bwd(const hsnf4_lora_bwd_args* probs, int n, int64_t T, int r, float alpha,
                   void* workspace, size_t ws_bytes, void* stream) {
  static const char* fn = "lora_group_bwd";
  if (!probs) return fail(HSNF4_ERR_INVALID, "%s: probs is NULL", fn);
  int rc = check_group(fn, n, T, r, alpha);
  if (!rc) rc = check_gemm_tokens(kGemmDx, T, r);
  if (rc) return rc;
  for (int i = 0; i < n; ++i) {
    const hsnf4_lora_bwd_args& p = probs[i];
    rc = check_weight(fn, i, p.W);
    if (!rc)
      rc = check_ptrs(fn, {{p.X, "X"}, {p.t_save, "t_save"}, {p.A, "A"}, {p.B, "B"},
                           {p.dY, "dY"}, {p.dX, "dX"}, {p.dA, "dA"}, {p.dB, "dB"}});
    if (!rc) rc = check_dropout(fn, i, p.dropout_p);
    if (rc) return rc;
  }
  {
    int32_t formats[8];
    for (int i = 0; i < n; ++i) formats[i] = probs[i].W.format;
    rc = check_one_format(fn, n, formats);
    if (rc) return rc;
  }
  BwdLayout L;
  bwd_layout(probs, n, T, r, &L);
  rc = check_workspace(fn, workspace, ws_bytes, L.total);
  if (rc) return rc;
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const float s = alpha / static_cast<float>(r);
  ProjectDesc pd[8];
  GemmProblemDesc gd[8];
  GradDesc grd[16];
  DropDesc dd[8], da[8];
  int nd = 0;
  for (int i = 0; i < n; ++i) {
    const hsnf4_lora_bwd_args& p = probs[i];
    float* u = reinterpret_cast<float*>(ws + L.u[i]);
    const bool drop = p.dropout_p > 0.0f;
    // with dropout: X_d recomputed from the forward's (seed, offset) feeds
    // dA; the GEMM's rank-r slice is zero and the masked adapter term of dX
    // is added after it
    const void* xl = drop ? static_cast<const void*>(ws + L.xd[i]) : p.X;
    if (drop) {
      // the apply pass records the keep mask; the dX pass reads it back
      dd[nd] = {p.X, ws + L.xd[i], nullptr, nullptr, p.W.k_in, p.dropout_p, p.dropout_seed,
                p.dropout_offset, ws + L.bits[i]};
      da[nd] = {nullptr, p.dX, u, p.A, p.W.k_in, p.dropout_p, p.dropout_seed, p.dropout_offset,
                ws + L.bits[i]};
      ++nd;
    }
    // u and the forward's t as two bf16 parts each: the gradient kernel's operands
    const size_t part = round_up(static_cast<size_t>(T) * r_padded(r) * 2, 256);
    uint8_t* u_hi = ws + L.parts[i];
    uint8_t* u_lo = u_hi + part;
    uint8_t* t_hi = u_lo + part;
    uint8_t* t_lo = t_hi + part;
    pd[i] = {p.dY, p.W.n_out, p.B, false, u, ws + L.su[i], drop, u_hi, u_lo, p.t_save, t_hi,
             t_lo};
    gd[i] = {p.W.codes, p.W.absmax, p.W.n_out, p.W.k_in, p.dY, p.A, ws + L.su[i], p.dX,
             p.W.format == HSNF4_BASE_BF16};
    grd[2 * i] = {p.dY, p.W.n_out, t_hi, t_lo, p.dB, true};  // dB = s dY^T t    [n_out, r]
    grd[2 * i + 1] = {xl, p.W.k_in, u_hi, u_lo, p.dA, false};  // dA = s u^T X(_d) [r, k_in]
  }
  if (nd) {
    rc = cuda_status(launch_dropout_apply(dd, nd, T, st), "lora_group_bwd: dropout launch");
    if (rc) return rc;
  }
  rc = cuda_status(launch_lora_project_group(pd, n, T, r, s, ws + L.prj, st),
                   "lora_group_bwd: projection launch");
  if (rc) return rc;
  // The adapter gradients need only u, t, X and dY: they run before the dX
  // GEMM, while the dY the projection has just read (and X) are still in L2,
  // instead of after the GEMM has streamed the base through it.
  rc = cuda_status(launch_lora_grad_group(grd, 2 * n, T, r, s, st),
                   "lora_group_bwd: gradient launch");
  if (rc) return rc;
  rc = launch_lora_gemm_group(kGemmDx, gd, n, T, r, ws + L.gemm, L.total - L.gemm, st);
  if (rc) return rc;
  if (nd)
    rc = cuda_status(launch_dx_dropout_add(da, nd, T, r, s, st),
                     "lora_group_bwd: dropout dX launch");
  return rc;
}

int lora_merge(const hsnf4_nf4_weight* W, const void* A, const void* B, int r, float alpha,
               void* W_out, void* stream) {
  static const char* fn = "lora_merge";
  if (!W) return fail(HSNF4_ERR_INVALID, "%s: W is NULL", fn);
  int rc = check_weight(fn, 0, *W);
  if (rc) return rc;
  if (r < 8 || r > 64 || r % 8)
    return fail(HSNF4_ERR_INVALID, "%s: rank must be a multiple of 8 in [8, 64] (got %d)", fn, r);
  if (!isfinite(alpha)) return fail(HSNF4_ERR_INVALID, "%s: alpha is not finite", fn);
  rc = check_ptrs(fn, {{A, "A"}, {B, "B"}, {W_out, "W_out"}});
  if (rc) return rc;
  if (W_out == W->codes) return fail(HSNF4_ERR_INVALID, "%s: W_out aliases the base", fn);
  return cuda_status(launch_lora_merge(W->codes, W->absmax, W->format == HSNF4_BASE_BF16,
                                       W->n_out, W->k_in, A, B, r,
                                       alpha / static_cast<float>(r), W_out,
                                       static_cast<cudaStream_t>(stream)),
                     "lora_merge launch");
}

int lora_dropout_apply(const void* X, int64_t T, int64_t k_in, float p, uint64_t seed,
                       uint64_t offset, void* X_d, void* stream) {
  static const char* fn = "lora_dropout_apply";
  int rc = check_nf4_shape(fn, T, k_in);
  if (!rc) rc = check_dropout(fn, 0, p);
  if (!rc) rc = check_ptrs(fn, {{X, "X"}, {X_d, "X_d"}});
  if (rc) return rc;
  DropDesc d = {X, X_d, nullptr, nullptr, k_in, p, seed, offset};
  return cuda_status(launch_dropout_apply(&d, 1, T, static_cast<cudaStream_t>(stream)),
                     "lora_dropout_apply launch");
}

// ---------------------------------------------------------------- decoder glue

static int check_rows(const char* fn, int64_t T, int64_t n) {
  if (T < 1 || n < 8 || n % 8 || T > (int64_t(1) << 31) || n > (int64_t(1) << 30))
    return fail(HSNF4_ERR_INVALID, "%s: need T >= 1 and n a positive multiple of 8 (got T=%lld, "
                "n=%lld)", fn, (long long)T, (long long)n);
  return HSNF4_OK;
}

static int check_elems(const char* fn, int64_t n) {
  if (n < 8 || n % 8)
    return fail(HSNF4_ERR_INVALID, "%s: need a positive multiple of 8 elements (got %lld)", fn,
                (long long)n);
  return HSNF4_OK;
}

static int check_opt(const char* fn, const void* p, const char* name) {
  if (p && !aligned16(p)) return fail(HSNF4_ERR_INVALID, "%s: %s is not 16-byte aligned", fn, name);
  return HSNF4_OK;
}

int decoder_rmsnorm_fwd(const void* xa, const void* xb, const void* g, void* h_out, void* y,
                        int64_t T, int64_t n, float eps, void* stream) {
  static const char* fn = "decoder_rmsnorm_fwd";
  int rc = check_rows(fn, T, n);
  if (!rc) rc = check_ptrs(fn, {{xa, "xa"}, {g, "g"}, {y, "y"}});
  if (!rc) rc = check_opt(fn, xb, "xb");
  if (!rc && xb) rc = check_ptrs(fn, {{h_out, "h_out"}});
  if (!rc && !(eps >= 0.0f)) rc = fail(HSNF4_ERR_INVALID, "%s: eps must be >= 0", fn);
  if (rc) return rc;
  return cuda_status(launch_rmsnorm_fwd(xa, xb, g, h_out, y, T, n, eps,
                                        static_cast<cudaStream_t>(stream)),
                     "decoder_rmsnorm_fwd launch");
}

int decoder_rmsnorm_bwd(const void* x, const void* g, const void* dy1, const void* dy2,
                        const void* dy3, const void* dres, void* dx, int64_t T, int64_t n,
                        float eps, void* stream) {
  static const char* fn = "decoder_rmsnorm_bwd";
  int rc = check_rows(fn, T, n);
  if (!rc) rc = check_ptrs(fn, {{x, "x"}, {g, "g"}, {dy1, "dy1"}, {dx, "dx"}});
  if (!rc) rc = check_opt(fn, dy2, "dy2");
  if (!rc) rc = check_opt(fn, dy3, "dy3");
  if (!rc) rc = check_opt(fn, dres, "dres");
  if (!rc && !(eps >= 0.0f)) rc = fail(HSNF4_ERR_INVALID, "%s: eps must be >= 0", fn);
  if (rc) return rc;
  return cuda_status(launch_rmsnorm_bwd(x, g, dy1, dy2, dy3, dres, dx, T, n, eps,
                                        static_cast<cudaStream_t>(stream)),
                     "decoder_rmsnorm_bwd launch");
}

int decoder_swiglu_fwd(const void* a, const void* b, void* m, int64_t n, void* stream) {
  static const char* fn = "decoder_swiglu_fwd";
  int rc = check_elems(fn, n);
  if (!rc) rc = check_ptrs(fn, {{a, "a"}, {b, "b"}, {m, "m"}});
  if (rc) return rc;
  return cuda_status(launch_silu_mul_fwd(a, b, m, n, static_cast<cudaStream_t>(stream)),
                     "decoder_swiglu_fwd launch");
}

int decoder_swiglu_bwd(const void* a, const void* b, const void* dm, void* da, void* db, int64_t n,
                       void* stream) {
  static const char* fn = "decoder_swiglu_bwd";
  int rc = check_elems(fn, n);
  if (!rc) rc = check_ptrs(fn, {{a, "a"}, {b, "b"}, {dm, "dm"}, {da, "da"}, {db, "db"}});
  if (rc) return rc;
  return cuda_status(launch_silu_mul_bwd(a, b, dm, da, db, n, static_cast<cudaStream_t>(stream)),
                     "decoder_swiglu_bwd launch");
}

int decoder_add(const void* x, const void* y, void* out, int64_t n, void* stream) {
  static const char* fn = "decoder_add";
  int rc = check_elems(fn, n);
  if (!rc) rc = check_ptrs(fn, {{x, "x"}, {y, "y"}, {out, "out"}});
  if (rc) return rc;
  return cuda_status(launch_add(x, y, out, n, static_cast<cudaStream_t>(stream)),
                     "decoder_add launch");
}

static int check_attn(const char* fn, int64_t T, int H, int KV) {
  if (T < 1 || T > 32768 || H < 1 || KV < 1 || H % KV)
    return fail(HSNF4_ERR_INVALID, "%s: need 1 <= T <= 32768 and H a multiple of KV (got T=%lld, "
                "H=%d, KV=%d)", fn, (long long)T, H, KV);
  return HSNF4_OK;
}

int decoder_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                          int64_t T, int H, int KV, void* stream) {
  static const char* fn = "decoder_attention_fwd";
  int rc = check_attn(fn, T, H, KV);
  if (!rc) rc = check_ptrs(fn, {{q, "q"}, {k, "k"}, {v, "v"}, {o, "o"}, {lse, "lse"}});
  if (rc) return rc;
  return cuda_status(launch_attention_fwd(q, k, v, o, lse, T, H, KV, 1.0f / sqrtf(128.0f),
                                          static_cast<cudaStream_t>(stream)),
                     "decoder_attention_fwd launch");
}

size_t decoder_attention_scratch_bytes(int64_t T, int H) {
  if (T < 1 || H < 1) return 0;
  // row dots [H, T] (rounded up to 64 floats), then fp32 dK, dV partials [2H][T][128]
  return (static_cast<size_t>(T) * H + 63) / 64 * 64 * 4 + static_cast<size_t>(T) * H * 2 * 128 * 4;
}

int decoder_attention_bwd(const void* q, const void* k, const void* v, const void* o,
                          const float* lse, const void* dout, void* dq, void* dk, void* dv,
                          float* scratch, int64_t T, int H, int KV, void* stream) {
  static const char* fn = "decoder_attention_bwd";
  int rc = check_attn(fn, T, H, KV);
  if (!rc)
    rc = check_ptrs(fn, {{q, "q"}, {k, "k"}, {v, "v"}, {o, "o"}, {lse, "lse"}, {dout, "dout"},
                         {dq, "dq"}, {dk, "dk"}, {dv, "dv"}, {scratch, "scratch"}});
  if (rc) return rc;
  return cuda_status(launch_attention_bwd(q, k, v, o, lse, dout, dq, dk, dv, scratch, T, H, KV,
                                          1.0f / sqrtf(128.0f), static_cast<cudaStream_t>(stream)),
                     "decoder_attention_bwd launch");
}

static hsnf4_lora_fwd_args one_fwd(const hsnf4_nf4_weight* W, const void* X, const void* A,
                                   const void* B, void* Y, float* t_save) {
  hsnf4_lora_fwd_args a;
  memset(&a, 0, sizeof a);  // no dropout
  a.W = *W;
  a.X = X;
  a.A = A;
  a.B = B;
  a.Y = Y;
  a.t_save = t_save;
  return a;
}

size_t lora_linear_fwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r) {
  hsnf4_nf4_weight W = {nullptr, nullptr, n_out, k_in, HSNF4_BASE_NF4, 0};
  hsnf4_lora_fwd_args a = one_fwd(&W, nullptr, nullptr, nullptr, nullptr, nullptr);
  return lora_group_fwd_workspace(&a, 1, T, r);
}

size_t lora_linear_bwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r) {
  hsnf4_lora_bwd_args a;
  memset(&a, 0, sizeof a);
  a.W.n_out = n_out;
  a.W.k_in = k_in;
  return lora_group_bwd_workspace(&a, 1, T, r);
}

int lora_linear_fwd(const hsnf4_nf4_weight* W, const void* X, int64_t T, const void* A,
                    const void* B, int r, float alpha, void* Y, float* t_save, void* workspace,
                    size_t ws_bytes, void* stream) {
  if (!W) return fail(HSNF4_ERR_INVALID, "lora_linear_fwd: W is NULL");
  hsnf4_lora_fwd_args a = one_fwd(W, X, A, B, Y, t_save);
  return lora_group_fwd(&a, 1, T, r, alpha, workspace, ws_bytes, stream);
}

int lora_linear_bwd(const hsnf4_nf4_weight* W, const void* X, const float* t_save, int64_t T,
                    const void* A, const void* B, int r, float alpha, const void* dY, void* dX,
                    float* dA, float* dB, void* workspace, size_t ws_bytes, void* stream) {
  if (!W) return fail(HSNF4_ERR_INVALID, "lora_linear_bwd: W is NULL");
  hsnf4_lora_bwd_args a;
  memset(&a, 0, sizeof a);  // no dropout
  a.W = *W;
  a.X = X;
  a.t_save = t_save;
  a.A = A;
  a.B = B;
  a.dY = dY;
  a.dX = dX;
  a.dA = dA;
  a.dB = dB;
  return lora_group_bwd(&a, 1, T, r, alpha, workspace, ws_bytes, stream);
}

}  // extern "C"
