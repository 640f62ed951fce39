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
// NormalFloat-4 (the "nf4" type of the Poros API reference; values from the
// published construction): standard-normal quantiles at probabilities
// delta - j (delta - 1/2) / 8, j = 0..7 (positive side) and
// delta - j (delta - 1/2) / 7, j = 0..6 (negative side, mirrored), plus 0,
// divided by the quantile at delta = 1 - (1/32 + 1/30) / 2.
// The quantile is found by Newton's method on Phi(x) - p with
// Phi(x) = erfc(-x / sqrt 2) / 2 and Phi'(x) = exp(-x^2 / 2) / sqrt(2 pi),
// iterated to a fixed point in double; each ratio is rounded once to fp32.

static double newton_quantile(double p) {
  const double inv_sqrt2 = 0.70710678118654752440;
  const double inv_sqrt_2pi = 0.39894228040143267794;
  double x = 0.0;
  for (int it = 0; it < 200; ++it) {
    const double f = 0.5 * erfc(-x * inv_sqrt2) - p;
    const double d = inv_sqrt_2pi * exp(-0.5 * x * x);
    const double nx = x - f / d;
    if (nx == x) break;
    if (it > 60 && fabs(nx - x) <= 4e-16 * fabs(x)) {  // settled to rounding noise
      x = 0.5 * (x + nx);
      break;
    }
    x = nx;
  }
  return x;
}

static Nf4Codebook derive_codebook() {
  Nf4Codebook cb;
  const double delta = 1.0 - 0.5 * (1.0 / 32.0 + 1.0 / 30.0);
  const double top = newton_quantile(delta);
  for (int j = 0; j < 7; ++j)
    cb.v[j] = static_cast<float>(-newton_quantile(delta - j * (delta - 0.5) / 7.0) / top);
  cb.v[7] = 0.0f;
  for (int j = 0; j < 8; ++j)
    cb.v[15 - j] = static_cast<float>(newton_quantile(delta - j * (delta - 0.5) / 8.0) / top);
  cb.v[0] = -1.0f;
  cb.v[15] = 1.0f;
  return cb;
}

const Nf4Codebook& codebook() {
  static Nf4Codebook cb;
  static std::once_flag once;
  std::call_once(once, [] { cb = derive_codebook(); });
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
  uint32_t f = 0;
  rc = cuda_status(read_gemm_flags(&f), "hsnf4_device_status: read flags");
  if (rc) return rc;
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

static int check_lora(const char* fn, const hsnf4_nf4_weight* W, int64_t T, int r) {
  if (!W) return fail(HSNF4_ERR_INVALID, "%s: W is NULL", fn);
  if (W->n_out < 64 || W->n_out % 64 || W->k_in < 64 || W->k_in % 64)
    return fail(HSNF4_ERR_INVALID,
                "%s: n_out and k_in must be positive multiples of 64 (got %lld x %lld)", fn,
                (long long)W->n_out, (long long)W->k_in);
  if (W->n_out > (1 << 30) || W->k_in > (1 << 30))
    return fail(HSNF4_ERR_INVALID, "%s: weight dimension too large", fn);
  if (T < 1 || T > (int64_t(1) << 30))
    return fail(HSNF4_ERR_INVALID, "%s: T must be in [1, 2^30] (got %lld)", fn, (long long)T);
  if (r < 8 || r > 64 || r % 8)
    return fail(HSNF4_ERR_INVALID, "%s: rank must be a multiple of 8 in [8, 64] (got %d)", fn, r);
  return check_ptrs(fn, {{W->codes, "W->codes"}, {W->absmax, "W->absmax"}});
}

size_t lora_linear_fwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r) {
  (void)n_out;
  (void)k_in;
  if (T < 1 || r < 1) return 0;
  return round_up(static_cast<size_t>(T) * r_padded(r) * 2, 256) +  // s*t, bf16
         round_up(static_cast<size_t>(T) * r * 4, 256);             // t, fp32 (if no t_save)
}

size_t lora_linear_bwd_workspace(int64_t T, int64_t n_out, int64_t k_in, int r) {
  (void)n_out;
  (void)k_in;
  if (T < 1 || r < 1) return 0;
  return round_up(static_cast<size_t>(T) * r_padded(r) * 2, 256) +  // s*u, bf16
         round_up(static_cast<size_t>(T) * r * 4, 256);             // u, fp32
}

int lora_linear_fwd(const hsnf4_nf4_weight* W, const void* X, int64_t T, const void* A,
                    const void* B, int r, float alpha, void* Y, float* t_save, void* workspace,
                    size_t ws_bytes, void* stream) {
  static const char* fn = "lora_linear_fwd";
  int rc = check_lora(fn, W, T, r);
  if (rc) return rc;
  rc = check_ptrs(fn, {{X, "X"}, {A, "A"}, {B, "B"}, {Y, "Y"}, {workspace, "workspace"}});
  if (rc) return rc;
  if (t_save && !aligned16(t_save)) return fail(HSNF4_ERR_INVALID, "%s: t_save misaligned", fn);
  if (!isfinite(alpha)) return fail(HSNF4_ERR_INVALID, "%s: alpha is not finite", fn);
  const size_t need = lora_linear_fwd_workspace(T, W->n_out, W->k_in, r);
  if (ws_bytes < need)
    return fail(HSNF4_ERR_OOM, "%s: workspace too small: need %zu bytes, given %zu", fn, need,
                ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(HSNF4_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rp = r_padded(r);
  const float s = alpha / static_cast<float>(r);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* ts = ws;
  float* t_out = t_save ? t_save
                        : reinterpret_cast<float*>(ws + round_up(static_cast<size_t>(T) * rp * 2, 256));
  rc = cuda_status(launch_lora_project(X, T, W->k_in, A, true, r, rp, s, t_out, ts, st),
                   "lora_linear_fwd: project launch");
  if (rc) return rc;
  return launch_lora_gemm(kGemmFwd, W, X, T, B, r, rp, ts, Y, st);
}

int lora_linear_bwd(const hsnf4_nf4_weight* W, const void* X, const float* t_save, int64_t T,
                    const void* A, const void* B, int r, float alpha, const void* dY, void* dX,
                    float* dA, float* dB, void* workspace, size_t ws_bytes, void* stream) {
  static const char* fn = "lora_linear_bwd";
  int rc = check_lora(fn, W, T, r);
  if (rc) return rc;
  rc = check_ptrs(fn, {{X, "X"}, {t_save, "t_save"}, {A, "A"}, {B, "B"}, {dY, "dY"}, {dX, "dX"},
                       {dA, "dA"}, {dB, "dB"}, {workspace, "workspace"}});
  if (rc) return rc;
  if (!isfinite(alpha)) return fail(HSNF4_ERR_INVALID, "%s: alpha is not finite", fn);
  const size_t need = lora_linear_bwd_workspace(T, W->n_out, W->k_in, r);
  if (ws_bytes < need)
    return fail(HSNF4_ERR_OOM, "%s: workspace too small: need %zu bytes, given %zu", fn, need,
                ws_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(HSNF4_ERR_INVALID, "%s: workspace must be 256-byte aligned", fn);
  cudaStream_t st = static_cast<cudaStream_t>(stream);
  const int rp = r_padded(r);
  const float s = alpha / static_cast<float>(r);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* su = ws;
  float* u = reinterpret_cast<float*>(ws + round_up(static_cast<size_t>(T) * rp * 2, 256));
  rc = cuda_status(launch_lora_project(dY, T, W->n_out, B, false, r, rp, s, u, su, st),
                   "lora_linear_bwd: project launch");
  if (rc) return rc;
  rc = launch_lora_gemm(kGemmDx, W, dY, T, A, r, rp, su, dX, st);
  if (rc) return rc;
  rc = cuda_status(launch_lora_grad(dY, T, W->n_out, t_save, r, s, dB, true, st),
                   "lora_linear_bwd: dB launch");
  if (rc) return rc;
  return cuda_status(launch_lora_grad(X, T, W->k_in, u, r, s, dA, false, st),
                     "lora_linear_bwd: dA launch");
}

}  // extern "C"
