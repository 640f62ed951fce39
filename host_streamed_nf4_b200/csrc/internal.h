// internal.h -- host-side declarations shared by the library's translation
// units (not part of the public ABI; see include/hsnf4.h for that).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "hsnf4.h"
#include "nf4_device.cuh"

namespace hsnf4 {

// Record a failure for this thread (hsnf4_last_error) and return `status`.
int fail(int status, const char* fmt, ...) __attribute__((format(printf, 2, 3)));

// Map a CUDA error to HSNF4_ERR_CUDA with the call's name, or HSNF4_OK.
int cuda_status(cudaError_t e, const char* what);

// The NormalFloat-4 codebook the kernels use (the published NF4 values).
const Nf4Codebook& codebook();

// Host-side fault injection sites (hsnf4_inject_fault).
enum FaultSite { kFaultNone = 0, kFaultCopyEnqueue = 1, kFaultEventRecord = 2 };
// True (and the injection is consumed) if the pending fault is at `site`.
bool take_fault(FaultSite site);

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline size_t round_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- launchers (enqueue only; arguments already validated) ----

cudaError_t launch_nf4_quantize(const void* w, int64_t n_out, int64_t k_in, void* codes,
                                float* absmax, cudaStream_t st);
cudaError_t launch_nf4_dequant(const void* codes, const float* absmax, int64_t n_out,
                               int64_t k_in, void* out, cudaStream_t st);

// ---- rank-r projections, grouped (lora_rank.cu): t_q = Z_q Adp_q^T (fp32
// [T, r]) and zs_q = bf16(s * t_q) ([T, r_pad], pad columns 0).  Adp is
// A [r, C] (r_major, forward) or B [C, r] (backward).  Optional outputs:
// hi/lo, the two bf16 parts of t_q ([T, r_pad] each); split_hi/lo, the two
// bf16 parts of split_src (fp32 [T, r]).  No workspace.
struct ProjectDesc {
  const void* Z;
  int64_t C;
  const void* adp;
  bool r_major;
  float* t_out;
  void* zs;
  bool zero_zs = false;  // write zs = 0 (the GEMM's rank-r slice then adds nothing)
  void* hi = nullptr;
  void* lo = nullptr;
  const float* split_src = nullptr;
  void* split_hi = nullptr;
  void* split_lo = nullptr;
};
size_t project_workspace_bytes(const ProjectDesc* d, int n, int64_t T, int r);
cudaError_t launch_lora_project_group(const ProjectDesc* d, int n, int64_t T, int r, float s,
                                      void* ws, cudaStream_t st);

// ---- adapter gradients, grouped (lora_rank.cu): out_q = s Z_q^T V_q, Z
// bf16 [T, C], V = V_hi + V_lo (bf16 [T, r_pad] each); out is [C, r]
// (c_major, dB) or [r, C] (dA).
struct GradDesc {
  const void* Z;
  int64_t C;
  const void* V_hi;
  const void* V_lo;
  float* out;
  bool c_major;
};
cudaError_t launch_lora_grad_group(const GradDesc* d, int n, int64_t T, int r, float s,
                                   cudaStream_t st);
cudaError_t read_rank_flags(uint32_t* flags);
cudaError_t read_merge_flags(uint32_t* flags);

// 2-D TMA descriptor of a row-major tensor [outer][inner] (row_bytes apart)
// with a box of box_inner x box_outer elements; false if the driver refuses.
bool encode_tma_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle sw);

enum GemmMode { kGemmFwd = 0, kGemmDx = 1 };

// ---- fused NF4 dequant + tcgen05 GEMM with the rank-r slice, grouped:
//  fwd: out[T, n_out] = act[T, k_in] deq(W)^T + lo_b[T, r_pad] lo_a[n_out, r]^T
//  dx : out[T, k_in]  = act[T, n_out] deq(W) + lo_b[T, r_pad] lo_a[r, k_in]
// lo_b is the pre-scaled bf16 rank-r factor (s*t or s*u).
struct GemmProblemDesc {
  const void* codes;
  const float* absmax;
  int64_t n_out, k_in;
  const void* act;
  const void* lo_a;
  const void* lo_b;
  void* out;
  bool dense;  // codes is a bf16 [n_out, k_in] weight (no absmax, no dequant)
};
size_t gemm_workspace_bytes(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r);
int gemm_plan_info(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r,
                   hsnf4_gemm_plan_info* out);
// HSNF4_OK if the fused GEMM takes T tokens at rank r in this mode (a tiling
// fits shared memory and T spans at most 64 token tiles); else the error,
// recorded.  Needs only the sizes, so callers check it before any launch.
int check_gemm_tokens(GemmMode mode, int64_t T, int r);
int launch_lora_gemm_group(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r,
                           void* workspace, size_t ws_bytes, cudaStream_t st);

cudaError_t launch_selftest_stall(cudaStream_t st);

// W' = deq(W) + s B A -> bf16 [N, K] (dense: base is a bf16 weight)
cudaError_t launch_lora_merge(const void* base, const float* absmax, bool dense, int64_t N,
                              int64_t K, const void* A, const void* B, int r, float s, void* out,
                              cudaStream_t st);

// Process-wide count of kernels this library launched (hsnf4_kernel_launches).
void count_launch();

// Launch with programmatic stream serialization: the kernel's CTAs may start
// before the previous kernel in the stream completes.  Only for kernels that
// call pdl_wait_then_release() before any global-memory access.
template <typename Params>
inline cudaError_t launch_pdl(void (*kernel)(Params), dim3 grid, dim3 block, size_t smem,
                              cudaStream_t st, const Params& p) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, p);
}

// ---- LoRA dropout, grouped (lora_dropout.cu): apply writes out = X_d;
// dx add updates out = dX += keep * scale * s * (u A).
struct DropDesc {
  const void* X;
  void* out;
  const float* u;
  const void* A;
  int64_t K;
  float p;
  uint64_t seed, offset;
  // optional keep mask, one byte per 8 consecutive elements (bit i: element
  // 8g + i): apply writes it, dx add reads it instead of re-running Philox
  uint8_t* bits = nullptr;
};
cudaError_t launch_dropout_apply(const DropDesc* d, int n, int64_t T, cudaStream_t st);
cudaError_t launch_dx_dropout_add(const DropDesc* d, int n, int64_t T, int r, float s,
                                  cudaStream_t st);

// ---- decoder glue (glue.cu, attention.cu)
cudaError_t launch_rmsnorm_fwd(const void* xa, const void* xb, const void* g, void* h_out,
                               void* y, int64_t T, int64_t n, float eps, cudaStream_t st);
cudaError_t launch_rmsnorm_bwd(const void* x, const void* g, const void* dy1, const void* dy2,
                               const void* dy3, const void* dres, void* dx, int64_t T, int64_t n,
                               float eps, cudaStream_t st);
cudaError_t launch_silu_mul_fwd(const void* a, const void* b, void* m, int64_t n,
                                cudaStream_t st);
cudaError_t launch_silu_mul_bwd(const void* a, const void* b, const void* dm, void* da, void* db,
                                int64_t n, cudaStream_t st);
cudaError_t launch_add(const void* x, const void* y, void* out, int64_t n, cudaStream_t st);
cudaError_t launch_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int64_t T, int H, int KV, float scale, cudaStream_t st);
cudaError_t launch_attention_bwd(const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                 float* D, int64_t T, int H, int KV, float scale,
                                 cudaStream_t st);

// Kernel timing (hsnf4_profile): bracket a launch with prof_begin/prof_end.
enum ProfKind {
  kProfGemmFwd = 0,
  kProfGemmDx = 1,
  kProfDequant = 2,
  kProfMerge = 3,
  kProfProject = 4,
  kProfGrad = 5,
  kProfKinds = 6
};
bool profiling();
void* prof_begin(cudaStream_t st, int kind);
void prof_end(void* token, int kind, double work, cudaStream_t st);

// Read and clear the device failure flags the GEMM kernels record.
cudaError_t read_gemm_flags(uint32_t* flags);

}  // namespace hsnf4
