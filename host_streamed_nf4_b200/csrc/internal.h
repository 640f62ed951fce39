// internal.h -- host-side declarations shared by the library's translation
// units (not part of the public ABI; see include/hsnf4.h for that).
#pragma once

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

// The NormalFloat-4 codebook the kernels use (derived once, in double).
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

// t = Z Adp^T (fp32 [T, r]) and zs = bf16(s * t) [T, r_pad] (pad columns 0).
// adp_rows_major: adapter stored [r, C] (A) if true, [C, r] (B) if false.
cudaError_t launch_lora_project(const void* Z, int64_t T, int64_t C, const void* adp,
                                bool adp_r_major, int r, int r_pad, float s, float* t_out,
                                void* zs, cudaStream_t st);

// out = s * Z^T V: Z bf16 [T, C], V fp32 [T, r].  out_c_major: out is [C, r]
// (dB) if true, [r, C] (dA) if false.
cudaError_t launch_lora_grad(const void* Z, int64_t T, int64_t C, const float* V, int r,
                             float s, float* out, bool out_c_major, cudaStream_t st);

enum GemmMode { kGemmFwd = 0, kGemmDx = 1 };

// Fused NF4 dequant + tcgen05 GEMM with the rank-r slice.
//  fwd: out[T, n_out] = act[T, k_in] deq(W)^T + lo_b[T, r_pad] lo_a[n_out, r]^T
//  dx : out[T, k_in]  = act[T, n_out] deq(W) + lo_b[T, r_pad] lo_a[r, k_in]
// lo_b is the pre-scaled bf16 rank-r factor (s*t or s*u).
int launch_lora_gemm(GemmMode mode, const hsnf4_nf4_weight* W, const void* act, int64_t T,
                     const void* lo_a, int r, int r_pad, const void* lo_b, void* out,
                     cudaStream_t st);

cudaError_t launch_selftest_stall(cudaStream_t st);

// Kernel timing (hsnf4_profile): bracket a launch with prof_begin/prof_end.
enum ProfKind { kProfGemmFwd = 0, kProfGemmDx = 1, kProfDequant = 2, kProfKinds = 3 };
bool profiling();
void* prof_begin(cudaStream_t st);
void prof_end(void* token, int kind, double work, cudaStream_t st);

// Read and clear the device failure flags the GEMM kernels record.
cudaError_t read_gemm_flags(uint32_t* flags);

}  // namespace hsnf4
