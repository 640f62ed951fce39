// lora_aux.cu -- the rank-r pieces of the LoRA linear around the fused GEMM.
//
//   project:  t = Z Adp^T   (Z bf16 [T, C], adapter [r, C] or [C, r])
//             writes t (fp32) and zs = bf16(s * t) padded to r_pad columns,
//             the operand of the GEMM's rank-r slice.
//             forward:  t = X A^T   (Adp = A, [r, k_in])
//             backward: u = dY B    (Adp = B, [n_out, r])
//   grad:     out = s Z^T V (Z bf16 [T, C], V fp32 [T, r])
//             dB = s dY^T t  ([n_out, r]),   dA = s u^T X  ([r, k_in])
//
// These are skinny (r <= 64) and bound by reading Z once; they run on the
// CUDA cores with fp32 accumulation.  Every output is reduced in a fixed
// order (per-thread strided partial sums, a fixed butterfly inside a warp,
// then warps in index order), so results are bitwise reproducible.
#include <cuda_bf16.h>

#include "internal.h"

namespace hsnf4 {

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xFFFF0000u); }
__device__ __forceinline__ float bf16_at(const uint16_t* p, int64_t i) {
  return __uint_as_float(static_cast<uint32_t>(__ldg(p + i)) << 16);
}

// ---------------------------------------------------------------- project
// CTA = 256 threads and TT token rows.  Thread x walks the contraction
// index c = x, x+256, ... and keeps TT*R partial sums; the partials are then
// combined by a butterfly within each warp and by warp index through shared
// memory.

template <int R, int TT, bool R_MAJOR>
__global__ void __launch_bounds__(256) lora_project_kernel(
    const uint16_t* __restrict__ Z, int64_t T, int64_t C, const uint16_t* __restrict__ adp,
    int r_pad, float s, float* __restrict__ t_out, uint16_t* __restrict__ zs) {
  __shared__ float red[8][TT * R];
  const int64_t t0 = static_cast<int64_t>(blockIdx.x) * TT;
  float acc[TT][R];
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) acc[i][j] = 0.0f;

  for (int64_t c = threadIdx.x; c < C; c += 256) {
    float a[R];
    if (R_MAJOR) {
#pragma unroll
      for (int j = 0; j < R; ++j) a[j] = bf16_at(adp, j * C + c);
    } else {
      const uint4* row = reinterpret_cast<const uint4*>(adp + c * R);  // R % 8 == 0
#pragma unroll
      for (int q = 0; q < R / 8; ++q) {
        const uint4 v = __ldg(row + q);
        a[8 * q + 0] = bf16_lo(v.x); a[8 * q + 1] = bf16_hi(v.x);
        a[8 * q + 2] = bf16_lo(v.y); a[8 * q + 3] = bf16_hi(v.y);
        a[8 * q + 4] = bf16_lo(v.z); a[8 * q + 5] = bf16_hi(v.z);
        a[8 * q + 6] = bf16_lo(v.w); a[8 * q + 7] = bf16_hi(v.w);
      }
    }
#pragma unroll
    for (int i = 0; i < TT; ++i) {
      const float z = (t0 + i < T) ? bf16_at(Z, (t0 + i) * C + c) : 0.0f;
#pragma unroll
      for (int j = 0; j < R; ++j) acc[i][j] = fmaf(z, a[j], acc[i][j]);
    }
  }
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
#pragma unroll
  for (int i = 0; i < TT; ++i)
#pragma unroll
    for (int j = 0; j < R; ++j) {
      float v = acc[i][j];
#pragma unroll
      for (int o = 16; o >= 1; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
      if (lane == 0) red[warp][i * R + j] = v;
    }
  __syncthreads();
  for (int k = threadIdx.x; k < TT * R; k += 256) {
    float v = red[0][k];
#pragma unroll
    for (int w = 1; w < 8; ++w) v += red[w][k];
    const int i = k / R, j = k % R;
    const int64_t t = t0 + i;
    if (t < T) {
      t_out[t * R + j] = v;
      const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(s, v));
      zs[t * r_pad + j] = *reinterpret_cast<const uint16_t*>(&b);
    }
  }
  // zero the padding columns of zs
  for (int k = threadIdx.x; k < TT * (r_pad - R); k += 256) {
    const int i = k / (r_pad - R), j = R + k % (r_pad - R);
    if (t0 + i < T) zs[(t0 + i) * r_pad + j] = 0;
  }
}

template <int R, bool R_MAJOR>
static cudaError_t project_r(const void* Z, int64_t T, int64_t C, const void* adp, int r_pad,
                             float s, float* t_out, void* zs, cudaStream_t st) {
  constexpr int TT = (R <= 16) ? 4 : (R <= 32 ? 2 : 1);
  const int64_t grid = (T + TT - 1) / TT;
  lora_project_kernel<R, TT, R_MAJOR><<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint16_t*>(Z), T, C, static_cast<const uint16_t*>(adp), r_pad, s, t_out,
      static_cast<uint16_t*>(zs));
  return cudaGetLastError();
}

template <bool R_MAJOR>
static cudaError_t project_dispatch(const void* Z, int64_t T, int64_t C, const void* adp, int r,
                                    int r_pad, float s, float* t_out, void* zs,
                                    cudaStream_t st) {
  switch (r) {
    case 8: return project_r<8, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 16: return project_r<16, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 24: return project_r<24, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 32: return project_r<32, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 40: return project_r<40, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 48: return project_r<48, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 56: return project_r<56, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    case 64: return project_r<64, R_MAJOR>(Z, T, C, adp, r_pad, s, t_out, zs, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_lora_project(const void* Z, int64_t T, int64_t C, const void* adp,
                                bool adp_r_major, int r, int r_pad, float s, float* t_out,
                                void* zs, cudaStream_t st) {
  return adp_r_major ? project_dispatch<true>(Z, T, C, adp, r, r_pad, s, t_out, zs, st)
                     : project_dispatch<false>(Z, T, C, adp, r, r_pad, s, t_out, zs, st);
}

// ---------------------------------------------------------------- grad
// CTA = 32 columns x 8 token groups.  Thread (x, g) sums tokens g, g+8, ...
// in increasing order for column c0+x and all R rank indices; the 8 group
// partials are then added in group order.  V is staged through shared memory
// in chunks of 64 tokens.

constexpr int kGradCols = 32;
constexpr int kGradGroups = 8;
constexpr int kGradChunk = 64;

template <int R, bool OUT_C_MAJOR>
__global__ void __launch_bounds__(256) lora_grad_kernel(const uint16_t* __restrict__ Z, int64_t T,
                                                        int64_t C, const float* __restrict__ V,
                                                        float s, float* __restrict__ out) {
  __shared__ float vs[kGradChunk * R];
  __shared__ float part[kGradCols][R + 1];
  const int x = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * kGradCols + x;
  const bool live = c < C;
  float acc[R];
#pragma unroll
  for (int j = 0; j < R; ++j) acc[j] = 0.0f;
  for (int64_t tc = 0; tc < T; tc += kGradChunk) {
    const int n = static_cast<int>((T - tc < kGradChunk) ? (T - tc) : kGradChunk);
    __syncthreads();
    for (int k = threadIdx.x; k < n * R; k += 256) vs[k] = __ldg(V + tc * R + k);
    __syncthreads();
    for (int i = g; i < n; i += kGradGroups) {
      const float z = live ? bf16_at(Z, (tc + i) * C + c) : 0.0f;
#pragma unroll
      for (int j = 0; j < R; ++j) acc[j] = fmaf(z, vs[i * R + j], acc[j]);
    }
  }
  // add the group partials in group order 0..7
  for (int q = 0; q < kGradGroups; ++q) {
    if (g == q) {
#pragma unroll
      for (int j = 0; j < R; ++j) part[x][j] = (q == 0) ? acc[j] : part[x][j] + acc[j];
    }
    __syncthreads();
  }
  for (int k = threadIdx.x; k < kGradCols * R; k += 256) {
    const int cx = k / R, j = k % R;
    const int64_t cc = static_cast<int64_t>(blockIdx.x) * kGradCols + cx;
    if (cc < C) {
      const float v = __fmul_rn(s, part[cx][j]);
      if (OUT_C_MAJOR)
        out[cc * R + j] = v;
      else
        out[static_cast<int64_t>(j) * C + cc] = v;
    }
  }
}

template <int R, bool OUT_C_MAJOR>
static cudaError_t grad_r(const void* Z, int64_t T, int64_t C, const float* V, float s,
                          float* out, cudaStream_t st) {
  const int64_t grid = (C + kGradCols - 1) / kGradCols;
  lora_grad_kernel<R, OUT_C_MAJOR><<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint16_t*>(Z), T, C, V, s, out);
  return cudaGetLastError();
}

template <bool OUT_C_MAJOR>
static cudaError_t grad_dispatch(const void* Z, int64_t T, int64_t C, const float* V, int r,
                                 float s, float* out, cudaStream_t st) {
  switch (r) {
    case 8: return grad_r<8, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 16: return grad_r<16, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 24: return grad_r<24, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 32: return grad_r<32, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 40: return grad_r<40, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 48: return grad_r<48, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 56: return grad_r<56, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    case 64: return grad_r<64, OUT_C_MAJOR>(Z, T, C, V, s, out, st);
    default: return cudaErrorInvalidValue;
  }
}

cudaError_t launch_lora_grad(const void* Z, int64_t T, int64_t C, const float* V, int r,
                             float s, float* out, bool out_c_major, cudaStream_t st) {
  return out_c_major ? grad_dispatch<true>(Z, T, C, V, r, s, out, st)
                     : grad_dispatch<false>(Z, T, C, V, r, s, out, st);
}

}  // namespace hsnf4
