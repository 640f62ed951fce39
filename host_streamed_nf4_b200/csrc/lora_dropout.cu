// lora_dropout.cu -- LoRA dropout on the adapter branch (Poros API
// reference: lora_dropout, default 0.05), for a group of problems per launch.
//
//   apply:   X_d = keep ? bf16_rne(fp32(x) * scale) : +0       (bf16 [T, K])
//            the input of t = X_d A^T (forward) and of dA = s u^T X_d
//            (backward, recomputed from the same (seed, offset));
//   dx add:  dX += keep * scale * s * (u A)                      (bf16 [T, K])
//            the adapter term of the input gradient, which the mask makes
//            elementwise, added after the fused GEMM has written dY deq(W)
//            (the GEMM's rank-r slice is zero in this mode).
//
// The mask is recomputed, never stored: element e = t K + k takes word e % 4
// of the Philox block of e / 4 (philox.cuh).  An apply thread owns 8
// consecutive elements of one row (16 bytes of bf16, two Philox blocks); a
// dx-add thread the same 8 columns of 4 consecutive rows.  Both kernels
// are HBM-bound elementwise passes: apply reads 2 B and writes 2 B per
// element, dx add reads 2 B and writes 2 B (u and A are re-read from L2).
#include <cuda_bf16.h>

#include "internal.h"
#include "philox.cuh"

namespace hsnf4 {

constexpr int kMaxDrop = 16;

struct DropProblem {
  const uint16_t* X;   // apply: input [T, K];  dx add: unused
  uint16_t* out;       // apply: X_d [T, K];    dx add: dX [T, K] (read and written)
  const float* u;      // dx add: u fp32 [T, r]
  const uint16_t* A;   // dx add: A bf16 [r, K]
  int64_t groups;      // work items: T * K / 8 (apply), ceil(T / 4) * K / 8 (dx add)
  int64_t g0;          // first group index of this problem in the launch
  int64_t K;
  uint64_t seed, offset;
  uint32_t thr;
  float scale;
};

struct DropParams {
  DropProblem p[kMaxDrop];
  int n, r, T;
  float s;
  int64_t total;  // work items over all problems
};

__device__ __forceinline__ int drop_problem(const DropParams& P, int64_t g) {
  int q = 0;
  while (q + 1 < P.n && g >= P.p[q + 1].g0) ++q;
  return q;
}

// keep bits of the 8 elements 8g .. 8g+7 (bit i = element 8g + i)
__device__ __forceinline__ uint32_t keep8(const DropProblem& pr, int64_t g) {
  uint32_t bits = 0;
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const Philox4 w = dropout_words(static_cast<uint64_t>(2 * g + h), pr.seed, pr.offset);
#pragma unroll
    for (int i = 0; i < 4; ++i)
      bits |= ((w.w[i] >> 8) >= pr.thr ? 1u : 0u) << (4 * h + i);
  }
  return bits;
}

__global__ void __launch_bounds__(256) lora_dropout_apply(const __grid_constant__ DropParams P) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < P.total;
       g += stride) {
    const DropProblem& pr = P.p[drop_problem(P, g)];
    const int64_t lg = g - pr.g0;
    const uint32_t keep = keep8(pr, lg);
    const uint4 x = __ldg(reinterpret_cast<const uint4*>(pr.X) + lg);
    const uint32_t xs[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float lo = __fmul_rn(__uint_as_float(xs[h] << 16), pr.scale);
      const float hi = __fmul_rn(__uint_as_float(xs[h] & 0xFFFF0000u), pr.scale);
      const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
      uint32_t bits = *reinterpret_cast<const uint32_t*>(&v);
      if (!((keep >> (2 * h)) & 1u)) bits &= 0xFFFF0000u;
      if (!((keep >> (2 * h + 1)) & 1u)) bits &= 0x0000FFFFu;
      o[h] = bits;
    }
    reinterpret_cast<uint4*>(pr.out)[lg] = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

// dx add: a thread owns 8 consecutive columns of 4 consecutive tokens, so
// each 16-byte row of A serves 32 elements
__global__ void __launch_bounds__(256) lora_dx_dropout_add(const __grid_constant__ DropParams P) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < P.total;
       g += stride) {
    const DropProblem& pr = P.p[drop_problem(P, g)];
    const int64_t lg = g - pr.g0;
    const int64_t k8 = pr.K / 8;
    const int64_t t0 = (lg / k8) * 4, k0 = (lg % k8) * 8;
    const int nt = static_cast<int>((P.T - t0) < 4 ? (P.T - t0) : 4);
    // adapter term: lora[tt][i] = sum_j u[t0 + tt, j] A[j, k0 + i]
    float lora[4][8];
#pragma unroll
    for (int tt = 0; tt < 4; ++tt)
#pragma unroll
      for (int i = 0; i < 8; ++i) lora[tt][i] = 0.0f;
    for (int j0 = 0; j0 < P.r; j0 += 4) {  // r % 8 == 0
      // four rows of A and the four tokens' u[j0 .. j0 + 3], all loads first
      uint4 a[4];
      float4 uq[4];
#pragma unroll
      for (int jj = 0; jj < 4; ++jj)
        a[jj] = __ldg(reinterpret_cast<const uint4*>(pr.A + (j0 + jj) * pr.K + k0));
#pragma unroll
      for (int tt = 0; tt < 4; ++tt)
        uq[tt] = tt < nt ? __ldg(reinterpret_cast<const float4*>(pr.u + (t0 + tt) * P.r + j0))
                         : make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int jj = 0; jj < 4; ++jj) {
        const uint32_t as[4] = {a[jj].x, a[jj].y, a[jj].z, a[jj].w};
        float af[8];
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          af[2 * h] = __uint_as_float(as[h] << 16);
          af[2 * h + 1] = __uint_as_float(as[h] & 0xFFFF0000u);
        }
#pragma unroll
        for (int tt = 0; tt < 4; ++tt) {
          const float uj = jj == 0 ? uq[tt].x : jj == 1 ? uq[tt].y : jj == 2 ? uq[tt].z : uq[tt].w;
#pragma unroll
          for (int i = 0; i < 8; ++i) lora[tt][i] = __fmaf_rn(uj, af[i], lora[tt][i]);
        }
      }
    }
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      if (tt >= nt) break;
      const int64_t e8 = ((t0 + tt) * pr.K + k0) / 8;  // this row segment's 8-element group
      const uint32_t keep = keep8(pr, e8);
      uint4* dst = reinterpret_cast<uint4*>(pr.out) + e8;
      const uint4 d = *dst;
      const uint32_t ds[4] = {d.x, d.y, d.z, d.w};
      uint32_t o[4];
#pragma unroll
      for (int h = 0; h < 4; ++h) {
        float lo = __uint_as_float(ds[h] << 16), hi = __uint_as_float(ds[h] & 0xFFFF0000u);
        if ((keep >> (2 * h)) & 1u)
          lo = __fadd_rn(lo, __fmul_rn(__fmul_rn(P.s, lora[tt][2 * h]), pr.scale));
        if ((keep >> (2 * h + 1)) & 1u)
          hi = __fadd_rn(hi, __fmul_rn(__fmul_rn(P.s, lora[tt][2 * h + 1]), pr.scale));
        const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
        o[h] = *reinterpret_cast<const uint32_t*>(&v);
      }
      *dst = make_uint4(o[0], o[1], o[2], o[3]);
    }
  }
}

static cudaError_t launch_drop(bool dx, const DropDesc* d, int n, int64_t T, int r, float s,
                               cudaStream_t st) {
  if (n < 1 || n > kMaxDrop) return cudaErrorInvalidValue;
  DropParams P;
  memset(&P, 0, sizeof P);
  P.n = n;
  P.r = r;
  P.T = static_cast<int>(T);
  P.s = s;
  int64_t g = 0;
  for (int q = 0; q < n; ++q) {
    DropProblem& pr = P.p[q];
    const DropoutParams dp = make_dropout(d[q].p, d[q].seed, d[q].offset);
    pr.X = static_cast<const uint16_t*>(d[q].X);
    pr.out = static_cast<uint16_t*>(d[q].out);
    pr.u = d[q].u;
    pr.A = static_cast<const uint16_t*>(d[q].A);
    pr.K = d[q].K;
    // apply: one item per 8 elements; dx add: 8 columns x 4 tokens
    pr.groups = dx ? (T + 3) / 4 * (d[q].K / 8) : T * d[q].K / 8;
    pr.g0 = g;
    pr.seed = dp.seed;
    pr.offset = dp.offset;
    pr.thr = dp.thr;
    pr.scale = dp.scale;
    g += pr.groups;
  }
  P.total = g;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (g + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 16) grid = static_cast<int64_t>(sms) * 16;
  if (grid < 1) grid = 1;
  count_launch();
  if (dx)
    lora_dx_dropout_add<<<static_cast<unsigned>(grid), 256, 0, st>>>(P);
  else
    lora_dropout_apply<<<static_cast<unsigned>(grid), 256, 0, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_dropout_apply(const DropDesc* d, int n, int64_t T, cudaStream_t st) {
  return launch_drop(false, d, n, T, 0, 0.0f, st);
}

cudaError_t launch_dx_dropout_add(const DropDesc* d, int n, int64_t T, int r, float s,
                                  cudaStream_t st) {
  return launch_drop(true, d, n, T, r, s, st);
}

}  // namespace hsnf4
