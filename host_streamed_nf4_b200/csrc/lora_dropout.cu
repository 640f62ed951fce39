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
// The mask is recomputed from (seed, offset), never kept across calls:
// element e = t K + k takes word e % 4 of the Philox block of e / 4
// (philox.cuh).  Within one backward call the apply pass also writes the
// mask as one byte per 8 elements to workspace, and the dx add that follows
// reads those bytes instead of running Philox a second time.  An apply thread owns 8
// consecutive elements of one row (16 bytes of bf16, two Philox blocks); a
// dx-add thread the same 8 columns of 4 consecutive rows.  Both kernels
// are HBM-bound elementwise passes: apply reads 2 B and writes 2 B per
// element, dx add reads 2 B and writes 2 B (u and A are re-read from L2).
#include <cuda_bf16.h>

#include "internal.h"
#include "ptx.cuh"
#include "philox.cuh"

namespace hsnf4 {

constexpr int kMaxDrop = 16;

struct DropProblem {
  const uint16_t* X;   // apply: input [T, K];  dx add: unused
  uint16_t* out;       // apply: X_d [T, K];    dx add: dX [T, K] (read and written)
  const float* u;      // dx add: u fp32 [T, r]
  const uint16_t* A;   // dx add: A bf16 [r, K]
  uint8_t* bits;       // keep mask bytes [T * K / 8], or null (apply: written; dx add: read)
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
  pdl_wait_then_release();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; g < P.total;
       g += stride) {
    const DropProblem& pr = P.p[drop_problem(P, g)];
    const int64_t lg = g - pr.g0;
    const uint32_t keep = keep8(pr, lg);
    if (pr.bits) pr.bits[lg] = static_cast<uint8_t>(keep);
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

// dx add: a CTA owns a tile of 32 tokens x 256 columns of one problem.  It
// stages the tile's slice of A ([r, 256] bf16) and of u ([32, r] fp32) in
// shared memory once, while each thread's dX rows and mask bytes are already
// in flight; thread (token group w, column group l) then forms its 4 tokens
// x 8 columns of u A from shared memory and updates dX.
constexpr int kDxTok = 32, kDxCols = 256, kDxMaxR = 64;

__global__ void __launch_bounds__(256) lora_dx_dropout_add(const __grid_constant__ DropParams P) {
  __shared__ __align__(16) uint16_t a_s[kDxMaxR * kDxCols];  // A[j][c], this tile's columns
  __shared__ __align__(16) float u_s[kDxTok * kDxMaxR];      // u[t][j], this tile's tokens
  pdl_wait_then_release();
  const int q = drop_problem(P, blockIdx.x);
  const DropProblem& pr = P.p[q];
  const int64_t local = static_cast<int64_t>(blockIdx.x) - pr.g0;
  const int64_t col_tiles = (pr.K + kDxCols - 1) / kDxCols;
  const int tt0 = static_cast<int>(local / col_tiles) * kDxTok;
  const int64_t c0 = (local % col_tiles) * kDxCols;
  const int width = static_cast<int>((pr.K - c0) < kDxCols ? (pr.K - c0) : kDxCols);
  const int tid = threadIdx.x, l = tid & 31, w = tid >> 5;
  const int r = P.r;
  const int t0 = tt0 + w * 4, k0 = l * 8;  // this thread's tokens and columns (tile-relative)
  const bool col_ok = k0 < width;

  // this thread's dX rows and mask bytes first: their latency overlaps the staging
  uint4 d[4];
  uint32_t keep[4];
#pragma unroll
  for (int tt = 0; tt < 4; ++tt) {
    d[tt] = make_uint4(0, 0, 0, 0);
    keep[tt] = 0;
    if (col_ok && t0 + tt < P.T) {
      const int64_t e8 = (static_cast<int64_t>(t0 + tt) * pr.K + c0 + k0) / 8;
      d[tt] = reinterpret_cast<const uint4*>(pr.out)[e8];
      keep[tt] = pr.bits ? static_cast<uint32_t>(__ldg(pr.bits + e8)) : keep8(pr, e8);
    }
  }
  // stage A[:, c0 .. c0 + 255] (16-byte pieces) and u[tt0 .. tt0 + 31, :]
  for (int v = tid; v < r * (kDxCols / 8); v += 256) {
    const int j = v / (kDxCols / 8), cc = (v % (kDxCols / 8)) * 8;
    uint4 x = make_uint4(0, 0, 0, 0);
    if (cc < width) x = __ldg(reinterpret_cast<const uint4*>(pr.A + static_cast<int64_t>(j) * pr.K +
                                                             c0 + cc));
    *reinterpret_cast<uint4*>(a_s + j * kDxCols + cc) = x;
  }
  for (int v = tid; v < kDxTok * r / 4; v += 256) {
    const int t = v / (r / 4), jq = (v % (r / 4)) * 4;
    float4 x = make_float4(0.f, 0.f, 0.f, 0.f);
    if (tt0 + t < P.T) x = __ldg(reinterpret_cast<const float4*>(pr.u + static_cast<int64_t>(tt0 + t) * r + jq));
    *reinterpret_cast<float4*>(u_s + t * r + jq) = x;
  }
  __syncthreads();
  if (!col_ok) return;
  // adapter term: lora[tt][i] = sum_j u[t0 + tt, j] A[j, k0 + i], in j order
  float lora[4][8];
#pragma unroll
  for (int tt = 0; tt < 4; ++tt)
#pragma unroll
    for (int i = 0; i < 8; ++i) lora[tt][i] = 0.0f;
  for (int j = 0; j < r; ++j) {
    const uint4 a = *reinterpret_cast<const uint4*>(a_s + j * kDxCols + k0);
    const uint32_t as[4] = {a.x, a.y, a.z, a.w};
    float af[8];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      af[2 * h] = __uint_as_float(as[h] << 16);
      af[2 * h + 1] = __uint_as_float(as[h] & 0xFFFF0000u);
    }
#pragma unroll
    for (int tt = 0; tt < 4; ++tt) {
      const float uj = u_s[(w * 4 + tt) * r + j];
#pragma unroll
      for (int i = 0; i < 8; ++i) lora[tt][i] = __fmaf_rn(uj, af[i], lora[tt][i]);
    }
  }
#pragma unroll
  for (int tt = 0; tt < 4; ++tt) {
    if (t0 + tt >= P.T) break;
    const int64_t e8 = (static_cast<int64_t>(t0 + tt) * pr.K + c0 + k0) / 8;
    const uint32_t ds[4] = {d[tt].x, d[tt].y, d[tt].z, d[tt].w};
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      float lo = __uint_as_float(ds[h] << 16), hi = __uint_as_float(ds[h] & 0xFFFF0000u);
      if ((keep[tt] >> (2 * h)) & 1u)
        lo = __fadd_rn(lo, __fmul_rn(__fmul_rn(P.s, lora[tt][2 * h]), pr.scale));
      if ((keep[tt] >> (2 * h + 1)) & 1u)
        hi = __fadd_rn(hi, __fmul_rn(__fmul_rn(P.s, lora[tt][2 * h + 1]), pr.scale));
      const __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
      o[h] = *reinterpret_cast<const uint32_t*>(&v);
    }
    reinterpret_cast<uint4*>(pr.out)[e8] = make_uint4(o[0], o[1], o[2], o[3]);
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
    pr.bits = d[q].bits;
    pr.K = d[q].K;
    // apply: one item per 8 elements; dx add: one CTA per 32 tokens x 256 columns
    pr.groups = dx ? (T + kDxTok - 1) / kDxTok * ((d[q].K + kDxCols - 1) / kDxCols)
                   : T * d[q].K / 8;
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
  if (dx) grid = g;  // one CTA per tile
  if (grid < 1) grid = 1;
  return launch_pdl(dx ? lora_dx_dropout_add : lora_dropout_apply,
                    dim3(static_cast<unsigned>(grid)), dim3(256), 0, st, P);
}

cudaError_t launch_dropout_apply(const DropDesc* d, int n, int64_t T, cudaStream_t st) {
  return launch_drop(false, d, n, T, 0, 0.0f, st);
}

cudaError_t launch_dx_dropout_add(const DropDesc* d, int n, int64_t T, int r, float s,
                                  cudaStream_t st) {
  return launch_drop(true, d, n, T, r, s, st);
}

}  // namespace hsnf4
