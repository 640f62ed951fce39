// lora_aux.cu -- the rank-r pieces of the LoRA linear around the fused GEMM,
// for a group of independent problems per launch.
//
//   project:  t = Z Adp^T   (Z bf16 [T, C]; adapter A [r, C] or B [C, r])
//             writes t (fp32 [T, r]) and zs = bf16(s * t) ([T, r_pad], pad
//             columns zero), the operand of the GEMM's rank-r slice.
//             forward:  t = X A^T  (Adp = A);   backward: u = dY B  (Adp = B)
//   grad:     out = s Z^T V (Z bf16 [T, C], V fp32 [T, r])
//             dB = s dY^T t  ([n_out, r]),   dA = s u^T X  ([r, k_in])
//
// project multiplies exact bf16 inputs on the tensor cores (mma.sync
// m16n8k16, fp32 accumulate) over 64-token x 128-column chunks and writes a
// partial per chunk; a second pass adds the chunks in chunk order.  grad keeps
// V in fp32 and runs on the CUDA cores with 4 x 4 register tiles; each output
// is a fixed-order sum.  Both are bound by reading Z once.
#include <cuda_bf16.h>

#include "internal.h"

namespace hsnf4 {

constexpr int kMaxAux = 16;

// ---------------------------------------------------------------- project

constexpr int kPrjTok = 64;   // tokens per chunk
constexpr int kPrjCols = 128; // contraction columns per chunk
constexpr int kPrjLd = kPrjCols + 8;  // padded smem row (bf16): conflict-free fragment loads

struct PrjProblem {
  const uint16_t* Z;
  const uint16_t* adp;
  float* t_out;
  uint16_t* zs;
  float* partial;  // [chunks][T][r_pad]
  int64_t C;
  int r_major, chunks, item0;  // item0: first CTA index of this problem
};

struct PrjParams {
  PrjProblem p[kMaxAux];
  int n, T, r, r_pad, t_tiles;
  float s;
};

__device__ __forceinline__ int find_problem(const int* item0, int n, int item) {
  int q = 0;
  while (q + 1 < n && item >= item0[q + 1]) ++q;
  return q;
}

__device__ __forceinline__ void mma_bf16_16816(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                               uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) lora_project_chunks(const __grid_constant__ PrjParams P) {
  __shared__ __align__(16) uint16_t zs_tile[kPrjTok * kPrjLd];
  __shared__ __align__(16) uint16_t ad_tile[64 * kPrjLd];
  int item0[kMaxAux];
#pragma unroll
  for (int q = 0; q < kMaxAux; ++q) item0[q] = q < P.n ? P.p[q].item0 : 0x7fffffff;
  const int q = find_problem(item0, P.n, blockIdx.x);
  const PrjProblem& pr = P.p[q];
  const int local = blockIdx.x - pr.item0;
  const int tt = local % P.t_tiles, chunk = local / P.t_tiles;
  const int t0 = tt * kPrjTok;
  const int64_t c0 = static_cast<int64_t>(chunk) * kPrjCols;
  const int R = P.r_pad;
  const int tid = threadIdx.x;

  // Z chunk: 64 rows x 128 columns, 16-byte loads (C % 64 == 0, so a chunk is
  // 64 or 128 columns wide)
  const int width = static_cast<int>((pr.C - c0) < kPrjCols ? (pr.C - c0) : kPrjCols);
  for (int v = tid; v < kPrjTok * (kPrjCols / 8); v += 256) {
    const int row = v / (kPrjCols / 8), col = (v % (kPrjCols / 8)) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (t0 + row < P.T && col < width)
      val = __ldg(reinterpret_cast<const uint4*>(pr.Z + static_cast<int64_t>(t0 + row) * pr.C +
                                                 c0 + col));
    *reinterpret_cast<uint4*>(zs_tile + row * kPrjLd + col) = val;
  }
  // adapter chunk as [j][c] (bf16), rows j >= r zero
  if (pr.r_major) {
    for (int v = tid; v < R * (kPrjCols / 8); v += 256) {
      const int j = v / (kPrjCols / 8), col = (v % (kPrjCols / 8)) * 8;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (j < P.r && col < width)
        val = __ldg(reinterpret_cast<const uint4*>(pr.adp + static_cast<int64_t>(j) * pr.C + c0 +
                                                   col));
      *reinterpret_cast<uint4*>(ad_tile + j * kPrjLd + col) = val;
    }
  } else {
    // B is [C, r]: each 16-byte load holds 8 consecutive j of one column c
    const int per_row = P.r / 8;
    for (int v = tid; v < kPrjCols * (R / 8); v += 256) {
      const int c = v / (R / 8), jq = (v % (R / 8)) * 8;
      uint4 val = make_uint4(0, 0, 0, 0);
      if (c < width && jq < P.r)
        val = __ldg(reinterpret_cast<const uint4*>(pr.adp + (c0 + c) * P.r) + jq / 8);
      (void)per_row;
      const uint32_t w[4] = {val.x, val.y, val.z, val.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        ad_tile[(jq + 2 * e) * kPrjLd + c] = static_cast<uint16_t>(w[e] & 0xFFFFu);
        ad_tile[(jq + 2 * e + 1) * kPrjLd + c] = static_cast<uint16_t>(w[e] >> 16);
      }
    }
  }
  __syncthreads();

  // warp tiles: 16 tokens x 8 rank columns over the chunk's 128 columns
  const int warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int n_tiles = (kPrjTok / 16) * (R / 8);
  for (int wt = warp; wt < n_tiles; wt += 8) {
    const int m0 = (wt % (kPrjTok / 16)) * 16, n0 = (wt / (kPrjTok / 16)) * 8;
    float c[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
    for (int k0 = 0; k0 < kPrjCols; k0 += 16) {
      const uint16_t* ar = zs_tile + (m0 + g) * kPrjLd + k0 + 2 * qd;
      const uint16_t* br = ad_tile + (n0 + g) * kPrjLd + k0 + 2 * qd;
      const uint32_t a0 = *reinterpret_cast<const uint32_t*>(ar);
      const uint32_t a1 = *reinterpret_cast<const uint32_t*>(ar + 8 * kPrjLd);
      const uint32_t a2 = *reinterpret_cast<const uint32_t*>(ar + 8);
      const uint32_t a3 = *reinterpret_cast<const uint32_t*>(ar + 8 * kPrjLd + 8);
      const uint32_t b0 = *reinterpret_cast<const uint32_t*>(br);
      const uint32_t b1 = *reinterpret_cast<const uint32_t*>(br + 8);
      mma_bf16_16816(c, a0, a1, a2, a3, b0, b1);
    }
    float* part = pr.partial + static_cast<int64_t>(chunk) * P.T * R;
    const int ta = t0 + m0 + g, tb = ta + 8, j = n0 + 2 * qd;
    if (ta < P.T) *reinterpret_cast<float2*>(part + static_cast<int64_t>(ta) * R + j) = make_float2(c[0], c[1]);
    if (tb < P.T) *reinterpret_cast<float2*>(part + static_cast<int64_t>(tb) * R + j) = make_float2(c[2], c[3]);
  }
}

// t[q][t][j] = sum over chunks (in order) of the partials; zs = bf16(s * t)
__global__ void __launch_bounds__(256) lora_project_sum(const __grid_constant__ PrjParams P) {
  const int per = P.T * P.r_pad;
  const int64_t idx = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  if (idx >= static_cast<int64_t>(per) * P.n) return;
  const int q = static_cast<int>(idx / per), e = static_cast<int>(idx % per);
  const PrjProblem& pr = P.p[q];
  const int t = e / P.r_pad, j = e % P.r_pad;
  uint16_t out = 0;
  if (j < P.r) {
    float v = 0.0f;
    for (int ch = 0; ch < pr.chunks; ++ch) v += __ldg(pr.partial + static_cast<int64_t>(ch) * per + e);
    pr.t_out[static_cast<int64_t>(t) * P.r + j] = v;
    const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(P.s, v));
    out = *reinterpret_cast<const uint16_t*>(&b);
  }
  pr.zs[static_cast<int64_t>(t) * P.r_pad + j] = out;
}

size_t project_workspace_bytes(const ProjectDesc* d, int n, int64_t T, int r) {
  const int r_pad = (r + 15) / 16 * 16;
  size_t total = 0;
  for (int q = 0; q < n; ++q) {
    const int64_t chunks = (d[q].C + kPrjCols - 1) / kPrjCols;
    total += round_up(static_cast<size_t>(chunks) * T * r_pad * 4, 256);
  }
  return total;
}

cudaError_t launch_lora_project_group(const ProjectDesc* d, int n, int64_t T, int r, float s,
                                      void* ws, cudaStream_t st) {
  if (n < 1 || n > kMaxAux) return cudaErrorInvalidValue;
  PrjParams P;
  memset(&P, 0, sizeof P);
  P.n = n;
  P.T = static_cast<int>(T);
  P.r = r;
  P.r_pad = (r + 15) / 16 * 16;
  P.s = s;
  P.t_tiles = static_cast<int>((T + kPrjTok - 1) / kPrjTok);
  uint8_t* w = static_cast<uint8_t*>(ws);
  int items = 0;
  for (int q = 0; q < n; ++q) {
    PrjProblem& p = P.p[q];
    p.Z = static_cast<const uint16_t*>(d[q].Z);
    p.adp = static_cast<const uint16_t*>(d[q].adp);
    p.t_out = d[q].t_out;
    p.zs = static_cast<uint16_t*>(d[q].zs);
    p.C = d[q].C;
    p.r_major = d[q].r_major ? 1 : 0;
    p.chunks = static_cast<int>((d[q].C + kPrjCols - 1) / kPrjCols);
    p.partial = reinterpret_cast<float*>(w);
    w += round_up(static_cast<size_t>(p.chunks) * T * P.r_pad * 4, 256);
    p.item0 = items;
    items += p.chunks * P.t_tiles;
  }
  lora_project_chunks<<<items, 256, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t outs = static_cast<int64_t>(n) * T * P.r_pad;
  lora_project_sum<<<static_cast<unsigned>((outs + 255) / 256), 256, 0, st>>>(P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- grad
// CTA = 64 columns.  Thread (cq, jq, tg): columns 4cq..4cq+3, rank indices
// 4jq..4jq+3 of the current 16-block, tokens t = tg (mod 4) in increasing
// order; the 4 token groups are then added in group order.

constexpr int kGrdCols = 64;
constexpr int kGrdTok = 64;

struct GrdProblem {
  const uint16_t* Z;
  const float* V;
  float* out;
  int64_t C;
  int c_major, item0;
};

struct GrdParams {
  GrdProblem p[kMaxAux];
  int n, T, r;
  float s;
};

__global__ void __launch_bounds__(256) lora_grad_group(const __grid_constant__ GrdParams P) {
  __shared__ __align__(16) uint16_t zt[kGrdTok * kGrdCols];
  __shared__ __align__(16) float vt[kGrdTok * 16];
  __shared__ __align__(16) float red[4][kGrdCols][16 + 1];
  int item0[kMaxAux];
#pragma unroll
  for (int q = 0; q < kMaxAux; ++q) item0[q] = q < P.n ? P.p[q].item0 : 0x7fffffff;
  const int q = find_problem(item0, P.n, blockIdx.x);
  const GrdProblem& pr = P.p[q];
  const int64_t c0 = static_cast<int64_t>(blockIdx.x - pr.item0) * kGrdCols;
  const int tid = threadIdx.x;
  const int cq = tid & 15, jq = (tid >> 4) & 3, tg = tid >> 6;
  const int width = static_cast<int>((pr.C - c0) < kGrdCols ? (pr.C - c0) : kGrdCols);

  for (int jb = 0; jb < P.r; jb += 16) {
    const int jn = (P.r - jb) < 16 ? (P.r - jb) : 16;  // 8 or 16
    float acc[4][4];
#pragma unroll
    for (int a = 0; a < 4; ++a)
#pragma unroll
      for (int b = 0; b < 4; ++b) acc[a][b] = 0.0f;
    for (int tc = 0; tc < P.T; tc += kGrdTok) {
      const int nt = (P.T - tc) < kGrdTok ? (P.T - tc) : kGrdTok;
      __syncthreads();
      for (int v = tid; v < kGrdTok * (kGrdCols / 8); v += 256) {
        const int row = v / (kGrdCols / 8), col = (v % (kGrdCols / 8)) * 8;
        uint4 val = make_uint4(0, 0, 0, 0);
        if (row < nt && col < width)
          val = __ldg(reinterpret_cast<const uint4*>(pr.Z + static_cast<int64_t>(tc + row) * pr.C +
                                                     c0 + col));
        *reinterpret_cast<uint4*>(zt + row * kGrdCols + col) = val;
      }
      for (int v = tid; v < kGrdTok * 16; v += 256) {
        const int row = v >> 4, j = v & 15;
        vt[v] = (row < nt && j < jn) ? __ldg(pr.V + static_cast<int64_t>(tc + row) * P.r + jb + j)
                                     : 0.0f;
      }
      __syncthreads();
      for (int i = tg; i < nt; i += 4) {
        const uint2 zz = *reinterpret_cast<const uint2*>(zt + i * kGrdCols + cq * 4);
        const float z[4] = {__uint_as_float(zz.x << 16), __uint_as_float(zz.x & 0xFFFF0000u),
                            __uint_as_float(zz.y << 16), __uint_as_float(zz.y & 0xFFFF0000u)};
        const float4 vv = *reinterpret_cast<const float4*>(vt + i * 16 + jq * 4);
        const float w[4] = {vv.x, vv.y, vv.z, vv.w};
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) acc[a][b] = fmaf(z[a], w[b], acc[a][b]);
      }
    }
    // token groups 0..3 added in order
    for (int g = 0; g < 4; ++g) {
      if (tg == g) {
#pragma unroll
        for (int a = 0; a < 4; ++a)
#pragma unroll
          for (int b = 0; b < 4; ++b) {
            float& dst = red[0][cq * 4 + a][jq * 4 + b];
            dst = (g == 0) ? acc[a][b] : dst + acc[a][b];
          }
      }
      __syncthreads();
    }
    for (int v = tid; v < kGrdCols * 16; v += 256) {
      const int cl = v >> 4, j = v & 15;
      if (cl < width && j < jn) {
        const float val = __fmul_rn(P.s, red[0][cl][j]);
        const int64_t c = c0 + cl;
        if (pr.c_major)
          pr.out[c * P.r + jb + j] = val;
        else
          pr.out[static_cast<int64_t>(jb + j) * pr.C + c] = val;
      }
    }
    __syncthreads();
  }
}

cudaError_t launch_lora_grad_group(const GradDesc* d, int n, int64_t T, int r, float s,
                                   cudaStream_t st) {
  if (n < 1 || n > kMaxAux) return cudaErrorInvalidValue;
  GrdParams P;
  memset(&P, 0, sizeof P);
  P.n = n;
  P.T = static_cast<int>(T);
  P.r = r;
  P.s = s;
  int items = 0;
  for (int q = 0; q < n; ++q) {
    GrdProblem& p = P.p[q];
    p.Z = static_cast<const uint16_t*>(d[q].Z);
    p.V = d[q].V;
    p.out = d[q].out;
    p.C = d[q].C;
    p.c_major = d[q].c_major ? 1 : 0;
    p.item0 = items;
    items += static_cast<int>((d[q].C + kGrdCols - 1) / kGrdCols);
  }
  lora_grad_group<<<items, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace hsnf4
