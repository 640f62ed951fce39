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
// m16n8k16, fp32 accumulate) over 64-token x 128..1024-column chunks and
// writes a partial per chunk; a second pass adds the chunks in chunk order.  grad also
// runs on mma.sync: Z is exact in bf16 and the fp32 V is split into
// V = hi + lo (two bf16 numbers, |lo| <= 2^-9 |V|), both multiplied, so each
// product keeps ~16 significant bits and accumulates in fp32, in a fixed
// token order.  Both are bound by reading Z once.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"

namespace hsnf4 {

constexpr int kMaxAux = 16;

// ---------------------------------------------------------------- project
// CTA = 64 tokens x one chunk of the contraction (128 to 1024 columns),
// walked in 128-column sub-chunks through a 3-stage cp.async ring in shared
// memory, so two sub-chunks are in flight while one is multiplied.  Warp
// tiles of 16 tokens x 8 rank columns keep their accumulators across the
// sub-chunks; one fp32 partial per chunk.  The launch takes the widest chunk
// that still gives every SM four CTAs (two resident, two waves), so short
// token counts keep the grid wide and long ones keep the partial sums few.

constexpr int kPrjTok = 64;          // tokens per CTA
constexpr int kPrjSub = 128;         // columns per sub-chunk (one ring stage)
constexpr int kPrjColsMax = 1024;    // widest chunk
constexpr int kPrjColsMin = kPrjSub; // narrowest chunk (sizes the workspace)
constexpr int kPrjLd = kPrjSub + 8;  // padded smem row (bf16): conflict-free fragment loads
constexpr int kPrjStages = 3;
constexpr int kPrjZBytes = kPrjTok * kPrjLd * 2;   // Z tile [64][136]
// adapter tile: A [r, C] staged [j][136] (<= 64 rows), B [C, r] staged [c][R + 8]
constexpr int kPrjABytes = (64 * kPrjLd * 2) > (kPrjSub * 72 * 2) ? (64 * kPrjLd * 2)
                                                                 : (kPrjSub * 72 * 2);
constexpr int kPrjStageBytes = kPrjZBytes + kPrjABytes;
constexpr int kPrjSmem = kPrjStages * kPrjStageBytes;

struct PrjProblem {
  const uint16_t* Z;
  const uint16_t* adp;
  float* t_out;
  uint16_t* zs;
  float* partial;  // [chunks][T][r_pad]
  int64_t C;
  int r_major, chunks, item0;  // item0: first CTA index of this problem
  int zero_zs;
};

struct PrjParams {
  PrjProblem p[kMaxAux];
  int n, T, r, r_pad, t_tiles, cols;  // cols: chunk width
  float s;
};

// index of the problem whose CTA range holds `item` (problems are laid out
// back to back; the scan reads the kernel parameters in place)
template <typename Prob>
__device__ __forceinline__ int find_problem(const Prob* p, int n, int item) {
  int q = 0;
  while (q + 1 < n && item >= p[q + 1].item0) ++q;
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

// 16-byte global -> shared copy; src_bytes 0 writes zeros and reads nothing
__device__ __forceinline__ void cp_async16(uint32_t dst, const void* src, int src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(dst), "l"(src),
               "r"(src_bytes)
               : "memory");
}
__device__ __forceinline__ void cp_async_commit() {
  asm volatile("cp.async.commit_group;" ::: "memory");
}
template <int N>
__device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

__device__ __forceinline__ void ldmatrix_x2_trans(uint32_t& d0, uint32_t& d1, uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
               : "=r"(d0), "=r"(d1)
               : "r"(addr));
}

// Issue the copies of one sub-chunk [c0, c0 + 128) into a ring stage: the Z
// tile (64 x 128 bf16 = 1024 16-byte pieces, 4 per thread) and the adapter
// tile (at most 1024 pieces, 4 per thread).  Rows past T, columns past C and
// rank indices past r are written as zeros.
__device__ __forceinline__ void prj_issue(const PrjParams& P, const PrjProblem& pr, int t0,
                                          int64_t c0, uint32_t stage) {
  const int tid = threadIdx.x, R = P.r_pad;
  const int width = static_cast<int>((pr.C - c0) < kPrjSub ? (pr.C - c0) : kPrjSub);
  const uint32_t zt = stage, at = stage + kPrjZBytes;
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const int v = tid + k * 256;
    const int row = v >> 4, col = (v & 15) * 8;
    const bool ok = t0 + row < P.T && col < width;
    const uint16_t* src = ok ? pr.Z + static_cast<int64_t>(t0 + row) * pr.C + c0 + col : pr.Z;
    cp_async16(zt + (row * kPrjLd + col) * 2, src, ok ? 16 : 0);
  }
  if (pr.r_major) {  // A [r, C]: stage row j holds A[j, c0 .. c0 + 127]
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v = tid + k * 256;
      const int j = v >> 4, col = (v & 15) * 8;
      if (j < R) {
        const bool ok = j < P.r && col < width;
        const uint16_t* src = ok ? pr.adp + static_cast<int64_t>(j) * pr.C + c0 + col : pr.adp;
        cp_async16(at + (j * kPrjLd + col) * 2, src, ok ? 16 : 0);
      }
    }
  } else {  // B [C, r]: stage row c holds B[c0 + c, 0 .. R - 1]
    const int per_row = R / 8;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v = tid + k * 256;
      const int c = v / per_row, jq = (v % per_row) * 8;
      if (c < kPrjSub) {
        const bool ok = c < width && jq < P.r;
        const uint16_t* src = ok ? pr.adp + (c0 + c) * P.r + jq : pr.adp;
        cp_async16(at + (c * (R + 8) + jq) * 2, src, ok ? 16 : 0);
      }
    }
  }
}

__global__ void __launch_bounds__(256, 2) lora_project_chunks(const __grid_constant__ PrjParams P) {
  extern __shared__ __align__(128) uint8_t prj_smem[];
  const int q = find_problem(P.p, P.n, blockIdx.x);
  const PrjProblem& pr = P.p[q];
  const int local = blockIdx.x - pr.item0;
  const int tt = local % P.t_tiles, chunk = local / P.t_tiles;
  const int t0 = tt * kPrjTok;
  const int64_t cb = static_cast<int64_t>(chunk) * P.cols;
  const int64_t ce = (cb + P.cols) < pr.C ? (cb + P.cols) : pr.C;
  const int n_sub = static_cast<int>((ce - cb + kPrjSub - 1) / kPrjSub);
  const int R = P.r_pad;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int n_tiles = (kPrjTok / 16) * (R / 8);  // 8 .. 32 warp tiles
  const uint32_t base = static_cast<uint32_t>(__cvta_generic_to_shared(prj_smem));
  float acc[4][4];
#pragma unroll
  for (int w = 0; w < 4; ++w)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[w][e] = 0.0f;

#pragma unroll
  for (int i = 0; i < kPrjStages - 1; ++i) {
    if (i < n_sub) prj_issue(P, pr, t0, cb + static_cast<int64_t>(i) * kPrjSub,
                             base + i * kPrjStageBytes);
    cp_async_commit();
  }
  for (int i = 0; i < n_sub; ++i) {
    cp_async_wait<kPrjStages - 2>();  // this thread's copies of sub-chunk i landed
    __syncthreads();                  // everyone's did; stage (i - 1) is free again
    const int nx = i + kPrjStages - 1;
    if (nx < n_sub) prj_issue(P, pr, t0, cb + static_cast<int64_t>(nx) * kPrjSub,
                              base + (nx % kPrjStages) * kPrjStageBytes);
    cp_async_commit();
    const uint8_t* stage = prj_smem + (i % kPrjStages) * kPrjStageBytes;
    const uint16_t* zt = reinterpret_cast<const uint16_t*>(stage);
    const uint16_t* at = reinterpret_cast<const uint16_t*>(stage + kPrjZBytes);
    const uint32_t at_u32 = base + (i % kPrjStages) * kPrjStageBytes + kPrjZBytes;
#pragma unroll
    for (int w = 0; w < 4; ++w) {
      const int wt = warp + 8 * w;
      if (wt >= n_tiles) break;
      const int m0 = (wt % (kPrjTok / 16)) * 16, n0 = (wt / (kPrjTok / 16)) * 8;
#pragma unroll
      for (int k0 = 0; k0 < kPrjSub; k0 += 16) {
        const uint16_t* ar = zt + (m0 + g) * kPrjLd + k0 + 2 * qd;
        uint32_t b0, b1;
        if (pr.r_major) {
          const uint16_t* br = at + (n0 + g) * kPrjLd + k0 + 2 * qd;
          b0 = *reinterpret_cast<const uint32_t*>(br);
          b1 = *reinterpret_cast<const uint32_t*>(br + 8);
        } else {  // rows k0 .. k0 + 15 of the [c][R + 8] tile, columns n0 .. n0 + 7
          ldmatrix_x2_trans(b0, b1, at_u32 + ((k0 + (lane & 15)) * (R + 8) + n0) * 2);
        }
        mma_bf16_16816(acc[w], *reinterpret_cast<const uint32_t*>(ar),
                       *reinterpret_cast<const uint32_t*>(ar + 8 * kPrjLd),
                       *reinterpret_cast<const uint32_t*>(ar + 8),
                       *reinterpret_cast<const uint32_t*>(ar + 8 * kPrjLd + 8), b0, b1);
      }
    }
  }
  cp_async_wait<0>();
  float* part = pr.partial + static_cast<int64_t>(chunk) * P.T * R;
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int wt = warp + 8 * w;
    if (wt >= n_tiles) break;
    const int m0 = (wt % (kPrjTok / 16)) * 16, n0 = (wt / (kPrjTok / 16)) * 8;
    const int ta = t0 + m0 + g, tb = ta + 8, j = n0 + 2 * qd;
    if (ta < P.T)
      *reinterpret_cast<float2*>(part + static_cast<int64_t>(ta) * R + j) =
          make_float2(acc[w][0], acc[w][1]);
    if (tb < P.T)
      *reinterpret_cast<float2*>(part + static_cast<int64_t>(tb) * R + j) =
          make_float2(acc[w][2], acc[w][3]);
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
    // loads run ahead in batches of 8; the adds stay in chunk order
    float v = 0.0f;
    const float* src = pr.partial + e;
    int ch = 0;
    for (; ch + 8 <= pr.chunks; ch += 8) {
      float x[8];
#pragma unroll
      for (int k = 0; k < 8; ++k) x[k] = __ldg(src + static_cast<int64_t>(ch + k) * per);
#pragma unroll
      for (int k = 0; k < 8; ++k) v += x[k];
    }
    for (; ch < pr.chunks; ++ch) v += __ldg(src + static_cast<int64_t>(ch) * per);
    pr.t_out[static_cast<int64_t>(t) * P.r + j] = v;
    const __nv_bfloat16 b = __float2bfloat16_rn(__fmul_rn(P.s, v));
    out = pr.zero_zs ? 0 : *reinterpret_cast<const uint16_t*>(&b);
  }
  pr.zs[static_cast<int64_t>(t) * P.r_pad + j] = out;
}

size_t project_workspace_bytes(const ProjectDesc* d, int n, int64_t T, int r) {
  const int r_pad = (r + 15) / 16 * 16;
  size_t total = 0;
  for (int q = 0; q < n; ++q) {
    const int64_t chunks = (d[q].C + kPrjColsMin - 1) / kPrjColsMin;
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
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  auto grid_for = [&](int cols) {
    int64_t items = 0;
    for (int q = 0; q < n; ++q) items += (d[q].C + cols - 1) / cols * P.t_tiles;
    return items;
  };
  P.cols = kPrjColsMax;
  while (P.cols > kPrjColsMin && grid_for(P.cols) < 4 * sms) P.cols /= 2;
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
    p.zero_zs = d[q].zero_zs ? 1 : 0;
    p.chunks = static_cast<int>((d[q].C + P.cols - 1) / P.cols);
    p.partial = reinterpret_cast<float*>(w);
    w += round_up(static_cast<size_t>(p.chunks) * T * P.r_pad * 4, 256);
    p.item0 = items;
    items += p.chunks * P.t_tiles;
  }
  static cudaError_t smem_rc = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    smem_rc = cudaFuncSetAttribute(lora_project_chunks,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize, kPrjSmem);
  });
  if (smem_rc != cudaSuccess) return smem_rc;
  count_launch();
  lora_project_chunks<<<items, 256, kPrjSmem, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const int64_t outs = static_cast<int64_t>(n) * T * P.r_pad;
  count_launch();
  lora_project_sum<<<static_cast<unsigned>((outs + 255) / 256), 256, 0, st>>>(P);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- grad
// out[c, j] = s * sum_t Z[t, c] V[t, j] as D = A B with A = Z^T (16 columns
// c x 16 tokens per mma) and B = V (16 tokens x 8 rank indices).  A CTA owns
// 64 columns and one 16-wide rank block: 8 warps, each a 16 x 8 output tile,
// over all tokens in chunks of 64 (Z chunk staged row-major and read with
// ldmatrix.trans; V staged transposed as bf16 hi and lo parts).

constexpr int kGrdCols = 64;
constexpr int kGrdTok = 64;
constexpr int kGrdLdZ = kGrdCols + 8;   // padded Z row (bf16): conflict-free ldmatrix
constexpr int kGrdLdV = kGrdTok + 8;    // padded V^T row (bf16)

struct GrdProblem {
  const uint16_t* Z;
  const float* V;
  float* out;
  int64_t C;
  int c_major, item0;
};

struct GrdParams {
  GrdProblem p[kMaxAux];
  int n, T, r, jblocks;
  float s;
};

__device__ __forceinline__ void ldmatrix_x4_trans(uint32_t (&d)[4], const void* smem_row) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(d[0]), "=r"(d[1]), "=r"(d[2]), "=r"(d[3])
               : "r"(static_cast<uint32_t>(__cvta_generic_to_shared(smem_row))));
}

__global__ void __launch_bounds__(256) lora_grad_group(const __grid_constant__ GrdParams P) {
  __shared__ __align__(16) uint16_t zt[kGrdTok * kGrdLdZ];
  __shared__ __align__(16) uint16_t vhi[16 * kGrdLdV];
  __shared__ __align__(16) uint16_t vlo[16 * kGrdLdV];
  const int q = find_problem(P.p, P.n, blockIdx.x);
  const GrdProblem& pr = P.p[q];
  const int local = blockIdx.x - pr.item0;
  const int jb = (local % P.jblocks) * 16;
  const int64_t c0 = static_cast<int64_t>(local / P.jblocks) * kGrdCols;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int mt = (warp & 3) * 16, nt = (warp >> 2) * 8;  // this warp's 16 columns, 8 ranks
  const int width = static_cast<int>((pr.C - c0) < kGrdCols ? (pr.C - c0) : kGrdCols);
  const int jn = (P.r - jb) < 16 ? (P.r - jb) : 16;

  float acc[4] = {0.f, 0.f, 0.f, 0.f};
  // register staging of token chunks: Z 64 x 64 bf16 (2 x 16 B per thread)
  // and V 64 x 16 fp32 (4 per thread).  Two sets, so that the loads of the
  // next two chunks are in flight while one is multiplied.
  uint4 zr[2][2];
  float vr[2][4];
  auto load = [&](int set, int tc) {
    const int nt_tok = (P.T - tc) < kGrdTok ? (P.T - tc) : kGrdTok;
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = tid + k * 256;
      const int row = v >> 3, col = (v & 7) * 8;
      zr[set][k] = make_uint4(0, 0, 0, 0);
      if (row < nt_tok && col < width)
        zr[set][k] = __ldg(reinterpret_cast<const uint4*>(
            pr.Z + static_cast<int64_t>(tc + row) * pr.C + c0 + col));
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v = tid + k * 256;
      const int row = v >> 4, j = v & 15;
      vr[set][k] = (row < nt_tok && j < jn)
                       ? __ldg(pr.V + static_cast<int64_t>(tc + row) * P.r + jb + j)
                       : 0.0f;
    }
  };
  auto chunk = [&](int set, int tc) {
    __syncthreads();
#pragma unroll
    for (int k = 0; k < 2; ++k) {
      const int v = tid + k * 256;
      *reinterpret_cast<uint4*>(zt + (v >> 3) * kGrdLdZ + (v & 7) * 8) = zr[set][k];
    }
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const int v = tid + k * 256;
      const int row = v >> 4, j = v & 15;
      const __nv_bfloat16 hi = __float2bfloat16_rn(vr[set][k]);
      const __nv_bfloat16 lo = __float2bfloat16_rn(__fsub_rn(vr[set][k], __bfloat162float(hi)));
      vhi[j * kGrdLdV + row] = *reinterpret_cast<const uint16_t*>(&hi);
      vlo[j * kGrdLdV + row] = *reinterpret_cast<const uint16_t*>(&lo);
    }
    __syncthreads();
    if (tc + 2 * kGrdTok < P.T) load(set, tc + 2 * kGrdTok);  // refill the set just staged
#pragma unroll
    for (int k0 = 0; k0 < kGrdTok; k0 += 16) {
      // A = Z^T: submatrices (c 0-7 | 8-15) x (t 0-7 | 8-15), each the transpose
      // of an 8 x 8 block of the row-major Z chunk
      uint32_t a[4];
      const int mrow = lane & 7, which = lane >> 3;  // which: 0..3 -> (c+0,t+0) (c+8,t+0) (c+0,t+8) (c+8,t+8)
      const uint16_t* src = zt + (k0 + mrow + (which >> 1) * 8) * kGrdLdZ + mt + (which & 1) * 8;
      ldmatrix_x4_trans(a, src);
      const uint32_t bh0 = *reinterpret_cast<const uint32_t*>(vhi + (nt + g) * kGrdLdV + k0 + 2 * qd);
      const uint32_t bh1 = *reinterpret_cast<const uint32_t*>(vhi + (nt + g) * kGrdLdV + k0 + 8 + 2 * qd);
      const uint32_t bl0 = *reinterpret_cast<const uint32_t*>(vlo + (nt + g) * kGrdLdV + k0 + 2 * qd);
      const uint32_t bl1 = *reinterpret_cast<const uint32_t*>(vlo + (nt + g) * kGrdLdV + k0 + 8 + 2 * qd);
      mma_bf16_16816(acc, a[0], a[1], a[2], a[3], bh0, bh1);
      mma_bf16_16816(acc, a[0], a[1], a[2], a[3], bl0, bl1);
    }
  };
  load(0, 0);
  if (kGrdTok < P.T) load(1, kGrdTok);
  for (int tc = 0; tc < P.T; tc += 2 * kGrdTok) {  // chunk order (and sum order) unchanged
    chunk(0, tc);
    if (tc + kGrdTok < P.T) chunk(1, tc + kGrdTok);
  }
  // acc: (c = mt+g, j = nt+2qd, +1) and (c = mt+g+8, same j)
#pragma unroll
  for (int h = 0; h < 2; ++h) {
    const int cl = mt + g + 8 * h;
    if (cl >= width) continue;
    const int64_t c = c0 + cl;
#pragma unroll
    for (int e = 0; e < 2; ++e) {
      const int j = nt + 2 * qd + e;
      if (j >= jn) continue;
      const float val = __fmul_rn(P.s, acc[2 * h + e]);
      if (pr.c_major)
        pr.out[c * P.r + jb + j] = val;
      else
        pr.out[static_cast<int64_t>(jb + j) * pr.C + c] = val;
    }
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
  P.jblocks = (r + 15) / 16;
  int items = 0;
  for (int q = 0; q < n; ++q) {
    GrdProblem& p = P.p[q];
    p.Z = static_cast<const uint16_t*>(d[q].Z);
    p.V = d[q].V;
    p.out = d[q].out;
    p.C = d[q].C;
    p.c_major = d[q].c_major ? 1 : 0;
    p.item0 = items;
    items += static_cast<int>((d[q].C + kGrdCols - 1) / kGrdCols) * P.jblocks;
  }
  count_launch();
  lora_grad_group<<<items, 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace hsnf4
