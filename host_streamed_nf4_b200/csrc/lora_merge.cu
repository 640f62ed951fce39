// lora_merge.cu -- merge the adapter into the frozen base (Poros API
// reference, PorosModel.merge_and_unload):
//
//     W'[n, k] = bf16_rne( fp32( deq(W)[n, k] + s * sum_j B[n, j] A[j, k] ) )
//
// with deq(W) the bf16 value of the base (NF4: bf16_rne(codebook * absmax);
// dense base: the weight itself) and s = alpha / r.  The rank-r sum runs on
// the tensor cores (mma.sync m16n8k16: exact bf16 products, fp32
// accumulate), is scaled by s in fp32, added to deq(W) in fp32 and rounded
// once to bf16.
//
// CTA = 32 rows x 128 columns of W'.  B's 32 x r rows and A's r x 128
// columns are staged in shared memory; the 8 warps compute the 32 x 128
// fp32 product into shared memory; then each thread expands 2 x 8
// consecutive base elements (one 32-bit code word each), adds the product
// and writes 16 bytes.  HBM traffic is the base read plus W' written (A and
// B are re-read from L2).
#include <cuda_bf16.h>

#include "internal.h"
#include "nf4_device.cuh"

namespace hsnf4 {

constexpr int kMrgRows = 32;
constexpr int kMrgCols = 128;
constexpr int kMrgLdA = kMrgCols + 8;  // A tile [r][136] bf16
constexpr int kMrgLdS = kMrgCols + 4;  // product tile [32][132] fp32

struct MergeParams {
  const void* base;      // NF4 codes (uint8) or dense bf16 weight
  const float* absmax;   // NF4 only
  const uint16_t* A;     // bf16 [r, K]
  const uint16_t* B;     // bf16 [N, r]
  uint16_t* out;         // bf16 [N, K]
  int64_t N, K;
  int r, r_pad, dense, col_tiles;
  float s;
  Nf4Codebook cb;
};

__device__ __forceinline__ void mrg_mma(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t a2,
                                        uint32_t a3, uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}

__global__ void __launch_bounds__(256) lora_merge_kernel(const __grid_constant__ MergeParams P) {
  __shared__ __align__(16) uint16_t bs[kMrgRows * 72];     // B tile [32][R + 8], R <= 64
  __shared__ __align__(16) uint16_t as[64 * kMrgLdA];      // A tile [R][136]
  __shared__ __align__(16) float ps[kMrgRows * kMrgLdS];   // s-free product [32][132]
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int g = lane >> 2, qd = lane & 3;
  const int R = P.r_pad, ldb = R + 8;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x / P.col_tiles) * kMrgRows;
  const int64_t k0 = static_cast<int64_t>(blockIdx.x % P.col_tiles) * kMrgCols;

  // ---- the base bytes of this thread's two 8-element groups, loaded first so
  // that their DRAM latency overlaps the staging and the product below
  uint4 wraw[2];
  float wabs[2];
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int v = tid + i * 256;
    const int row = v >> 4, col = (v & 15) * 8;
    wraw[i] = make_uint4(0, 0, 0, 0);
    wabs[i] = 0.0f;
    if (k0 + col >= P.K) continue;
    const int64_t e = (n0 + row) * P.K + k0 + col;
    if (P.dense) {
      wraw[i] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(P.base) + e));
    } else {
      wraw[i].x = __ldg(reinterpret_cast<const uint32_t*>(static_cast<const uint8_t*>(P.base) +
                                                          e / 2));
      wabs[i] = __ldg(P.absmax + e / 64);
    }
  }

  // ---- stage B rows n0.. (j < r, zeros up to R) and A columns k0.. (rows j < r)
  for (int v = tid; v < kMrgRows * (R / 8); v += 256) {
    const int row = v / (R / 8), jq = (v % (R / 8)) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (jq < P.r) val = __ldg(reinterpret_cast<const uint4*>(P.B + (n0 + row) * P.r + jq));
    *reinterpret_cast<uint4*>(bs + row * ldb + jq) = val;
  }
  for (int v = tid; v < R * (kMrgCols / 8); v += 256) {
    const int j = v / (kMrgCols / 8), col = (v % (kMrgCols / 8)) * 8;
    uint4 val = make_uint4(0, 0, 0, 0);
    if (j < P.r && k0 + col < P.K)
      val = __ldg(reinterpret_cast<const uint4*>(P.A + static_cast<int64_t>(j) * P.K + k0 + col));
    *reinterpret_cast<uint4*>(as + j * kMrgLdA + col) = val;
  }
  __syncthreads();

  // ---- product tile: 2 x 16 warp tiles of 16 rows x 8 columns, 4 per warp
  const uint32_t as_u32 = static_cast<uint32_t>(__cvta_generic_to_shared(as));
#pragma unroll
  for (int w = 0; w < 4; ++w) {
    const int wt = warp + 8 * w;
    const int m0 = (wt & 1) * 16, c0 = (wt >> 1) * 8;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int j0 = 0; j0 < R; j0 += 16) {
      const uint16_t* ar = bs + (m0 + g) * ldb + j0 + 2 * qd;
      uint32_t b0, b1;
      asm volatile("ldmatrix.sync.aligned.m8n8.x2.trans.shared.b16 {%0,%1}, [%2];"
                   : "=r"(b0), "=r"(b1)
                   : "r"(as_u32 + ((j0 + (lane & 15)) * kMrgLdA + c0) * 2));
      mrg_mma(acc, *reinterpret_cast<const uint32_t*>(ar),
              *reinterpret_cast<const uint32_t*>(ar + 8 * ldb),
              *reinterpret_cast<const uint32_t*>(ar + 8),
              *reinterpret_cast<const uint32_t*>(ar + 8 * ldb + 8), b0, b1);
    }
    *reinterpret_cast<float2*>(ps + (m0 + g) * kMrgLdS + c0 + 2 * qd) = make_float2(acc[0], acc[1]);
    *reinterpret_cast<float2*>(ps + (m0 + g + 8) * kMrgLdS + c0 + 2 * qd) =
        make_float2(acc[2], acc[3]);
  }
  __syncthreads();

  // ---- expand the base, add s * product, round once, 16-byte stores
#pragma unroll
  for (int i = 0; i < 2; ++i) {
    const int v = tid + i * 256;                 // 512 groups of 8 elements
    const int row = v >> 4, col = (v & 15) * 8;
    if (k0 + col >= P.K) continue;
    const int64_t e = (n0 + row) * P.K + k0 + col;  // first element of the group
    uint32_t wv[4];
    if (P.dense) {
      wv[0] = wraw[i].x, wv[1] = wraw[i].y, wv[2] = wraw[i].z, wv[3] = wraw[i].w;
    } else {
      const uint4 w = nf4_dequant8(wraw[i].x, nf4_make_table(P.cb, wabs[i]));
      wv[0] = w.x, wv[1] = w.y, wv[2] = w.z, wv[3] = w.w;
    }
    const float* pr = ps + row * kMrgLdS + col;
    uint32_t o[4];
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float lo = __uint_as_float(wv[h] << 16), hi = __uint_as_float(wv[h] & 0xFFFF0000u);
      const __nv_bfloat162 m = __floats2bfloat162_rn(__fadd_rn(lo, __fmul_rn(P.s, pr[2 * h])),
                                                     __fadd_rn(hi, __fmul_rn(P.s, pr[2 * h + 1])));
      o[h] = *reinterpret_cast<const uint32_t*>(&m);
    }
    *reinterpret_cast<uint4*>(P.out + e) = make_uint4(o[0], o[1], o[2], o[3]);
  }
}

cudaError_t launch_lora_merge(const void* base, const float* absmax, bool dense, int64_t N,
                              int64_t K, const void* A, const void* B, int r, float s, void* out,
                              cudaStream_t st) {
  MergeParams P;
  P.base = base;
  P.absmax = absmax;
  P.A = static_cast<const uint16_t*>(A);
  P.B = static_cast<const uint16_t*>(B);
  P.out = static_cast<uint16_t*>(out);
  P.N = N;
  P.K = K;
  P.r = r;
  P.r_pad = (r + 15) / 16 * 16;
  P.dense = dense ? 1 : 0;
  P.s = s;
  P.cb = codebook();
  P.col_tiles = static_cast<int>((K + kMrgCols - 1) / kMrgCols);
  const int64_t grid = (N / kMrgRows) * P.col_tiles;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  void* prof = prof_begin(st);
  count_launch();
  lora_merge_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(P);
  const cudaError_t e = cudaGetLastError();
  // algorithmic bytes per element: the base read (0.5625 B NF4, 2 B dense) + 2 B written
  if (prof) prof_end(prof, kProfMerge, (dense ? 4.0 : 2.5625) * static_cast<double>(N) * K, st);
  return e;
}

}  // namespace hsnf4
