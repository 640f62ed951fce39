// nf4_codec.cu -- NF4 quantize+pack and standalone dequantize (sm_100a).
//
// Both are HBM-bound streaming kernels: quantize reads 2 B and writes
// 0.5625 B per element; dequantize reads 0.5625 B and writes 2 B.  Each warp
// owns whole 64-element blocks so that the block's absmax is a warp-level
// reduction and every global access is a contiguous, 16-byte vector.
#include <cuda_bf16.h>

#include "internal.h"

namespace hsnf4 {

// ---------------------------------------------------------------- quantize
// Poros API reference (quantization="nf4") names the data type; the
// codebook, block length (64), fp32 absmax, nibble order and the nearest /
// lower-index-on-ties rule are this library's fixed reading.
//
// One warp quantizes 2 blocks (128 elements): lane l handles elements
// 4l..4l+3 of the pair (an 8-byte load), so lanes 0..15 form block 0 and
// lanes 16..31 block 1.  absmax = max|w| over the 16 lanes (exact: max is
// order independent); x = w / absmax with IEEE division; the code is the
// first index of the minimum fp32 distance |x - c_i|.

__device__ __forceinline__ int nearest_code(const Nf4Codebook& cb, float x) {
  int best = 0;
  float bd = fabsf(__fsub_rn(x, cb.v[0]));
#pragma unroll
  for (int i = 1; i < 16; ++i) {
    const float d = fabsf(__fsub_rn(x, cb.v[i]));
    if (d < bd) {
      bd = d;
      best = i;
    }
  }
  return best;
}

__global__ void __launch_bounds__(256) nf4_quantize_kernel(const uint2* __restrict__ w,
                                                           uint16_t* __restrict__ codes,
                                                           float* __restrict__ absmax,
                                                           int64_t n_pairs, int64_t n_blocks,
                                                           Nf4Codebook cb) {
  const int lane = threadIdx.x & 31;
  const int64_t warp = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) >> 5;
  const int64_t nwarps = (static_cast<int64_t>(gridDim.x) * blockDim.x) >> 5;
  for (int64_t pr = warp; pr < n_pairs; pr += nwarps) {
    const int64_t blk = pr * 2 + (lane >> 4);
    const bool live = blk < n_blocks;  // the last pair may hold one block
    uint2 v = make_uint2(0, 0);
    if (live) v = w[pr * 32 + lane];
    float x[4];
    x[0] = __uint_as_float(v.x << 16);
    x[1] = __uint_as_float(v.x & 0xFFFF0000u);
    x[2] = __uint_as_float(v.y << 16);
    x[3] = __uint_as_float(v.y & 0xFFFF0000u);
    float a = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
#pragma unroll
    for (int o = 8; o >= 1; o >>= 1) a = fmaxf(a, __shfl_xor_sync(0xffffffffu, a, o));
    int c[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) c[i] = (a == 0.0f) ? 7 : nearest_code(cb, __fdiv_rn(x[i], a));
    // bytes (e0 hi | e1 lo), (e2 hi | e3 lo) -> little-endian 16-bit word
    const uint16_t packed =
        static_cast<uint16_t>(((c[0] << 4) | c[1]) | (((c[2] << 4) | c[3]) << 8));
    if (live) {
      codes[pr * 32 + lane] = packed;
      if ((lane & 15) == 0) absmax[blk] = a;
    }
  }
}

cudaError_t launch_nf4_quantize(const void* w, int64_t n_out, int64_t k_in, void* codes,
                                float* absmax, cudaStream_t st) {
  const int64_t n_blocks = n_out * k_in / 64;
  const int64_t n_pairs = (n_blocks + 1) / 2;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t warps_needed = n_pairs;
  int64_t grid = (warps_needed + 7) / 8;
  const int64_t cap = static_cast<int64_t>(sms) * 16;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  // The last pair may hold a single block: give the kernel an even-sized
  // view only when the element count allows it (n_blocks even), otherwise
  // the guarded lanes skip the missing half.
  count_launch();
  nf4_quantize_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint2*>(w), static_cast<uint16_t*>(codes), absmax, n_pairs, n_blocks,
      codebook());
  return cudaGetLastError();
}

// ---------------------------------------------------------------- dequant
// A lane expands 8 elements (4 code bytes -> 16 output bytes); 8 lanes cover
// one 64-element block and build that block's bf16 table.  A warp therefore
// reads 128 contiguous code bytes and writes 512 contiguous output bytes.

__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint32_t* __restrict__ codes,
                                                          const float* __restrict__ absmax,
                                                          uint4* __restrict__ out,
                                                          int64_t n_groups, Nf4Codebook cb) {
  const int64_t tid = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t g = tid; g < n_groups; g += stride) {  // g = group of 8 elements
    const uint32_t cw = __ldg(codes + g);
    const float a = __ldg(absmax + (g >> 3));
    const Nf4Table t = nf4_make_table(cb, a);
    out[g] = nf4_dequant8(cw, t);
  }
}

cudaError_t launch_nf4_dequant(const void* codes, const float* absmax, int64_t n_out,
                               int64_t k_in, void* out, cudaStream_t st) {
  const int64_t n_groups = n_out * k_in / 8;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (n_groups + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 8;
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  void* prof = prof_begin(st);
  count_launch();
  nf4_dequant_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint32_t*>(codes), absmax, static_cast<uint4*>(out), n_groups,
      codebook());
  const cudaError_t e = cudaGetLastError();
  // algorithmic bytes: 0.5 B codes + 4/64 B absmax read, 2 B written per element
  if (prof) prof_end(prof, kProfDequant, 2.5625 * static_cast<double>(n_out) * k_in, st);
  return e;
}

}  // namespace hsnf4
