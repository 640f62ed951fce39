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
// A lane expands 32 elements per step: one 16-byte code load (half a
// 64-element block), one absmax, one bf16 table, 64 output bytes.  The
// warp's 2 KiB of output for the step goes through a per-warp shared-memory
// stage, so that every global store instruction writes 512 contiguous bytes
// (lane l stores the 16-byte pieces l, l + 32, l + 64, l + 96); the stage
// slots are XOR-swizzled so both the writes and the reads are free of bank
// conflicts.  Each lane has the code loads of two steps in flight.

__device__ __forceinline__ int dq_slot(int s) { return s ^ ((s >> 3) & 7); }

__device__ __forceinline__ void dq_step(const uint4 cw, const float a, bool active,
                                        const Nf4Codebook& cb, uint4* __restrict__ stage,
                                        uint4* __restrict__ out, int64_t qw, int64_t n_quads,
                                        int lane) {
  if (active) {
    const Nf4Table t = nf4_make_table(cb, a);
    stage[dq_slot(4 * lane + 0)] = nf4_dequant8(cw.x, t);
    stage[dq_slot(4 * lane + 1)] = nf4_dequant8(cw.y, t);
    stage[dq_slot(4 * lane + 2)] = nf4_dequant8(cw.z, t);
    stage[dq_slot(4 * lane + 3)] = nf4_dequant8(cw.w, t);
  }
  __syncwarp();
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const int sl = lane + 32 * j;  // the warp's 16-byte piece sl: quad qw + sl / 4
    if (qw + (sl >> 2) < n_quads) out[4 * qw + sl] = stage[dq_slot(sl)];
  }
  __syncwarp();
}

__global__ void __launch_bounds__(256) nf4_dequant_kernel(const uint4* __restrict__ codes,
                                                          const float* __restrict__ absmax,
                                                          uint4* __restrict__ out,
                                                          int64_t n_quads, Nf4Codebook cb) {
  __shared__ uint4 stage_all[8][128];  // per warp: 32 lanes x 4 pieces
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint4* stage = stage_all[warp];
  const int64_t step = static_cast<int64_t>(gridDim.x) * 256;  // quads per grid-wide step
  // qw: first quad of this warp's step (warp-uniform, so the loop is too)
  int64_t qw = static_cast<int64_t>(blockIdx.x) * 256 + warp * 32;
  for (; qw < n_quads; qw += 2 * step) {
    const int64_t q0 = qw + lane, q1 = qw + step + lane;
    const bool a0 = q0 < n_quads, a1 = q1 < n_quads;
    uint4 c0 = make_uint4(0, 0, 0, 0), c1 = c0;
    float m0 = 0.0f, m1 = 0.0f;
    if (a0) {
      c0 = __ldg(codes + q0);
      m0 = __ldg(absmax + (q0 >> 1));
    }
    if (a1) {
      c1 = __ldg(codes + q1);
      m1 = __ldg(absmax + (q1 >> 1));
    }
    dq_step(c0, m0, a0, cb, stage, out, qw, n_quads, lane);
    if (qw + step < n_quads) dq_step(c1, m1, a1, cb, stage, out, qw + step, n_quads, lane);
  }
}

cudaError_t launch_nf4_dequant(const void* codes, const float* absmax, int64_t n_out,
                               int64_t k_in, void* out, cudaStream_t st) {
  const int64_t n_quads = n_out * k_in / 32;  // k_in % 64 == 0
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (n_quads + 255) / 256;
  const int64_t cap = static_cast<int64_t>(sms) * 4;  // resident at 52 registers: one wave
  if (grid > cap) grid = cap;
  if (grid < 1) grid = 1;
  void* prof = prof_begin(st, kProfDequant);
  count_launch();
  nf4_dequant_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(
      static_cast<const uint4*>(codes), absmax, static_cast<uint4*>(out), n_quads, codebook());
  const cudaError_t e = cudaGetLastError();
  // algorithmic bytes: 0.5 B codes + 4/64 B absmax read, 2 B written per element
  if (prof) prof_end(prof, kProfDequant, 2.5625 * static_cast<double>(n_out) * k_in, st);
  return e;
}

}  // namespace hsnf4
