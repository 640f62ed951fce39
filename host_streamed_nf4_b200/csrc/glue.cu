// glue.cu -- the elementwise and row-wise pieces of a decoder layer around
// its seven projections (pre-norm Qwen2.5 / Llama-3.1 layer; the pages
// rematerialize each block of layers in the backward -- Poros on consumer
// GPUs, "OOM playbook").  Compute dtype bf16: every output is rounded once to
// bf16 from fp32 arithmetic.
//
//   rmsnorm_fwd:  h = bf16(xa + xb) (written when xb is given, the residual
//                 add), y = bf16(h * g / sqrt(mean h^2 + eps))
//   rmsnorm_bwd:  dx = bf16(dres + r (g . w) - r^3 h (sum g w h) / n),
//                 w = dy1 + dy2 + dy3 (fp32 sum of the branches' bf16 grads)
//   silu_mul:     m = bf16(silu(a) b); da = bf16(dm b s (1 + a (1 - s))),
//                 db = bf16(dm a s), s = 1 / (1 + e^-a)
//   add:          out = bf16(x + y)
//
// A row (one token) per CTA for the norms, 8 elements per thread otherwise;
// reductions are in a fixed order (thread partials, warp shuffles, then the
// warps in index order), so results do not depend on timing.
#include <cuda_bf16.h>

#include "internal.h"

namespace hsnf4 {

namespace {

__device__ __forceinline__ void unpack8(const uint4 v, float (&f)[8]) {
  const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    f[2 * h] = __uint_as_float(w[h] << 16);
    f[2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
  }
}

__device__ __forceinline__ uint4 pack8(const float (&f)[8]) {
  uint32_t w[4];
#pragma unroll
  for (int h = 0; h < 4; ++h) {
    const __nv_bfloat162 b = __floats2bfloat162_rn(f[2 * h], f[2 * h + 1]);
    w[h] = *reinterpret_cast<const uint32_t*>(&b);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 ld8(const uint16_t* p, int64_t i) {
  return __ldg(reinterpret_cast<const uint4*>(p) + i);
}

// sum over the CTA (256 threads) in a fixed order; every thread gets it
__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  __syncthreads();  // red may still be read by a previous call
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < 8; ++w) s += red[w];
  return s;
}

__global__ void __launch_bounds__(256) rmsnorm_fwd_kernel(const uint16_t* __restrict__ xa,
                                                          const uint16_t* __restrict__ xb,
                                                          const uint16_t* __restrict__ g,
                                                          uint16_t* __restrict__ h_out,
                                                          uint16_t* __restrict__ y, int n,
                                                          float eps) {
  __shared__ float red[8];
  const int64_t row = blockIdx.x;
  const int n8 = n / 8;
  const int64_t base = row * n8;
  float ss = 0.0f;
  for (int c = threadIdx.x; c < n8; c += 256) {
    float x[8];
    unpack8(ld8(xa, base + c), x);
    if (xb) {
      float b[8];
      unpack8(ld8(xb, base + c), b);
#pragma unroll
      for (int e = 0; e < 8; ++e) x[e] = __fadd_rn(x[e], b[e]);
      const uint4 hv = pack8(x);
      reinterpret_cast<uint4*>(h_out)[base + c] = hv;
      unpack8(hv, x);  // the norm reads the bf16 residual sum
    }
#pragma unroll
    for (int e = 0; e < 8; ++e) ss = __fmaf_rn(x[e], x[e], ss);
  }
  ss = block_sum(ss, red);
  const float r = 1.0f / sqrtf(__fadd_rn(__fdiv_rn(ss, static_cast<float>(n)), eps));
  for (int c = threadIdx.x; c < n8; c += 256) {
    float x[8], gv[8];
    unpack8(xb ? reinterpret_cast<const uint4*>(h_out)[base + c] : ld8(xa, base + c), x);
    unpack8(ld8(g, c), gv);
#pragma unroll
    for (int e = 0; e < 8; ++e) x[e] = __fmul_rn(__fmul_rn(x[e], r), gv[e]);
    reinterpret_cast<uint4*>(y)[base + c] = pack8(x);
  }
}

__global__ void __launch_bounds__(256) rmsnorm_bwd_kernel(
    const uint16_t* __restrict__ x, const uint16_t* __restrict__ g,
    const uint16_t* __restrict__ dy1, const uint16_t* __restrict__ dy2,
    const uint16_t* __restrict__ dy3, const uint16_t* __restrict__ dres,
    uint16_t* __restrict__ dx, int n, float eps) {
  __shared__ float red[8];
  const int64_t row = blockIdx.x;
  const int n8 = n / 8;
  const int64_t base = row * n8;
  float ss = 0.0f, wx = 0.0f;
  auto load_w = [&](int c, float (&w)[8]) {
    float gv[8];
    unpack8(ld8(dy1, base + c), w);
    if (dy2) {
      float t[8];
      unpack8(ld8(dy2, base + c), t);
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = __fadd_rn(w[e], t[e]);
    }
    if (dy3) {
      float t[8];
      unpack8(ld8(dy3, base + c), t);
#pragma unroll
      for (int e = 0; e < 8; ++e) w[e] = __fadd_rn(w[e], t[e]);
    }
    unpack8(ld8(g, c), gv);
#pragma unroll
    for (int e = 0; e < 8; ++e) w[e] = __fmul_rn(w[e], gv[e]);
  };
  for (int c = threadIdx.x; c < n8; c += 256) {
    float xv[8], w[8];
    unpack8(ld8(x, base + c), xv);
    load_w(c, w);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      ss = __fmaf_rn(xv[e], xv[e], ss);
      wx = __fmaf_rn(w[e], xv[e], wx);
    }
  }
  ss = block_sum(ss, red);
  wx = block_sum(wx, red);
  const float r = 1.0f / sqrtf(__fadd_rn(__fdiv_rn(ss, static_cast<float>(n)), eps));
  const float k = __fdiv_rn(__fmul_rn(__fmul_rn(__fmul_rn(r, r), r), wx), static_cast<float>(n));
  for (int c = threadIdx.x; c < n8; c += 256) {
    float xv[8], w[8], o[8];
    unpack8(ld8(x, base + c), xv);
    load_w(c, w);
    float res[8] = {0, 0, 0, 0, 0, 0, 0, 0};
    if (dres) unpack8(ld8(dres, base + c), res);
#pragma unroll
    for (int e = 0; e < 8; ++e)
      o[e] = __fadd_rn(res[e], __fsub_rn(__fmul_rn(r, w[e]), __fmul_rn(k, xv[e])));
    reinterpret_cast<uint4*>(dx)[base + c] = pack8(o);
  }
}

__device__ __forceinline__ float sigmoidf_(float a) { return 1.0f / (1.0f + expf(-a)); }

__global__ void __launch_bounds__(256) silu_mul_fwd_kernel(const uint16_t* __restrict__ a,
                                                           const uint16_t* __restrict__ b,
                                                           uint16_t* __restrict__ m,
                                                           int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    float av[8], bv[8], o[8];
    unpack8(ld8(a, i), av);
    unpack8(ld8(b, i), bv);
#pragma unroll
    for (int e = 0; e < 8; ++e) o[e] = __fmul_rn(__fmul_rn(av[e], sigmoidf_(av[e])), bv[e]);
    reinterpret_cast<uint4*>(m)[i] = pack8(o);
  }
}

__global__ void __launch_bounds__(256) silu_mul_bwd_kernel(const uint16_t* __restrict__ a,
                                                           const uint16_t* __restrict__ b,
                                                           const uint16_t* __restrict__ dm,
                                                           uint16_t* __restrict__ da,
                                                           uint16_t* __restrict__ db,
                                                           int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    float av[8], bv[8], gv[8], oa[8], ob[8];
    unpack8(ld8(a, i), av);
    unpack8(ld8(b, i), bv);
    unpack8(ld8(dm, i), gv);
#pragma unroll
    for (int e = 0; e < 8; ++e) {
      const float s = sigmoidf_(av[e]);
      const float ds = __fmul_rn(s, __fadd_rn(1.0f, __fmul_rn(av[e], __fsub_rn(1.0f, s))));
      oa[e] = __fmul_rn(__fmul_rn(gv[e], bv[e]), ds);
      ob[e] = __fmul_rn(gv[e], __fmul_rn(av[e], s));
    }
    reinterpret_cast<uint4*>(da)[i] = pack8(oa);
    reinterpret_cast<uint4*>(db)[i] = pack8(ob);
  }
}

__global__ void __launch_bounds__(256) add_kernel(const uint16_t* __restrict__ x,
                                                  const uint16_t* __restrict__ y,
                                                  uint16_t* __restrict__ out, int64_t n8) {
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n8;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    float xv[8], yv[8];
    unpack8(ld8(x, i), xv);
    unpack8(ld8(y, i), yv);
#pragma unroll
    for (int e = 0; e < 8; ++e) xv[e] = __fadd_rn(xv[e], yv[e]);
    reinterpret_cast<uint4*>(out)[i] = pack8(xv);
  }
}

unsigned elementwise_grid(int64_t n8) {
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (n8 + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 16) grid = static_cast<int64_t>(sms) * 16;
  return static_cast<unsigned>(grid < 1 ? 1 : grid);
}

}  // namespace

cudaError_t launch_rmsnorm_fwd(const void* xa, const void* xb, const void* g, void* h_out,
                               void* y, int64_t T, int64_t n, float eps, cudaStream_t st) {
  count_launch();
  rmsnorm_fwd_kernel<<<static_cast<unsigned>(T), 256, 0, st>>>(
      static_cast<const uint16_t*>(xa), static_cast<const uint16_t*>(xb),
      static_cast<const uint16_t*>(g), static_cast<uint16_t*>(h_out), static_cast<uint16_t*>(y),
      static_cast<int>(n), eps);
  return cudaGetLastError();
}

cudaError_t launch_rmsnorm_bwd(const void* x, const void* g, const void* dy1, const void* dy2,
                               const void* dy3, const void* dres, void* dx, int64_t T, int64_t n,
                               float eps, cudaStream_t st) {
  count_launch();
  rmsnorm_bwd_kernel<<<static_cast<unsigned>(T), 256, 0, st>>>(
      static_cast<const uint16_t*>(x), static_cast<const uint16_t*>(g),
      static_cast<const uint16_t*>(dy1), static_cast<const uint16_t*>(dy2),
      static_cast<const uint16_t*>(dy3), static_cast<const uint16_t*>(dres),
      static_cast<uint16_t*>(dx), static_cast<int>(n), eps);
  return cudaGetLastError();
}

cudaError_t launch_silu_mul_fwd(const void* a, const void* b, void* m, int64_t n,
                                cudaStream_t st) {
  count_launch();
  silu_mul_fwd_kernel<<<elementwise_grid(n / 8), 256, 0, st>>>(
      static_cast<const uint16_t*>(a), static_cast<const uint16_t*>(b), static_cast<uint16_t*>(m),
      n / 8);
  return cudaGetLastError();
}

cudaError_t launch_silu_mul_bwd(const void* a, const void* b, const void* dm, void* da, void* db,
                                int64_t n, cudaStream_t st) {
  count_launch();
  silu_mul_bwd_kernel<<<elementwise_grid(n / 8), 256, 0, st>>>(
      static_cast<const uint16_t*>(a), static_cast<const uint16_t*>(b),
      static_cast<const uint16_t*>(dm), static_cast<uint16_t*>(da), static_cast<uint16_t*>(db),
      n / 8);
  return cudaGetLastError();
}

cudaError_t launch_add(const void* x, const void* y, void* out, int64_t n, cudaStream_t st) {
  count_launch();
  add_kernel<<<elementwise_grid(n / 8), 256, 0, st>>>(static_cast<const uint16_t*>(x),
                                                       static_cast<const uint16_t*>(y),
                                                       static_cast<uint16_t*>(out), n / 8);
  return cudaGetLastError();
}

}  // namespace hsnf4
