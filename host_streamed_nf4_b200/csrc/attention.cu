// attention.cu -- causal scaled dot-product attention with grouped KV heads,
// forward and backward, for the decoder layer around the projections
// (head_dim 128, the Qwen2.5 / Llama-3.1 families').
//
//   o_i = sum_{j <= i} softmax_j(scale q_i . k_j) v_j      per query head h,
//   keys/values of KV head h / (H / KV);  lse_i = log sum_{j <= i} e^{scale q_i.k_j}
//
// Tensor cores via mma.sync m16n8k16 (bf16 in, fp32 accumulate), 64-query x
// 64-key tiles double-buffered through cp.async (the next tile loads while
// this one is multiplied), 4 warps of 16 rows, online softmax in registers (exp2 with
// the scale folded into log2 units); the probabilities are rounded to bf16
// for the P.V product.  Backward in two kernels without atomics, so results
// are run-to-run identical: dQ per (query tile, head) over its key tiles;
// dK and dV per (key tile, query head) over the query tiles, as fp32
// partials that a last kernel adds over the query heads of each KV group in
// head order; D_i = sum_c dO_ic O_ic precomputed.
#include <cuda_bf16.h>

#include <mutex>

#include "internal.h"

namespace hsnf4 {

namespace {

constexpr int kD = 128;          // head dim
constexpr int kBM = 64;          // query rows per CTA
constexpr int kBN = 64;          // key rows per tile
constexpr int kLd = kD + 8;      // padded smem row (bf16)
constexpr int kTileBytes = 64 * kLd * 2;
constexpr float kLog2e = 1.4426950408889634f;

struct AttnArgs {
  const uint16_t* q;  // [T, H*d]
  const uint16_t* k;  // [T, KV*d]
  const uint16_t* v;
  const uint16_t* o;  // [T, H*d] (backward)
  const uint16_t* dout;
  uint16_t* out;      // forward: o;  backward: dq
  uint16_t* dk;
  uint16_t* dv;
  float* lse;         // [H, T]
  const float* D;     // [H, T]
  float* part;        // backward: per-head fp32 dK, dV partials [2H][T][128]
  int T, H, KV;
  float scale;
};

__device__ __forceinline__ uint32_t su32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mma16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void ldm_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldm_x4_t(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ uint32_t pack_bf16(float lo, float hi) {
  const __nv_bfloat162 b = __floats2bfloat162_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&b);
}

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

// 64 rows x 128 columns of a row-major [T, stride] bf16 tensor (rows from
// r0, columns from c0) into a padded smem tile with cp.async; rows past T
// are written as zeros.
__device__ __forceinline__ void load_tile_async(uint16_t* dst, const uint16_t* src, int r0, int T,
                                                int64_t stride, int c0) {
  for (int v = threadIdx.x; v < 64 * 16; v += blockDim.x) {
    const int row = v >> 4, col = (v & 15) * 8;
    const bool in = r0 + row < T;
    const uint16_t* s = in ? src + static_cast<int64_t>(r0 + row) * stride + c0 + col : src;
    cp_async16(su32(dst + row * kLd + col), s, in ? 16 : 0);
  }
}

// A fragments (16 rows m0.., k16 step k0) of a row-major [.][kLd] smem tile
__device__ __forceinline__ void frag_a(uint32_t (&a)[4], const uint16_t* tile, int m0, int k0) {
  const int lane = threadIdx.x & 31;
  ldm_x4(a, su32(tile + (m0 + (lane & 15)) * kLd + k0 + (lane >> 4) * 8));
}

// B fragments for D = X Y^T with Y row-major [n][k] in smem: n-tile n0 (8 rows),
// k16 steps k0 and k0 + 16 -> b[0], b[1] (step k0), b[2], b[3] (step k0 + 16)
__device__ __forceinline__ void frag_bt(uint32_t (&b)[4], const uint16_t* tile, int n0, int k0) {
  const int lane = threadIdx.x & 31;
  ldm_x4(b, su32(tile + (n0 + (lane & 7)) * kLd + k0 + (lane >> 3) * 8));
}

// B fragments for D = X Y with Y row-major [k][n] in smem: k16 step k0,
// n-tiles n0 and n0 + 8 -> b[0], b[1] (n0), b[2], b[3] (n0 + 8)
__device__ __forceinline__ void frag_b(uint32_t (&b)[4], const uint16_t* tile, int k0, int n0) {
  const int lane = threadIdx.x & 31;
  ldm_x4_t(b, su32(tile + (k0 + (lane & 7) + ((lane >> 3) & 1) * 8) * kLd + n0 + (lane >> 4) * 8));
}

// S[16 x 64] = X_w (16 rows at m0 of tile X) . Y^T (64 rows of tile Y), both [.][128]
__device__ __forceinline__ void gemm_xyt(float (&s)[8][4], const uint16_t* X, int m0,
                                         const uint16_t* Y) {
#pragma unroll
  for (int j = 0; j < 8; ++j)
#pragma unroll
    for (int e = 0; e < 4; ++e) s[j][e] = 0.0f;
#pragma unroll
  for (int k0 = 0; k0 < kD; k0 += 32) {
    uint32_t a0[4], a1[4];
    frag_a(a0, X, m0, k0);
    frag_a(a1, X, m0, k0 + 16);
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      uint32_t b[4];
      frag_bt(b, Y, j * 8, k0);
      mma16816(s[j], a0, b[0], b[1]);
      mma16816(s[j], a1, b[2], b[3]);
    }
  }
}

// acc[16 x 128] += P (16 x 64, register accumulator layout, rounded to bf16) . Y (64 x 128 tile)
__device__ __forceinline__ void gemm_py(float (&acc)[16][4], const float (&p)[8][4],
                                        const uint16_t* Y) {
#pragma unroll
  for (int kk = 0; kk < 4; ++kk) {  // keys 16 kk .. 16 kk + 15
    uint32_t a[4];
    a[0] = pack_bf16(p[2 * kk][0], p[2 * kk][1]);
    a[1] = pack_bf16(p[2 * kk][2], p[2 * kk][3]);
    a[2] = pack_bf16(p[2 * kk + 1][0], p[2 * kk + 1][1]);
    a[3] = pack_bf16(p[2 * kk + 1][2], p[2 * kk + 1][3]);
#pragma unroll
    for (int n = 0; n < 8; ++n) {  // head-dim columns 16 n .. 16 n + 15
      uint32_t b[4];
      frag_b(b, Y, kk * 16, n * 16);
      mma16816(acc[2 * n], a, b[0], b[1]);
      mma16816(acc[2 * n + 1], a, b[2], b[3]);
    }
  }
}

// ---------------------------------------------------------------- forward
__global__ void __launch_bounds__(128) attn_fwd_kernel(const __grid_constant__ AttnArgs P) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);
  uint16_t* KV = Qs + 64 * kLd;  // K0 V0 K1 V1: the next tile loads during this one
  const int qt = blockIdx.x, h = blockIdx.y, kh = h / (P.H / P.KV);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, qd = lane & 3;
  const int m0 = warp * 16;
  const int64_t qs = static_cast<int64_t>(P.H) * kD, ks = static_cast<int64_t>(P.KV) * kD;
  load_tile_async(Qs, P.q, qt * kBM, P.T, qs, h * kD);
  load_tile_async(KV, P.k, 0, P.T, ks, kh * kD);
  load_tile_async(KV + 64 * kLd, P.v, 0, P.T, ks, kh * kD);
  cp_async_commit();
  const float c = P.scale * kLog2e;
  float m[2] = {-INFINITY, -INFINITY}, l[2] = {0.0f, 0.0f};
  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.0f;
  const int rows[2] = {qt * kBM + m0 + g, qt * kBM + m0 + g + 8};
  for (int kt = 0; kt <= qt; ++kt) {
    const uint16_t* Ks = KV + ((kt & 1) * 2) * 64 * kLd;
    const uint16_t* Vs = Ks + 64 * kLd;
    if (kt < qt) {  // the other buffer was released at the end of the previous tile
      uint16_t* Kn = KV + (((kt + 1) & 1) * 2) * 64 * kLd;
      load_tile_async(Kn, P.k, (kt + 1) * kBN, P.T, ks, kh * kD);
      load_tile_async(Kn + 64 * kLd, P.v, (kt + 1) * kBN, P.T, ks, kh * kD);
    }
    cp_async_commit();
    cp_async_wait<1>();  // everything but the group just committed: tile kt is in
    __syncthreads();
    float s[8][4];
    gemm_xyt(s, Qs, m0, Ks);
#pragma unroll
    for (int hr = 0; hr < 2; ++hr) {
      float mx = m[hr];
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          const int key = kt * kBN + j * 8 + 2 * qd + e;
          float& x = s[j][2 * hr + e];
          x = (key <= rows[hr] && key < P.T) ? x * c : -INFINITY;
          mx = fmaxf(mx, x);
        }
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
      mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
      // a fully masked row keeps -inf: use 0 as the reference so exp2 gives 0
      const float ref = mx == -INFINITY ? 0.0f : mx;
      const float corr = exp2f(m[hr] - ref);
      float sum = 0.0f;
#pragma unroll
      for (int j = 0; j < 8; ++j)
#pragma unroll
        for (int e = 0; e < 2; ++e) {
          float& x = s[j][2 * hr + e];
          x = exp2f(x - ref);
          sum += x;
        }
      sum += __shfl_xor_sync(0xffffffffu, sum, 1);
      sum += __shfl_xor_sync(0xffffffffu, sum, 2);
      l[hr] = l[hr] * corr + sum;
      m[hr] = mx;
#pragma unroll
      for (int n = 0; n < 16; ++n) {
        acc[n][2 * hr] *= corr;
        acc[n][2 * hr + 1] *= corr;
      }
    }
    gemm_py(acc, s, Vs);
    __syncthreads();  // this buffer is refilled by the next iteration's prefetch
  }
  // normalize and write o (bf16) and lse (natural log)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const int row = rows[hr];
    if (row >= P.T) continue;
    const float inv = 1.0f / l[hr];
    uint16_t* dst = P.out + static_cast<int64_t>(row) * qs + h * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * qd) =
          pack_bf16(acc[n][2 * hr] * inv, acc[n][2 * hr + 1] * inv);
    if (qd == 0) P.lse[static_cast<int64_t>(h) * P.T + row] = (m[hr] + log2f(l[hr])) / kLog2e;
  }
}

// D[h][i] = sum_c dO[i, h, c] O[i, h, c]: a warp per (row, head)
__global__ void __launch_bounds__(256) attn_bwd_dot_kernel(const __grid_constant__ AttnArgs P) {
  const int64_t w = (static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  if (w >= static_cast<int64_t>(P.T) * P.H) return;
  const int row = static_cast<int>(w / P.H), h = static_cast<int>(w % P.H);
  const int64_t off = static_cast<int64_t>(row) * P.H * kD + h * kD + lane * 4;
  const uint2 a = __ldg(reinterpret_cast<const uint2*>(P.dout + off));
  const uint2 b = __ldg(reinterpret_cast<const uint2*>(P.o + off));
  float s = __uint_as_float(a.x << 16) * __uint_as_float(b.x << 16) +
            __uint_as_float(a.x & 0xFFFF0000u) * __uint_as_float(b.x & 0xFFFF0000u) +
            __uint_as_float(a.y << 16) * __uint_as_float(b.y << 16) +
            __uint_as_float(a.y & 0xFFFF0000u) * __uint_as_float(b.y & 0xFFFF0000u);
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
  if (lane == 0) const_cast<float*>(P.D)[static_cast<int64_t>(h) * P.T + row] = s;
}

// ---------------------------------------------------------------- dQ
__global__ void __launch_bounds__(128) attn_bwd_dq_kernel(const __grid_constant__ AttnArgs P) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* Qs = reinterpret_cast<uint16_t*>(smem);
  uint16_t* dOs = Qs + 64 * kLd;
  uint16_t* KV = dOs + 64 * kLd;  // K0 V0 K1 V1
  const int qt = blockIdx.x, h = blockIdx.y, kh = h / (P.H / P.KV);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, qd = lane & 3;
  const int m0 = warp * 16;
  const int64_t qs = static_cast<int64_t>(P.H) * kD, ks = static_cast<int64_t>(P.KV) * kD;
  load_tile_async(Qs, P.q, qt * kBM, P.T, qs, h * kD);
  load_tile_async(dOs, P.dout, qt * kBM, P.T, qs, h * kD);
  load_tile_async(KV, P.k, 0, P.T, ks, kh * kD);
  load_tile_async(KV + 64 * kLd, P.v, 0, P.T, ks, kh * kD);
  cp_async_commit();
  const float c = P.scale * kLog2e;
  const int rows[2] = {qt * kBM + m0 + g, qt * kBM + m0 + g + 8};
  float lse2[2], Dr[2];
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    const bool in = rows[hr] < P.T;
    lse2[hr] = in ? P.lse[static_cast<int64_t>(h) * P.T + rows[hr]] * kLog2e : 0.0f;
    Dr[hr] = in ? P.D[static_cast<int64_t>(h) * P.T + rows[hr]] : 0.0f;
  }
  float acc[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[n][e] = 0.0f;
  for (int kt = 0; kt <= qt; ++kt) {
    const uint16_t* Ks = KV + ((kt & 1) * 2) * 64 * kLd;
    const uint16_t* Vs = Ks + 64 * kLd;
    if (kt < qt) {
      uint16_t* Kn = KV + (((kt + 1) & 1) * 2) * 64 * kLd;
      load_tile_async(Kn, P.k, (kt + 1) * kBN, P.T, ks, kh * kD);
      load_tile_async(Kn + 64 * kLd, P.v, (kt + 1) * kBN, P.T, ks, kh * kD);
    }
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[8][4], dp[8][4];
    gemm_xyt(s, Qs, m0, Ks);    // S = Q K^T
    gemm_xyt(dp, dOs, m0, Vs);  // dP = dO V^T
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1, key = kt * kBN + j * 8 + 2 * qd + (e & 1);
        const bool on = key <= rows[hr] && key < P.T && rows[hr] < P.T;
        const float p = on ? exp2f(s[j][e] * c - lse2[hr]) : 0.0f;
        s[j][e] = p * (dp[j][e] - Dr[hr]);  // dS
      }
    gemm_py(acc, s, Ks);  // dQ += dS K
    __syncthreads();
  }
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    if (rows[hr] >= P.T) continue;
    uint16_t* dst = P.out + static_cast<int64_t>(rows[hr]) * qs + h * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n)
      *reinterpret_cast<uint32_t*>(dst + n * 8 + 2 * qd) =
          pack_bf16(acc[n][2 * hr] * P.scale, acc[n][2 * hr + 1] * P.scale);
  }
}

// ---------------------------------------------------------------- dK, dV
// Per CTA one key tile and one QUERY head: S^T = K Q^T (keys x queries), P^T
// from the saved lse, 16 keys per warp; the head's fp32 dK, dV partials go to
// scratch and a second kernel adds the heads of each KV group in head order.
__global__ void __launch_bounds__(128) attn_bwd_dkdv_kernel(const __grid_constant__ AttnArgs P) {
  extern __shared__ __align__(16) uint8_t smem[];
  uint16_t* Ks = reinterpret_cast<uint16_t*>(smem);
  uint16_t* Vs = Ks + 64 * kLd;
  uint16_t* QD = Vs + 64 * kLd;  // Q0 dO0 Q1 dO1: the next query tile loads during this one
  float* LD = reinterpret_cast<float*>(QD + 4 * 64 * kLd);  // per buffer: lse [64], D [64]
  const int kt = blockIdx.x, h = blockIdx.y, kh = h / (P.H / P.KV);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31, g = lane >> 2, qd = lane & 3;
  const int m0 = warp * 16;
  const int64_t qs = static_cast<int64_t>(P.H) * kD, ks = static_cast<int64_t>(P.KV) * kD;
  auto stage = [&](int qt, int b) {  // query tile qt into buffer b
    uint16_t* q = QD + (b * 2) * 64 * kLd;
    load_tile_async(q, P.q, qt * kBM, P.T, qs, h * kD);
    load_tile_async(q + 64 * kLd, P.dout, qt * kBM, P.T, qs, h * kD);
    for (int i = threadIdx.x; i < 64; i += blockDim.x) {
      const int row = qt * kBM + i;
      LD[b * 128 + i] = row < P.T ? P.lse[static_cast<int64_t>(h) * P.T + row] * kLog2e : 0.0f;
      LD[b * 128 + 64 + i] = row < P.T ? P.D[static_cast<int64_t>(h) * P.T + row] : 0.0f;
    }
  };
  load_tile_async(Ks, P.k, kt * kBN, P.T, ks, kh * kD);
  load_tile_async(Vs, P.v, kt * kBN, P.T, ks, kh * kD);
  stage(kt, 0);
  cp_async_commit();
  const float c = P.scale * kLog2e;
  const int keys[2] = {kt * kBN + m0 + g, kt * kBN + m0 + g + 8};
  float dk[16][4], dv[16][4];
#pragma unroll
  for (int n = 0; n < 16; ++n)
#pragma unroll
    for (int e = 0; e < 4; ++e) dk[n][e] = dv[n][e] = 0.0f;
  const int q_tiles = (P.T + kBM - 1) / kBM;
  for (int qt = kt; qt < q_tiles; ++qt) {
    const int b = (qt - kt) & 1;
    const uint16_t* Qs = QD + (b * 2) * 64 * kLd;
    const uint16_t* dOs = Qs + 64 * kLd;
    const float* lse_s = LD + b * 128;
    const float* D_s = lse_s + 64;
    if (qt + 1 < q_tiles) stage(qt + 1, b ^ 1);
    cp_async_commit();
    cp_async_wait<1>();
    __syncthreads();
    float s[8][4];
    gemm_xyt(s, Ks, m0, Qs);  // S^T = K Q^T
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int hr = e >> 1, qi = j * 8 + 2 * qd + (e & 1), row = qt * kBM + qi;
        const bool on = keys[hr] <= row && row < P.T && keys[hr] < P.T;
        s[j][e] = on ? exp2f(s[j][e] * c - lse_s[qi]) : 0.0f;  // P^T
      }
    gemm_py(dv, s, dOs);  // dV += P^T dO
    float dp[8][4];
    gemm_xyt(dp, Vs, m0, dOs);  // dP^T = V dO^T
#pragma unroll
    for (int j = 0; j < 8; ++j)
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int qi = j * 8 + 2 * qd + (e & 1);
        s[j][e] = s[j][e] * (dp[j][e] - D_s[qi]);  // dS^T
      }
    gemm_py(dk, s, Qs);  // dK += dS^T Q
    __syncthreads();
  }
  // this head's partials: part[h][key][c] (dK unscaled), part[H + h][key][c] (dV)
#pragma unroll
  for (int hr = 0; hr < 2; ++hr) {
    if (keys[hr] >= P.T) continue;
    float* pk = P.part + (static_cast<int64_t>(h) * P.T + keys[hr]) * kD;
    float* pv = P.part + (static_cast<int64_t>(P.H + h) * P.T + keys[hr]) * kD;
#pragma unroll
    for (int n = 0; n < 16; ++n) {
      *reinterpret_cast<float2*>(pk + n * 8 + 2 * qd) = make_float2(dk[n][2 * hr], dk[n][2 * hr + 1]);
      *reinterpret_cast<float2*>(pv + n * 8 + 2 * qd) = make_float2(dv[n][2 * hr], dv[n][2 * hr + 1]);
    }
  }
}

// dK[key, kh] = scale sum_{h in group kh} part_k[h][key], dV likewise (head order)
__global__ void __launch_bounds__(256) attn_bwd_kv_reduce_kernel(const __grid_constant__ AttnArgs P) {
  const int grp = P.H / P.KV;
  const int64_t n4 = static_cast<int64_t>(P.T) * P.KV * (kD / 4);
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x; i < n4;
       i += static_cast<int64_t>(gridDim.x) * 256) {
    const int c4 = static_cast<int>(i % (kD / 4));
    const int64_t rk = i / (kD / 4);
    const int kh = static_cast<int>(rk % P.KV);
    const int64_t key = rk / P.KV;
    float4 a = make_float4(0.f, 0.f, 0.f, 0.f), b = a;
    for (int hh = 0; hh < grp; ++hh) {
      const int h = kh * grp + hh;
      const float4 x = *reinterpret_cast<const float4*>(
          P.part + (static_cast<int64_t>(h) * P.T + key) * kD + c4 * 4);
      const float4 y = *reinterpret_cast<const float4*>(
          P.part + (static_cast<int64_t>(P.H + h) * P.T + key) * kD + c4 * 4);
      a.x += x.x, a.y += x.y, a.z += x.z, a.w += x.w;
      b.x += y.x, b.y += y.y, b.z += y.z, b.w += y.w;
    }
    const int64_t o = key * P.KV * kD + kh * kD + c4 * 4;
    *reinterpret_cast<uint2*>(P.dk + o) =
        make_uint2(pack_bf16(a.x * P.scale, a.y * P.scale), pack_bf16(a.z * P.scale, a.w * P.scale));
    *reinterpret_cast<uint2*>(P.dv + o) = make_uint2(pack_bf16(b.x, b.y), pack_bf16(b.z, b.w));
  }
}

template <typename K>
cudaError_t set_smem(K kernel, int bytes, std::once_flag& once, cudaError_t& rc) {
  std::call_once(once, [&] {
    rc = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes);
  });
  return rc;
}

}  // namespace

cudaError_t launch_attention_fwd(const void* q, const void* k, const void* v, void* o, float* lse,
                                 int64_t T, int H, int KV, float scale, cudaStream_t st) {
  static std::once_flag once;
  static cudaError_t rc = cudaSuccess;
  const int smem = 5 * kTileBytes;  // Q + double-buffered K, V
  if (set_smem(attn_fwd_kernel, smem, once, rc) != cudaSuccess) return rc;
  AttnArgs P{};
  P.q = static_cast<const uint16_t*>(q);
  P.k = static_cast<const uint16_t*>(k);
  P.v = static_cast<const uint16_t*>(v);
  P.out = static_cast<uint16_t*>(o);
  P.lse = lse;
  P.T = static_cast<int>(T);
  P.H = H;
  P.KV = KV;
  P.scale = scale;
  count_launch();
  attn_fwd_kernel<<<dim3(static_cast<unsigned>((T + kBM - 1) / kBM), H), 128, smem, st>>>(P);
  return cudaGetLastError();
}

cudaError_t launch_attention_bwd(const void* q, const void* k, const void* v, const void* o,
                                 const float* lse, const void* dout, void* dq, void* dk, void* dv,
                                 float* D, int64_t T, int H, int KV, float scale,
                                 cudaStream_t st) {
  static std::once_flag once_q, once_kv;
  static cudaError_t rc_q = cudaSuccess, rc_kv = cudaSuccess;
  const int smem_q = 6 * kTileBytes, smem_kv = 6 * kTileBytes + 2 * 2 * 64 * 4;
  if (set_smem(attn_bwd_dq_kernel, smem_q, once_q, rc_q) != cudaSuccess) return rc_q;
  if (set_smem(attn_bwd_dkdv_kernel, smem_kv, once_kv, rc_kv) != cudaSuccess) return rc_kv;
  AttnArgs P{};
  P.q = static_cast<const uint16_t*>(q);
  P.k = static_cast<const uint16_t*>(k);
  P.v = static_cast<const uint16_t*>(v);
  P.o = static_cast<const uint16_t*>(o);
  P.dout = static_cast<const uint16_t*>(dout);
  P.out = static_cast<uint16_t*>(dq);
  P.dk = static_cast<uint16_t*>(dk);
  P.dv = static_cast<uint16_t*>(dv);
  P.lse = const_cast<float*>(lse);
  P.D = D;
  P.T = static_cast<int>(T);
  P.H = H;
  P.KV = KV;
  P.scale = scale;
  // partials after the row dots, on a 256-byte boundary (float4 loads)
  P.part = D + (static_cast<int64_t>(H) * T + 63) / 64 * 64;
  const int64_t warps = T * H;
  count_launch();
  attn_bwd_dot_kernel<<<static_cast<unsigned>((warps * 32 + 255) / 256), 256, 0, st>>>(P);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  const unsigned tiles = static_cast<unsigned>((T + kBM - 1) / kBM);
  count_launch();
  attn_bwd_dq_kernel<<<dim3(tiles, H), 128, smem_q, st>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  count_launch();
  attn_bwd_dkdv_kernel<<<dim3(tiles, H), 128, smem_kv, st>>>(P);
  e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  int64_t grid = (T * KV * (kD / 4) + 255) / 256;
  if (grid > static_cast<int64_t>(sms) * 8) grid = static_cast<int64_t>(sms) * 8;
  count_launch();
  attn_bwd_kv_reduce_kernel<<<static_cast<unsigned>(grid), 256, 0, st>>>(P);
  return cudaGetLastError();
}

}  // namespace hsnf4
