// lora_rank.cu -- the rank-r pieces of the LoRA linear around the fused GEMM
// (sm_100a: TMA tiles, tcgen05 MMA into tensor memory), for a group of
// independent problems per launch.
//
//   project:  t = Z Adp^T         Z bf16 [T, C]; Adp = A [r, C] (forward,
//             t = X A^T) or B [C, r] (backward, u = dY B).  Writes t (fp32
//             [T, r]), zs = bf16(s t) ([T, r_pad], pad columns 0: the
//             operand of the GEMM's rank-r slice) and, in the backward, the
//             bf16 parts t = hi + lo of u and of the forward's t (the
//             adapter-gradient operands below).
//   grad:     out = s Z^T V        Z bf16 [T, C], V = hi + lo ([T, r_pad]
//             bf16 each).  dB = s dY^T t ([n_out, r]); dA = s u^T X ([r, k_in]).
//
// Both are bound by reading Z once from HBM (Poros API reference: the LoRA
// adapters of rank lora_rank on every projection; the pages print no kernel,
// so the design here is this library's own).  Problems of a group that read
// the same Z (q, k, v, gate and up share their input) are stacked along the
// MMA's N side, so their shared input is read once for all of them.
//
// project: two passes.  Pass 1 is persistent: an item is one group's 128
// tokens x one slice of the contraction (slices sized so that every SM gets
// a few items); warp 0 streams 64-column steps of Z and of the stacked
// adapters through a ring of shared-memory stages (TMA, 128B swizzle; B read
// MN-major with a 32B swizzle) without pausing between items, warp 1 issues
// tcgen05.mma.cta_group::1 (M = 128 tokens, N = stacked ranks) into one of
// two TMEM accumulators, and four warps write the other accumulator to the
// item's fp32 partial meanwhile.  Pass 2 adds each token's partials, a warp
// per token, in an order fixed by the sizes (deterministic, no atomics) and
// writes the outputs.
//
// grad (persistent, same roles): an item is 128 columns c of Z over every
// token, D[c, j] = sum_t Z[t, c] V[t, j], with Z read MN-major (the same
// shared-memory tile a K-major read would use, another descriptor) and V
// MN-major.  The fp32
// factor V enters as two exact bf16 parts, both multiplied, so every
// product keeps ~16 significant bits and accumulates in fp32 in token order.
//
// Every wait is bounded: a wait that runs out records a flag in
// g_rank_flags (read by hsnf4_device_status), drains what its CTA started
// and lets the kernel finish.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>
#include <utility>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace hsnf4 {

__device__ unsigned int g_rank_flags;

enum : unsigned int {
  kRkFlagProducer = 1u << 8,
  kRkFlagMma = 1u << 9,
  kRkFlagEpilogue = 1u << 10,
  kRkFlagDrain = 1u << 11,
};

constexpr int kRkMaxGroups = 8;
constexpr int kRkMaxProbs = 8;
constexpr int kRkMaxN = 128;      // stacked ranks per item (two TMEM accumulators fit)
constexpr int kRkZBytes = 128 * 128;  // 128 rows x 64 bf16

__device__ __forceinline__ uint16_t bf16_bits_rn(float x) {
  const __nv_bfloat16 b = __float2bfloat16_rn(x);
  return *reinterpret_cast<const uint16_t*>(&b);
}

// x = hi + lo with hi = bf16(x), lo = bf16(x - hi) (the difference is exact
// in fp32): two bf16 numbers carrying ~16 significant bits of x.
__device__ __forceinline__ void split_bf16(float x, uint16_t& hi, uint16_t& lo) {
  const __nv_bfloat16 h = __float2bfloat16_rn(x);
  hi = *reinterpret_cast<const uint16_t*>(&h);
  lo = bf16_bits_rn(__fsub_rn(x, __bfloat162float(h)));
}

// TMEM columns to allocate for n accumulator columns (a power of two >= 32)
__host__ __device__ inline int tmem_cols_for(int n) {
  int c = 32;
  while (c < n) c <<= 1;
  return c;
}

// ---------------------------------------------------------------- project

struct RkProjProb {
  CUtensorMap map_adp;  // fwd: A [r, C], box {64, r_pad}, 128B swizzle (K-major rows j)
                        // bwd: B [C, r], box {16, 64}, 32B swizzle (MN-major: j contiguous)
  float* t_out;         // fp32 [T, r]
  uint16_t* zs;         // bf16 [T, r_pad] = s t (0 if zero_zs)
  uint16_t* hi;         // optional bf16 [T, r_pad]: the two parts of t
  uint16_t* lo;
  const float* split_src;  // optional fp32 [T, r] (the forward's t) ...
  uint16_t* split_hi;      // ... written as two bf16 parts [T, r_pad]
  uint16_t* split_lo;
  int zero_zs;
};

struct RkProjGroup {
  CUtensorMap map_z;  // Z bf16 [T, C], box {64, 128}, 128B swizzle
  float* part;        // fp32 partials [t_tiles * 128][chunks][N] of this group
  int nk;             // 64-column steps of the contraction
  int chunks;         // slices of the contraction (ceil(nk / L))
  int n_prob;         // problems stacked on this Z (N = n_prob * r_pad)
  int prob[kRkMaxProbs];
  int item0;          // first item of this group (t_tiles * chunks items)
  int out0;           // first thread of this group in the reduce pass
};

constexpr int kPrjStagesMax = 8;
constexpr int kPrjThreads = 192;

struct RkProjParams {
  RkProjGroup g[kRkMaxGroups];
  RkProjProb p[kRkMaxProbs];
  int n_groups, n_items, n_out, T, r, r_pad, bwd, max_n, stages, tmem_cols, L;
  float s;
};

// Pass 1 (persistent).  An item is one group's 128-token tile x one slice of
// L contraction steps; CTA b takes items b, b + gridDim.x, ...  Warp 0
// streams the items' steps through the ring without pausing between items,
// warp 1 issues each item's MMAs into one of two TMEM accumulators, and
// warps 2..5 write the other accumulator (the previous item) to the item's
// fp32 partial in global memory meanwhile.
__global__ void __launch_bounds__(kPrjThreads, 1) lora_project_tc(const __grid_constant__ RkProjParams P) {
  extern __shared__ uint8_t rk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rk_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[kPrjStagesMax], empty[kPrjStagesMax], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int R = P.r_pad;
  const int S = P.stages;
  const int stage_bytes = kRkZBytes + P.max_n * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = P.tmem_cols;
  // item -> (group, token tile, chunk, first step, steps)
  auto item = [&](int it, int& gi, int& tt, int& ch, int& k_lo, int& nsteps) {
    gi = 0;
    while (gi + 1 < P.n_groups && it >= P.g[gi + 1].item0) ++gi;
    const RkProjGroup& G = P.g[gi];
    const int local = it - G.item0;
    tt = local / G.chunks;
    ch = local % G.chunks;
    k_lo = ch * P.L;
    nsteps = min(P.L, G.nk - k_lo);
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, static_cast<uint32_t>(2 * tcols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait_then_release();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  int last_load = -1;
  bool mma_issued = false;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (the whole
    // warp: lane 0 waits for the stage and arms its barrier, then the lanes
    // issue the step's boxes side by side)
    int g = 0, s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
      int gi, tt, ch, k_lo, nsteps;
      item(it, gi, tt, ch, k_lo, nsteps);
      const RkProjGroup& G = P.g[gi];
      const int N = G.n_prob * R;
      const int n_adp = P.bwd ? R / 16 : G.n_prob;  // adapter boxes per step
      for (int k = 0; k < nsteps; ++k, ++g) {
        if (lane == 0 && g >= S)
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_p, &g_rank_flags, kRkFlagProducer);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + s * stage_bytes;
        const int kc = (k_lo + k) * 64;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kRkZBytes + N * 128));
        __syncwarp();
        uint8_t* ad = st + kRkZBytes;
        if (lane == 0) {
          tma_load_2d(st, &G.map_z, &full[s], kc, tt * 128);
        } else if (lane <= n_adp) {
          const int a = lane - 1;
          if (!P.bwd)
            tma_load_2d(ad + a * R * 128, &P.p[G.prob[a]].map_adp, &full[s], kc, 0);
          else
            tma_load_2d(ad + a * 64 * 32, &P.p[G.prob[0]].map_adp, &full[s], a * 16, kc);
        }
        last_load = g;
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer
    if (lane == 0) {
      const uint64_t a0 = make_sdesc(smem_u32(smem), 16, 1024, kLayoutSw128);
      // adapters: K-major rows (forward A) or MN-major 16-rank atoms 2 KiB
      // apart (backward B); a 16-wide K step is 32 B along a row, or 16 rows
      // of 32 B
      const uint64_t b0 = P.bwd ? make_sdesc(smem_u32(smem + kRkZBytes), 64 * 32, 256, kLayoutSw32)
                                : make_sdesc(smem_u32(smem + kRkZBytes), 16, 1024, kLayoutSw128);
      const uint32_t b_k16 = P.bwd ? (512 >> 4) : (32 >> 4);
      int s = 0, li = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x, ++li) {
        int gi, tt, ch, k_lo, nsteps;
        item(it, gi, tt, ch, k_lo, nsteps);
        const int N = P.g[gi].n_prob * R;
        const uint32_t idesc = make_idesc_bf16(128, N, 0, P.bwd ? 1 : 0);
        const int b = li & 1;
        const uint32_t acc = tmem + static_cast<uint32_t>(b * tcols);
        if (li >= 2) {  // the epilogue has drained this accumulator's previous item
          if (!mbar_wait(&acc_empty[b], ((li >> 1) - 1) & 1, abort_p, &g_rank_flags,
                         kRkFlagMma))
            break;
          tc_fence_after();
        }
        for (int k = 0; k < nsteps; ++k) {
          if (!mbar_wait(&full[s], ph, abort_p, &g_rank_flags, kRkFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((s * stage_bytes) >> 4);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16)
            umma_bf16(acc, a0 + so + k16 * 2, b0 + so + k16 * b_k16, idesc,
                      (k > 0 || k16 > 0) ? 1u : 0u);
          mma_issued = true;
          umma_commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[b]);
      }
    }
  } else {
    // ---------------------------------------------- epilogue (warps 2..5)
    const int q4 = warp & 3;         // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;  // accumulator row = token row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    int li = 0;
    for (int it = blockIdx.x; it < P.n_items; it += gridDim.x, ++li) {
      int gi, tt, ch, k_lo, nsteps;
      item(it, gi, tt, ch, k_lo, nsteps);
      const RkProjGroup& G = P.g[gi];
      const int N = G.n_prob * R;
      const int b = li & 1;
      if (!mbar_wait(&acc_full[b], (li >> 1) & 1, abort_p, &g_rank_flags, kRkFlagEpilogue))
        break;
      tc_fence_after();
      // partials of a token are contiguous over slices: [token][slice][N]
      float* dst = G.part + (static_cast<int64_t>(tt * 128 + row) * G.chunks + ch) * N;
      for (int c0 = 0; c0 < N; c0 += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + static_cast<uint32_t>(b * tcols) + lane_base + static_cast<uint32_t>(c0), v);
        tmem_wait_ld();
#pragma unroll
        for (int j = 0; j < 16; j += 4)
          __stcg(reinterpret_cast<float4*>(dst + c0 + j),
                 make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                             __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3])));
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
  }

  __syncthreads();  // every thread sees the final abort word
  if (*abort_p) {
    volatile int never = 0;
    if (warp == 0 && lane == 0)
      for (int g = (last_load - S + 1 > 0 ? last_load - S + 1 : 0); g <= last_load; ++g)
        if (!mbar_wait(&full[g % S], (g / S) & 1, &never, &g_rank_flags, kRkFlagDrain)) break;
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(&drain);
      mbar_wait(&drain, 0, &never, &g_rank_flags, kRkFlagDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(2 * tcols));
  }
}

// Pass 2: one warp per (group, token); the token's partials are contiguous
// ([slice][N]).  With Q = N / 4 column quads rounded up to a power of two,
// lane l takes quad l % Q and adds the slices l / Q, l / Q + 32 / Q, ... in
// order; a fixed butterfly then adds the 32 / Q lane sums of each quad (the
// order depends only on the sizes, never on timing).  The lanes holding a
// quad's total write t, s t and the optional bf16 parts.
__global__ void __launch_bounds__(256) lora_project_reduce(const __grid_constant__ RkProjParams P) {
  pdl_wait_then_release();
  const int idx = static_cast<int>(blockIdx.x) * 8 + static_cast<int>(threadIdx.x >> 5);
  const int lane = threadIdx.x & 31;
  if (idx >= P.n_out) return;
  int gi = 0;
  while (gi + 1 < P.n_groups && idx >= P.g[gi + 1].out0) ++gi;
  const RkProjGroup& G = P.g[gi];
  const int R = P.r_pad, N = G.n_prob * R, quads = N / 4;
  const int t = idx - G.out0;
  int Q = 1;
  while (Q < quads) Q <<= 1;
  const int S = 32 / Q;  // lanes per quad
  const int q4 = lane % Q, sub = lane / Q;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (q4 < quads) {
    const float4* src =
        reinterpret_cast<const float4*>(G.part + static_cast<int64_t>(t) * G.chunks * N) + q4;
    // sixteen loads in flight (the tail of a batch predicated off), then the
    // adds in slice order
    for (int ch0 = sub; ch0 < G.chunks; ch0 += 16 * S) {
      float4 v[16];
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (ch0 + k * S < G.chunks) v[k] = __ldcg(src + static_cast<int64_t>(ch0 + k * S) * quads);
#pragma unroll
      for (int k = 0; k < 16; ++k)
        if (ch0 + k * S < G.chunks) {
          acc.x += v[k].x;
          acc.y += v[k].y;
          acc.z += v[k].z;
          acc.w += v[k].w;
        }
    }
  }
  for (int m = Q; m < 32; m <<= 1) {
    acc.x += __shfl_xor_sync(0xffffffffu, acc.x, m);
    acc.y += __shfl_xor_sync(0xffffffffu, acc.y, m);
    acc.z += __shfl_xor_sync(0xffffffffu, acc.z, m);
    acc.w += __shfl_xor_sync(0xffffffffu, acc.w, m);
  }
  if (sub != 0 || q4 >= quads) return;
  const int c = q4 * 4;
  const int q = c / R, j = c % R;  // 4 columns of problem q, ranks j .. j + 3
  const RkProjProb& pr = P.p[G.prob[q]];
  const float a[4] = {acc.x, acc.y, acc.z, acc.w};
  uint16_t zsv[4], hv[4], lv[4];
#pragma unroll
  for (int e4 = 0; e4 < 4; ++e4) {
    const bool real = j + e4 < P.r;
    if (real) pr.t_out[static_cast<int64_t>(t) * P.r + j + e4] = a[e4];
    zsv[e4] = (real && !pr.zero_zs) ? bf16_bits_rn(__fmul_rn(P.s, a[e4])) : 0;
    split_bf16(real ? a[e4] : 0.0f, hv[e4], lv[e4]);
  }
  const int64_t o = static_cast<int64_t>(t) * R + j;
  *reinterpret_cast<uint2*>(pr.zs + o) =
      make_uint2(zsv[0] | (uint32_t(zsv[1]) << 16), zsv[2] | (uint32_t(zsv[3]) << 16));
  if (pr.hi) {
    *reinterpret_cast<uint2*>(pr.hi + o) =
        make_uint2(hv[0] | (uint32_t(hv[1]) << 16), hv[2] | (uint32_t(hv[3]) << 16));
    *reinterpret_cast<uint2*>(pr.lo + o) =
        make_uint2(lv[0] | (uint32_t(lv[1]) << 16), lv[2] | (uint32_t(lv[3]) << 16));
  }
  if (pr.split_src) {  // the forward's t of the same token, as two bf16 parts
#pragma unroll
    for (int e4 = 0; e4 < 4; ++e4) {
      const float x = (j + e4 < P.r) ? pr.split_src[static_cast<int64_t>(t) * P.r + j + e4] : 0.f;
      split_bf16(x, hv[e4], lv[e4]);
    }
    *reinterpret_cast<uint2*>(pr.split_hi + o) =
        make_uint2(hv[0] | (uint32_t(hv[1]) << 16), hv[2] | (uint32_t(hv[3]) << 16));
    *reinterpret_cast<uint2*>(pr.split_lo + o) =
        make_uint2(lv[0] | (uint32_t(lv[1]) << 16), lv[2] | (uint32_t(lv[3]) << 16));
  }
}

// ---------------------------------------------------------------- grad

struct RkGradProb {
  CUtensorMap map_hi;  // V hi: bf16 [T, r_pad], box {16, 64}, 32B swizzle
  CUtensorMap map_lo;  // V lo: the same
  float* out;          // [C, r] (c_major: dB) or [r, C] (dA)
  int c_major;
};

struct RkGradGroup {
  CUtensorMap map_z;  // Z bf16 [T, C], box {64, 64}, 128B swizzle (read MN-major)
  int64_t C;
  int n_prob;
  int prob[kRkMaxProbs];
  int cta0;           // first CTA of this group (ceil(C / 128) CTAs)
};

struct RkGradParams {
  RkGradGroup g[2 * kRkMaxGroups];
  RkGradProb p[2 * kRkMaxProbs];
  int n_groups, n_items, T, r, r_pad, nk, max_n, stages, tmem_cols;
  float s;
};

constexpr int kGrdStagesMax = 8;
constexpr int kGrdMT = 2;                   // 128-row M tiles per item
constexpr int kGrdCols = 128 * kGrdMT;      // columns of Z per item
constexpr int kGrdZBytes = kGrdMT * 16384;  // Z per step: kGrdCols x 64 tokens

// Persistent: CTA b takes items b, b + gridDim.x, ... (an item = one group's
// 128-column tile over every token).  Warp 0 streams the items' steps
// through the ring without pausing between items, warp 1 issues each item's
// MMAs into one of two TMEM accumulators, and warps 2..5 drain the other
// accumulator (the previous item) meanwhile, so loads stay in flight across
// item boundaries.
constexpr int kGrdThreads = 192;

__global__ void __launch_bounds__(kGrdThreads, 1) lora_grad_tc(const __grid_constant__ RkGradParams P) {
  extern __shared__ uint8_t rk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rk_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[kGrdStagesMax], empty[kGrdStagesMax], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const int R = P.r_pad;
  const int S = P.stages;
  const int stage_bytes = kGrdZBytes + 2 * P.max_n * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = P.tmem_cols;  // per accumulator; 2 x kGrdMT of them
  const int nsteps = P.nk;
  // item -> (group, first column)
  auto item_of = [&](int it, int& gi, int& c0) {
    gi = 0;
    while (gi + 1 < P.n_groups && it >= P.g[gi + 1].cta0) ++gi;
    c0 = (it - P.g[gi].cta0) * kGrdCols;
  };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, static_cast<uint32_t>(2 * kGrdMT * tcols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  pdl_wait_then_release();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  int last_load = -1;
  bool mma_issued = false;

  if (warp == 0) {
    // ---------------------------------------------- TMA producer (the whole
    // warp: lane 0 waits for the stage and arms its barrier, then the lanes
    // issue the step's boxes side by side)
    int g = 0, s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x) {
      int gi, c0;
      item_of(it, gi, c0);
      const RkGradGroup& G = P.g[gi];
      const int vbytes = G.n_prob * R * 128;
      const int n_atoms = G.n_prob * (R / 16);  // 16-rank V atoms per part
      for (int i = 0; i < nsteps; ++i, ++g) {
        if (lane == 0 && g >= S)
          ok = mbar_wait(&empty[s], ph ^ 1u, abort_p, &g_rank_flags, kRkFlagProducer);
        ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + s * stage_bytes;
        const int tk = i * 64;
        if (lane == 0)
          mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(kGrdZBytes + 2 * vbytes));
        __syncwarp();
        // Z: per 128-column M tile two 64-column atoms (rows = tokens), the
        // MN-major operand layout; the tiles of an item are adjacent columns.
        // The first lanes load them, the next lanes the V atoms (hi parts,
        // then lo parts), one box per lane.
        for (int box = lane; box < 2 * kGrdMT + 2 * n_atoms; box += 32) {
          if (box < 2 * kGrdMT) {
            tma_load_2d(st + box * 8192, &G.map_z, &full[s], c0 + 64 * box, tk);
          } else {
            const int v = box - 2 * kGrdMT;
            const int part = v / n_atoms, atom = v % n_atoms;  // part 0: hi, 1: lo
            const RkGradProb& pr = P.p[G.prob[atom / (R / 16)]];
            tma_load_2d(st + kGrdZBytes + part * vbytes + atom * 2048,
                        part ? &pr.map_lo : &pr.map_hi, &full[s], (atom % (R / 16)) * 16, tk);
          }
        }
        last_load = g;
        if (++s == S) {
          s = 0;
          ph ^= 1u;
        }
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer
    if (lane == 0) {
      // A = Z MN-major: two 64-column atoms 8 KiB apart (LBO), 8-token groups
      // 1 KiB apart (SBO), 16 tokens = 2 KiB per K step.  B = V MN-major, 32B
      // swizzle: 16-rank atoms 2 KiB apart (LBO), 8-token groups 256 B apart
      // (SBO), 16 tokens = 512 B per K step; the lo parts follow the hi parts.
      const uint64_t a0 = make_sdesc(smem_u32(smem), 64 * 128, 1024, kLayoutSw128);
      const uint64_t b0 = make_sdesc(smem_u32(smem + kGrdZBytes), 2048, 256, kLayoutSw32);
      int s = 0, li = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (int it = blockIdx.x; it < P.n_items && ok; it += gridDim.x, ++li) {
        int gi, c0;
        item_of(it, gi, c0);
        const int N = P.g[gi].n_prob * R;
        const uint32_t idesc = make_idesc_bf16(128, N, 1, 1);
        const uint32_t lo_off = static_cast<uint32_t>(N * 128) >> 4;  // V lo after V hi
        const int b = li & 1;
        const uint32_t acc = tmem + static_cast<uint32_t>(b * kGrdMT * tcols);
        if (li >= 2) {  // the epilogue has drained these accumulators' previous item
          if (!mbar_wait(&acc_empty[b], ((li >> 1) - 1) & 1, abort_p, &g_rank_flags,
                         kRkFlagMma))
            break;
          tc_fence_after();
        }
        for (int i = 0; i < nsteps; ++i) {
          if (!mbar_wait(&full[s], ph, abort_p, &g_rank_flags, kRkFlagMma)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint64_t so = static_cast<uint64_t>((s * stage_bytes) >> 4);
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint64_t bd = b0 + so + k16 * (512 >> 4);
#pragma unroll
            for (int m = 0; m < kGrdMT; ++m) {
              const uint64_t ad = a0 + so + (m * 16384 >> 4) + k16 * (2048 >> 4);
              const uint32_t d = acc + static_cast<uint32_t>(m * tcols);
              umma_bf16(d, ad, bd, idesc, (i > 0 || k16 > 0) ? 1u : 0u);
              umma_bf16(d, ad, bd + lo_off, idesc, 1u);
            }
          }
          mma_issued = true;
          umma_commit(&empty[s]);
          if (++s == S) {
            s = 0;
            ph ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit(&acc_full[b]);
      }
    }
  } else {
    // ---------------------------------------------- epilogue (warps 2..5)
    const int q4 = warp & 3;                      // TMEM lane quarter of this warp
    const int row = q4 * 32 + lane;               // accumulator row = column c0 + row
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    int li = 0;
    for (int it = blockIdx.x; it < P.n_items; it += gridDim.x, ++li) {
      int gi, c0;
      item_of(it, gi, c0);
      const RkGradGroup& G = P.g[gi];
      const int b = li & 1;
      if (!mbar_wait(&acc_full[b], (li >> 1) & 1, abort_p, &g_rank_flags, kRkFlagEpilogue))
        break;
      tc_fence_after();
      for (int m = 0; m < kGrdMT; ++m) {
      const int c = c0 + m * 128 + row;
      const uint32_t accm = tmem + static_cast<uint32_t>((b * kGrdMT + m) * tcols) + lane_base;
      for (int q = 0; q < G.n_prob; ++q) {
        const RkGradProb& pr = P.p[G.prob[q]];
        for (int jc = 0; jc < R; jc += 16) {
          uint32_t v[16];
          tmem_ld16(accm + static_cast<uint32_t>(q * R + jc), v);
          tmem_wait_ld();
          if (c >= G.C) continue;
          if (pr.c_major) {  // dB [C, r]: this thread's row, 16 consecutive ranks
            float* o = pr.out + static_cast<int64_t>(c) * P.r + jc;
            if (P.r - jc >= 16 && (P.r % 4) == 0) {
#pragma unroll
              for (int j = 0; j < 16; j += 4)
                *reinterpret_cast<float4*>(o + j) =
                    make_float4(__fmul_rn(P.s, __uint_as_float(v[j])),
                                __fmul_rn(P.s, __uint_as_float(v[j + 1])),
                                __fmul_rn(P.s, __uint_as_float(v[j + 2])),
                                __fmul_rn(P.s, __uint_as_float(v[j + 3])));
            } else {
#pragma unroll
              for (int j = 0; j < 16; ++j)
                if (jc + j < P.r) o[j] = __fmul_rn(P.s, __uint_as_float(v[j]));
            }
          } else {  // dA [r, C]: one column, coalesced across the warp
#pragma unroll
            for (int j = 0; j < 16; ++j)
              if (jc + j < P.r)
                pr.out[static_cast<int64_t>(jc + j) * G.C + c] =
                    __fmul_rn(P.s, __uint_as_float(v[j]));
          }
        }
      }
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);
    }
  }

  __syncthreads();  // every thread sees the final abort word
  if (*abort_p) {
    volatile int never = 0;
    if (warp == 0 && lane == 0)
      for (int g = (last_load - S + 1 > 0 ? last_load - S + 1 : 0); g <= last_load; ++g)
        if (!mbar_wait(&full[g % S], (g / S) & 1, &never, &g_rank_flags, kRkFlagDrain)) break;
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(&drain);
      mbar_wait(&drain, 0, &never, &g_rank_flags, kRkFlagDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(2 * kGrdMT * tcols));
  }
}

// ---------------------------------------------------------------- host side

static int project_stage_bytes(int N) { return kRkZBytes + N * 128; }
static int grad_stage_bytes(int N) { return kGrdZBytes + 2 * N * 128; }

constexpr int kRkMaxSmem = 200 * 1024 + 1024;

static cudaError_t rk_configure() {
  static cudaError_t rc = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    rc = cudaFuncSetAttribute(lora_project_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kRkMaxSmem);
    if (rc == cudaSuccess)
      rc = cudaFuncSetAttribute(lora_grad_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                kRkMaxSmem);
  });
  return rc;
}

// Problems reading the same Z (same pointer and width) share one item; a
// group takes as many problems as fit kRkMaxN stacked ranks.
template <typename GetZ>
static int stack_groups(int n, int r_pad, GetZ getz, int (*members)[kRkMaxProbs], int* counts) {
  int ng = 0;
  int gid[16];
  for (int q = 0; q < n; ++q) {
    int found = -1;
    for (int g = 0; g < ng; ++g) {
      const int first = members[g][0];
      if (getz(first).first == getz(q).first && getz(first).second == getz(q).second &&
          (counts[g] + 1) * r_pad <= kRkMaxN) {
        found = g;
        break;
      }
    }
    if (found < 0) {
      found = ng++;
      counts[found] = 0;
    }
    members[found][counts[found]++] = q;
    gid[q] = found;
  }
  (void)gid;
  return ng;
}

// The launch plan of a projection group: the stacked groups, the slice
// length L (steps) and each group's partial offset; fills P (maps aside) and
// returns the partial bytes (0 for invalid sizes).
struct PrjPlan {
  int ng, L, t_tiles, max_n;
  int members[kRkMaxGroups][kRkMaxProbs], counts[kRkMaxGroups];
  int64_t part_off[kRkMaxGroups];  // bytes
  int64_t part_bytes;
};

static bool prj_plan(const ProjectDesc* d, int n, int64_t T, int r, PrjPlan* pl) {
  if (n < 1 || n > kRkMaxProbs || T < 1 || r < 1) return false;
  const int R = (r + 15) / 16 * 16;
  const bool bwd = !d[0].r_major;
  if (bwd) {  // backward problems read distinct dY: one problem per group
    pl->ng = n;
    for (int q = 0; q < n; ++q) {
      pl->members[q][0] = q;
      pl->counts[q] = 1;
    }
  } else {
    pl->ng = stack_groups(n, R, [&](int q) { return std::make_pair(d[q].Z, d[q].C); },
                          pl->members, pl->counts);
  }
  pl->t_tiles = static_cast<int>((T + 127) / 128);
  int64_t total_steps = 0;
  pl->max_n = 0;
  for (int g = 0; g < pl->ng; ++g) {
    total_steps += static_cast<int64_t>(pl->t_tiles) * (d[pl->members[g][0]].C / 64);
    pl->max_n = std::max(pl->max_n, pl->counts[g] * R);
  }
  // slices of about total / (4 x SMs) steps: every SM gets a few items and
  // long contractions are cut into many
  int dev = 0, sms = 148;
  if (cudaGetDevice(&dev) == cudaSuccess)
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  else
    cudaGetLastError();
  pl->L = static_cast<int>(std::max<int64_t>(4, (total_steps + 4 * sms - 1) / (4 * sms)));
  int64_t off = 0;
  for (int g = 0; g < pl->ng; ++g) {
    const int64_t nk = d[pl->members[g][0]].C / 64;
    const int64_t chunks = (nk + pl->L - 1) / pl->L;
    pl->part_off[g] = off;
    off += static_cast<int64_t>(round_up(
        static_cast<size_t>(pl->t_tiles * chunks * 128 * pl->counts[g] * R) * 4, 256));
  }
  pl->part_bytes = off;
  return true;
}

size_t project_workspace_bytes(const ProjectDesc* d, int n, int64_t T, int r) {
  PrjPlan pl;
  if (!prj_plan(d, n, T, r, &pl)) return 0;
  return static_cast<size_t>(pl.part_bytes);
}

cudaError_t launch_lora_project_group(const ProjectDesc* d, int n, int64_t T, int r, float s,
                                      void* ws, cudaStream_t st) {
  if (n < 1 || n > kRkMaxProbs) return cudaErrorInvalidValue;
  cudaError_t e = rk_configure();
  if (e != cudaSuccess) return e;
  static RkProjParams P;  // large: built on the host, copied into the launch
  static PrjPlan pl;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  if (!prj_plan(d, n, T, r, &pl)) return cudaErrorInvalidValue;
  if (pl.part_bytes > 0 && !ws) return cudaErrorInvalidValue;
  memset(&P, 0, sizeof P);
  const bool bwd = !d[0].r_major;
  P.T = static_cast<int>(T);
  P.r = r;
  P.r_pad = (r + 15) / 16 * 16;
  P.s = s;
  P.bwd = bwd ? 1 : 0;
  P.L = pl.L;
  const int R = P.r_pad;
  for (int q = 0; q < n; ++q) {
    RkProjProb& p = P.p[q];
    bool ok;
    if (!bwd)  // A [r, C]: rows j (r_pad of them, the rest zero-filled), 64 columns a step
      ok = encode_tma_2d(&p.map_adp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q].adp, d[q].C, r,
                         d[q].C * 2, 64, R, CU_TENSOR_MAP_SWIZZLE_128B);
    else  // B [C, r]: 16 ranks (32 bytes) x 64 rows c per box
      ok = encode_tma_2d(&p.map_adp, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q].adp, r, d[q].C,
                         static_cast<uint64_t>(r) * 2, 16, 64, CU_TENSOR_MAP_SWIZZLE_32B);
    if (!ok) return cudaErrorInvalidValue;
    p.t_out = d[q].t_out;
    p.zs = static_cast<uint16_t*>(d[q].zs);
    p.hi = static_cast<uint16_t*>(d[q].hi);
    p.lo = static_cast<uint16_t*>(d[q].lo);
    p.split_src = d[q].split_src;
    p.split_hi = static_cast<uint16_t*>(d[q].split_hi);
    p.split_lo = static_cast<uint16_t*>(d[q].split_lo);
    p.zero_zs = d[q].zero_zs ? 1 : 0;
  }
  int items = 0, outs = 0;
  double bytes = 0;
  for (int g = 0; g < pl.ng; ++g) {
    RkProjGroup& G = P.g[g];
    const int q0 = pl.members[g][0];
    if (!encode_tma_2d(&G.map_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q0].Z, d[q0].C, T,
                       d[q0].C * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    G.part = reinterpret_cast<float*>(static_cast<uint8_t*>(ws) + pl.part_off[g]);
    G.nk = static_cast<int>(d[q0].C / 64);
    G.chunks = (G.nk + pl.L - 1) / pl.L;
    G.n_prob = pl.counts[g];
    for (int k = 0; k < pl.counts[g]; ++k) G.prob[k] = pl.members[g][k];
    G.item0 = items;
    items += pl.t_tiles * G.chunks;
    G.out0 = outs;
    outs += static_cast<int>(T);  // one warp per token
    bytes += 2.0 * T * d[q0].C;
  }
  P.n_groups = pl.ng;
  P.n_items = items;
  P.n_out = outs;
  P.max_n = pl.max_n;
  P.tmem_cols = tmem_cols_for(pl.max_n);
  const int stage = project_stage_bytes(pl.max_n);
  P.stages = std::max(2, std::min(kPrjStagesMax, (190 * 1024) / stage));
  const int smem = P.stages * stage + 1024;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(items, sms);
  void* prof = prof_begin(st, kProfProject);
  e = launch_pdl(lora_project_tc, dim3(grid), dim3(kPrjThreads), smem, st, P);
  if (e == cudaSuccess)
    e = launch_pdl(lora_project_reduce, dim3((outs + 7) / 8), dim3(256), 0, st, P);
  prof_end(prof, kProfProject, bytes, st);
  return e;
}

cudaError_t launch_lora_grad_group(const GradDesc* d, int n, int64_t T, int r, float s,
                                   cudaStream_t st) {
  if (n < 1 || n > 2 * kRkMaxProbs) return cudaErrorInvalidValue;
  cudaError_t e = rk_configure();
  if (e != cudaSuccess) return e;
  static RkGradParams P;
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&P, 0, sizeof P);
  P.T = static_cast<int>(T);
  P.r = r;
  P.r_pad = (r + 15) / 16 * 16;
  P.s = s;
  P.nk = static_cast<int>((T + 63) / 64);
  const int R = P.r_pad;
  for (int q = 0; q < n; ++q) {
    RkGradProb& p = P.p[q];
    if (!encode_tma_2d(&p.map_hi, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q].V_hi, R, T,
                       static_cast<uint64_t>(R) * 2, 16, 64, CU_TENSOR_MAP_SWIZZLE_32B) ||
        !encode_tma_2d(&p.map_lo, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q].V_lo, R, T,
                       static_cast<uint64_t>(R) * 2, 16, 64, CU_TENSOR_MAP_SWIZZLE_32B))
      return cudaErrorInvalidValue;
    p.out = d[q].out;
    p.c_major = d[q].c_major ? 1 : 0;
  }
  // problems reading the same Z with the same output orientation share an item
  int members[2 * kRkMaxGroups][kRkMaxProbs], counts[2 * kRkMaxGroups];
  const int ng = stack_groups(
      n, R,
      [&](int q) {
        return std::make_pair(d[q].Z, d[q].C * 2 + (d[q].c_major ? 1 : 0));
      },
      members, counts);
  int ctas = 0, max_n = 0;
  double bytes = 0;
  for (int g = 0; g < ng; ++g) {
    RkGradGroup& G = P.g[g];
    const int q0 = members[g][0];
    if (!encode_tma_2d(&G.map_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q0].Z, d[q0].C, T,
                       d[q0].C * 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    G.C = d[q0].C;
    G.n_prob = counts[g];
    for (int k = 0; k < counts[g]; ++k) G.prob[k] = members[g][k];
    G.cta0 = ctas;  // first item of this group
    ctas += static_cast<int>((d[q0].C + kGrdCols - 1) / kGrdCols);
    max_n = std::max(max_n, counts[g] * R);
    bytes += 2.0 * T * d[q0].C;
  }
  P.n_groups = ng;
  P.n_items = ctas;
  P.max_n = max_n;
  P.tmem_cols = tmem_cols_for(max_n);
  // ring: as many stages as fit about 190 KiB (one CTA per SM)
  const int stage = grad_stage_bytes(max_n);
  P.stages = std::max(2, std::min(kGrdStagesMax, (190 * 1024) / stage));
  const int smem = P.stages * stage + 1024;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int grid = std::min(ctas, sms);
  void* prof = prof_begin(st, kProfGrad);
  e = launch_pdl(lora_grad_tc, dim3(grid), dim3(kGrdThreads), smem, st, P);
  prof_end(prof, kProfGrad, bytes, st);
  return e;
}

cudaError_t read_rank_flags(uint32_t* flags) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_rank_flags, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_rank_flags, &z, sizeof z);
  }
  return e;
}

}  // namespace hsnf4
