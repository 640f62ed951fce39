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
// project: a CTA takes 128 tokens x one slice of the contraction.  Warp 0
// streams 64-column steps of Z and of the stacked adapters through a ring of
// shared-memory stages (TMA, 128B swizzle), warp 1 issues
// tcgen05.mma.cta_group::1 (M = 128 tokens, N = stacked ranks, bf16 in,
// fp32 accumulate in TMEM).  The CS CTAs of a thread-block cluster split the
// contraction of one token tile; each writes its fp32 partial to its own
// shared memory and the cluster adds the CS partials through distributed
// shared memory in slice order, so the sum never depends on timing and no
// second pass or atomic is needed.
//
// grad: a CTA takes 128 columns c of Z and every token: D[c, j] =
// sum_t Z[t, c] V[t, j] with Z read MN-major (the same shared-memory tile a
// K-major read would use, another descriptor) and V MN-major.  The fp32
// factor V enters as two exact bf16 parts, both multiplied, so every
// product keeps ~16 significant bits and accumulates in fp32 in token order.
//
// Every wait is bounded: a wait that runs out records a flag in
// g_rank_flags (read by hsnf4_device_status), drains what its CTA started
// and lets the kernel finish.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <map>
#include <mutex>
#include <tuple>
#include <utility>

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

constexpr int kRkThreads = 128;   // 4 warps: TMEM lanes 0..127 = tile rows
constexpr int kRkStages = 4;
constexpr int kRkMaxGroups = 8;
constexpr int kRkMaxProbs = 8;
constexpr int kRkMaxN = 128;      // stacked ranks per item (the partial tile fits the ring)
constexpr int kRkZBytes = 128 * 128;  // 128 rows x 64 bf16

__device__ __forceinline__ float4 ld_dsmem_f32x4(uint32_t local_addr, uint32_t rank) {
  float4 v;
  asm volatile(
      "{\n\t.reg .b32 ra;\n\t"
      "mapa.shared::cluster.u32 ra, %4, %5;\n\t"
      "ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [ra];\n\t}"
      : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
      : "r"(local_addr), "r"(rank)
      : "memory");
  return v;
}

__device__ __forceinline__ uint32_t cluster_nctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_nctarank;" : "=r"(r));
  return r;
}

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
  int nk;             // 64-column steps of the contraction
  int n_prob;         // problems stacked on this Z (N = n_prob * r_pad)
  int prob[kRkMaxProbs];
  int cluster0;       // first cluster of this group (t_tiles clusters each)
};

struct RkProjParams {
  RkProjGroup g[kRkMaxGroups];
  RkProjProb p[kRkMaxProbs];
  int n_groups, T, r, r_pad, t_tiles, bwd;
  float s;
};

__global__ void __launch_bounds__(kRkThreads, 1) lora_project_tc(const __grid_constant__ RkProjParams P) {
  extern __shared__ uint8_t rk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rk_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[kRkStages], empty[kRkStages], done, drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  const uint32_t CS = cluster_nctarank();
  const uint32_t crank = cluster_ctarank();
  const int cluster = static_cast<int>(blockIdx.x / CS);
  int gi = 0;
  while (gi + 1 < P.n_groups && cluster >= P.g[gi + 1].cluster0) ++gi;
  const RkProjGroup& G = P.g[gi];
  const int tt = cluster - G.cluster0;
  const int t0 = tt * 128;
  const int R = P.r_pad;
  const int N = G.n_prob * R;
  const int k_lo = static_cast<int>(static_cast<int64_t>(crank) * G.nk / CS);
  const int k_hi = static_cast<int>(static_cast<int64_t>(crank + 1) * G.nk / CS);
  const int nsteps = k_hi - k_lo;
  const int stage_bytes = kRkZBytes + N * 128;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = tmem_cols_for(N);

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRkStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, static_cast<uint32_t>(tcols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  int last_load = -1;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    // ---------------------------------------------- TMA producer
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % kRkStages;
      if (i >= kRkStages &&
          !mbar_wait(&empty[s], ((i / kRkStages) - 1) & 1, abort_p, &g_rank_flags,
                     kRkFlagProducer))
        break;
      uint8_t* st = smem + s * stage_bytes;
      const int kc = (k_lo + i) * 64;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(stage_bytes));
      tma_load_2d(st, &G.map_z, &full[s], kc, t0);
      uint8_t* ad = st + kRkZBytes;
      if (!P.bwd) {
        for (int q = 0; q < G.n_prob; ++q)
          tma_load_2d(ad + q * R * 128, &P.p[G.prob[q]].map_adp, &full[s], kc, 0);
      } else {
        for (int a = 0; a < R / 16; ++a)
          tma_load_2d(ad + a * 64 * 32, &P.p[G.prob[0]].map_adp, &full[s], a * 16, kc);
      }
      last_load = i;
    }
  } else if (warp == 1 && lane == 0) {
    // ---------------------------------------------- MMA issuer
    const uint32_t idesc = make_idesc_bf16(128, N, 0, P.bwd ? 1 : 0);
    const uint64_t a0 = make_sdesc(smem_u32(smem), 16, 1024, kLayoutSw128);
    const uint64_t b0 = P.bwd ? make_sdesc(smem_u32(smem + kRkZBytes), 64 * 32, 256, kLayoutSw32)
                              : make_sdesc(smem_u32(smem + kRkZBytes), 16, 1024, kLayoutSw128);
    // per 16-wide K step: 32 bytes along a 128B-swizzled row (K-major), or
    // 16 rows of 32 bytes (MN-major, 32B swizzle)
    const uint32_t b_k16 = P.bwd ? (512 >> 4) : (32 >> 4);
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % kRkStages;
      if (!mbar_wait(&full[s], (i / kRkStages) & 1, abort_p, &g_rank_flags, kRkFlagMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t ad = a0 + static_cast<uint64_t>((s * stage_bytes) >> 4);
      const uint64_t bd = b0 + static_cast<uint64_t>((s * stage_bytes) >> 4);
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16)
        umma_bf16(tmem, ad + k16 * 2, bd + k16 * b_k16, idesc, (i > 0 || k16 > 0) ? 1u : 0u);
      mma_issued = true;
      umma_commit(&empty[s]);
    }
    if (ok && nsteps > 0) umma_commit(&done);
  }
  __syncwarp();

  // ---------------------------------------------- accumulator -> own partial
  // The ring is free once the last MMA completed: the partial tile (fp32
  // [128][N + 4]: rows 16-byte aligned, the pad spreads rows over banks)
  // reuses it.
  float* part = reinterpret_cast<float*>(smem);
  const int PS = N + 4;
  const int row = threadIdx.x;  // TMEM lane = token row of the tile
  bool have = nsteps > 0;
  if (have)
    have = mbar_wait(&done, 0, abort_p, &g_rank_flags, kRkFlagEpilogue);
  if (have) {
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    for (int c0 = 0; c0 < N; c0 += 16) {
      uint32_t v[16];
      tmem_ld16(tmem + lane_base + static_cast<uint32_t>(c0), v);
      tmem_wait_ld();
#pragma unroll
      for (int j = 0; j < 16; j += 4)
        *reinterpret_cast<float4*>(part + row * PS + c0 + j) =
            make_float4(__uint_as_float(v[j]), __uint_as_float(v[j + 1]),
                        __uint_as_float(v[j + 2]), __uint_as_float(v[j + 3]));
    }
  } else if (!*abort_p) {
    for (int c = 0; c < N; c += 4)
      *reinterpret_cast<float4*>(part + row * PS + c) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
  __syncthreads();  // every thread sees the final abort word
  if (*abort_p) {
    // drain what this CTA started before its shared memory and TMEM go away
    volatile int never = 0;
    if (warp == 0 && lane == 0)
      for (int i = (last_load - kRkStages + 1 > 0 ? last_load - kRkStages + 1 : 0);
           i <= last_load; ++i)
        if (!mbar_wait(&full[i % kRkStages], (i / kRkStages) & 1, &never, &g_rank_flags,
                       kRkFlagDrain))
          break;
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(&drain);
      mbar_wait(&drain, 0, &never, &g_rank_flags, kRkFlagDrain);
    }
  }
  tc_fence_before();
  cluster_sync();  // every CTA's partial written (or this cluster gave up)

  // ---------------------------------------------- ordered cluster sum
  // This CTA owns rows [crank * 128 / CS, (crank + 1) * 128 / CS) of the
  // token tile; each thread takes 4 consecutive columns of one row and adds
  // the CS partials in slice order.
  const int r_lo = static_cast<int>(crank * 128 / CS), r_hi = static_cast<int>((crank + 1) * 128 / CS);
  const int quads = N / 4;
  const bool failed = *abort_p != 0;
  for (int e = threadIdx.x; e < (r_hi - r_lo) * quads && !failed; e += kRkThreads) {
    const int rr = r_lo + e / quads, c = (e % quads) * 4;
    const int t = t0 + rr;
    if (t >= P.T) continue;
    const uint32_t addr = smem_u32(part + rr * PS + c);
    float4 acc = ld_dsmem_f32x4(addr, 0);
    for (uint32_t src = 1; src < CS; ++src) {
      const float4 v = ld_dsmem_f32x4(addr, src);
      acc.x += v.x;
      acc.y += v.y;
      acc.z += v.z;
      acc.w += v.w;
    }
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
    if (pr.split_src) {  // the forward's t of the same rows, as two bf16 parts
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
  tc_fence_before();
  cluster_sync();  // no CTA leaves while a peer may still read its partial
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(tcols));
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
  int n_groups, T, r, r_pad, nk;
  float s;
};

__global__ void __launch_bounds__(kRkThreads, 1) lora_grad_tc(const __grid_constant__ RkGradParams P) {
  extern __shared__ uint8_t rk_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(rk_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t full[kRkStages], empty[kRkStages], done, drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;

  int gi = 0;
  while (gi + 1 < P.n_groups && static_cast<int>(blockIdx.x) >= P.g[gi + 1].cta0) ++gi;
  const RkGradGroup& G = P.g[gi];
  const int c0 = (static_cast<int>(blockIdx.x) - G.cta0) * 128;
  const int R = P.r_pad;
  const int N = G.n_prob * R;
  const int vbytes = N * 64 * 2;                 // one V part of a step: N ranks x 64 tokens
  const int stage_bytes = kRkZBytes + 2 * vbytes;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int tcols = tmem_cols_for(N);
  const int nsteps = P.nk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kRkStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&done, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, static_cast<uint32_t>(tcols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  int last_load = -1;
  bool mma_issued = false;

  if (warp == 0 && lane == 0) {
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % kRkStages;
      if (i >= kRkStages &&
          !mbar_wait(&empty[s], ((i / kRkStages) - 1) & 1, abort_p, &g_rank_flags,
                     kRkFlagProducer))
        break;
      uint8_t* st = smem + s * stage_bytes;
      const int tk = i * 64;
      mbar_arrive_expect_tx(&full[s], static_cast<uint32_t>(stage_bytes));
      // Z: two 64-column atoms (rows = tokens), the MN-major operand layout
      tma_load_2d(st, &G.map_z, &full[s], c0, tk);
      tma_load_2d(st + kRkZBytes / 2, &G.map_z, &full[s], c0 + 64, tk);
      uint8_t* vh = st + kRkZBytes;
      for (int q = 0; q < G.n_prob; ++q) {
        const RkGradProb& pr = P.p[G.prob[q]];
        for (int a = 0; a < R / 16; ++a) {
          const int atom = q * (R / 16) + a;
          tma_load_2d(vh + atom * 2048, &pr.map_hi, &full[s], a * 16, tk);
          tma_load_2d(vh + vbytes + atom * 2048, &pr.map_lo, &full[s], a * 16, tk);
        }
      }
      last_load = i;
    }
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = make_idesc_bf16(128, N, 1, 1);
    // A = Z MN-major: two 64-column atoms 8 KiB apart (LBO), 8-token groups
    // 1 KiB apart (SBO), 16 tokens = 2 KiB per K step.  B = V MN-major, 32B
    // swizzle: 16-rank atoms 2 KiB apart (LBO), 8-token groups 256 B apart
    // (SBO), 16 tokens = 512 B per K step.
    const uint64_t a0 = make_sdesc(smem_u32(smem), 64 * 128, 1024, kLayoutSw128);
    const uint64_t bh0 = make_sdesc(smem_u32(smem + kRkZBytes), 2048, 256, kLayoutSw32);
    const uint64_t bl0 = make_sdesc(smem_u32(smem + kRkZBytes + vbytes), 2048, 256, kLayoutSw32);
    bool ok = true;
    for (int i = 0; i < nsteps; ++i) {
      const int s = i % kRkStages;
      if (!mbar_wait(&full[s], (i / kRkStages) & 1, abort_p, &g_rank_flags, kRkFlagMma)) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint64_t so = static_cast<uint64_t>((s * stage_bytes) >> 4);
#pragma unroll
      for (int k16 = 0; k16 < 4; ++k16) {
        umma_bf16(tmem, a0 + so + k16 * (2048 >> 4), bh0 + so + k16 * (512 >> 4), idesc,
                  (i > 0 || k16 > 0) ? 1u : 0u);
        umma_bf16(tmem, a0 + so + k16 * (2048 >> 4), bl0 + so + k16 * (512 >> 4), idesc, 1u);
      }
      mma_issued = true;
      umma_commit(&empty[s]);
    }
    if (ok && nsteps > 0) umma_commit(&done);
  }
  __syncwarp();

  // ---------------------------------------------- epilogue: row c of D
  const int c = c0 + static_cast<int>(threadIdx.x);
  bool ok = nsteps > 0 && mbar_wait(&done, 0, abort_p, &g_rank_flags, kRkFlagEpilogue);
  if (ok) {
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    for (int q = 0; q < G.n_prob; ++q) {
      const RkGradProb& pr = P.p[G.prob[q]];
      for (int jc = 0; jc < R; jc += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + lane_base + static_cast<uint32_t>(q * R + jc), v);
        tmem_wait_ld();
        if (c >= G.C) continue;
#pragma unroll
        for (int j = 0; j < 16; ++j) {
          if (jc + j >= P.r) break;
          const float val = __fmul_rn(P.s, __uint_as_float(v[j]));
          if (pr.c_major)
            pr.out[static_cast<int64_t>(c) * P.r + jc + j] = val;
          else
            pr.out[static_cast<int64_t>(jc + j) * G.C + c] = val;
        }
      }
    }
  }
  __syncthreads();  // every thread sees the final abort word
  if (*abort_p) {
    volatile int never = 0;
    if (warp == 0 && lane == 0)
      for (int i = (last_load - kRkStages + 1 > 0 ? last_load - kRkStages + 1 : 0);
           i <= last_load; ++i)
        if (!mbar_wait(&full[i % kRkStages], (i / kRkStages) & 1, &never, &g_rank_flags,
                       kRkFlagDrain))
          break;
    if (warp == 1 && lane == 0 && mma_issued) {
      umma_commit(&drain);
      mbar_wait(&drain, 0, &never, &g_rank_flags, kRkFlagDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(tcols));
  }
}

// ---------------------------------------------------------------- host side

static int project_stage_bytes(int N) { return kRkZBytes + N * 128; }
static int grad_stage_bytes(int N) { return kRkZBytes + 2 * N * 128; }

constexpr int kRkMaxSmem = kRkStages * (kRkZBytes + 2 * kRkMaxN * 128) + 1024;

static cudaError_t rk_configure() {
  static cudaError_t rc = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    rc = cudaFuncSetAttribute(lora_project_tc, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kRkMaxSmem);
    if (rc == cudaSuccess)
      rc = cudaFuncSetAttribute(lora_project_tc, cudaFuncAttributeNonPortableClusterSizeAllowed,
                                1);
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

size_t project_workspace_bytes(const ProjectDesc*, int, int64_t, int) { return 0; }

cudaError_t launch_lora_project_group(const ProjectDesc* d, int n, int64_t T, int r, float s,
                                      void*, cudaStream_t st) {
  if (n < 1 || n > kRkMaxProbs) return cudaErrorInvalidValue;
  cudaError_t e = rk_configure();
  if (e != cudaSuccess) return e;
  static RkProjParams P;  // large: built on the host, copied into the launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&P, 0, sizeof P);
  const bool bwd = !d[0].r_major;
  P.T = static_cast<int>(T);
  P.r = r;
  P.r_pad = (r + 15) / 16 * 16;
  P.s = s;
  P.bwd = bwd ? 1 : 0;
  P.t_tiles = static_cast<int>((T + 127) / 128);
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
  // backward problems read distinct dY: one problem per group there
  int members[kRkMaxGroups][kRkMaxProbs], counts[kRkMaxGroups];
  int ng;
  if (bwd) {
    ng = n;
    for (int q = 0; q < n; ++q) {
      members[q][0] = q;
      counts[q] = 1;
    }
  } else {
    ng = stack_groups(n, R, [&](int q) { return std::make_pair(d[q].Z, d[q].C); }, members,
                      counts);
  }
  // cluster size: the widest (16, else 8) whose grid still fits about two
  // waves; every cluster splits one token tile's contraction
  int max_n = 0, cl = 0;
  for (int g = 0; g < ng; ++g) {
    RkProjGroup& G = P.g[g];
    const int q0 = members[g][0];
    if (!encode_tma_2d(&G.map_z, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d[q0].Z, d[q0].C, T,
                       d[q0].C * 2, 64, 128, CU_TENSOR_MAP_SWIZZLE_128B))
      return cudaErrorInvalidValue;
    G.nk = static_cast<int>(d[q0].C / 64);
    G.n_prob = counts[g];
    for (int k = 0; k < counts[g]; ++k) G.prob[k] = members[g][k];
    G.cluster0 = cl;
    cl += P.t_tiles;
    max_n = std::max(max_n, counts[g] * R);
  }
  P.n_groups = ng;
  int nk_max = 0;
  for (int g = 0; g < ng; ++g) nk_max = std::max(nk_max, P.g[g].nk);
  const int smem = kRkStages * project_stage_bytes(max_n) + 1024;
  cudaLaunchConfig_t cfg = {};
  cfg.blockDim = dim3(kRkThreads);
  cfg.dynamicSmemBytes = static_cast<size_t>(smem);
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  // cluster size: the one with the smallest estimated time, counting the
  // rounds of clusters the GPU can hold at once and the longest slice
  // (decided once per launch shape)
  static std::map<std::tuple<int, int, int, int>, int> cs_cache;
  int dev = 0;
  cudaGetDevice(&dev);
  const auto key = std::make_tuple(dev, cl, nk_max, smem);
  int CS = 0;
  int64_t best = 0;
  const auto hit = cs_cache.find(key);
  if (hit != cs_cache.end()) CS = hit->second;
  for (int cs : {16, 8, 4}) {
    if (hit != cs_cache.end()) break;
    attr[0].val.clusterDim.x = cs;
    cfg.gridDim = dim3(static_cast<unsigned>(cl * cs));
    int active = 0;
    if (cudaOccupancyMaxActiveClusters(&active, lora_project_tc, &cfg) != cudaSuccess ||
        active < 1) {
      cudaGetLastError();  // a size the device cannot co-schedule: not a launch error
      continue;
    }
    const int64_t rounds = (cl + active - 1) / active;
    const int64_t cost = rounds * ((nk_max + cs - 1) / cs + 6);
    if (CS == 0 || cost < best) {
      CS = cs;
      best = cost;
    }
  }
  if (CS == 0) return cudaErrorInvalidConfiguration;
  cs_cache[key] = CS;
  attr[0].val.clusterDim.x = CS;
  cfg.gridDim = dim3(static_cast<unsigned>(cl * CS));
  double bytes = 0;
  for (int g = 0; g < ng; ++g) bytes += 2.0 * T * d[members[g][0]].C;
  void* prof = prof_begin(st);
  count_launch();
  e = cudaLaunchKernelEx(&cfg, lora_project_tc, P);
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
    G.cta0 = ctas;
    ctas += static_cast<int>((d[q0].C + 127) / 128);
    max_n = std::max(max_n, counts[g] * R);
    bytes += 2.0 * T * d[q0].C;
  }
  P.n_groups = ng;
  const int smem = kRkStages * grad_stage_bytes(max_n) + 1024;
  void* prof = prof_begin(st);
  count_launch();
  lora_grad_tc<<<ctas, kRkThreads, smem, st>>>(P);
  e = cudaGetLastError();
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
