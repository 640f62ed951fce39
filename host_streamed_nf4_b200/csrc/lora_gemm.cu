// lora_gemm.cu -- fused NF4 dequant + tcgen05 GEMM with the rank-r LoRA term
// folded into the same tensor-core accumulation (sm_100a), for a group of
// independent LoRA linears in one persistent launch.
//
// Forward of a LoRA linear (Poros API reference, lora_rank/lora_alpha; the
// frozen base is only read -- HN comment on host-RAM streaming):
//     Y[T, n_out] = X[T, k_in] deq(W)^T + (s t)[T, r] B[n_out, r]^T
// Backward, input gradient:
//     dX[T, k_in] = dY[T, n_out] deq(W) + (s u)[T, r] A[r, k_in]
//
// Both are computed transposed, with the weight on the MMA's M side so that
// each 128-row slab of W is dequantized once for up to 512 tokens:
//     fwd: D[n, t] = sum_k deq(W)[n, k] X[t, k]      (A operand K-major)
//     dx : D[k, t] = sum_n deq(W)[n, k] dY[t, n]     (A operand MN-major)
// The rank-r term is one more K-slice of the same accumulator:
//     fwd: D[n, t] += sum_j B[n, j] (s t)[t, j]
//     dx : D[k, t] += sum_j A[j, k] (s u)[t, j]
//
// The kernel runs as clusters of two CTAs on neighbouring SMs that share
// every MMA (tcgen05 cta_group::2, M = 256): each CTA dequantizes its own
// 128 rows of the 256-row tile and holds half of each token block, and the
// even CTA issues one instruction for both.  Per SM that halves the MMA
// instructions and the activation bytes staged per K step.  Each CTA fills
// its own rings with its own barriers; the odd CTA's otherwise idle MMA
// warp forwards "my half of stage g is ready" (and "my epilogue drained
// the accumulator") to the even CTA's pair barriers, and the MMA
// completion is committed to the matching barriers of both CTAs.
//
// Work units are (problem, 256-row tile, token tile, K split).  The host
// assigns them to persistent CTA pairs longest-first (static,
// deterministic).  A problem whose units are long and few is split along K:
// each piece writes its fp32 tile to workspace, and the pieces are added in
// split order, so the sum does not depend on timing.  In a longest-first
// plan the pieces are among the first units to run: each counts itself on
// the tile's arrival word, and the last to arrive adds the pieces and writes
// the output while its pair goes on with later units.  In a stream-K plan a
// tile's first piece often ends its pair's share, so the pieces are added
// by lora_splitk_reduce, spread over the whole GPU, after the kernel.
//
// CTA roles (15 warps, the same in both CTAs of a pair):
//   warps 0-3, 4-7   two dequant warpgroups taking alternate K steps: raw
//                    codes (smem) -> bf16 A tile in the UMMA 128B-swizzled
//                    layout, one 64-element block (one 128-byte line) per
//                    thread;
//   warps 8-11       epilogue: TMEM -> registers -> smem transpose ->
//                    coalesced bf16 rows of the output (or fp32 partials,
//                    and in a longest-first plan the sum of a split tile's
//                    partials by its last piece);
//   warp 12          TMA producer of the activation tiles and rank-r operands;
//   warp 13          TMA producer of the raw code tiles;
//   warp 14          TMEM owner; UMMA issuer of the pair (even CTA) or the
//                    forwarder of the odd CTA's ready signals.
// Every wait is bounded (ptx.cuh); a timed-out wait records a flag in
// g_gemm_flags, the CTA drains what it started and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <unistd.h>

#include <algorithm>
#include <array>
#include <atomic>
#include <chrono>
#include <climits>
#include <cstddef>
#include <map>
#include <tuple>
#include <mutex>
#include <queue>
#include <vector>

#include "internal.h"
#include "ptx.cuh"

namespace hsnf4 {

__device__ unsigned int g_gemm_flags;

enum : unsigned int {
  kFlagProducer = 1u,
  kFlagDequant = 2u,
  kFlagMma = 4u,
  kFlagLora = 8u,
  kFlagEpilogue = 16u,
  kFlagDrain = 32u,
  kFlagSelftest = 64u,
  kFlagArrive = 128u,
};

constexpr int kTileM = 128;                    // rows of one CTA (W rows or k_in columns)
constexpr int kPairM = 2 * kTileM;             // rows of the pair's MMA (one unit)
constexpr int kStepK = 64;                     // contraction per pipeline step
constexpr int kCodeBytes = 4096;               // raw codes of one step (128 x 64 / 2)
constexpr int kATileBytes = kTileM * 128;      // dequantized bf16 A tile
constexpr int kStageElems = 16 * kTileM;       // epilogue transpose buffer: 16 tokens x 128 rows
constexpr int kStageBufs = 4;                  // ... a ring of 4: two per 32-token step
constexpr int kMaxSmem = 232448;               // 227 KiB opt-in per block
constexpr int kThreads = 15 * 32;
constexpr int kWarpEpi = 8, kWarpProdX = 12, kWarpProdC = 13, kWarpMma = 14;

struct GemmProblem {
  CUtensorMap map_act;    // X / dY: bf16 [T, contraction], box {64, min(BN/2,128)}, 128B swizzle
  CUtensorMap map_codes;  // uint8 [n_out, k_in/2]; box {32, 128} fwd (32B swizzle), {64, 64}
                          // dx (64B swizzle); dense:
                          // bf16 [n_out, k_in], box {64, 128} fwd, {64, 64} dx, 128B swizzle
  CUtensorMap map_lo_a;   // fwd: B [n_out, r] box {16, 128} 32B; dx: A [r, k_in] box {64, r_pad} 128B
  CUtensorMap map_lo_b;   // s*t or s*u: bf16 [T, r_pad], box {16, min(BN/2,128)}, 32B swizzle
  CUtensorMap map_out;    // output bf16 [T, m_total], box {128 rows, 16 tokens}, no swizzle
  const float* absmax;
  uint16_t* out;          // bf16 [T, m_total]
  float* partial;         // split-K partial tiles (fp32 [BN tokens][128 rows] each), or null
  unsigned long long* arrive;  // split problems: one arrival word per 128-row half-tile
  int n_out, k_in, m_total, nk, kblocks, m_tiles;  // m_tiles: 256-row tiles
  int splits;             // partial slots per tile: the most K segments any tile has
};

constexpr int kMaxProblems = 8;
constexpr int kMaxPairs = 80;
constexpr int kMaxUnits = 2560;
constexpr int kMaxSplits = 8;  // pieces of one tile at most (the planners' limit)

struct GemmParams {
  GemmProblem prob[kMaxProblems];
  Nf4Codebook cb;
  int T, BN, r_pad, n_acc, sx, sc, sa, tmem_cols;
  int n_buf;  // TMEM accumulator buffers: 2 (BN <= 256: the epilogue of a unit
              // overlaps the next unit's MMAs) or 1 (BN = 512 fills TMEM)
  int dense;  // 1: map_codes is the bf16 weight, TMA-loaded straight into the A ring
  uint16_t pair_off[kMaxPairs + 1];  // units of pair c: units[pair_off[c] .. pair_off[c+1])
  // problem(3) | K segment(3) | pieces of the tile - 1 (3) | the tile's last
  // piece adds the pieces (1; else lora_splitk_reduce does, after the
  // kernel) | token tile(6) | row tile(16)
  uint32_t units[kMaxUnits];
  uint32_t unit_k[kMaxUnits];  // first K step(15) | end K step(15) | writes a partial(1)
  // this launch's tag of the arrival words (56 bits, never reused in the
  // process; a word holding another tag counts as no arrivals)
  unsigned long long token;
};
static_assert(sizeof(GemmParams) <= 32764, "kernel parameter block");

__host__ __device__ inline uint32_t pack_unit_k(int kb0, int kb1, bool partial) {
  return static_cast<uint32_t>(kb0) | (static_cast<uint32_t>(kb1) << 15) |
         (partial ? (1u << 30) : 0u);
}

__host__ __device__ inline uint32_t pack_unit(int p, int s, int tt, int mt) {
  return (static_cast<uint32_t>(p) << 29) | (static_cast<uint32_t>(s) << 26) |
         (static_cast<uint32_t>(tt) << 16) | static_cast<uint32_t>(mt);
}
// the pieces of the unit's tile and whether its last piece adds them
__host__ __device__ inline uint32_t with_pieces(uint32_t u, int nseg, bool fixup) {
  return u | (static_cast<uint32_t>(nseg - 1) << 23) | (fixup ? (1u << 22) : 0u);
}
__host__ __device__ inline int unit_problem(uint32_t u) { return static_cast<int>(u >> 29); }
__host__ __device__ inline int unit_segment(uint32_t u) { return static_cast<int>((u >> 26) & 7); }
__host__ __device__ inline int unit_tt(uint32_t u) { return static_cast<int>((u >> 16) & 63); }
__host__ __device__ inline int unit_mt(uint32_t u) { return static_cast<int>(u & 0xFFFF); }

// A work unit: one K segment [kb0, kb1) of one (problem, token tile, 256-row
// tile).  A tile cut into nseg segments has each write an fp32 partial
// (slot `split` of the tile); the nseg partials are added in segment order
// by the last of them to finish (longest-first plans) or by a second pass.
struct Unit {
  int p, split, tt, mt, kb0, kb1, nseg;
  bool partial, fixup;
};

__device__ __forceinline__ Unit unpack_unit(const GemmParams& P, int ui) {
  const uint32_t u = P.units[ui], k = P.unit_k[ui];
  Unit r;
  r.p = unit_problem(u);
  r.split = unit_segment(u);
  r.tt = unit_tt(u);
  r.mt = unit_mt(u);
  r.nseg = static_cast<int>((u >> 23) & 7) + 1;
  r.fixup = ((u >> 22) & 1u) != 0;
  r.kb0 = k & 0x7FFF;
  r.kb1 = (k >> 15) & 0x7FFF;
  r.partial = ((k >> 30) & 1u) != 0;
  return r;
}

struct SmemPlan {
  int x_bytes, a_off, c_off, la_off, lb_off, st_off, bar_off, total;
};

__host__ __device__ inline SmemPlan smem_plan(int mode, int BN, int sx, int sc, int sa, int r_pad) {
  SmemPlan p;
  const int slices = r_pad / 16;
  p.x_bytes = (BN / 2) * 128;  // this CTA's half of the token block
  p.a_off = sx * p.x_bytes;
  p.c_off = p.a_off + sa * kATileBytes;
  p.la_off = p.c_off + sc * kCodeBytes;
  const int la = (mode == kGemmFwd) ? slices * 4096 : 2 * r_pad * 128;
  p.lb_off = p.la_off + la;
  p.st_off = p.lb_off + slices * (BN / 2) * 32;
  p.bar_off = p.st_off + kStageBufs * kStageElems * 2;
  p.total = p.bar_off + (2 * sx + 2 * sc + 2 * sa + 16) * 8 + 32;
  return p;
}

__device__ __forceinline__ void named_sync(int id, int n) {
  asm volatile("bar.sync %0, %1;" ::"r"(id), "r"(n) : "memory");
}

// named barrier that also ANDs a predicate over its n threads: every thread
// leaves with the same answer, so a group that leaves its loop on a failed
// wait leaves it together and never strands the others at a barrier
__device__ __forceinline__ bool named_sync_and(int id, int n, bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred pi, po;\n\t"
      "setp.ne.u32 pi, %1, 0;\n\t"
      "bar.red.and.pred po, %2, %3, pi;\n\t"
      "selp.u32 %0, 1, 0, po;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "r"(id), "r"(n)
      : "memory");
  return r != 0;
}

// Position in a ring of n stages: the stage and the parity of the phase in
// which it is filled this round.  Stepping it costs a compare, where
// g % n and g / n by a run-time n would cost a division on every K step of
// the critical path.
struct Ring {
  int s = 0;
  uint32_t ph = 0;
  __device__ __forceinline__ void step(int n) {
    if (++s == n) {
      s = 0;
      ph ^= 1u;
    }
  }
  __device__ __forceinline__ void step2(int n) {  // two stages at once (n >= 2)
    s += 2;
    if (s >= n) {
      s -= n;
      ph ^= 1u;
    }
  }
};

// Counts one piece of a split tile on the tile's arrival word: the word
// holds this launch's token in its high 56 bits and the pieces counted so
// far in its low 8; a word holding another token (memory never written, or
// a launch that stopped early) counts as none.  The piece that completes
// the count gets true and clears the word, so a completed launch leaves
// every word 0 (a replayed graph reuses its token).  Every failed
// compare-and-swap means another piece was counted, so at most nseg - 1
// attempts fail.
__device__ __forceinline__ bool piece_arrive(unsigned long long* w, unsigned long long token,
                                             int nseg) {
  const unsigned long long tag = token << 8;
  unsigned long long cur = *reinterpret_cast<volatile unsigned long long*>(w);
  for (int attempt = 0; attempt <= 2 * kMaxSplits; ++attempt) {
    const unsigned long long nxt = (cur & ~0xFFull) == tag ? cur + 1 : (tag | 1ull);
    const unsigned long long prev = atomicCAS(w, cur, nxt);
    if (prev == cur) {
      if ((nxt & 0xFFull) != static_cast<unsigned long long>(nseg)) return false;
      atomicExch(w, 0ull);
      return true;
    }
    cur = prev;
  }
  atomicOr(&g_gemm_flags, kFlagArrive);
  return false;
}

template <int MODE>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
    lora_gemm_kernel(const __grid_constant__ GemmParams P) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int BN = P.BN, SX = P.sx, SC = P.sc, SA = P.sa;
  const SmemPlan plan = smem_plan(MODE, BN, SX, SC, SA, P.r_pad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int slices = P.r_pad / 16;
  const uint32_t crank = cluster_ctarank();  // 0: issues the pair's MMAs; 1: forwards
  const int pair = static_cast<int>(blockIdx.x >> 1);
  const int u_begin = P.pair_off[pair], u_end = P.pair_off[pair + 1];
  // This CTA's share of a token block: per accumulator h (tokens t0 + 256 h
  // .. + min(256, BN - 256 h)) the half starting crank * box_rows further,
  // staged as rows h * box_rows .. of the X tile and of each rank-r slice.
  const int half_rows = BN / 2;
  const int box_rows = half_rows < 128 ? half_rows : 128;
  const int row0 = static_cast<int>(crank) * kTileM;  // this CTA's rows within a unit

  uint8_t* lora_a = smem + plan.la_off;
  uint8_t* lora_b = smem + plan.lb_off;
  uint16_t* stage = reinterpret_cast<uint16_t*>(smem + plan.st_off);
  uint64_t* x_full = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint64_t* x_empty = x_full + SX;
  uint64_t* c_full = x_empty + SX;
  uint64_t* c_empty = c_full + SC;
  uint64_t* a_full = c_empty + SC;
  uint64_t* a_empty = a_full + SA;
  uint64_t* lora_full = a_empty + SA;
  uint64_t* lora_empty = lora_full + 1;
  uint64_t* acc_full = lora_empty + 1;  // [2]
  uint64_t* acc_empty = acc_full + 2;   // [2]
  uint64_t* drain_bar = acc_empty + 2;
  // the even CTA's view of the odd CTA (arrived on by its forwarder)
  uint64_t* pair_full = drain_bar + 1;  // [4]: both halves of K step g staged (ring of SP)
  uint64_t* pair_lora = pair_full + 4;  // the odd CTA's rank-r operands staged
  uint64_t* pair_acc = pair_lora + 1;   // [2]: the odd CTA's epilogue drained buffer b
  const int SP = SX < SA ? SX : SA;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(pair_acc + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto x_tile = [&](int s) { return smem + s * plan.x_bytes; };
  auto a_tile = [&](int s) { return smem + plan.a_off + s * kATileBytes; };
  auto c_tile = [&](int s) { return smem + plan.c_off + s * kCodeBytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < SX; ++s) {
      mbar_init(&x_full[s], 1);
      mbar_init(&x_empty[s], 1);
    }
    for (int s = 0; s < SC; ++s) {
      mbar_init(&c_full[s], 1);
      mbar_init(&c_empty[s], 4);  // one arrival per warp of the consuming warpgroup
    }
    for (int s = 0; s < SA; ++s) {
      mbar_init(&a_full[s], P.dense ? 1 : 4);  // TMA (dense) or the 4 warps of a warpgroup
      mbar_init(&a_empty[s], 1);
    }
    mbar_init(lora_full, 1);
    mbar_init(lora_empty, 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 128);
    }
    mbar_init(drain_bar, 1);
    for (int s = 0; s < 4; ++s) mbar_init(&pair_full[s], 1);
    mbar_init(pair_lora, 1);
    for (int b = 0; b < 2; ++b) mbar_init(&pair_acc[b], 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kWarpMma) {  // both CTAs: one allocation of the same columns in each TMEM
    tmem_alloc_pair(tmem_slot, static_cast<uint32_t>(P.tmem_cols));
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA arrive
  tc_fence_after();
  pdl_wait_then_release();
  const uint32_t tmem = *tmem_slot;

  int last_x = -1, last_c = -1, last_l = -1;  // producers: last issued sequence numbers
  bool mma_started = false;

  if (warp == kWarpProdX) {
    // -------------------------------------------------- activations + rank-r operands
    if (lane == 0) {
      int g = 0, lu = 0;
      Ring xr;
      const uint32_t lora_tx = static_cast<uint32_t>(plan.st_off - plan.la_off);
      bool ok = true;
      for (int ui = u_begin; ui < u_end && ok; ++ui, ++lu) {
        const Unit U = unpack_unit(P, ui);
        const GemmProblem& pr = P.prob[U.p];
        const int m0 = U.mt * kPairM + row0, t0 = U.tt * BN;
        for (int kb = U.kb0; kb < U.kb1; ++kb, ++g, xr.step(SX)) {
          const int s = xr.s;
          if (g >= SX && !mbar_wait(&x_empty[s], xr.ph ^ 1u, abort_flag, &g_gemm_flags,
                                    kFlagProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&x_full[s], static_cast<uint32_t>(half_rows * 128));
          for (int h = 0; h < P.n_acc; ++h)
            tma_load_2d(x_tile(s) + h * box_rows * 128, &pr.map_act, &x_full[s], kb * kStepK,
                        t0 + h * 256 + static_cast<int>(crank) * box_rows);
          last_x = g;
        }
        if (!ok) break;
        // rank-r operands after the unit's activation tiles: the previous
        // unit's rank-r slice has long been consumed by then
        if (lu > 0 && !mbar_wait(lora_empty, (lu - 1) & 1, abort_flag, &g_gemm_flags,
                                 kFlagProducer))
          break;
        mbar_arrive_expect_tx(lora_full, lora_tx);
        if (MODE == kGemmFwd) {
          for (int j = 0; j < slices; ++j)
            tma_load_2d(lora_a + j * 4096, &pr.map_lo_a, lora_full, j * 16, m0);
        } else {
          for (int h = 0; h < 2; ++h)
            tma_load_2d(lora_a + h * P.r_pad * 128, &pr.map_lo_a, lora_full, m0 + h * 64, 0);
        }
        for (int j = 0; j < slices; ++j)
          for (int h = 0; h < P.n_acc; ++h)
            tma_load_2d(lora_b + j * half_rows * 32 + h * box_rows * 32, &pr.map_lo_b, lora_full,
                        j * 16, t0 + h * 256 + static_cast<int>(crank) * box_rows);
        last_l = lu;
      }
    }
  } else if (warp == kWarpProdC) {
    // -------------------------------------------------- raw code tiles, or (dense base) the
    // bf16 weight tiles straight into the A ring: the 128B-swizzled TMA box is
    // the UMMA operand layout the dequant warps would have written
    if (lane == 0) {
      int g = 0;
      Ring cr;  // over the A ring (dense base) or the code ring
      const int CS = P.dense ? SA : SC;
      bool ok = true;
      for (int ui = u_begin; ui < u_end && ok; ++ui) {
        const Unit U = unpack_unit(P, ui);
        const GemmProblem& pr = P.prob[U.p];
        const int m0 = U.mt * kPairM + row0;
        for (int kb = U.kb0; kb < U.kb1; ++kb, ++g, cr.step(CS)) {
          if (P.dense) {
            const int s = cr.s;
            if (g >= SA && !mbar_wait(&a_empty[s], cr.ph ^ 1u, abort_flag, &g_gemm_flags,
                                      kFlagProducer)) {
              ok = false;
              break;
            }
            mbar_arrive_expect_tx(&a_full[s], static_cast<uint32_t>(kATileBytes));
            if (MODE == kGemmFwd) {
              tma_load_2d(a_tile(s), &pr.map_codes, &a_full[s], kb * kStepK, m0);
            } else {
              for (int h = 0; h < 2; ++h)
                tma_load_2d(a_tile(s) + h * (kATileBytes / 2), &pr.map_codes, &a_full[s],
                            m0 + h * 64, kb * kStepK);
            }
            last_c = g;
            continue;
          }
          const int s = cr.s;
          if (g >= SC && !mbar_wait(&c_empty[s], cr.ph ^ 1u, abort_flag, &g_gemm_flags,
                                    kFlagProducer)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(&c_full[s], static_cast<uint32_t>(kCodeBytes));
          if (MODE == kGemmFwd)
            tma_load_2d(c_tile(s), &pr.map_codes, &c_full[s], kb * 32, m0);
          else
            tma_load_2d(c_tile(s), &pr.map_codes, &c_full[s], m0 / 2, kb * kStepK);
          last_c = g;
        }
      }
    }
  } else if (warp == kWarpMma && crank == 1) {
    // -------------------------------------------------- forwarder (odd CTA)
    // Mirrors the issuer's order: before a unit, "my epilogue drained this
    // buffer"; per K step, "my X and A halves of step g are staged"; after
    // the unit's K steps, "my rank-r operands are staged".
    if (lane == 0) {
      const int NB = P.n_buf;
      int lu = 0;
      Ring xr, ar, pr_;
      bool ok = true;
      for (int ui = u_begin; ui < u_end && ok; ++ui, ++lu) {
        const Unit U = unpack_unit(P, ui);
        const int buf = NB > 1 ? (lu & 1) : 0;
        if (lu >= NB) {
          if (!mbar_wait(&acc_empty[buf], ((lu / NB) - 1) & 1, abort_flag, &g_gemm_flags,
                         kFlagMma))
            break;
          mbar_arrive_cluster(&pair_acc[buf], 0);
        }
        for (int kb = U.kb0; kb < U.kb1; ++kb, xr.step(SX), ar.step(SA), pr_.step(SP)) {
          ok = mbar_wait(&x_full[xr.s], xr.ph, abort_flag, &g_gemm_flags, kFlagMma) &&
               mbar_wait(&a_full[ar.s], ar.ph, abort_flag, &g_gemm_flags, kFlagMma);
          if (!ok) break;
          mbar_arrive_cluster(&pair_full[pr_.s], 0);
        }
        if (!ok) break;
        if (!mbar_wait(lora_full, lu & 1, abort_flag, &g_gemm_flags, kFlagLora)) break;
        mbar_arrive_cluster(pair_lora, 0);
      }
    }
  } else if (warp == kWarpMma) {
    // -------------------------------------------------- UMMA issuer of the pair (even CTA)
    if (lane == 0) {
      // All descriptors are computed once: per stage and per 16-wide K step
      // only the start-address field changes (in 16-byte units; shared
      // addresses stay below 256 KiB, so the 14-bit field never carries).
      // They address this CTA's shared memory; the odd CTA's operands sit
      // at the same offsets in its own.
      //   fwd A: 128 rows x 128 B lines (K-major, 8-row groups 1 KiB apart);
      //          a 16-wide K step is 32 B further along each line.
      //   dx  A: two 64-column atoms 8 KiB apart (LBO), 8-row groups 1 KiB
      //          apart (SBO); a 16-row K step is 2 KiB further.
      //   B (activations): K-major, 8-row groups 1 KiB apart; accumulator
      //          h reads this CTA's rows h*128.. (16 KiB further).
      const uint64_t a_desc0 =
          (MODE == kGemmFwd) ? make_sdesc(smem_u32(a_tile(0)), 16, 1024, kLayoutSw128)
                             : make_sdesc(smem_u32(a_tile(0)), 64 * 128, 1024, kLayoutSw128);
      const uint64_t b_desc0 = make_sdesc(smem_u32(x_tile(0)), 16, 1024, kLayoutSw128);
      const uint32_t a_k16 = (MODE == kGemmFwd) ? (32 >> 4) : (2048 >> 4);
      const uint32_t a_stage = kATileBytes >> 4, b_stage = plan.x_bytes >> 4;
      const uint32_t b_half = static_cast<uint32_t>(box_rows * 128) >> 4;
      const uint32_t lb_half = static_cast<uint32_t>(box_rows * 32) >> 4;
      const int n0 = BN < 256 ? BN : 256;
      const uint32_t idesc0 = make_idesc_bf16(kPairM, n0, MODE == kGemmDx ? 1 : 0, 0);
      const uint32_t idesc1 =
          make_idesc_bf16(kPairM, BN > 256 ? BN - 256 : 16, MODE == kGemmDx ? 1 : 0, 0);
      const bool two = P.n_acc > 1;
      const int NB = P.n_buf;
      constexpr uint16_t kBoth = 3;  // commit to the barriers of both CTAs
      int lu = 0;
      Ring xr, ar, pr_;
      bool ok = true;
      for (int ui = u_begin; ui < u_end && ok; ++ui, ++lu) {
        const Unit U = unpack_unit(P, ui);
        const int buf = NB > 1 ? (lu & 1) : 0;
        const uint32_t acc0 = tmem + static_cast<uint32_t>(buf * 256);
        if (lu >= NB) {  // both epilogues have drained this buffer's previous unit
          const uint32_t ph = ((lu / NB) - 1) & 1;
          ok = mbar_wait(&acc_empty[buf], ph, abort_flag, &g_gemm_flags, kFlagMma) &&
               mbar_wait(&pair_acc[buf], ph, abort_flag, &g_gemm_flags, kFlagMma);
          if (!ok) break;
          tc_fence_after();
        }
        for (int kb = U.kb0; kb < U.kb1; ++kb, xr.step(SX), ar.step(SA), pr_.step(SP)) {
          const int sx = xr.s, sa = ar.s;
          ok = mbar_wait(&x_full[sx], xr.ph, abort_flag, &g_gemm_flags, kFlagMma) &&
               mbar_wait(&a_full[sa], ar.ph, abort_flag, &g_gemm_flags, kFlagMma) &&
               mbar_wait(&pair_full[pr_.s], pr_.ph, abort_flag, &g_gemm_flags, kFlagMma);
          if (!ok) break;
          tc_fence_after();
          const uint64_t ad = a_desc0 + static_cast<uint64_t>(sa * a_stage);
          const uint64_t bd = b_desc0 + static_cast<uint64_t>(sx * b_stage);
          const uint32_t first = (kb > U.kb0) ? 1u : 0u;
#pragma unroll
          for (int k16 = 0; k16 < 4; ++k16) {
            const uint32_t acc = (k16 > 0) ? 1u : first;
            umma_bf16_pair(acc0, ad + k16 * a_k16, bd + k16 * 2, idesc0, acc);
            if (two)
              umma_bf16_pair(acc0 + 256, ad + k16 * a_k16, bd + b_half + k16 * 2, idesc1, acc);
          }
          mma_started = true;
          umma_commit_pair(&x_empty[sx], kBoth);
          umma_commit_pair(&a_empty[sa], kBoth);
        }
        if (!ok) break;
        ok = mbar_wait(lora_full, lu & 1, abort_flag, &g_gemm_flags, kFlagLora) &&
             mbar_wait(pair_lora, lu & 1, abort_flag, &g_gemm_flags, kFlagLora);
        if (!ok) break;
        if (U.split == 0) {  // the rank-r slice is added once, by split 0
          tc_fence_after();
          const uint32_t la = smem_u32(lora_a), lb = smem_u32(lora_b);
          for (int j = 0; j < slices; ++j) {
            const uint64_t adesc =
                (MODE == kGemmFwd) ? make_sdesc(la + j * 4096, 16, 256, kLayoutSw32)
                                   : make_sdesc(la + j * 2048, P.r_pad * 128, 1024, kLayoutSw128);
            const uint64_t bdesc = make_sdesc(lb + j * half_rows * 32, 16, 256, kLayoutSw32);
            umma_bf16_pair(acc0, adesc, bdesc, idesc0, 1u);
            if (two) umma_bf16_pair(acc0 + 256, adesc, bdesc + lb_half, idesc1, 1u);
          }
          mma_started = true;
        }
        umma_commit_pair(lora_empty, kBoth);
        umma_commit_pair(&acc_full[buf], kBoth);
      }
    }
  } else if (warp < kWarpEpi && P.dense) {
    // dense base: the weight arrives as bf16, the dequant warps have no work
  } else if (warp < kWarpEpi) {
    // -------------------------------------------------- dequant (two warpgroups)
    const int grp = warp >> 2;        // 0 or 1: takes the K steps with g % 2 == grp
    const int i = threadIdx.x & 127;  // this thread's line of the A tile
    const int line = (MODE == kGemmFwd) ? i : ((i >> 6) * 64 + (i & 63));
    // this thread's two 16-byte chunks of the step's code tile.  The tile is
    // TMA-swizzled so that a warp's loads hit distinct banks: fwd rows of 32 B
    // (32B swizzle: chunk c of row w at c ^ ((w >> 2) & 1)), dx rows of 64 B
    // (64B swizzle: chunk c of row w at c ^ ((w >> 1) & 3))
    int code_chunk0, code_chunk1;  // in 16-byte units from the tile start
    if (MODE == kGemmFwd) {
      const int sw = (i >> 2) & 1;
      code_chunk0 = i * 2 + (0 ^ sw);
      code_chunk1 = i * 2 + (1 ^ sw);
    } else {
      const int row = i & 63, h = i >> 6, sw = (row >> 1) & 3;
      code_chunk0 = row * 4 + ((2 * h) ^ sw);
      code_chunk1 = row * 4 + ((2 * h + 1) ^ sw);
    }
    // this thread's absmax for K step kb of unit U (0 past the weight's edge)
    auto absmax_at = [&](const Unit& U, int kb) -> float {
      const GemmProblem& pr = P.prob[U.p];
      const int m0 = U.mt * kPairM + row0;
      if (MODE == kGemmFwd) {
        const int row = m0 + i;
        return row < pr.n_out ? __ldg(pr.absmax + static_cast<int64_t>(row) * pr.kblocks + kb)
                              : 0.0f;
      }
      const int row = kb * kStepK + (i & 63);
      const int kblk = m0 / 64 + (i >> 6);
      return kblk < pr.kblocks ? __ldg(pr.absmax + static_cast<int64_t>(row) * pr.kblocks + kblk)
                               : 0.0f;
    };
    // advance (ui, kb, U) by `steps` K steps of this CTA's sequence; false at its end
    auto advance = [&](int& ui, int& kb, Unit& U, int steps) -> bool {
      kb += steps;
      while (kb >= U.kb1) {
        const int over = kb - U.kb1;
        if (++ui >= u_end) return false;
        U = unpack_unit(P, ui);
        kb = U.kb0 + over;
      }
      return true;
    };
    // This warpgroup's K steps are g = grp, grp + 2, ...  The absmax of the
    // next one is loaded while the current one waits and expands, so the
    // global-load latency is off the per-step path.
    int ui = u_begin, kb = 0, g = grp;
    Unit U{};
    bool have = ui < u_end;
    if (have) {
      U = unpack_unit(P, ui);
      kb = U.kb0;
      have = advance(ui, kb, U, grp);
    }
    float a_next = have ? absmax_at(U, kb) : 0.0f;
    bool ok = true;
    Ring cr, ar;  // this warpgroup's stages: grp, grp + 2, ... (both rings hold >= 2)
    cr.s = grp;
    ar.s = grp;
    while (have && ok) {
      const float a = a_next;
      const int gc = g;
      have = advance(ui, kb, U, 2);
      g += 2;
      if (have) a_next = absmax_at(U, kb);
      const int sc = cr.s, sa = ar.s;
      const uint32_t phc = cr.ph, pha = ar.ph;
      cr.step2(SC);
      ar.step2(SA);
      if (!mbar_wait(&c_full[sc], phc, abort_flag, &g_gemm_flags, kFlagDequant)) {
        ok = false;
        break;
      }
      const uint4* src = reinterpret_cast<const uint4*>(c_tile(sc));
      const uint4 c0 = src[code_chunk0], c1 = src[code_chunk1];
      // the warp's code loads have returned (the reduction consumes every
      // lane's words) before lane 0 releases the code stage to the producer
      const uint32_t dep = __reduce_or_sync(
          0xffffffffu, c0.x ^ c0.y ^ c0.z ^ c0.w ^ c1.x ^ c1.y ^ c1.z ^ c1.w);
      if (lane == 0) mbar_arrive_after(&c_empty[sc], dep);
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const Nf4Table tab = nf4_make_table(P.cb, a);
      if (gc >= SA && !mbar_wait(&a_empty[sa], pha ^ 1u, abort_flag, &g_gemm_flags,
                                 kFlagDequant)) {
        ok = false;
        break;
      }
      uint8_t* dst = a_tile(sa) + line * 128;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint4 v = nf4_dequant8(words[w], tab);
        *reinterpret_cast<uint4*>(dst + ((w ^ (line & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();  // each thread's tile writes -> visible to the MMA (async proxy)
      __syncwarp();
      if (lane == 0) mbar_arrive(&a_full[sa]);
    }
  } else {
    // -------------------------------------------------- epilogue (warps 8..11)
    const int q = warp - kWarpEpi;              // TMEM lane quarter
    const int i = threadIdx.x - kWarpEpi * 32;  // 0..127: TMEM lane = tile row
    const uint32_t lane_base = static_cast<uint32_t>(q * 32) << 16;
    int lu = 0;
    int epi_step = 0;  // 32-token output steps so far (picks the staging buffer pair)
    for (int ui = u_begin; ui < u_end; ++ui, ++lu) {
      const Unit U = unpack_unit(P, ui);
      const GemmProblem& pr = P.prob[U.p];
      const int m0 = U.mt * kPairM + row0, t0 = U.tt * BN;
      const int NB = P.n_buf;
      const int buf = NB > 1 ? (lu & 1) : 0;
      const uint32_t acc0 = tmem + static_cast<uint32_t>(buf * 256) + lane_base;
      const bool ok = mbar_wait(&acc_full[buf], (lu / NB) & 1, abort_flag, &g_gemm_flags,
                                kFlagEpilogue);
      // all four warps go on or stop together (the tile loop below meets at
      // a named barrier; tcgen05.ld is warp-collective)
      if (!named_sync_and(1, 128, ok)) break;
      tc_fence_after();
      // this CTA's 128-row half of the unit's tile
      const int tile = (U.tt * pr.m_tiles + U.mt) * 2 + static_cast<int>(crank);
      if (U.partial) {
        // this piece's fp32 tile -> workspace, token-major ([BN][128]) so that
        // a warp's 32 rows of one token are 128 contiguous bytes
        float* const slots = pr.partial + static_cast<int64_t>(tile) * pr.splits * kTileM * BN + i;
        float* const mine = slots + static_cast<int64_t>(U.split) * kTileM * BN;
        for (int c = 0; c < BN; c += 16) {
          uint32_t v[16];
          tmem_ld16(acc0 + static_cast<uint32_t>(c), v);
          tmem_wait_ld();
#pragma unroll
          for (int j = 0; j < 16; ++j)
            __stcg(mine + static_cast<int64_t>(c + j) * kTileM, __uint_as_float(v[j]));
        }
        tc_fence_before();
        mbar_arrive(&acc_empty[buf]);
        // Once every thread's rows are visible at device scope, thread 0
        // counts the piece on this half-tile's arrival word; the piece that
        // completes the count adds the tile's pieces in split order (their
        // rows read from L2) and writes the bf16 output like a whole tile.
        // Halves wholly past the output's edge have nothing to write.
        if (!U.fixup || m0 >= pr.m_total) continue;
        __threadfence();
        named_sync(1, 128);
        const int nseg = U.nseg;
        bool last = true;
        if (i == 0) {
          last = piece_arrive(pr.arrive + tile, P.token, nseg);
          __threadfence();
        }
        if (!named_sync_and(1, 128, last)) continue;
        for (int c = 0; c < BN; c += 32) {
          float v[32];
#pragma unroll
          for (int j = 0; j < 32; ++j) v[j] = __ldcg(slots + static_cast<int64_t>(c + j) * kTileM);
          for (int sp = 1; sp < nseg; ++sp) {
            const float* q = slots + static_cast<int64_t>(sp) * kTileM * BN;
#pragma unroll
            for (int j = 0; j < 32; ++j) v[j] += __ldcg(q + static_cast<int64_t>(c + j) * kTileM);
          }
          uint16_t* sb = stage + (epi_step & 1) * 2 * kStageElems;
#pragma unroll
          for (int j = 0; j < 32; ++j) {
            const __nv_bfloat16 b = __float2bfloat16_rn(v[j]);
            sb[j * kTileM + i] = *reinterpret_cast<const uint16_t*>(&b);
          }
          fence_proxy_async_smem();
          if (i == 0) bulk_wait_group_read<0>();
          named_sync(1, 128);
          if (i == 0) {
            for (int h = 0; h < 2; ++h)
              if (t0 + c + 16 * h < P.T)
                tma_store_2d(&pr.map_out, sb + h * kStageElems, m0, t0 + c + 16 * h);
            bulk_commit_group();
          }
          ++epi_step;
        }
        continue;
      }
      // 32 tokens per step: one TMEM load, a transpose into two 16-token x
      // 128-row bf16 buffers (sb[token j][row i]) of a ring of four, and two
      // TMA tile stores issued by thread 0 (rows and tokens past the output's
      // edge are not written).  Buffers alternate in pairs: before the step's
      // barrier thread 0 waits until the previous step's stores have read
      // their buffers, which the next step overwrites.
      for (int c = 0; c < BN; c += 32) {
        uint32_t v[32];
        tmem_ld32(acc0 + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
        uint16_t* sb = stage + (epi_step & 1) * 2 * kStageElems;
#pragma unroll
        for (int j = 0; j < 32; ++j) {
          const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[j]));
          sb[j * kTileM + i] = *reinterpret_cast<const uint16_t*>(&b);
        }
        fence_proxy_async_smem();
        if (i == 0) bulk_wait_group_read<0>();
        named_sync(1, 128);
        if (i == 0) {
          for (int h = 0; h < 2; ++h)
            if (t0 + c + 16 * h < P.T)
              tma_store_2d(&pr.map_out, sb + h * kStageElems, m0, t0 + c + 16 * h);
          bulk_commit_group();
        }
        ++epi_step;
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[buf]);
    }
    if (i == 0) bulk_wait_group_read<0>();  // the output stores have read smem before it goes away
  }

  // -------------------------------------------------- teardown
  __syncthreads();
  if (*abort_flag) {
    // drain what this CTA started before its shared memory and TMEM go away
    volatile int never = 0;
    if (warp == kWarpProdX && lane == 0) {
      for (int g = (last_x - SX + 1 > 0 ? last_x - SX + 1 : 0); g <= last_x; ++g)
        if (!mbar_wait(&x_full[g % SX], (g / SX) & 1, &never, &g_gemm_flags, kFlagDrain)) break;
      if (last_l >= 0) mbar_wait(lora_full, last_l & 1, &never, &g_gemm_flags, kFlagDrain);
    }
    if (warp == kWarpProdC && lane == 0) {
      const int S = P.dense ? SA : SC;
      uint64_t* full = P.dense ? a_full : c_full;
      for (int g = (last_c - S + 1 > 0 ? last_c - S + 1 : 0); g <= last_c; ++g)
        if (!mbar_wait(&full[g % S], (g / S) & 1, &never, &g_gemm_flags, kFlagDrain)) break;
    }
    if (warp == kWarpMma && lane == 0 && mma_started) {  // the even CTA's issued MMAs
      umma_commit_pair(drain_bar, 1);
      mbar_wait(drain_bar, 0, &never, &g_gemm_flags, kFlagDrain);
    }
  }
  tc_fence_before();
  // neither CTA leaves while the pair's MMAs may still read its shared memory
  // or a forwarder may still arrive on the even CTA's barriers
  cluster_sync();
  if (warp == kWarpMma) {
    tc_fence_after();
    tmem_dealloc_pair(tmem, static_cast<uint32_t>(P.tmem_cols));
  }
}

// One thread waits on a barrier nothing arrives at: the bounded wait must
// give up, flag it and let the kernel finish.
__global__ void selftest_stall_kernel() {
  __shared__ uint64_t bar;
  __shared__ int abort_word;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    abort_word = 0;
    fence_mbar_init();
    mbar_wait(&bar, 0, &abort_word, &g_gemm_flags, kFlagSelftest);
  }
}

cudaError_t launch_selftest_stall(cudaStream_t st) {
  count_launch();
  selftest_stall_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
}

// Adds the K-split partial tiles of a stream-K launch in split order and
// writes the bf16 outputs.  One CTA per (problem tile, 8-token slice);
// thread i owns row pair (2i, 2i+1) of the tile.
struct ReduceTile {
  const float* part;  // [splits][BN][128] of this tile
  uint16_t* out;      // output base
  int m0, t0, M, splits;
};

constexpr int kReduceTok = 8;
constexpr int kMaxReduceTiles = 768;  // 32 B each: the parameter block stays < 32 KiB

struct ReduceParams {
  ReduceTile tile[kMaxReduceTiles];
  int n_tiles, BN, T;
};

__global__ void __launch_bounds__(128) lora_splitk_reduce(const __grid_constant__ ReduceParams R) {
  pdl_wait_then_release();
  // CTA: one tile, 8 tokens; warp w the tokens 2w, 2w + 1 of them; lane l
  // rows 4l .. 4l + 3 (one 16-byte piece of each partial, 512 contiguous
  // bytes per token across the warp).  All of a token's split loads are in
  // flight before the adds, which stay in split order.
  const int slices = R.BN / kReduceTok;
  const int tix = blockIdx.x / slices, slice = blockIdx.x % slices;
  const ReduceTile& tl = R.tile[tix];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  const int i = lane * 4;
  const int row = tl.m0 + i;  // m_total is a multiple of 64: rows i .. i + 3 are all in or out
  if (row >= tl.M) return;
#pragma unroll
  for (int jj = 0; jj < 2; ++jj) {
    const int c = slice * kReduceTok + w * 2 + jj;
    const int t = tl.t0 + c;
    if (t >= R.T) continue;
    float4 v[kMaxSplits];
#pragma unroll
    for (int s = 0; s < kMaxSplits; ++s)
      if (s < tl.splits)
        v[s] = __ldcg(reinterpret_cast<const float4*>(
            tl.part + (static_cast<int64_t>(s) * R.BN + c) * kTileM + i));
    float4 acc = v[0];
#pragma unroll
    for (int s = 1; s < kMaxSplits; ++s)
      if (s < tl.splits) {
        acc.x += v[s].x;
        acc.y += v[s].y;
        acc.z += v[s].z;
        acc.w += v[s].w;
      }
    const __nv_bfloat162 lo = __floats2bfloat162_rn(acc.x, acc.y);
    const __nv_bfloat162 hi = __floats2bfloat162_rn(acc.z, acc.w);
    uint2 o;
    o.x = *reinterpret_cast<const uint32_t*>(&lo);
    o.y = *reinterpret_cast<const uint32_t*>(&hi);
    *reinterpret_cast<uint2*>(tl.out + static_cast<int64_t>(t) * tl.M + row) = o;
  }
}

// ---------------------------------------------------------------- host side

static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

bool encode_tma_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
                   uint64_t outer, uint64_t row_bytes, uint32_t box_inner, uint32_t box_outer,
                   CUtensorMapSwizzle sw) {
  auto fn = encode_fn();
  if (!fn) return false;
  cuuint64_t dims[2] = {inner, outer};
  cuuint64_t strides[1] = {row_bytes};
  cuuint32_t box[2] = {box_inner, box_outer};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, dt, 2, const_cast<void*>(base), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE>
static int configure_once() {
  static int rc = -1;
  static std::once_flag once;
  std::call_once(once, [] {
    rc = cudaFuncSetAttribute(lora_gemm_kernel<MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                              kMaxSmem) == cudaSuccess
             ? 0
             : 1;
  });
  return rc;
}

static int sm_count() {
  int dev = 0, n = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
  return n;
}

struct Tiling {
  int BN, sx, sc, sa;
};

// Token tile (<= 256 and a multiple of 16, or 512) and ring depths that fit
// in shared memory.
static bool choose_tiling(GemmMode mode, int64_t T, int r_pad, Tiling* t) {
  const int64_t t16 = (T + 15) / 16 * 16;
  // 512 tokens (one TMEM buffer) beats 256 with double-buffered TMEM by
  // ~1.5x at T = 512 on B200: each dequantized W tile feeds twice the MMAs
  const int first = t16 > 256 ? 512 : static_cast<int>(t16);
  for (int bn : {first, 256}) {
    if (bn > first) continue;
    for (int x : {4, 3, 2}) {
      if (smem_plan(mode, bn, x, 4, 3, r_pad).total + 1024 <= kMaxSmem) {
        *t = {bn, x, 4, 3};
        return true;
      }
    }
  }
  return false;
}

// Cost model of a unit in K steps: its K steps plus a fixed overhead (the
// epilogue and the pipeline refill), plus the fp32 partial-tile write when
// the tile is split along K.
constexpr int64_t kUnitOverhead = 8;
constexpr int64_t kSplitOverhead = 4;

static int64_t unit_cost(int64_t ksteps, int splits) {
  return ksteps + kUnitOverhead + (splits > 1 ? kSplitOverhead : 0);
}

// Makespan of the longest-first assignment of these units to `sms` CTAs.
static int64_t lpt_makespan(std::vector<int64_t>& costs, int sms) {
  std::sort(costs.begin(), costs.end(), std::greater<int64_t>());
  std::priority_queue<int64_t, std::vector<int64_t>, std::greater<int64_t>> heap;
  const size_t G = std::min<size_t>(costs.size(), static_cast<size_t>(sms));
  for (size_t c = 0; c < G; ++c) heap.push(0);
  int64_t mk = 0;
  for (int64_t c : costs) {
    int64_t l = heap.top();
    heap.pop();
    l += c;
    mk = std::max(mk, l);
    heap.push(l);
  }
  return mk;
}

// The LPT plan's objective for K splits `sp` (per problem): the simulated
// makespan of the longest-first schedule (in K steps) plus the split tiles'
// partial reads by their last pieces, charged at ~16 KiB per K step per SM.
static int64_t lpt_objective(const std::vector<int64_t>& tiles, const std::vector<int64_t>& nk,
                             const std::vector<int>& sp, int BN, int sms) {
  std::vector<int64_t> costs;
  double reduce_bytes = 0;
  for (size_t p = 0; p < tiles.size(); ++p) {
    for (int s = 0; s < sp[p]; ++s) {
      const int64_t ks = (s + 1) * nk[p] / sp[p] - s * nk[p] / sp[p];
      costs.insert(costs.end(), static_cast<size_t>(tiles[p]), unit_cost(ks, sp[p]));
    }
    if (sp[p] > 1) reduce_bytes += static_cast<double>(tiles[p]) * sp[p] * kPairM * BN * 4;
  }
  if (costs.size() > static_cast<size_t>(kMaxUnits)) return INT64_MAX;  // over the unit limit
  const int64_t reduce =
      reduce_bytes > 0 ? 4 + static_cast<int64_t>(reduce_bytes / (16384.0 * sms)) : 0;
  return lpt_makespan(costs, sms / 2) + reduce;  // units run on CTA pairs
}

// K splits per problem for the LPT plan.  Search: starting from no splits,
// repeatedly add one split to the problem holding the longest unit (pieces
// of at least 16 K steps, at most 8 splits), keeping the best objective seen.
static int64_t plan_splits(const std::vector<int64_t>& tiles, const std::vector<int64_t>& nk,
                           int BN, int sms, std::vector<int>* splits) {
  const size_t n = tiles.size();
  std::vector<int> cur(n, 1);
  *splits = cur;
  int64_t best = lpt_objective(tiles, nk, cur, BN, sms);
  for (int it = 0; it < 24; ++it) {
    int worst = -1;
    int64_t worst_cost = -1;
    for (size_t p = 0; p < n; ++p) {
      const int64_t c = unit_cost(nk[p] / cur[p] + (nk[p] % cur[p] ? 1 : 0), cur[p]);
      if (c > worst_cost && cur[p] < kMaxSplits && nk[p] / (cur[p] + 1) >= 16) {
        worst = static_cast<int>(p);
        worst_cost = c;
      }
    }
    if (worst < 0) break;
    cur[worst] += 1;
    const int64_t obj = lpt_objective(tiles, nk, cur, BN, sms);
    if (obj < best) {
      best = obj;
      *splits = cur;
    }
  }
  return best;
}

// The stream-K plan: every pair gets an equal share C = ceil(W / G) of all
// K steps, walking the tiles in (problem, token tile, row tile) order and
// cutting a tile's K range where a share ends (no piece shorter than
// kMinSegment steps).  A tile cut into pieces has each write an fp32 partial.
// Balances launches with fewer tiles than pairs, or tiles that do not
// divide evenly among them, at the cost of the partials.
struct Segment {
  int p, tt, mt, kb0, kb1, seg, nseg, pair;
};
constexpr int kMinSegment = 8;

static int64_t streamk_cut(const std::vector<int64_t>& mt_n, const std::vector<int64_t>& nk,
                           int t_tiles, int BN, int G, int sms, int64_t C,
                           std::vector<Segment>* out);

static int64_t streamk_segments(const std::vector<int64_t>& mt_n, const std::vector<int64_t>& nk,
                                int t_tiles, int BN, int G, int sms, std::vector<Segment>* out) {
  int64_t W = 0;
  for (size_t p = 0; p < nk.size(); ++p) W += mt_n[p] * t_tiles * nk[p];
  // the smallest share that leaves the last pair no more than the others
  // (pieces are never cut below kMinSegment, so an exact W / G can overflow)
  int64_t best = INT64_MAX;
  std::vector<Segment> trial;
  for (int64_t C = (W + G - 1) / G, step = std::max<int64_t>(1, C / 32), it = 0; it < 24;
       ++it, C += step) {
    const int64_t obj = streamk_cut(mt_n, nk, t_tiles, BN, G, sms, C, &trial);
    if (obj < best) {
      best = obj;
      *out = trial;
    }
  }
  return best;
}

static int64_t streamk_cut(const std::vector<int64_t>& mt_n, const std::vector<int64_t>& nk,
                           int t_tiles, int BN, int G, int sms, int64_t C,
                           std::vector<Segment>* out) {
  out->clear();
  int pair = 0;
  int64_t load = 0;
  std::vector<int64_t> cost(G, 0);
  double reduce_bytes = 0;
  for (size_t p = 0; p < nk.size(); ++p)
    for (int tt = 0; tt < t_tiles; ++tt)
      for (int mt = 0; mt < mt_n[p]; ++mt) {
        const size_t first = out->size();
        int kb = 0, seg = 0;
        while (kb < nk[p]) {
          if (pair < G - 1 && load > 0 && C - load < kMinSegment) {
            ++pair;
            load = 0;
          }
          int64_t take = pair == G - 1 ? nk[p] - kb : std::min<int64_t>(nk[p] - kb, C - load);
          if (nk[p] - kb - take < kMinSegment) take = nk[p] - kb;  // no sliver left behind
          out->push_back({static_cast<int>(p), tt, mt, kb, static_cast<int>(kb + take), seg, 0,
                          pair});
          kb += static_cast<int>(take);
          load += take;
          ++seg;
          if (pair < G - 1 && load >= C) {
            ++pair;
            load = 0;
          }
        }
        for (size_t i = first; i < out->size(); ++i) {
          Segment& s = (*out)[i];
          s.nseg = seg;
          cost[s.pair] += unit_cost(s.kb1 - s.kb0, seg);
        }
        if (seg > 1) reduce_bytes += static_cast<double>(seg) * kPairM * BN * 4;
        if (seg > kMaxSplits) return INT64_MAX;  // a tile's last piece adds at most kMaxSplits
      }
  if (out->size() > static_cast<size_t>(kMaxUnits)) return INT64_MAX;
  const int64_t reduce =
      reduce_bytes > 0 ? 4 + static_cast<int64_t>(reduce_bytes / (16384.0 * sms)) : 0;
  return *std::max_element(cost.begin(), cost.end()) + reduce;
}

// The launch's work plan: LPT over uniform K splits, or stream-K where the
// cost model puts it at least 4% lower.  Deterministic in the shapes and the
// SM count.
struct GemmPlan {
  bool stream_k = false;
  std::vector<int> splits;       // LPT: K splits per problem
  std::vector<int> slots;        // partial slots per tile of each problem (1: no partials)
  std::vector<size_t> part_base;
  std::vector<size_t> arrive_base;  // arrival words of the split problems' half-tiles
  size_t need = 0;               // workspace bytes of the partials and arrival words
};

static void plan_dims(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int BN,
                      std::vector<int64_t>* mt_n, std::vector<int64_t>* nk, int* t_tiles) {
  *t_tiles = static_cast<int>((T + BN - 1) / BN);
  mt_n->assign(n, 0);
  nk->assign(n, 0);
  for (int p = 0; p < n; ++p) {
    const int64_t mdim = (mode == kGemmFwd) ? probs[p].n_out : probs[p].k_in;
    const int64_t contraction = (mode == kGemmFwd) ? probs[p].k_in : probs[p].n_out;
    (*mt_n)[p] = (mdim + kPairM - 1) / kPairM;
    (*nk)[p] = contraction / kStepK;
  }
}

static int plan_pairs(int sms) { return std::min(sms / 2, kMaxPairs); }

static GemmPlan make_plan(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int BN) {
  const int sms = sm_count();
  std::vector<int64_t> mt_n, nk;
  int t_tiles = 0;
  plan_dims(mode, probs, n, T, BN, &mt_n, &nk, &t_tiles);
  std::vector<int64_t> tiles(n);
  for (int p = 0; p < n; ++p) tiles[p] = mt_n[p] * t_tiles;
  GemmPlan pl;
  const int64_t lpt = plan_splits(tiles, nk, BN, sms, &pl.splits);
  std::vector<Segment> segs;
  const int64_t sk = streamk_segments(mt_n, nk, t_tiles, BN, plan_pairs(sms), sms, &segs);
  // stream-K only for a clear predicted gain: measured on Qwen2.5-72B decoder
  // launches, the model undercharges the partial tiles (their epilogue and
  // the reduce pass), so predicted gains of ~3% turned into losses of ~5%
  pl.stream_k = sk < lpt - lpt / 25;
  pl.slots.assign(n, 1);
  if (pl.stream_k) {
    for (const Segment& s : segs) pl.slots[s.p] = std::max(pl.slots[s.p], s.nseg);
  } else {
    for (int p = 0; p < n; ++p) pl.slots[p] = pl.splits[p];
  }
  pl.part_base.assign(n, 0);
  pl.arrive_base.assign(n, 0);
  for (int p = 0; p < n; ++p) {
    if (pl.slots[p] <= 1) continue;
    pl.part_base[p] = pl.need;
    pl.need += round_up(static_cast<size_t>(tiles[p]) * pl.slots[p] * kPairM * BN * 4, 256);
    pl.arrive_base[p] = pl.need;
    pl.need += round_up(static_cast<size_t>(tiles[p]) * 2 * sizeof(unsigned long long), 256);
  }
  return pl;
}

// make_plan results, cached by (mode, T, BN, SM count, shapes)
static GemmPlan cached_plan(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T,
                            int BN) {
  static std::mutex mu;
  static std::map<std::vector<int64_t>, GemmPlan> cache;
  std::vector<int64_t> key = {static_cast<int64_t>(mode), T, BN, sm_count()};
  for (int p = 0; p < n; ++p) {
    key.push_back(probs[p].n_out);
    key.push_back(probs[p].k_in);
  }
  std::lock_guard<std::mutex> lk(mu);
  auto it = cache.find(key);
  if (it != cache.end()) return it->second;
  GemmPlan pl = make_plan(mode, probs, n, T, BN);
  if (cache.size() > 4096) cache.clear();
  cache.emplace(key, pl);
  return pl;
}

size_t gemm_workspace_bytes(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r) {
  Tiling tl;
  if (!choose_tiling(mode, T, (r + 15) / 16 * 16, &tl)) return 0;
  return cached_plan(mode, probs, n, T, tl.BN).need;
}

// The launch's work units per CTA pair, in order: (unit code, K range) of
// each.  nseg: the K pieces of each tile cut into several (problem, token
// tile, row tile).  HSNF4_OK or the error, recorded.
using PairUnits = std::vector<std::vector<std::pair<uint32_t, uint32_t>>>;
using TilePieces = std::map<std::tuple<int, int, int>, int>;

static int build_units(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int BN,
                       const GemmPlan& L, PairUnits* per, TilePieces* nseg) {
  std::vector<int64_t> mt_n, nks;
  int t_tiles_p = 0;
  plan_dims(mode, probs, n, T, BN, &mt_n, &nks, &t_tiles_p);
  for (int p = 0; p < n; ++p)
    if (mt_n[p] > (1 << 16) || nks[p] >= (1 << 15))
      return fail(HSNF4_ERR_INVALID, "lora gemm: problem %d exceeds the tile index range", p);

  const int sms = sm_count();
  const int t_tiles = t_tiles_p;
  per->clear();
  nseg->clear();
  if (L.stream_k) {
    std::vector<Segment> segs;
    const int G = plan_pairs(sms);
    if (streamk_segments(mt_n, nks, t_tiles, BN, G, sms, &segs) == INT64_MAX)
      return fail(HSNF4_ERR_INVALID, "lora gemm: no stream-K plan within the unit limit");
    per->assign(G, {});
    for (const Segment& sg : segs) {
      (*per)[sg.pair].push_back({pack_unit(sg.p, sg.seg, sg.tt, sg.mt),
                              pack_unit_k(sg.kb0, sg.kb1, sg.nseg > 1)});
      if (sg.nseg > 1) (*nseg)[{sg.p, sg.tt, sg.mt}] = sg.nseg;
    }
  } else {
    // units, longest first, each to the least loaded pair so far
    struct U {
      int64_t cost;
      uint32_t code, k;
    };
    std::vector<U> units;
    for (int p = 0; p < n; ++p) {
      const int S = L.splits[p];
      for (int sp = 0; sp < S; ++sp) {
        const int kb0 = static_cast<int>(sp * nks[p] / S);
        const int kb1 = static_cast<int>((sp + 1) * nks[p] / S);
        const int64_t cost = unit_cost(kb1 - kb0, S);
        for (int tt = 0; tt < t_tiles; ++tt)
          for (int mt = 0; mt < mt_n[p]; ++mt) {
            units.push_back({cost, pack_unit(p, sp, tt, mt), pack_unit_k(kb0, kb1, S > 1)});
            if (S > 1) (*nseg)[{p, tt, mt}] = S;
          }
      }
    }
    if (units.size() > static_cast<size_t>(kMaxUnits))
      return fail(HSNF4_ERR_INVALID, "lora gemm: %zu work units exceed the per-launch limit %d",
                  units.size(), kMaxUnits);
    std::stable_sort(units.begin(), units.end(),
                     [](const U& a, const U& b) { return a.cost > b.cost; });
    // persistent CTA pairs: one per two SMs
    const int G = static_cast<int>(std::min<size_t>(units.size(), plan_pairs(sms)));
    per->assign(G, {});
    using Load = std::pair<int64_t, int>;
    std::priority_queue<Load, std::vector<Load>, std::greater<Load>> heap;
    for (int c = 0; c < G; ++c) heap.push({0, c});
    for (const U& u : units) {
      Load top = heap.top();
      heap.pop();
      (*per)[top.second].push_back({u.code, u.k});
      heap.push({top.first + u.cost, top.second});
    }
  }
  return HSNF4_OK;
}

// Split tiles whose last piece adds the pieces in the kernel: those whose
// every piece has at least kFixupCover K steps of cover in its pair -- the
// pair's later units plus the steps by which the pair finishes before the
// busiest pair -- so the adding (reads of the other pieces from L2) overlaps
// other work or idle time.  The others (a stream-K share's first piece, a
// launch with no more units than pairs) are added by the reduce pass after
// the kernel.
using FixupTiles = std::map<std::tuple<int, int, int>, bool>;
constexpr int64_t kFixupCover = 32;

static int64_t unit_steps(uint32_t kk) {
  return static_cast<int64_t>((kk >> 15) & 0x7FFF) - static_cast<int64_t>(kk & 0x7FFF);
}

static FixupTiles fixup_tiles(const PairUnits& per, const TilePieces& nseg) {
  FixupTiles fixup;
  for (const auto& kv : nseg) fixup[kv.first] = true;
  int64_t busiest = 0;
  for (const auto& pair : per) {
    int64_t steps = 0;
    for (const auto& uk : pair) steps += unit_steps(uk.second);
    busiest = std::max(busiest, steps);
  }
  for (const auto& pair : per) {
    int64_t cover = busiest;  // after the current unit: later units + the pair's slack
    for (const auto& uk : pair) cover -= unit_steps(uk.second);
    for (auto it = pair.rbegin(); it != pair.rend(); ++it) {
      const uint32_t u = it->first, kk = it->second;
      if ((kk >> 30) & 1u) {
        const std::tuple<int, int, int> key{unit_problem(u), unit_tt(u), unit_mt(u)};
        if (cover < kFixupCover) fixup[key] = false;
      }
      cover += unit_steps(kk);
    }
  }
  return fixup;
}

// Work-plan introspection (hsnf4_gemm_plan): the launch's units decoded
// back and checked, every tile's K range covered once by pieces in order.
int gemm_plan_info(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r,
                   hsnf4_gemm_plan_info* out) {
  Tiling tl;
  if (!choose_tiling(mode, T, (r + 15) / 16 * 16, &tl))
    return fail(HSNF4_ERR_INVALID, "lora gemm: no tiling fits shared memory (T=%lld, r=%d)",
                (long long)T, r);
  const GemmPlan L = cached_plan(mode, probs, n, T, tl.BN);
  PairUnits per;
  TilePieces nseg;
  const int rc = build_units(mode, probs, n, T, tl.BN, L, &per, &nseg);
  if (rc != HSNF4_OK) return rc;
  std::vector<int64_t> mt_n, nks;
  int t_tiles = 0;
  plan_dims(mode, probs, n, T, tl.BN, &mt_n, &nks, &t_tiles);
  memset(out, 0, sizeof *out);
  out->stream_k = L.stream_k ? 1 : 0;
  out->pairs = static_cast<int32_t>(per.size());
  out->split_tiles = static_cast<int32_t>(nseg.size());
  for (const auto& kv : fixup_tiles(per, nseg)) out->fixup_tiles += kv.second ? 1 : 0;
  out->min_pair_steps = INT64_MAX;
  // tile -> its pieces (segment index, kb0, kb1, writes a partial)
  std::map<std::tuple<int, int, int>, std::vector<std::array<int, 4>>> pieces;
  for (const auto& pair : per) {
    int64_t steps = 0;
    for (const auto& uk : pair) {
      const uint32_t u = uk.first, kk = uk.second;
      const int p = unit_problem(u), seg = unit_segment(u);
      const int tt = unit_tt(u), mt = unit_mt(u);
      const int kb0 = static_cast<int>(kk & 0x7FFF), kb1 = static_cast<int>((kk >> 15) & 0x7FFF);
      pieces[{p, tt, mt}].push_back({seg, kb0, kb1, static_cast<int>((kk >> 30) & 1)});
      steps += kb1 - kb0;
      out->units += 1;
    }
    out->total_steps += steps;
    out->max_pair_steps = std::max(out->max_pair_steps, steps);
    out->min_pair_steps = std::min(out->min_pair_steps, steps);
  }
  bool ok = true;
  int64_t tiles = 0;
  for (int p = 0; p < n; ++p) tiles += mt_n[p] * t_tiles;
  ok = ok && static_cast<int64_t>(pieces.size()) == tiles;
  for (auto& kv : pieces) {
    auto& v = kv.second;
    std::sort(v.begin(), v.end());
    const int np = static_cast<int>(v.size());
    const auto it = nseg.find(kv.first);
    ok = ok && (np > 1 ? (it != nseg.end() && it->second == np) : it == nseg.end());
    int kb = 0;
    for (int i = 0; i < np; ++i) {
      ok = ok && v[i][0] == i && v[i][1] == kb && v[i][2] > v[i][1] && v[i][3] == (np > 1);
      kb = v[i][2];
    }
    ok = ok && kb == nks[std::get<0>(kv.first)];
  }
  out->covered = ok ? 1 : 0;
  if (out->min_pair_steps == INT64_MAX) out->min_pair_steps = 0;
  return HSNF4_OK;
}

int check_gemm_tokens(GemmMode mode, int64_t T, int r) {
  Tiling tl;
  if (!choose_tiling(mode, T, (r + 15) / 16 * 16, &tl))
    return fail(HSNF4_ERR_INVALID, "lora gemm: no tiling fits shared memory (T=%lld, r=%d)",
                (long long)T, r);
  if ((T + tl.BN - 1) / tl.BN > 64)
    return fail(HSNF4_ERR_INVALID, "lora gemm: T=%lld exceeds %d tokens per launch",
                (long long)T, 64 * tl.BN);
  return HSNF4_OK;
}

// A tag for the arrival words of one launch: 56 bits, consecutive launches
// consecutive values from a start drawn once per process, so no two
// launches of the process share one and a word left by another process or
// never written matches only by a 2^-56 chance.
static unsigned long long next_launch_token() {
  static std::atomic<unsigned long long> next{0};
  static const unsigned long long start = [] {
    unsigned long long z = static_cast<unsigned long long>(
        std::chrono::steady_clock::now().time_since_epoch().count()) ^
        (static_cast<unsigned long long>(getpid()) << 32) ^
        reinterpret_cast<uintptr_t>(&next);
    z = (z ^ (z >> 30)) * 0xBF58476D1CE4E5B9ull;  // splitmix64 finaliser
    z = (z ^ (z >> 27)) * 0x94D049BB133111EBull;
    return z ^ (z >> 31);
  }();
  return (start + next.fetch_add(1)) & ((1ull << 56) - 1);
}

int launch_lora_gemm_group(GemmMode mode, const GemmProblemDesc* probs, int n, int64_t T, int r,
                           void* workspace, size_t ws_bytes, cudaStream_t st) {
  if (n < 1 || n > kMaxProblems)
    return fail(HSNF4_ERR_INVALID, "lora gemm: 1..%d problems per launch (got %d)", kMaxProblems,
                n);
  static GemmParams P;  // large: built on the host, copied into the launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&P, 0, offsetof(GemmParams, units));
  const int r_pad = (r + 15) / 16 * 16;
  Tiling tl;
  if (!choose_tiling(mode, T, r_pad, &tl))
    return fail(HSNF4_ERR_INVALID, "lora gemm: no tiling fits shared memory (T=%lld, r=%d)",
                (long long)T, r);
  const int BN = tl.BN;
  const int t_tiles = static_cast<int>((T + BN - 1) / BN);
  if (t_tiles > 64)
    return fail(HSNF4_ERR_INVALID, "lora gemm: T=%lld exceeds %d tokens per launch",
                (long long)T, 64 * BN);
  P.T = static_cast<int>(T);
  P.BN = BN;
  P.r_pad = r_pad;
  P.n_acc = (BN + 255) / 256;
  P.n_buf = BN <= 256 ? 2 : 1;
  P.sx = tl.sx;
  P.sc = tl.sc;
  P.sa = tl.sa;
  P.cb = codebook();
  P.dense = probs[0].dense ? 1 : 0;
  for (int p = 1; p < n; ++p)
    if (probs[p].dense != probs[0].dense)
      return fail(HSNF4_ERR_INVALID, "lora gemm: a group takes one base format");
  int tc = 32;
  while (tc < BN) tc <<= 1;
  P.tmem_cols = P.n_buf == 2 ? 512 : tc;  // two 256-column buffers, or one of BN
  const int sms = sm_count();
  const GemmPlan L = cached_plan(mode, probs, n, T, BN);
  if (L.need > ws_bytes || (L.need && !workspace))
    return fail(HSNF4_ERR_OOM, "lora gemm: workspace too small: need %zu bytes, given %zu",
                L.need, ws_bytes);
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  PairUnits per;
  TilePieces nseg;
  {
    const int rc = build_units(mode, probs, n, T, BN, L, &per, &nseg);
    if (rc != HSNF4_OK) return rc;
  }
  const int G = static_cast<int>(per.size());
  const FixupTiles fixup = fixup_tiles(per, nseg);
  bool any_reduce = false;
  for (const auto& kv : fixup) any_reduce = any_reduce || !kv.second;
  int k = 0;
  for (int c = 0; c < G; ++c) {
    P.pair_off[c] = static_cast<uint16_t>(k);
    for (const auto& uk : per[c]) {
      if (k == kMaxUnits)
        return fail(HSNF4_ERR_INVALID, "lora gemm: work units exceed the per-launch limit %d",
                    kMaxUnits);
      P.units[k] = uk.first;
      P.unit_k[k] = uk.second;
      if ((uk.second >> 30) & 1u) {  // a piece of a split tile: its pieces, who adds them
        const std::tuple<int, int, int> key{unit_problem(uk.first), unit_tt(uk.first),
                                            unit_mt(uk.first)};
        const auto it = nseg.find(key);
        if (it == nseg.end() || it->second < 2 || it->second > kMaxSplits)
          return fail(HSNF4_ERR_INVALID, "lora gemm: inconsistent split plan");
        P.units[k] = with_pieces(uk.first, it->second, fixup.at(key));
      }
      ++k;
    }
  }
  P.pair_off[G] = static_cast<uint16_t>(k);

  bool ok = true;
  // each CTA of a pair stages half of every 256-token accumulator block
  const int box_rows = BN / 2 < 128 ? BN / 2 : 128;
  for (int p = 0; p < n; ++p) {
    const GemmProblemDesc& d = probs[p];
    GemmProblem& g = P.prob[p];
    const int64_t contraction = (mode == kGemmFwd) ? d.k_in : d.n_out;
    g.absmax = d.absmax;
    g.out = static_cast<uint16_t*>(d.out);
    g.n_out = static_cast<int>(d.n_out);
    g.k_in = static_cast<int>(d.k_in);
    g.m_total = static_cast<int>((mode == kGemmFwd) ? d.n_out : d.k_in);
    g.nk = static_cast<int>(contraction / kStepK);
    g.kblocks = static_cast<int>(d.k_in / 64);
    g.m_tiles = (g.m_total + kPairM - 1) / kPairM;
    g.splits = L.slots[p];
    if (g.splits > 1) {
      g.partial = reinterpret_cast<float*>(ws + L.part_base[p]);
      g.arrive = reinterpret_cast<unsigned long long*>(ws + L.arrive_base[p]);
    }
    ok = ok && encode_tma_2d(&g.map_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.act, contraction, T,
                         contraction * 2, 64, box_rows, CU_TENSOR_MAP_SWIZZLE_128B);
    if (d.dense)  // bf16 [n_out, k_in]: 64 k x (128 rows fwd | 64 rows dx), 128B swizzle
      ok = ok && encode_tma_2d(&g.map_codes, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.codes, d.k_in,
                           d.n_out, d.k_in * 2, 64, mode == kGemmFwd ? 128 : 64,
                           CU_TENSOR_MAP_SWIZZLE_128B);
    if (mode == kGemmFwd) {
      if (!d.dense)
        ok = ok && encode_tma_2d(&g.map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, d.codes, d.k_in / 2,
                             d.n_out, d.k_in / 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_32B);
      ok = ok && encode_tma_2d(&g.map_lo_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.lo_a, r, d.n_out,
                           r * 2, 16, 128, CU_TENSOR_MAP_SWIZZLE_32B);
    } else {
      if (!d.dense)
        ok = ok && encode_tma_2d(&g.map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, d.codes, d.k_in / 2,
                             d.n_out, d.k_in / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_64B);
      ok = ok && encode_tma_2d(&g.map_lo_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.lo_a, d.k_in, r,
                           d.k_in * 2, 64, r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
    }
    ok = ok && encode_tma_2d(&g.map_lo_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.lo_b, r_pad, T,
                         r_pad * 2, 16, box_rows, CU_TENSOR_MAP_SWIZZLE_32B);
    ok = ok && encode_tma_2d(&g.map_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, d.out, g.m_total, T,
                             static_cast<uint64_t>(g.m_total) * 2, kTileM, 16,
                             CU_TENSOR_MAP_SWIZZLE_NONE);
  }
  if (!ok) return fail(HSNF4_ERR_CUDA, "lora gemm: cuTensorMapEncodeTiled failed");

  if (configure_once<kGemmFwd>() != 0 || configure_once<kGemmDx>() != 0)
    return fail(HSNF4_ERR_CUDA, "lora gemm: smem attribute");
  const int smem = smem_plan(mode, BN, tl.sx, tl.sc, tl.sa, r_pad).total + 1024;
  P.token = next_launch_token();
  void* prof = prof_begin(st, mode == kGemmFwd ? kProfGemmFwd : kProfGemmDx);
  cudaError_t e = launch_pdl(mode == kGemmFwd ? lora_gemm_kernel<kGemmFwd> : lora_gemm_kernel<kGemmDx>,
                             dim3(2 * G), dim3(kThreads), smem, st, P);  // G clusters of 2
  if (e == cudaSuccess && any_reduce) {
    // add the K-split partials in split order and write the bf16 outputs
    static ReduceParams R;
    R.n_tiles = 0;
    R.BN = BN;
    R.T = static_cast<int>(T);
    for (int p = 0; p < n; ++p) {
      const GemmProblem& g = P.prob[p];
      if (g.splits <= 1) continue;
      for (int tt = 0; tt < t_tiles; ++tt)
        for (int mt = 0; mt < g.m_tiles; ++mt) {
          const auto it = nseg.find({p, tt, mt});
          if (it == nseg.end()) continue;  // a tile in one piece wrote its output directly
          if (fixup.at({p, tt, mt})) continue;  // its last piece added the pieces
          for (int c = 0; c < 2; ++c) {  // the two 128-row halves of the pair's tile
            const int m0 = mt * kPairM + c * kTileM;
            if (m0 >= g.m_total) continue;
            if (R.n_tiles == kMaxReduceTiles) {
              e = launch_pdl(lora_splitk_reduce, dim3(R.n_tiles * (BN / kReduceTok)), dim3(128),
                             0, st, R);
              if (e != cudaSuccess) break;
              R.n_tiles = 0;
            }
            const int tile = (tt * g.m_tiles + mt) * 2 + c;
            R.tile[R.n_tiles++] = {g.partial + static_cast<int64_t>(tile) * g.splits * kTileM * BN,
                                   g.out, m0, tt * BN, g.m_total, it->second};
          }
        }
    }
    if (e == cudaSuccess && R.n_tiles)
      e = launch_pdl(lora_splitk_reduce, dim3(R.n_tiles * (BN / kReduceTok)), dim3(128), 0, st, R);
  }
  if (prof) {
    // algorithmic FLOPs: the base products plus the rank-r slices
    double flops = 0;
    for (int p = 0; p < n; ++p)
      flops += (mode == kGemmFwd) ? 2.0 * T * probs[p].n_out * (probs[p].k_in + r)
                                  : 2.0 * T * probs[p].k_in * (probs[p].n_out + r);
    prof_end(prof, mode == kGemmFwd ? kProfGemmFwd : kProfGemmDx, flops, st);
  }
  return cuda_status(e, "lora gemm launch");
}

cudaError_t read_gemm_flags(uint32_t* flags) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_gemm_flags, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_gemm_flags, &z, sizeof z);
  }
  return e;
}

}  // namespace hsnf4
