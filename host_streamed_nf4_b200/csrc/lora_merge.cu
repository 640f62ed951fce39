// lora_merge.cu -- merge the adapter into the frozen base (Poros API
// reference, PorosModel.merge_and_unload):
//
//     W'[n, k] = bf16_rne( fp32( deq(W)[n, k] + s * sum_j B[n, j] A[j, k] ) )
//
// with deq(W) the bf16 value of the base (NF4: bf16_rne(codebook * absmax);
// dense base: the weight itself) and s = alpha / r.  The rank-r sum runs on
// the tensor cores (exact bf16 products, fp32 accumulate), is scaled by s in
// fp32, added to deq(W) in fp32 and rounded once to bf16.
//
// Persistent CTAs (sm_100a), each taking 128 x 128 tiles of W' in turn.
// Warp 0 loads a tile's base (NF4 codes or bf16 weight), B's 128 rows and
// A's 128 columns with TMA into one of two stages; warp 1 issues r/16
// tcgen05 MMAs (M = 128 rows, N = 128 columns, K = 16 ranks each; B read
// K-major, A read MN-major) into a 128-column fp32 accumulator in tensor
// memory.  Two warpgroups then expand the tile, each thread one row of 64
// columns: it reads its product row back from tensor memory 16 columns at a
// time, expands the matching base bytes, adds, rounds and writes the bf16
// row into a 128B-swizzled staging box; each warp stores its own 32 rows
// with TMA as soon as it has written them, so no warp waits for another's
// rows or stores.  HBM traffic is the base read once plus W' written once;
// several CTAs per SM keep loads and stores in flight.
#include <cuda_bf16.h>

#include <algorithm>
#include <mutex>

#include "internal.h"
#include "nf4_device.cuh"
#include "ptx.cuh"

namespace hsnf4 {

__device__ unsigned int g_merge_flags;

enum : unsigned int {
  kMrgFlagLoad = 1u << 16,
  kMrgFlagMma = 1u << 17,
  kMrgFlagDrain = 1u << 18,
};

constexpr int kMrgTile = 128;
// Buffering per base format, and the CTAs per SM it allows (TMEM: 512
// columns per SM, kAccBufs x 128 per CTA; shared memory ~227 KB; registers
// 64 K).  NF4: one accumulator and one staging tile per warpgroup, three
// CTAs per SM (measured ~10% faster than two double-buffered CTAs: more
// expanding warps hide the waits).  Dense: the 32 KB base tiles allow two
// CTAs, each double-buffered.
template <bool DENSE>
struct MrgCfg {
  static constexpr int kAccBufs = DENSE ? 2 : 1;  // TMEM accumulators per CTA
  static constexpr int kOutBufs = DENSE ? 2 : 1;  // output staging tiles per warpgroup
  static constexpr int kCtasPerSm = DENSE ? 2 : 3;
  static_assert(kAccBufs * kMrgTile * kCtasPerSm <= 512, "TMEM columns per SM");
};
// columns per TMEM read of the expanding loop (8 or 16).  8: the NF4
// instance fits the 64 registers a thread has at three CTAs per SM without
// spilling (16 spilled one register and ran 3-4% slower).
constexpr int kMrgCols = 8;
static_assert(kMrgCols == 8 || kMrgCols == 16, "TMEM read width");

struct MergeParams {
  CUtensorMap map_base;  // NF4: codes uint8 [N, K/2], box {64, 128}, 64B swizzle
                         // dense: bf16 [N, K], box {64, 128}, 128B swizzle (two per tile)
  CUtensorMap map_a;     // A bf16 [r, K], box {64, r_pad}, 128B swizzle (MN-major operand)
  CUtensorMap map_b;     // B bf16 [N, r], box {16, 128}, 32B swizzle (K-major operand)
  CUtensorMap map_out;   // W' bf16 [N, K], box {64, 32} (one warp's rows), 128B swizzle
  const float* absmax;   // NF4 only: fp32 [N, K/64]
  int64_t N, K;
  int r_pad, dense, col_tiles, row_tiles;
  float s;
  Nf4Codebook cb;
};

// shared-memory plan (offsets from a 1 KiB-aligned base): two load stages
// (base tile, B slices, A atoms) and two output staging tiles
struct MergeSmem {
  int b, a, stage, out, total;  // b, a: offsets inside a stage
};

__host__ __device__ inline MergeSmem merge_smem(int dense, int r_pad) {
  MergeSmem m;
  m.b = dense ? 32768 : 8192;        // base tile: 128 x 128 bf16, or 128 x 64 code bytes
  m.a = m.b + (r_pad / 16) * 4096;   // B: r_pad / 16 slices of 128 rows x 32 B
  m.stage = m.a + 2 * r_pad * 128;   // A: two 64-column atoms of r_pad rows x 128 B
  m.out = 2 * m.stage;               // W': per buffer two 64-column boxes of 128 rows x 128 B
  m.total = m.out + (dense ? MrgCfg<true>::kOutBufs : MrgCfg<false>::kOutBufs) * 32768;
  return m;
}

constexpr int kMrgThreads = 320;  // producer, MMA issuer, two expanding warpgroups
constexpr int kMrgExpand = kMrgThreads - 64;  // the expanding threads (warps 2..9)
static_assert(kMrgExpand == 256, "two warpgroups expand the tile");

// Persistent: CTA b takes tiles b, b + gridDim.x, ...  Warp 0 loads the next
// tile into the other stage while the current one is processed; warp 1
// issues each tile's MMAs into a TMEM accumulator (MrgCfg: one or two per
// CTA); warps 2..9 (two warpgroups, one row of the tile per thread) expand
// it into staging boxes (one or two per warpgroup), each warp's 32 rows
// written out by a TMA store of its own while the next tile is expanded.
template <bool DENSE>
__global__ void __launch_bounds__(kMrgThreads, MrgCfg<DENSE>::kCtasPerSm)
    lora_merge_kernel(const __grid_constant__ MergeParams P) {
  extern __shared__ uint8_t mrg_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mrg_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t st_full[2], st_empty[2], acc_full[2], acc_empty[2], drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  constexpr int kMrgAccBufs = MrgCfg<DENSE>::kAccBufs, kMrgOutBufs = MrgCfg<DENSE>::kOutBufs;
  const MergeSmem L = merge_smem(DENSE, P.r_pad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int n_tiles = P.row_tiles * P.col_tiles;
  const int slices = P.r_pad / 16;

  if (threadIdx.x == 0) {
    for (int b = 0; b < 2; ++b) {
      mbar_init(&st_full[b], 1);
      mbar_init(&st_empty[b], 1 + kMrgExpand);  // the MMAs (commit) and the expanding threads
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], kMrgExpand);
    }
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kMrgAccBufs * kMrgTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  int last_load = -1;
  bool mma_issued = false;

  if (warp == 0) {
    // ---------------------------------------------- TMA loads of each tile
    if (lane == 0) {
      const uint32_t bytes = static_cast<uint32_t>(L.stage);
      int li = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++li) {
        const int s = li & 1;
        if (li >= 2 && !mbar_wait(&st_empty[s], ((li >> 1) - 1) & 1, abort_p, &g_merge_flags,
                                  kMrgFlagLoad))
          break;
        const int n0 = (tile / P.col_tiles) * kMrgTile, k0 = (tile % P.col_tiles) * kMrgTile;
        uint8_t* st = smem + s * L.stage;
        mbar_arrive_expect_tx(&st_full[s], bytes);
        if (DENSE) {
          tma_load_2d(st, &P.map_base, &st_full[s], k0, n0);
          tma_load_2d(st + 16384, &P.map_base, &st_full[s], k0 + 64, n0);
        } else {
          tma_load_2d(st, &P.map_base, &st_full[s], k0 / 2, n0);
        }
        for (int j = 0; j < slices; ++j)
          tma_load_2d(st + L.b + j * 4096, &P.map_b, &st_full[s], 16 * j, n0);
        for (int h = 0; h < 2; ++h)
          tma_load_2d(st + L.a + h * P.r_pad * 128, &P.map_a, &st_full[s], k0 + 64 * h, 0);
        last_load = li;
      }
    }
  } else if (warp == 1) {
    // ---------------------------------------------- MMA issuer
    if (lane == 0) {
      // D[n, k] = sum_j B[n, j] A[j, k]: A operand = B slice j (K-major, 32B
      // swizzle, 8-row groups 256 B apart); B operand = rows 16j.. of A
      // (MN-major, 128B swizzle: 64-column atoms r_pad * 128 B apart, 8-rank
      // groups 1 KiB apart, 16 ranks = 2 KiB per slice)
      const uint32_t idesc = make_idesc_bf16(kMrgTile, kMrgTile, 0, 1);
      int li = 0;
      for (int tile = blockIdx.x; tile < n_tiles; tile += gridDim.x, ++li) {
        const int s = li & 1, b = li % kMrgAccBufs;
        if (!mbar_wait(&st_full[s], (li >> 1) & 1, abort_p, &g_merge_flags, kMrgFlagMma)) break;
        if (li >= kMrgAccBufs &&
            !mbar_wait(&acc_empty[b], ((li / kMrgAccBufs) - 1) & 1, abort_p, &g_merge_flags,
                                  kMrgFlagMma))
          break;
        tc_fence_after();
        const uint8_t* st = smem + s * L.stage;
        for (int j = 0; j < slices; ++j) {
          const uint64_t ad = make_sdesc(smem_u32(st + L.b + j * 4096), 16, 256, kLayoutSw32);
          const uint64_t bd =
              make_sdesc(smem_u32(st + L.a + j * 2048), P.r_pad * 128, 1024, kLayoutSw128);
          umma_bf16(tmem + static_cast<uint32_t>(b * kMrgTile), ad, bd, idesc, j > 0 ? 1u : 0u);
        }
        mma_issued = true;
        umma_commit(&acc_full[b]);
        umma_commit(&st_empty[s]);  // B and A of this stage are read
      }
    }
  } else {
    // ---------------------------------------------- expand, add, round, store
    // warpgroup h (warps 2..5 or 6..9) takes columns 64 h .. 64 h + 63, one
    // row of the tile per thread; each warp stores its 32 rows of them
    const int h = (warp - 2) >> 2;
    const int q4 = warp & 3;           // TMEM lane quarter of this warp
    const int tid = q4 * 32 + lane;    // this thread's row of the tile
    const uint32_t lane_base = static_cast<uint32_t>(q4 * 32) << 16;
    // this row's absmax for the warpgroup's block of a tile, loaded one tile ahead
    auto absmax_of = [&](int tile) -> float {
      if (DENSE || tile >= n_tiles) return 0.f;
      const int n = (tile / P.col_tiles) * kMrgTile + tid, k0 = (tile % P.col_tiles) * kMrgTile;
      if (n >= P.N || k0 + 64 * h >= P.K) return 0.f;
      return __ldg(P.absmax + static_cast<int64_t>(n) * (P.K / 64) + k0 / 64 + h);
    };
    float am_next = absmax_of(blockIdx.x);
    int li = 0;
    bool ok = true;
    for (int tile = blockIdx.x; tile < n_tiles && ok; tile += gridDim.x, ++li) {
      const int s = li & 1, b = li % kMrgAccBufs, ob = li % kMrgOutBufs;
      const float am = am_next;
      am_next = absmax_of(tile + gridDim.x);
      const int n0 = (tile / P.col_tiles) * kMrgTile, k0 = (tile % P.col_tiles) * kMrgTile;
      ok = mbar_wait(&st_full[s], (li >> 1) & 1, abort_p, &g_merge_flags, kMrgFlagMma) &&
           mbar_wait(&acc_full[b], (li / kMrgAccBufs) & 1, abort_p, &g_merge_flags, kMrgFlagMma);
      // the staging rows this warp writes have been read by its earlier store
      // (issued by the same lane); a warp leaving on a failed wait leaves whole
      if (lane == 0) bulk_wait_group_read<kMrgOutBufs - 1>();
      if (!__all_sync(0xffffffffu, ok)) break;
      __syncwarp();
      tc_fence_after();
      const uint8_t* st = smem + s * L.stage;
      uint8_t* out_box = smem + L.out + ob * 32768 + h * 16384;
      Nf4Table tab;
      if (!DENSE) tab = nf4_make_table(P.cb, am);
      const uint64_t s2 = f32x2_pack(P.s, P.s);
      // this row's 64 code bytes of the warpgroup's 128 columns (NF4): 64-byte
      // code rows, 64B swizzle, 16-byte chunk q of row i at chunk q ^ ((i >> 1) & 3)
      uint32_t cw[8];
      if (!DENSE) {
#pragma unroll
        for (int q = 0; q < 2; ++q) {
          const int chunk = (2 * h + q) ^ ((tid >> 1) & 3);
          const uint4 x = *reinterpret_cast<const uint4*>(st + tid * 64 + chunk * 16);
          cw[4 * q] = x.x, cw[4 * q + 1] = x.y, cw[4 * q + 2] = x.z, cw[4 * q + 3] = x.w;
        }
        // once this row's codes are in registers (the stage's B and A are
        // read only by the MMAs, whose commit arrives too) the producer may
        // refill the stage while this tile is expanded
        mbar_arrive_after(&st_empty[s],
                          cw[0] ^ cw[1] ^ cw[2] ^ cw[3] ^ cw[4] ^ cw[5] ^ cw[6] ^ cw[7]);
      }
      // kMrgCols columns at a time; the product of the next kMrgCols is read
      // from tensor memory while these are expanded
      constexpr int C = kMrgCols, NCH = 64 / C;
      const uint32_t tcol = tmem + static_cast<uint32_t>(b * kMrgTile + 64 * h) + lane_base;
      uint32_t v[2][C];
      tmem_ld(tcol, v[0]);
      tmem_wait_ld_for(v[0]);
      const uint8_t* drow = st + h * 16384 + tid * 128;  // dense: this row's 128 B of the base
      uint8_t* orow = out_box + tid * 128;               // this row of the output box
#pragma unroll
      for (int j = 0; j < NCH; ++j) {
        if (j < NCH - 1) tmem_ld(tcol + static_cast<uint32_t>(C * (j + 1)), v[(j + 1) & 1]);
        const uint32_t(&acc)[C] = v[j & 1];
        // the base's C bf16 values of this row, columns C j .. C j + C - 1 of the block
        uint32_t w[C / 2];
#pragma unroll
        for (int q = 0; q < C / 8; ++q) {
          uint4 x;
          if constexpr (DENSE)  // 128B swizzle: 16-byte chunk q of row i at chunk q ^ (i & 7)
            x = *reinterpret_cast<const uint4*>(drow + ((((C / 8) * j + q) ^ (tid & 7)) * 16));
          else
            x = nf4_dequant8(cw[(C / 8) * j + q], tab);
          w[4 * q] = x.x, w[4 * q + 1] = x.y, w[4 * q + 2] = x.z, w[4 * q + 3] = x.w;
        }
        // fp32(deq + fp32(s * acc)), two columns per instruction, then one
        // rounding to bf16
        uint32_t o[C / 2];
#pragma unroll
        for (int e = 0; e < C / 2; ++e) {
          const uint64_t base = f32x2_pack_bits(w[e] << 16, w[e] & 0xFFFF0000u);
          const uint64_t pr = f32x2_pack_bits(acc[2 * e], acc[2 * e + 1]);
          o[e] = f32x2_to_bf16x2(f32x2_add_rn(base, f32x2_mul_rn(pr, s2)));
        }
        // the 128B-swizzled output box, same chunk rule as the dense base
#pragma unroll
        for (int q = 0; q < C / 8; ++q)
          *reinterpret_cast<uint4*>(orow + ((((C / 8) * j + q) ^ (tid & 7)) * 16)) =
              make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
        if (j < NCH - 1) tmem_wait_ld_for(v[(j + 1) & 1]);
      }
      tc_fence_before();
      mbar_arrive(&acc_empty[b]);            // the accumulator is read
      if (DENSE) mbar_arrive(&st_empty[s]);  // and this row of the base
      fence_proxy_async_smem();
      __syncwarp();
      if (lane == 0) {
        if (k0 + 64 * h < P.K && n0 + 32 * q4 < P.N)
          tma_store_2d(&P.map_out, out_box + q4 * 4096, k0 + 64 * h, n0 + 32 * q4);
        bulk_commit_group();
      }
    }
    if (lane == 0) bulk_wait_group_read<0>();  // the stores have read their staging boxes
  }

  __syncthreads();  // every thread sees the final abort word
  if (*abort_p && threadIdx.x == 0) {
    // drain what this CTA started before its shared memory and TMEM go away
    volatile int never = 0;
    for (int li = (last_load - 1 > 0 ? last_load - 1 : 0); li <= last_load; ++li)
      if (!mbar_wait(&st_full[li & 1], (li >> 1) & 1, &never, &g_merge_flags, kMrgFlagDrain))
        break;
  }
  if (*abort_p && warp == 1 && lane == 0 && mma_issued) {
    volatile int never = 0;
    umma_commit(&drain);
    mbar_wait(&drain, 0, &never, &g_merge_flags, kMrgFlagDrain);
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kMrgAccBufs * kMrgTile);
  }
}

cudaError_t launch_lora_merge(const void* base, const float* absmax, bool dense, int64_t N,
                              int64_t K, const void* A, const void* B, int r, float s, void* out,
                              cudaStream_t st) {
  static MergeParams P;  // built on the host, copied into the launch
  static std::mutex mu;
  std::lock_guard<std::mutex> lk(mu);
  memset(&P, 0, sizeof P);
  P.absmax = absmax;
  P.N = N;
  P.K = K;
  P.r_pad = (r + 15) / 16 * 16;
  P.dense = dense ? 1 : 0;
  P.s = s;
  P.cb = codebook();
  P.col_tiles = static_cast<int>((K + kMrgTile - 1) / kMrgTile);
  bool ok = dense ? encode_tma_2d(&P.map_base, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, base, K, N,
                                  K * 2, 64, kMrgTile, CU_TENSOR_MAP_SWIZZLE_128B)
                  : encode_tma_2d(&P.map_base, CU_TENSOR_MAP_DATA_TYPE_UINT8, base, K / 2, N,
                                  K / 2, 64, kMrgTile, CU_TENSOR_MAP_SWIZZLE_64B);
  ok = ok && encode_tma_2d(&P.map_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, A, K, r, K * 2, 64,
                           P.r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  ok = ok && encode_tma_2d(&P.map_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, B, r, N,
                           static_cast<uint64_t>(r) * 2, 16, kMrgTile, CU_TENSOR_MAP_SWIZZLE_32B);
  ok = ok && encode_tma_2d(&P.map_out, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, out, K, N, K * 2, 64,
                           32, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  const int smem = merge_smem(P.dense, P.r_pad).total + 1024;
  static cudaError_t attr_rc = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    attr_rc = cudaFuncSetAttribute(lora_merge_kernel<true>,
                                   cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   merge_smem(1, 64).total + 1024);
    if (attr_rc == cudaSuccess)
      attr_rc = cudaFuncSetAttribute(lora_merge_kernel<false>,
                                     cudaFuncAttributeMaxDynamicSharedMemorySize,
                                     merge_smem(0, 64).total + 1024);
  });
  if (attr_rc != cudaSuccess) return attr_rc;
  P.row_tiles = static_cast<int>((N + kMrgTile - 1) / kMrgTile);
  const int64_t tiles = static_cast<int64_t>(P.row_tiles) * P.col_tiles;
  if (tiles > 0x7fffffff) return cudaErrorInvalidConfiguration;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int per_sm = std::max(
      1, std::min(P.dense ? MrgCfg<true>::kCtasPerSm : MrgCfg<false>::kCtasPerSm,
                  (227 * 1024) / smem));
  const int grid = static_cast<int>(std::min<int64_t>(tiles, static_cast<int64_t>(per_sm) * sms));
  void* prof = prof_begin(st, kProfMerge);
  count_launch();
  if (P.dense)
    lora_merge_kernel<true><<<grid, kMrgThreads, smem, st>>>(P);
  else
    lora_merge_kernel<false><<<grid, kMrgThreads, smem, st>>>(P);
  const cudaError_t e = cudaGetLastError();
  // algorithmic bytes per element: the base read (0.5625 B NF4, 2 B dense) + 2 B written
  if (prof) prof_end(prof, kProfMerge, (dense ? 4.0 : 2.5625) * static_cast<double>(N) * K, st);
  return e;
}

cudaError_t read_merge_flags(uint32_t* flags) {
  unsigned int v = 0;
  cudaError_t e = cudaMemcpyFromSymbol(&v, g_merge_flags, sizeof v);
  if (e != cudaSuccess) return e;
  *flags = v;
  if (v) {
    const unsigned int z = 0;
    e = cudaMemcpyToSymbol(g_merge_flags, &z, sizeof z);
  }
  return e;
}

}  // namespace hsnf4
