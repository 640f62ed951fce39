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
// CTA = a 128 x 128 tile of W' (sm_100a).  One thread loads the tile's base
// (NF4 codes or bf16 weight), B's 128 rows and A's 128 columns with TMA,
// then issues r/16 tcgen05 MMAs (M = 128 rows, N = 128 columns, K = 16
// ranks each; B read K-major, A read MN-major) into a 128-column fp32
// accumulator in tensor memory.  Each of the 128 threads then owns one row:
// it reads its product row back from tensor memory 32 columns at a time,
// expands the matching base bytes, adds, rounds and writes the bf16 row into
// a staging tile that two TMA stores write out.  HBM traffic is the base read
// once plus W' written once; several CTAs per SM keep loads in flight.
#include <cuda_bf16.h>

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

struct MergeParams {
  CUtensorMap map_base;  // NF4: codes uint8 [N, K/2], box {64, 128}, 64B swizzle
                         // dense: bf16 [N, K], box {64, 128}, 128B swizzle (two per tile)
  CUtensorMap map_a;     // A bf16 [r, K], box {64, r_pad}, 128B swizzle (MN-major operand)
  CUtensorMap map_b;     // B bf16 [N, r], box {16, 128}, 32B swizzle (K-major operand)
  CUtensorMap map_out;   // W' bf16 [N, K], box {64, 128}, 128B swizzle
  const float* absmax;   // NF4 only: fp32 [N, K/64]
  int64_t N, K;
  int r_pad, dense, col_tiles;
  float s;
  Nf4Codebook cb;
};

// shared-memory plan of a tile (offsets from a 1 KiB-aligned base)
struct MergeSmem {
  int base, b, a, out, total;
};

__host__ __device__ inline MergeSmem merge_smem(int dense, int r_pad) {
  MergeSmem m;
  m.base = 0;
  m.b = dense ? 32768 : 8192;        // base tile: 128 x 128 bf16, or 128 x 64 code bytes
  m.a = m.b + (r_pad / 16) * 4096;   // B: r_pad / 16 slices of 128 rows x 32 B
  m.out = m.a + 2 * r_pad * 128;     // A: two 64-column atoms of r_pad rows x 128 B
  m.total = m.out + 2 * 16384;       // W': two 64-column boxes of 128 rows x 128 B
  return m;
}

__global__ void __launch_bounds__(128) lora_merge_kernel(const __grid_constant__ MergeParams P) {
  extern __shared__ uint8_t mrg_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(mrg_smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ uint64_t loaded, done, drain;
  __shared__ uint32_t tmem_slot;
  __shared__ int abort_flag;
  const MergeSmem L = merge_smem(P.dense, P.r_pad);
  const int tid = threadIdx.x, warp = tid >> 5;
  const int n0 = static_cast<int>(blockIdx.x / P.col_tiles) * kMrgTile;
  const int k0 = static_cast<int>(blockIdx.x % P.col_tiles) * kMrgTile;
  const int n = n0 + tid;  // this thread's row

  if (tid == 0) {
    mbar_init(&loaded, 1);
    mbar_init(&done, 1);
    mbar_init(&drain, 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(&tmem_slot, kMrgTile);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tmem_slot;
  volatile int* abort_p = &abort_flag;
  bool issued_load = false, issued_mma = false;

  // this thread's two absmax values (blocks k0/64 and k0/64 + 1 of row n),
  // loaded first so that their latency overlaps the tile loads
  float am[2] = {0.f, 0.f};
  if (!P.dense && n < P.N)
#pragma unroll
    for (int h = 0; h < 2; ++h)
      if (k0 + 64 * h < P.K) am[h] = __ldg(P.absmax + static_cast<int64_t>(n) * (P.K / 64) + k0 / 64 + h);

  if (tid == 0) {
    const int slices = P.r_pad / 16;
    const uint32_t bytes = static_cast<uint32_t>(L.total - 2 * 16384);
    mbar_arrive_expect_tx(&loaded, bytes);
    if (P.dense) {
      tma_load_2d(smem, &P.map_base, &loaded, k0, n0);
      tma_load_2d(smem + 16384, &P.map_base, &loaded, k0 + 64, n0);
    } else {
      tma_load_2d(smem, &P.map_base, &loaded, k0 / 2, n0);
    }
    for (int j = 0; j < slices; ++j) tma_load_2d(smem + L.b + j * 4096, &P.map_b, &loaded, 16 * j, n0);
    for (int h = 0; h < 2; ++h)
      tma_load_2d(smem + L.a + h * P.r_pad * 128, &P.map_a, &loaded, k0 + 64 * h, 0);
    issued_load = true;
    if (mbar_wait(&loaded, 0, abort_p, &g_merge_flags, kMrgFlagLoad)) {
      tc_fence_after();
      // D[n, k] = sum_j B[n, j] A[j, k]: A operand = B slice j (K-major,
      // 32B swizzle, 8-row groups 256 B apart); B operand = rows 16j.. of A
      // (MN-major, 128B swizzle: 64-column atoms r_pad * 128 B apart,
      // 8-rank groups 1 KiB apart, 16 ranks = 2 KiB per slice)
      const uint32_t idesc = make_idesc_bf16(kMrgTile, kMrgTile, 0, 1);
      for (int j = 0; j < slices; ++j) {
        const uint64_t ad = make_sdesc(smem_u32(smem + L.b + j * 4096), 16, 256, kLayoutSw32);
        const uint64_t bd =
            make_sdesc(smem_u32(smem + L.a + j * 2048), P.r_pad * 128, 1024, kLayoutSw128);
        umma_bf16(tmem, ad, bd, idesc, j > 0 ? 1u : 0u);
      }
      issued_mma = true;
      umma_commit(&done);
    }
  }
  __syncwarp();

  const bool ok = mbar_wait(&done, 0, abort_p, &g_merge_flags, kMrgFlagMma);
  if (ok) {
    tc_fence_after();
    const uint32_t lane_base = static_cast<uint32_t>(warp * 32) << 16;
    Nf4Table tab[2];
    if (!P.dense) {
      tab[0] = nf4_make_table(P.cb, am[0]);
      tab[1] = nf4_make_table(P.cb, am[1]);
    }
    uint8_t* out_row = smem + L.out;
#pragma unroll
    for (int c = 0; c < kMrgTile; c += 32) {
      uint32_t v[32];
      tmem_ld32(tmem + lane_base + static_cast<uint32_t>(c), v);
      tmem_wait_ld();
      // the base's 32 bf16 values of row n, columns c .. c + 31
      uint32_t w[16];
      if (P.dense) {
        const uint8_t* row = smem + (c / 64) * 16384 + tid * 128;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int chunk = ((c % 64) / 8 + q) ^ (tid & 7);
          const uint4 x = *reinterpret_cast<const uint4*>(row + chunk * 16);
          w[4 * q] = x.x, w[4 * q + 1] = x.y, w[4 * q + 2] = x.z, w[4 * q + 3] = x.w;
        }
      } else {
        // 64-byte code rows, 64B swizzle: 16-byte chunk q of row i sits at
        // chunk q ^ ((i >> 1) & 3)
        const int chunk = (c / 32) ^ ((tid >> 1) & 3);
        const uint4 x = *reinterpret_cast<const uint4*>(smem + tid * 64 + chunk * 16);
        const Nf4Table& t = tab[c / 64];
        const uint32_t cw[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const uint4 d = nf4_dequant8(cw[q], t);
          w[4 * q] = d.x, w[4 * q + 1] = d.y, w[4 * q + 2] = d.z, w[4 * q + 3] = d.w;
        }
      }
      uint32_t o[16];
#pragma unroll
      for (int h = 0; h < 16; ++h) {
        const float lo = __uint_as_float(w[h] << 16), hi = __uint_as_float(w[h] & 0xFFFF0000u);
        const __nv_bfloat162 m =
            __floats2bfloat162_rn(__fadd_rn(lo, __fmul_rn(P.s, __uint_as_float(v[2 * h]))),
                                  __fadd_rn(hi, __fmul_rn(P.s, __uint_as_float(v[2 * h + 1]))));
        o[h] = *reinterpret_cast<const uint32_t*>(&m);
      }
      // row n of the 128B-swizzled output box c / 64: 16-byte chunk q of
      // row i at chunk q ^ (i & 7)
      uint8_t* orow = out_row + (c / 64) * 16384 + tid * 128;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        const int chunk = ((c % 64) / 8 + q) ^ (tid & 7);
        *reinterpret_cast<uint4*>(orow + chunk * 16) =
            make_uint4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      }
    }
    fence_proxy_async_smem();
  }
  __syncthreads();
  if (tid == 0 && ok && !*abort_p) {
    for (int h = 0; h < 2; ++h)
      if (k0 + 64 * h < P.K) tma_store_2d(&P.map_out, smem + L.out + h * 16384, k0 + 64 * h, n0);
    bulk_commit_group();
    bulk_wait_group_all();
  }
  if (*abort_p && tid == 0) {
    // drain what this CTA started before its shared memory and TMEM go away
    volatile int never = 0;
    if (issued_load) mbar_wait(&loaded, 0, &never, &g_merge_flags, kMrgFlagDrain);
    if (issued_mma) {
      umma_commit(&drain);
      mbar_wait(&drain, 0, &never, &g_merge_flags, kMrgFlagDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem, kMrgTile);
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
                           kMrgTile, CU_TENSOR_MAP_SWIZZLE_128B);
  if (!ok) return cudaErrorInvalidValue;
  const int smem = merge_smem(P.dense, P.r_pad).total + 1024;
  static cudaError_t attr_rc = cudaSuccess;
  static std::once_flag once;
  std::call_once(once, [] {
    attr_rc = cudaFuncSetAttribute(lora_merge_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                   merge_smem(1, 64).total + 1024);
  });
  if (attr_rc != cudaSuccess) return attr_rc;
  const int64_t grid = ((N + kMrgTile - 1) / kMrgTile) * P.col_tiles;
  if (grid > 0x7fffffff) return cudaErrorInvalidConfiguration;
  void* prof = prof_begin(st);
  count_launch();
  lora_merge_kernel<<<static_cast<unsigned>(grid), 128, smem, st>>>(P);
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
