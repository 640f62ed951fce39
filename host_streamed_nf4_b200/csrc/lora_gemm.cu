// lora_gemm.cu -- fused NF4 dequant + tcgen05 GEMM with the rank-r LoRA term
// folded into the same tensor-core accumulation (sm_100a).
//
// Forward of a LoRA linear (Poros API reference, lora_rank/lora_alpha; the
// frozen base is only read -- HN comment on host-RAM streaming):
//     Y[T, n_out] = X[T, k_in] deq(W)^T + (s t)[T, r] B[n_out, r]^T
// Backward, input gradient:
//     dX[T, k_in] = dY[T, n_out] deq(W) + (s u)[T, r] A[r, k_in]
//
// Both are computed transposed, with the weight on the MMA's M side so that
// a CTA dequantizes one 128-row slab of W once for all of its tokens:
//     fwd: D[n, t] = sum_k deq(W)[n, k] X[t, k]      (A op K-major)
//     dx : D[k, t] = sum_n deq(W)[n, k] dY[t, n]     (A op MN-major)
// The rank-r term is one more K-slice of the same accumulator:
//     fwd: D[n, t] += sum_j B[n, j] (s t)[t, j]
//     dx : D[k, t] += sum_j A[j, k] (s u)[t, j]
//
// CTA roles (192 threads, one output tile of 128 x BN per CTA):
//   warp 4      TMA producer: activation tile (bf16, 128B swizzle) and the
//               raw code tile per 64-wide K step, plus the rank-r operands;
//   warp 5      TMEM owner and UMMA issuer (one elected thread);
//   warps 0..3  dequantize the code tile into the UMMA A-operand layout in
//               shared memory (one 64-element block = one 128-byte line per
//               thread), then run the epilogue (TMEM -> bf16 -> global).
// Every wait is bounded (ptx.cuh); a timed-out wait records a flag in
// g_gemm_flags, the CTA drains what it started and exits.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cudaTypedefs.h>

#include <mutex>

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
};

constexpr int kTileM = 128;     // rows of the MMA (W rows or k_in columns)
constexpr int kStepK = 64;      // contraction per pipeline stage
constexpr int kCodeBytes = 4096;          // raw codes of one stage (128 x 64 / 2)
constexpr int kATileBytes = kTileM * 128;  // dequantized bf16 A tile
constexpr int kMaxSmem = 232448;           // 227 KiB opt-in per block
constexpr int kThreads = 192;

struct GemmParams {
  CUtensorMap map_act;    // X / dY: bf16 [T, contraction], box {64, BN}, 128B swizzle
  CUtensorMap map_codes;  // uint8 [n_out, k_in/2]; box {32, 128} fwd, {64, 64} dx
  CUtensorMap map_lo_a;   // fwd: B [n_out, r] box {16, 128} 32B swz; dx: A [r, k_in] box {64, r_pad} 128B swz
  CUtensorMap map_lo_b;   // s*t or s*u: bf16 [T, r_pad], box {16, BN}, 32B swizzle
  const float* absmax;
  uint16_t* out;
  Nf4Codebook cb;
  int T, n_out, k_in, r_pad;
  int BN, stages, tmem_cols;
};

struct SmemPlan {
  int stage_bytes, lora_a_bytes, lora_b_bytes, bar_off, total;
};

__host__ __device__ inline SmemPlan smem_plan(int mode, int BN, int stages, int r_pad) {
  SmemPlan p;
  p.stage_bytes = BN * 128 + kATileBytes + kCodeBytes;
  const int slices = r_pad / 16;
  p.lora_a_bytes = (mode == kGemmFwd) ? slices * 4096 : 2 * r_pad * 128;
  p.lora_b_bytes = slices * BN * 32;
  p.bar_off = stages * p.stage_bytes + p.lora_a_bytes + p.lora_b_bytes;
  p.total = p.bar_off + (3 * stages + 3) * 8 + 16;
  return p;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1) lora_gemm_kernel(const __grid_constant__ GemmParams p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int S = p.stages, BN = p.BN;
  const SmemPlan plan = smem_plan(MODE, BN, S, p.r_pad);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int m0 = blockIdx.x * kTileM;  // W row (fwd) / k_in column (dx)
  const int t0 = blockIdx.y * BN;
  const int nk = (MODE == kGemmFwd) ? p.k_in / kStepK : p.n_out / kStepK;
  const int slices = p.r_pad / 16;
  const int kblocks = p.k_in / 64;  // absmax blocks per W row

  uint8_t* lora_a = smem + S * plan.stage_bytes;
  uint8_t* lora_b = lora_a + plan.lora_a_bytes;
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + plan.bar_off);
  uint64_t* deq = full + S;
  uint64_t* empty = deq + S;
  uint64_t* lora_bar = empty + S;
  uint64_t* acc_bar = lora_bar + 1;
  uint64_t* drain_bar = acc_bar + 1;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain_bar + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto act_tile = [&](int s) { return smem + s * plan.stage_bytes; };
  auto a_tile = [&](int s) { return smem + s * plan.stage_bytes + BN * 128; };
  auto code_tile = [&](int s) { return smem + s * plan.stage_bytes + BN * 128 + kATileBytes; };

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&deq[s], 128);
      mbar_init(&empty[s], 1);
    }
    mbar_init(lora_bar, 1);
    mbar_init(acc_bar, 1);
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 5) {
    tmem_alloc(tmem_slot, static_cast<uint32_t>(p.tmem_cols));
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tmem_slot;

  // idesc: M = 128, N = BN; fwd A is K-major, dx A is MN-major; B K-major.
  const uint32_t idesc = make_idesc_bf16(kTileM, BN, MODE == kGemmDx ? 1 : 0, 0);

  int issued_phase[8];  // producer: parity of the last load issued per stage (-1 none)
  bool mma_started = false;

  if (warp == 4) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int s = 0; s < 8; ++s) issued_phase[s] = -1;
      tma_prefetch_desc(&p.map_act);
      tma_prefetch_desc(&p.map_codes);
      mbar_arrive_expect_tx(lora_bar,
                            static_cast<uint32_t>(plan.lora_a_bytes + plan.lora_b_bytes));
      if (MODE == kGemmFwd) {
        for (int j = 0; j < slices; ++j)
          tma_load_2d(lora_a + j * 4096, &p.map_lo_a, lora_bar, j * 16, m0);
      } else {
        for (int h = 0; h < 2; ++h)
          tma_load_2d(lora_a + h * p.r_pad * 128, &p.map_lo_a, lora_bar, m0 + h * 64, 0);
      }
      for (int j = 0; j < slices; ++j)
        tma_load_2d(lora_b + j * BN * 32, &p.map_lo_b, lora_bar, j * 16, t0);
      const uint32_t stage_tx = static_cast<uint32_t>(BN * 128 + kCodeBytes);
      for (int kb = 0; kb < nk; ++kb) {
        const int s = kb % S, round = kb / S;
        if (kb >= S && !mbar_wait(&empty[s], (round - 1) & 1, abort_flag, &g_gemm_flags,
                                  kFlagProducer))
          break;
        mbar_arrive_expect_tx(&full[s], stage_tx);
        tma_load_2d(act_tile(s), &p.map_act, &full[s], kb * kStepK, t0);
        if (MODE == kGemmFwd)
          tma_load_2d(code_tile(s), &p.map_codes, &full[s], kb * 32, m0);
        else
          tma_load_2d(code_tile(s), &p.map_codes, &full[s], m0 / 2, kb * kStepK);
        issued_phase[s] = round & 1;
      }
    }
  } else if (warp == 5) {
    // ------------------------------------------------------------ UMMA issuer
    if (lane == 0) {
      bool ok = true;
      for (int kb = 0; kb < nk && ok; ++kb) {
        const int s = kb % S, ph = (kb / S) & 1;
        ok = mbar_wait(&full[s], ph, abort_flag, &g_gemm_flags, kFlagMma) &&
             mbar_wait(&deq[s], ph, abort_flag, &g_gemm_flags, kFlagMma);
        if (!ok) break;
        tc_fence_after();
        const uint32_t a_base = smem_u32(a_tile(s));
        const uint32_t b_base = smem_u32(act_tile(s));
#pragma unroll
        for (int k16 = 0; k16 < 4; ++k16) {
          // fwd A: 128 rows x 128 B lines (K-major, 8-row groups 1024 B apart);
          //        a 16-wide K step is 32 B further along each line.
          // dx  A: two 64-column atoms 8 KiB apart (LBO), 8-row groups 1 KiB
          //        apart (SBO); a 16-row K step is 2 KiB further.
          const uint64_t adesc =
              (MODE == kGemmFwd)
                  ? make_sdesc(a_base + k16 * 32, 16, 1024, kLayoutSw128)
                  : make_sdesc(a_base + k16 * 2048, 64 * 128, 1024, kLayoutSw128);
          const uint64_t bdesc = make_sdesc(b_base + k16 * 32, 16, 1024, kLayoutSw128);
          umma_bf16(tmem, adesc, bdesc, idesc, (kb > 0 || k16 > 0) ? 1u : 0u);
        }
        mma_started = true;
        umma_commit(&empty[s]);
      }
      if (ok && mbar_wait(lora_bar, 0, abort_flag, &g_gemm_flags, kFlagLora)) {
        tc_fence_after();
        const uint32_t la = smem_u32(lora_a), lb = smem_u32(lora_b);
        for (int j = 0; j < slices; ++j) {
          const uint64_t adesc =
              (MODE == kGemmFwd)
                  ? make_sdesc(la + j * 4096, 16, 256, kLayoutSw32)
                  : make_sdesc(la + j * 2048, p.r_pad * 128, 1024, kLayoutSw128);
          const uint64_t bdesc = make_sdesc(lb + j * BN * 32, 16, 256, kLayoutSw32);
          umma_bf16(tmem, adesc, bdesc, idesc, 1u);
        }
        mma_started = true;
        umma_commit(acc_bar);
      }
    }
  } else {
    // ------------------------------------------------------------ dequant
    const int i = threadIdx.x;  // 0..127
    const int line = (MODE == kGemmFwd) ? i : ((i >> 6) * 64 + (i & 63));
    const int code_off = (MODE == kGemmFwd) ? i * 32 : (i & 63) * 64 + (i >> 6) * 32;
    bool ok = true;
    for (int kb = 0; kb < nk; ++kb) {
      const int s = kb % S, ph = (kb / S) & 1;
      float a;
      if (MODE == kGemmFwd) {
        const int row = m0 + i;
        a = (row < p.n_out) ? __ldg(p.absmax + static_cast<int64_t>(row) * kblocks + kb) : 0.0f;
      } else {
        const int row = kb * kStepK + (i & 63);
        const int kblk = m0 / 64 + (i >> 6);
        a = (kblk < kblocks) ? __ldg(p.absmax + static_cast<int64_t>(row) * kblocks + kblk)
                             : 0.0f;
      }
      if (!mbar_wait(&full[s], ph, abort_flag, &g_gemm_flags, kFlagDequant)) {
        ok = false;
        break;
      }
      const uint4* src = reinterpret_cast<const uint4*>(code_tile(s) + code_off);
      const uint4 c0 = src[0], c1 = src[1];
      const uint32_t words[8] = {c0.x, c0.y, c0.z, c0.w, c1.x, c1.y, c1.z, c1.w};
      const Nf4Table tab = nf4_make_table(p.cb, a);
      uint8_t* dst = a_tile(s) + line * 128;
#pragma unroll
      for (int w = 0; w < 8; ++w) {
        const uint4 v = nf4_dequant8(words[w], tab);
        *reinterpret_cast<uint4*>(dst + ((w ^ (line & 7)) << 4)) = v;
      }
      fence_proxy_async_smem();
      mbar_arrive(&deq[s]);
    }
    // ------------------------------------------------------------ epilogue
    // tcgen05.ld is warp-collective: decide per warp, never per lane.
    ok = __all_sync(0xffffffffu, ok);
    if (ok) ok = __all_sync(0xffffffffu, mbar_wait(acc_bar, 0, abort_flag, &g_gemm_flags,
                                                   kFlagEpilogue));
    if (ok) {
      tc_fence_after();
      const int M = (MODE == kGemmFwd) ? p.n_out : p.k_in;
      const int row = m0 + warp * 32 + lane;
      for (int c = 0; c < BN; c += 16) {
        uint32_t v[16];
        tmem_ld16(tmem + (static_cast<uint32_t>(warp * 32) << 16) + static_cast<uint32_t>(c), v);
        tmem_wait_ld();
        if (row < M) {
#pragma unroll
          for (int j = 0; j < 16; ++j) {
            const int t = t0 + c + j;
            if (t < p.T) {
              const __nv_bfloat16 b = __float2bfloat16_rn(__uint_as_float(v[j]));
              p.out[static_cast<int64_t>(t) * M + row] = *reinterpret_cast<const uint16_t*>(&b);
            }
          }
        }
      }
    }
  }

  // ------------------------------------------------------------ teardown
  __syncthreads();
  if (*abort_flag) {
    // Drain what this CTA started before its shared memory and TMEM go away.
    if (warp == 4 && lane == 0) {
      for (int s = 0; s < S && s < 8; ++s)
        if (issued_phase[s] >= 0) {
          volatile int never = 0;
          if (!mbar_wait(&full[s], static_cast<uint32_t>(issued_phase[s]), &never,
                         &g_gemm_flags, kFlagDrain))
            break;
        }
    }
    if (warp == 5 && lane == 0 && mma_started) {
      umma_commit(drain_bar);
      volatile int never = 0;
      mbar_wait(drain_bar, 0, &never, &g_gemm_flags, kFlagDrain);
    }
  }
  tc_fence_before();
  __syncthreads();
  if (warp == 5) {
    tc_fence_after();
    tmem_dealloc(tmem, static_cast<uint32_t>(p.tmem_cols));
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
  selftest_stall_kernel<<<1, 32, 0, st>>>();
  return cudaGetLastError();
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

static bool encode_2d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t inner,
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

int launch_lora_gemm(GemmMode mode, const hsnf4_nf4_weight* W, const void* act, int64_t T,
                     const void* lo_a, int r, int r_pad, const void* lo_b, void* out,
                     cudaStream_t st) {
  const int64_t n_out = W->n_out, k_in = W->k_in;
  GemmParams p;
  memset(&p, 0, sizeof p);
  const int64_t bn16 = (T + 15) / 16 * 16;
  p.BN = static_cast<int>(bn16 < 256 ? bn16 : 256);
  p.T = static_cast<int>(T);
  p.n_out = static_cast<int>(n_out);
  p.k_in = static_cast<int>(k_in);
  p.r_pad = r_pad;
  p.absmax = W->absmax;
  p.out = static_cast<uint16_t*>(out);
  p.cb = codebook();
  int tc = 32;
  while (tc < p.BN) tc <<= 1;
  p.tmem_cols = tc;
  int stages = 4;
  while (stages > 2 && smem_plan(mode, p.BN, stages, r_pad).total + 1024 > kMaxSmem) --stages;
  p.stages = stages;
  const int smem = smem_plan(mode, p.BN, stages, r_pad).total + 1024;
  if (smem > kMaxSmem) return fail(HSNF4_ERR_INVALID, "lora gemm: shared memory plan %d B too large", smem);

  const int64_t contraction = (mode == kGemmFwd) ? k_in : n_out;
  bool ok = encode_2d(&p.map_act, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, act, contraction, T,
                      contraction * 2, 64, p.BN, CU_TENSOR_MAP_SWIZZLE_128B);
  if (mode == kGemmFwd) {
    ok = ok && encode_2d(&p.map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, k_in / 2, n_out,
                         k_in / 2, 32, 128, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && encode_2d(&p.map_lo_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lo_a, r, n_out, r * 2, 16,
                         128, CU_TENSOR_MAP_SWIZZLE_32B);
  } else {
    ok = ok && encode_2d(&p.map_codes, CU_TENSOR_MAP_DATA_TYPE_UINT8, W->codes, k_in / 2, n_out,
                         k_in / 2, 64, 64, CU_TENSOR_MAP_SWIZZLE_NONE);
    ok = ok && encode_2d(&p.map_lo_a, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lo_a, k_in, r, k_in * 2,
                         64, r_pad, CU_TENSOR_MAP_SWIZZLE_128B);
  }
  ok = ok && encode_2d(&p.map_lo_b, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, lo_b, r_pad, T, r_pad * 2,
                       16, p.BN, CU_TENSOR_MAP_SWIZZLE_32B);
  if (!ok) return fail(HSNF4_ERR_CUDA, "lora gemm: cuTensorMapEncodeTiled failed");

  const int64_t mdim = (mode == kGemmFwd) ? n_out : k_in;
  dim3 grid(static_cast<unsigned>((mdim + kTileM - 1) / kTileM),
            static_cast<unsigned>((T + p.BN - 1) / p.BN));
  cudaError_t e;
  if (configure_once<kGemmFwd>() != 0 || configure_once<kGemmDx>() != 0)
    return fail(HSNF4_ERR_CUDA, "lora gemm: smem attribute");
  void* prof = prof_begin(st);
  if (mode == kGemmFwd)
    lora_gemm_kernel<kGemmFwd><<<grid, kThreads, smem, st>>>(p);
  else
    lora_gemm_kernel<kGemmDx><<<grid, kThreads, smem, st>>>(p);
  e = cudaGetLastError();
  if (prof) {
    // algorithmic FLOPs: the base product plus the rank-r slice
    const double flops = (mode == kGemmFwd) ? 2.0 * T * n_out * (k_in + r)
                                            : 2.0 * T * k_in * (n_out + r);
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
