// noalloc.cu -- the LoRA forward for callers that cannot allocate device
// memory.
//
// lora_linear_fwd needs scratch (the scaled rank-r factor, the projection's
// chunk partials and, for long-K shapes, split-K partial tiles) and expects
// the caller to hand it in.  Some callers have no way
// to obtain device memory at the point where they run the layer: a runtime
// that reserves its whole device-memory budget at start-up and treats any
// later allocation as an error, a plugin or host callback that is not
// allowed to call into the allocator, or code whose memory is owned by a
// framework it cannot reach.  lora_linear_fwd_noalloc serves them with a
// fixed scratch area compiled into the library instead.
//
// The scratch is one file-scope __device__ array of kNoAllocScratchBytes.
// Every GPU that loads this library holds it until the process exits.  Host
// code cannot use the array's name as a device address (on the host it names
// a stand-in object), so the first call on each device looks the address up
// with cudaGetSymbolAddress while that device is current, checks the result
// and caches it, keyed by the current context's unique ID; later calls in
// the same context reuse it.  That first call should therefore come before
// any stream capture.  A new context on the device (after cudaDeviceReset,
// say) has a new ID, so its first call looks the address up again instead
// of using one from the old context.
//
// Every call shares the one array and the array keeps the last call's
// contents.  Nothing needs clearing: every scratch byte a call reads was
// written earlier in that same call, except the GEMM's K-split arrival
// words, which each launch tags with a fresh 56-bit value so that whatever
// an earlier call left in them counts as no arrivals.  Calls whose work
// overlaps on the GPU -- on different streams, or from different host
// threads -- race on the scratch; serialize them.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include <cstring>

#include "internal.h"

namespace hsnf4 {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// The current context's process-unique ID, through driver entry points the
// runtime hands out (no link against the driver library): 0 if no context
// is current or the entry points are missing.
static unsigned long long current_context_id() {
  using CtxGetCurrent = CUresult (*)(CUcontext*);
  using CtxGetId = CUresult (*)(CUcontext, unsigned long long*);
  static CtxGetCurrent get_current = nullptr;
  static CtxGetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<CtxGetCurrent>(p);
    p = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<CtxGetId>(p);
  });
  if (!get_current || !get_id) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || !ctx) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Device address of g_noalloc_scratch in the current context (looked up once
// per device and context), or nullptr with the error recorded.
static void* scratch_on_current_device() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
  static unsigned long long ctx_id[kMaxDevices] = {};
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) {
    cuda_status(e, "lora_linear_fwd_noalloc: cudaGetDevice");
    return nullptr;
  }
  if (dev < 0 || dev >= kMaxDevices) {
    fail(HSNF4_ERR_INVALID, "lora_linear_fwd_noalloc: device %d beyond the supported %d", dev,
         kMaxDevices);
    return nullptr;
  }
  std::lock_guard<std::mutex> lk(mu);
  const unsigned long long id = current_context_id();
  if (!addr[dev] || id == 0 || id != ctx_id[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                  "lora_linear_fwd_noalloc: cudaGetSymbolAddress of the scratch");
      return nullptr;
    }
    addr[dev] = p;
    // the lookup makes the device's context current if none was: read the
    // ID again, so the next call in this context reuses the address
    ctx_id[dev] = current_context_id();
  }
  return addr[dev];
}

}  // namespace hsnf4

using namespace hsnf4;

extern "C" int lora_linear_fwd_noalloc(const hsnf4_nf4_weight* W, const void* X, int64_t T,
                                       const void* A, const void* B, int r, float alpha, void* Y,
                                       float* t_save, void* stream) {
  static const char* fn = "lora_linear_fwd_noalloc";
  if (!W) return fail(HSNF4_ERR_INVALID, "%s: W is NULL", fn);
  hsnf4_lora_fwd_args a;
  memset(&a, 0, sizeof a);  // no dropout
  a.W = *W;
  a.X = X;
  a.A = A;
  a.B = B;
  a.Y = Y;
  a.t_save = t_save;
  // the size check needs only the shapes: nothing touches the GPU before it
  const size_t need = lora_group_fwd_workspace(&a, 1, T, r);
  if (need == 0)
    return fail(HSNF4_ERR_INVALID, "%s: invalid sizes (T=%lld, r=%d, %lld x %lld)", fn,
                (long long)T, r, (long long)W->n_out, (long long)W->k_in);
  if (need > kNoAllocScratchBytes)
    return fail(HSNF4_ERR_INVALID,
                "%s: T=%lld, W %lld x %lld, r=%d needs %zu bytes of scratch, beyond the built-in "
                "maximum of %zu; call lora_linear_fwd with a workspace instead",
                fn, (long long)T, (long long)W->n_out, (long long)W->k_in, r, need,
                kNoAllocScratchBytes);
  void* scratch = scratch_on_current_device();
  if (!scratch) return hsnf4_last_error(nullptr, 0);
  return lora_group_fwd(&a, 1, T, r, alpha, scratch, kNoAllocScratchBytes, stream);
}
