// noalloc.cu -- the LoRA forward for callers that cannot allocate device
// memory.
//
// lora_linear_fwd needs scratch (the scaled rank-r factor, the projection's
// chunk partials and, for long-K shapes, split-K partial tiles and their
// counters) and expects the caller to hand it in.  Some callers have no way
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
// and caches it; later calls reuse the cached address.  That first call
// should therefore come before any stream capture.
//
// Every call shares the one array and the array keeps the last call's
// contents; what must start at zero (the split-K arrival counters) is
// cleared on the stream by each call.  Calls whose work overlaps on the GPU
// -- on different streams, or from different host threads -- race on the
// scratch; serialize them.
#include <cuda_runtime.h>

#include <mutex>

#include <cstring>

#include "internal.h"

namespace hsnf4 {

constexpr size_t kNoAllocScratchBytes = size_t(64) << 20;  // 64 MiB

static __device__ __align__(256) uint8_t g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;

// Device address of g_noalloc_scratch on the current device (looked up once
// per device), or nullptr with the error recorded.
static void* scratch_on_current_device() {
  static std::mutex mu;
  static void* addr[kMaxDevices] = {};
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
  if (!addr[dev]) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || !p) {
      cuda_status(e != cudaSuccess ? e : cudaErrorInvalidSymbol,
                  "lora_linear_fwd_noalloc: cudaGetSymbolAddress of the scratch");
      return nullptr;
    }
    addr[dev] = p;
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
