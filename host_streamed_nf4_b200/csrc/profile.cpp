// profile.cpp -- CUDA-event timing of the library's own kernel launches,
// used to report achieved throughput against the roofline.
#include <cuda_runtime.h>
#include <string.h>

#include <atomic>
#include <mutex>
#include <string>
#include <vector>

#include "internal.h"

namespace hsnf4 {

namespace {

struct Rec {
  int kind;
  double work;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
unsigned g_kinds = 0;  // bit k: time launches of kind k
std::vector<Rec> g_recs;

const char* kKindName[kProfKinds] = {"lora_gemm_fwd", "lora_gemm_dx", "nf4_dequant",
                                      "lora_merge",    "lora_project", "lora_grad"};

}  // namespace

std::atomic<uint64_t> g_launches{0};

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

bool profiling() { return g_on; }

void* prof_begin(cudaStream_t st, int kind) {
  if (!g_on || !((g_kinds >> kind) & 1u)) return nullptr;
  cudaEvent_t a;
  if (cudaEventCreate(&a) != cudaSuccess) return nullptr;
  cudaEventRecord(a, st);
  return a;
}

void prof_end(void* token, int kind, double work, cudaStream_t st) {
  if (!token) return;
  cudaEvent_t b;
  if (cudaEventCreate(&b) != cudaSuccess) {
    cudaEventDestroy(static_cast<cudaEvent_t>(token));
    return;
  }
  cudaEventRecord(b, st);
  std::lock_guard<std::mutex> lk(g_mu);
  g_recs.push_back({kind, work, static_cast<cudaEvent_t>(token), b});
}

static void clear_locked() {
  for (auto& r : g_recs) {
    cudaEventDestroy(r.a);
    cudaEventDestroy(r.b);
  }
  g_recs.clear();
}

}  // namespace hsnf4

using namespace hsnf4;

extern "C" {

uint64_t hsnf4_kernel_launches(void) { return g_launches.load(std::memory_order_relaxed); }

int hsnf4_profile(int enable) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (enable) clear_locked();
  g_on = enable != 0;
  g_kinds = (1u << kProfKinds) - 1;
  return HSNF4_OK;
}

int hsnf4_profile_kinds(unsigned int kinds) {
  std::lock_guard<std::mutex> lk(g_mu);
  clear_locked();
  g_kinds = kinds & ((1u << kProfKinds) - 1);
  g_on = g_kinds != 0;
  return HSNF4_OK;
}

int hsnf4_profile_read(hsnf4_kernel_time* out, int max_out) {
  if (!out || max_out < 0) return -fail(HSNF4_ERR_INVALID, "hsnf4_profile_read: bad output");
  std::lock_guard<std::mutex> lk(g_mu);
  hsnf4_kernel_time acc[kProfKinds];
  memset(acc, 0, sizeof acc);
  for (int k = 0; k < kProfKinds; ++k) strncpy(acc[k].name, kKindName[k], sizeof acc[k].name - 1);
  for (auto& r : g_recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess)
      return -cuda_status(cudaGetLastError(), "hsnf4_profile_read: event sync");
    float ms = 0;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess)
      return -cuda_status(cudaGetLastError(), "hsnf4_profile_read: elapsed");
    acc[r.kind].launches += 1;
    acc[r.kind].total_ms += ms;
    acc[r.kind].work += r.work;
  }
  int n = 0;
  for (int k = 0; k < kProfKinds && n < max_out; ++k)
    if (acc[k].launches) out[n++] = acc[k];
  return n;
}

}  // extern "C"
