// profile.cpp -- optional per-kernel CUDA-event timing (hia_profile_begin/end).
#include <cuda_runtime.h>

#include <atomic>
#include <cstring>
#include <mutex>
#include <vector>

#include "kernels.h"

namespace {

const char* kNames[hia::kNumKernels] = {"rope2d_tables", "rope_rotate", "attn_fwd",  "bwd_pre",
                                        "attn_bwd",      "grad_finalize", "dw_reduce", "moe_prep",
                                        "moe_router",    "moe_scan",    "moe_gather", "moe_up_gate",
                                        "moe_down",      "moe_combine"};

struct Rec {
  int id;
  cudaEvent_t a, b;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<cudaEvent_t> g_pool;  // created once, reused
std::vector<Rec> g_recs;
size_t g_next = 0;
thread_local cudaEvent_t t_open[hia::kNumKernels] = {};

cudaEvent_t take() {
  if (g_next == g_pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    g_pool.push_back(e);
  }
  return g_pool[g_next++];
}

}  // namespace

namespace hia {

void prof_begin(KernelId id, cudaStream_t st) {
  if (!g_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t e = take();
  if (e && cudaEventRecord(e, st) == cudaSuccess) t_open[id] = e;
}

void prof_end(KernelId id, cudaStream_t st) {
  if (!g_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t a = t_open[id];
  t_open[id] = nullptr;
  if (!a) return;
  cudaEvent_t e = take();
  if (e && cudaEventRecord(e, st) == cudaSuccess) g_recs.push_back({int(id), a, e});
}

}  // namespace hia

extern "C" int hia_profile_begin(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_recs.clear();
  g_next = 0;
  g_on.store(true);
  return HIA_OK;
}

extern "C" int hia_profile_end(hia_kernel_time* out, int max_entries, int* n_out) {
  g_on.store(false);
  std::lock_guard<std::mutex> lk(g_mu);
  double tot[hia::kNumKernels] = {};
  int cnt[hia::kNumKernels] = {};
  int rc = HIA_OK;
  for (const Rec& r : g_recs) {
    float ms = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) {
      rc = HIA_ERR_CUDA;
      continue;
    }
    tot[r.id] += ms;
    cnt[r.id] += 1;
  }
  g_recs.clear();
  g_next = 0;
  int n = 0;
  for (int i = 0; i < hia::kNumKernels; ++i) {
    if (!cnt[i]) continue;
    if (out && n < max_entries) {
      std::memset(out[n].name, 0, sizeof(out[n].name));
      std::strncpy(out[n].name, kNames[i], sizeof(out[n].name) - 1);
      out[n].launches = cnt[i];
      out[n].total_ms = tot[i];
    }
    ++n;
  }
  if (n_out) *n_out = n;
  return rc;
}
