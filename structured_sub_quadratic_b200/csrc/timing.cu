// Per-kernel CUDA-event timing for benchmarks (see timing.cuh).
#include "monarch_attn.h"
#include "timing.cuh"

#include <atomic>
#include <cstring>
#include <mutex>
#include <string>
#include <vector>

namespace monarch {

namespace {

struct Pending {
  int slot;
  cudaEvent_t start, stop;
};

struct Slot {
  std::string name;
  double ms = 0.0;
  long launches = 0;
};

std::atomic<bool> g_enabled{false};
std::mutex g_mu;
std::vector<Slot> g_slots;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

int slot_of(const char* name) {
  for (size_t s = 0; s < g_slots.size(); ++s)
    if (g_slots[s].name == name) return (int)s;
  g_slots.push_back(Slot{name});
  return (int)g_slots.size() - 1;
}

}  // namespace

bool timing_enabled() { return g_enabled.load(std::memory_order_relaxed); }

KernelTimer::KernelTimer(const char* name, cudaStream_t stream) : stream_(stream) {
  if (!timing_enabled()) return;
  std::lock_guard<std::mutex> lock(g_mu);
  start_ = take_event();
  if (!start_) return;
  slot_ = slot_of(name);
  cudaEventRecord(start_, stream_);
}

void KernelTimer::stop() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaEvent_t stop = take_event();
  if (!stop) {
    g_pool.push_back(start_);
    return;
  }
  cudaEventRecord(stop, stream_);
  g_pending.push_back(Pending{slot_, start_, stop});
  slot_ = -1;
}

}  // namespace monarch

extern "C" {

int monarch_attn_timing_enable(int enable) {
  return monarch::g_enabled.exchange(enable != 0) ? 1 : 0;
}

int monarch_attn_timing_read(int max_kernels, char* names, int name_len, double* ms_total,
                             long* launches) {
  using namespace monarch;
  std::lock_guard<std::mutex> lock(g_mu);
  for (const Pending& p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.stop) != cudaSuccess ||
        cudaEventElapsedTime(&ms, p.start, p.stop) != cudaSuccess)
      return MONARCH_ERR_CUDA;
    g_slots[p.slot].ms += ms;
    g_slots[p.slot].launches += 1;
    g_pool.push_back(p.start);
    g_pool.push_back(p.stop);
  }
  g_pending.clear();
  const int n = (int)g_slots.size();
  for (int s = 0; s < n && s < max_kernels; ++s) {
    if (names && name_len > 0) {
      std::strncpy(names + (size_t)s * name_len, g_slots[s].name.c_str(), name_len - 1);
      names[(size_t)s * name_len + name_len - 1] = '\0';
    }
    if (ms_total) ms_total[s] = g_slots[s].ms;
    if (launches) launches[s] = g_slots[s].launches;
  }
  g_slots.clear();
  return n;
}

}  // extern "C"
