// wd_trace.cu — launch accounting and optional per-launch CUDA-event timing.
// Every kernel launch of the library is counted by class; with timing on,
// each launch is bracketed by two events recorded on its own stream, so a
// caller can read the device time of each kernel class over any region.
#include <atomic>
#include <mutex>
#include <vector>

#include "wd_internal.cuh"

namespace wd {

namespace {
struct Rec {
  cudaEvent_t a = nullptr, b = nullptr;
  int cls = 0;
};
std::mutex g_mu;
std::atomic<long long> g_counts[KC_COUNT];
std::atomic<bool> g_timing{false};
std::vector<Rec> g_pool;
size_t g_used = 0;
}  // namespace

Trace::Trace(int cls, cudaStream_t st) : cls_(cls), st_(st), slot_(-1) {
  g_counts[cls].fetch_add(1, std::memory_order_relaxed);
  if (!g_timing.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_used == g_pool.size()) {
    Rec r;
    if (cudaEventCreate(&r.a) != cudaSuccess || cudaEventCreate(&r.b) != cudaSuccess) return;
    g_pool.push_back(r);
  }
  slot_ = static_cast<int>(g_used++);
  g_pool[slot_].cls = cls;
  cudaEventRecord(g_pool[slot_].a, st_);
}

Trace::~Trace() {
  if (slot_ < 0) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEventRecord(g_pool[slot_].b, st_);
}

}  // namespace wd

extern "C" {

void wd_trace_enable(int on) { wd::g_timing.store(on != 0); }

wd_status wd_trace_read(int64_t* launches, double* total_ms) {
  using namespace wd;
  std::lock_guard<std::mutex> lk(g_mu);
  double ms[KC_COUNT] = {};
  for (size_t i = 0; i < g_used; ++i) {
    Rec& r = g_pool[i];
    if (cudaEventSynchronize(r.b) != cudaSuccess) { set_error("trace: event synchronize failed"); return WD_ERR_CUDA; }
    float t = 0.f;
    if (cudaEventElapsedTime(&t, r.a, r.b) == cudaSuccess) ms[r.cls] += t;
  }
  g_used = 0;
  for (int c = 0; c < KC_COUNT; ++c) {
    const long long n = g_counts[c].exchange(0);
    if (launches) launches[c] = n;
    if (total_ms) total_ms[c] = ms[c];
  }
  return WD_OK;
}

}  // extern "C"
