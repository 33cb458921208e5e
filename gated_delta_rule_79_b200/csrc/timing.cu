// Kernel timing for measurement: while enabled, every prefill call records a CUDA
// event on its stream when it starts and after each kernel it launches, so that a
// caller can split the time of a call among its kernels (the two-kernel paths
// launch a per-chunk prep kernel, then the state carry).  Recording is off unless
// gdr_timing_start() was called; it is process-wide and not meant for use inside
// stream capture.

#include <atomic>
#include <mutex>
#include <vector>

#include "gdr.h"
#include "launch.h"

namespace gdr {
namespace {

struct Mark {
  cudaEvent_t ev;
  int slot;   // -1: start of a call; i >= 0: end of the call's i-th kernel
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Mark> g_marks;

void clear_locked() {
  for (const Mark& m : g_marks) cudaEventDestroy(m.ev);
  g_marks.clear();
}

}  // namespace

void timing_mark(cudaStream_t stream, int slot) {
  if (!g_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on.load(std::memory_order_relaxed)) return;
  cudaEvent_t e;
  if (cudaEventCreate(&e) != cudaSuccess) return;
  if (cudaEventRecord(e, stream) != cudaSuccess) {
    cudaEventDestroy(e);
    return;
  }
  g_marks.push_back({e, slot});
}

}  // namespace gdr

extern "C" int gdr_timing_start(void) {
  std::lock_guard<std::mutex> lk(gdr::g_mu);
  gdr::clear_locked();
  gdr::g_on.store(true);
  return GDR_OK;
}

extern "C" int gdr_timing_stop(float* avg_ms, int max_kernels, int* ncalls) {
  std::lock_guard<std::mutex> lk(gdr::g_mu);
  gdr::g_on.store(false);
  constexpr int kMaxSlots = 8;
  double sum[kMaxSlots] = {0};
  int nslots = 0, calls = 0;
  bool ok = true;
  for (size_t i = 0; i < gdr::g_marks.size() && ok; ++i) {
    const gdr::Mark& m = gdr::g_marks[i];
    if (m.slot < 0) {
      ++calls;
      continue;
    }
    if (i == 0 || m.slot >= kMaxSlots) continue;
    float ms = 0.f;
    ok = cudaEventSynchronize(m.ev) == cudaSuccess &&
         cudaEventElapsedTime(&ms, gdr::g_marks[i - 1].ev, m.ev) == cudaSuccess;
    sum[m.slot] += ms;
    if (m.slot + 1 > nslots) nslots = m.slot + 1;
  }
  gdr::clear_locked();
  if (!ok) return -1;
  if (ncalls) *ncalls = calls;
  for (int s = 0; s < nslots && s < max_kernels && avg_ms; ++s)
    avg_ms[s] = calls ? (float)(sum[s] / calls) : 0.f;
  return nslots;
}
