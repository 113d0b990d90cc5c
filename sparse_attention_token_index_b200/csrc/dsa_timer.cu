// dsa_timer.cu — optional timing of the scoring kernel's launches.
//
// When armed by dsa_kernel_timer_start, the launchers of the scoring kernels
// (tensor-core and fp32 CUDA-core) record a CUDA event pair on the caller's
// stream around each launch, up to the armed number of launches.  The events
// are created when the timer is armed, so the timed calls themselves create
// nothing; while disarmed a launch pays one relaxed atomic load.
#include <atomic>
#include <mutex>
#include <vector>

#include "dsa_common.cuh"
#include "dsa_internal.h"

namespace dsa {
namespace {

std::mutex g_mu;
std::atomic<bool> g_armed{false};
std::vector<cudaEvent_t> g_ev;  // 2 per launch: start, end
int g_cap = 0;
int g_used = 0;

void destroy_events() {
  for (cudaEvent_t e : g_ev) cudaEventDestroy(e);
  g_ev.clear();
  g_cap = g_used = 0;
}

}  // namespace

TimerSlot timer_acquire() {
  TimerSlot s;
  if (!g_armed.load(std::memory_order_relaxed)) return s;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_armed.load(std::memory_order_relaxed) || g_used >= g_cap) return s;
  s.start = g_ev[2 * g_used];
  s.end = g_ev[2 * g_used + 1];
  ++g_used;
  return s;
}

}  // namespace dsa

extern "C" int dsa_kernel_timer_start(int max_launches) {
  using namespace dsa;
  if (max_launches < 1 || max_launches > (1 << 20)) return DSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  if (g_armed.load()) return DSA_ERR_INVALID_ARG;
  g_ev.assign(2 * (size_t)max_launches, nullptr);
  for (cudaEvent_t& e : g_ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      e = nullptr;
      for (cudaEvent_t& f : g_ev)
        if (f) cudaEventDestroy(f);
      g_ev.clear();
      return DSA_ERR_CUDA;
    }
  }
  g_cap = max_launches;
  g_used = 0;
  g_armed.store(true);
  return DSA_OK;
}

extern "C" int dsa_kernel_timer_stop(float* total_ms, int* launches) {
  using namespace dsa;
  if (!total_ms || !launches) return DSA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> lock(g_mu);
  if (!g_armed.load()) return DSA_ERR_INVALID_ARG;
  g_armed.store(false);
  double sum = 0.0;
  int r = DSA_OK;
  for (int i = 0; i < g_used && r == DSA_OK; ++i) {
    float ms = 0.f;
    if (cudaEventSynchronize(g_ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, g_ev[2 * i], g_ev[2 * i + 1]) != cudaSuccess)
      r = DSA_ERR_CUDA;
    sum += ms;
  }
  *total_ms = (float)sum;
  *launches = g_used;
  destroy_events();
  return r;
}
