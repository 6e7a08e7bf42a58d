// qlora_prof.cu -- launch counting and optional per-kernel-class device timing.
//
// Every kernel launch of the library goes through a ProfScope: the launch is
// counted per kernel class, and, while timing is enabled, bracketed by two
// CUDA events on the launching stream.  qlora_profile_read() waits for the
// recorded events, sums their elapsed times per class and resets.  Event
// objects are pooled and reused, so steady-state timing allocates nothing.
#include <atomic>
#include <mutex>
#include <vector>

#include "qlora_internal.h"

namespace qlora {

namespace {
struct Pending {
  int kc;
  cudaEvent_t a, b;
};
std::mutex g_mu;
std::atomic<int> g_enabled{0};
std::atomic<long long> g_launches[QLORA_KC_COUNT];
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_pool;

cudaEvent_t take_event() {
  if (!g_pool.empty()) {
    cudaEvent_t e = g_pool.back();
    g_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) {
    cudaGetLastError();
    return nullptr;
  }
  return e;
}
}  // namespace

ProfScope::ProfScope(int kc_, cudaStream_t st_) : kc(kc_), st(st_), a(nullptr) {
  g_launches[kc].fetch_add(1, std::memory_order_relaxed);
  if (!g_enabled.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  a = take_event();
  if (a) cudaEventRecord(static_cast<cudaEvent_t>(a), st);
}

ProfScope::~ProfScope() {
  if (!a) return;
  std::lock_guard<std::mutex> lk(g_mu);
  cudaEvent_t b = take_event();
  if (!b) {
    g_pool.push_back(static_cast<cudaEvent_t>(a));
    return;
  }
  cudaEventRecord(b, st);
  g_pending.push_back({kc, static_cast<cudaEvent_t>(a), b});
}

}  // namespace qlora

using namespace qlora;

extern "C" int qlora_profile_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_enabled.store(on ? 1 : 0);
  return QLORA_OK;
}

extern "C" int qlora_profile_read(double ms[QLORA_KC_COUNT], int64_t launches[QLORA_KC_COUNT]) {
  std::lock_guard<std::mutex> lk(g_mu);
  int rc = QLORA_OK;
  if (ms)
    for (int i = 0; i < QLORA_KC_COUNT; ++i) ms[i] = 0.0;
  for (const Pending& p : g_pending) {
    float t = 0.0f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&t, p.a, p.b) == cudaSuccess) {
      if (ms) ms[p.kc] += t;
    } else {
      cudaGetLastError();
      rc = QLORA_ERR_CUDA;
    }
    g_pool.push_back(p.a);
    g_pool.push_back(p.b);
  }
  g_pending.clear();
  for (int i = 0; i < QLORA_KC_COUNT; ++i) {
    const long long n = g_launches[i].exchange(0);
    if (launches) launches[i] = n;
  }
  return rc;
}
