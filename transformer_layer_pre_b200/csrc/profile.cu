// profile.cu — launch counter and event-pair timing of kernel classes.
#include <atomic>
#include <mutex>
#include <vector>

#include "../../include/tlp.h"
#include "profile.h"

namespace tlp {

namespace {

std::atomic<long long> g_launches{0};
std::atomic<int> g_enabled{0};
std::mutex g_mu;

struct Pair {
  cudaEvent_t a = nullptr, b = nullptr;
  int cls = 0;
};
std::vector<Pair> g_pairs;  // events are created once and reused
size_t g_used = 0;

}  // namespace

void count_launch(int n) { g_launches.fetch_add(n, std::memory_order_relaxed); }

ProfScope::ProfScope(int cls, cudaStream_t s) : slot_(-1), s_(s) {
  if (!g_enabled.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_used == g_pairs.size()) {
    Pair p;
    if (cudaEventCreate(&p.a) != cudaSuccess || cudaEventCreate(&p.b) != cudaSuccess) return;
    g_pairs.push_back(p);
  }
  slot_ = (int)g_used++;
  g_pairs[slot_].cls = cls;
  cudaEventRecord(g_pairs[slot_].a, s);
}

ProfScope::~ProfScope() {
  if (slot_ < 0) return;
  cudaEventRecord(g_pairs[slot_].b, s_);
}

}  // namespace tlp

using namespace tlp;

extern "C" {

void tl_profile_enable(int on) { g_enabled.store(on ? 1 : 0); }

int tl_profile_read(double* ms, long long* launches, int n) {
  std::lock_guard<std::mutex> lk(g_mu);
  cudaDeviceSynchronize();
  for (int c = 0; c < n && c < PC_COUNT; ++c) {
    if (ms) ms[c] = 0.0;
    if (launches) launches[c] = 0;
  }
  for (size_t i = 0; i < g_used; ++i) {
    const int c = g_pairs[i].cls;
    float t = 0.0f;
    if (c < n && cudaEventElapsedTime(&t, g_pairs[i].a, g_pairs[i].b) == cudaSuccess) {
      if (ms) ms[c] += t;
      if (launches) launches[c] += 1;
    }
  }
  g_used = 0;
  return PC_COUNT;
}

long long tl_launch_count(void) { return g_launches.load(); }

}  // extern "C"
