// Per-stage launch accounting and optional CUDA-event timing of every kernel
// the library launches (the measurement hook behind am_profile_*).
#include "am_internal.cuh"
#include "am_profile.cuh"

#include <atomic>
#include <mutex>
#include <vector>

namespace am {
namespace {

struct Rec {
  int stage;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_enabled = false;
std::vector<Rec> g_recs;
std::vector<cudaEvent_t> g_pool;
std::atomic<int64_t> g_launches{0};

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

}  // namespace

ProfScope::ProfScope(int stage, cudaStream_t s) : stage_(stage), s_(s), a_(nullptr) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (g_enabled) {
    a_ = take_event();
    if (a_) cudaEventRecord(a_, s_);
  }
}

ProfScope::~ProfScope() {
  g_launches.fetch_add(1);
  std::lock_guard<std::mutex> lk(g_mu);
  if (a_) {
    cudaEvent_t b = take_event();
    if (b) {
      cudaEventRecord(b, s_);
      g_recs.push_back({stage_, a_, b});
    } else {
      g_pool.push_back(a_);
    }
  }
}

}  // namespace am

using namespace am;

extern "C" {

am_status_t am_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_enabled = on != 0;
  return AM_OK;
}

am_status_t am_profile_collect(double* ms, int64_t* launches) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (ms)
    for (int k = 0; k < AM_STAGE_COUNT; ++k) ms[k] = 0.0;
  if (launches)
    for (int k = 0; k < AM_STAGE_COUNT; ++k) launches[k] = 0;
  am_status_t st = AM_OK;
  for (const Rec& r : g_recs) {
    float t = 0.f;
    if (cudaEventSynchronize(r.b) != cudaSuccess || cudaEventElapsedTime(&t, r.a, r.b) != cudaSuccess)
      st = AM_ERR_CUDA;
    if (ms && r.stage >= 0 && r.stage < AM_STAGE_COUNT) ms[r.stage] += t;
    if (launches && r.stage >= 0 && r.stage < AM_STAGE_COUNT) launches[r.stage] += 1;
    g_pool.push_back(r.a);
    g_pool.push_back(r.b);
  }
  g_recs.clear();
  return st;
}

int64_t am_kernel_launches(void) { return g_launches.load(); }

}  // extern "C"
