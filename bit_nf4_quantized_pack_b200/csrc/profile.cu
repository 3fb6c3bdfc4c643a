// Launch timing for measurement tools: when enabled, every kernel launch of
// the library is bracketed by a pair of CUDA events recorded on the stream it
// is launched on.  qlora_profile_read sums the elapsed times per kernel class.
#include <cuda_runtime.h>

#include <mutex>
#include <vector>

#include "profile.cuh"
#include "qlora_nf4.h"

namespace qnf4 {
namespace {

struct Pair {
  int id;
  cudaEvent_t a, b;
};

std::mutex g_mu;
bool g_on = false;
unsigned int g_mask = 0xFFFFFFFFu;
std::vector<Pair> g_pending;
std::vector<cudaEvent_t> g_free;
long long g_launches[kProfKinds] = {0};
long long g_total_launches = 0;
double g_ms[kProfKinds] = {0};

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

ProfScope::ProfScope(int id, cudaStream_t s) : id_(id), s_(s), a_(nullptr) {
  std::lock_guard<std::mutex> g(g_mu);
  ++g_total_launches;
  if (id_ >= 0 && id_ < kProfKinds) ++g_launches[id_];
  if (!g_on || id_ < 0 || id_ >= 32 || !((g_mask >> id_) & 1u)) return;
  a_ = take_event();
  if (a_) cudaEventRecord(static_cast<cudaEvent_t>(a_), s_);
}

ProfScope::~ProfScope() {
  std::lock_guard<std::mutex> g(g_mu);
  if (!g_on || !a_) return;
  cudaEvent_t b = take_event();
  if (!b) return;
  cudaEventRecord(b, s_);
  g_pending.push_back(Pair{id_, static_cast<cudaEvent_t>(a_), b});
}

bool prof_timing(int id) {
  std::lock_guard<std::mutex> g(g_mu);
  return g_on && id >= 0 && id < 32 && ((g_mask >> id) & 1u);
}

void prof_count_only(int id) {
  std::lock_guard<std::mutex> g(g_mu);
  ++g_total_launches;
  if (id >= 0 && id < kProfKinds) ++g_launches[id];
}

}  // namespace qnf4

extern "C" {

qlora_status qlora_profile_enable(int32_t on) {
  std::lock_guard<std::mutex> g(qnf4::g_mu);
  qnf4::g_on = on != 0;
  return QLORA_OK;
}

qlora_status qlora_profile_select(uint32_t kinds_mask) {
  std::lock_guard<std::mutex> g(qnf4::g_mu);
  qnf4::g_mask = kinds_mask;
  return QLORA_OK;
}

qlora_status qlora_profile_read(int32_t kind, double* total_ms, int64_t* launches) {
  if (kind < -1 || kind >= qnf4::kProfKinds || !total_ms || !launches) return QLORA_ERR_INVALID_ARG;
  std::lock_guard<std::mutex> g(qnf4::g_mu);
  for (auto& p : qnf4::g_pending) {
    if (cudaEventSynchronize(p.b) != cudaSuccess) return QLORA_ERR_CUDA;
    float ms = 0.0f;
    if (cudaEventElapsedTime(&ms, p.a, p.b) != cudaSuccess) return QLORA_ERR_CUDA;
    qnf4::g_ms[p.id] += ms;
    qnf4::g_free.push_back(p.a);
    qnf4::g_free.push_back(p.b);
  }
  qnf4::g_pending.clear();
  if (kind == -1) {
    double t = 0;
    for (int i = 0; i < qnf4::kProfKinds; ++i) t += qnf4::g_ms[i];
    *total_ms = t;
    *launches = qnf4::g_total_launches;
  } else {
    *total_ms = qnf4::g_ms[kind];
    *launches = qnf4::g_launches[kind];
  }
  return QLORA_OK;
}

qlora_status qlora_profile_reset(void) {
  std::lock_guard<std::mutex> g(qnf4::g_mu);
  for (int i = 0; i < qnf4::kProfKinds; ++i) {
    qnf4::g_ms[i] = 0;
    qnf4::g_launches[i] = 0;
  }
  qnf4::g_total_launches = 0;
  return QLORA_OK;
}

}  // extern "C"
