// Optional per-kernel timing: when enabled, every kernel launch of the
// library is bracketed by two CUDA events recorded on its own stream; reading
// the trace waits for those events and returns launches and total device
// milliseconds per kernel name.  Off by default (one branch per launch).
#include <atomic>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "common.cuh"

namespace vmoba {
namespace {

struct Pending {
  const char* name;
  cudaEvent_t a, b;
};

std::atomic<bool> g_on{false};
std::mutex g_mu;
std::vector<Pending> g_pending;
std::vector<cudaEvent_t> g_free;

cudaEvent_t take_event() {
  if (!g_free.empty()) {
    cudaEvent_t e = g_free.back();
    g_free.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
  return e;
}

}  // namespace

TraceScope::TraceScope(const char* name, cudaStream_t st) : stream_(st), a_(nullptr) {
  if (!g_on.load(std::memory_order_relaxed)) return;
  std::lock_guard<std::mutex> lock(g_mu);
  a_ = take_event();
  name_ = name;
  if (a_) cudaEventRecord(static_cast<cudaEvent_t>(a_), st);
}

TraceScope::~TraceScope() {
  if (!a_) return;
  std::lock_guard<std::mutex> lock(g_mu);
  cudaEvent_t b = take_event();
  if (!b) {
    g_free.push_back(static_cast<cudaEvent_t>(a_));
    return;
  }
  cudaEventRecord(b, stream_);
  g_pending.push_back(Pending{name_, static_cast<cudaEvent_t>(a_), b});
}

}  // namespace vmoba

extern "C" {

int vmoba_trace_enable(int on) {
  vmoba::g_on.store(on != 0);
  return VMOBA_OK;
}

int vmoba_trace_read(vmoba_trace_entry* out, int max_entries) {
  using namespace vmoba;
  std::lock_guard<std::mutex> lock(g_mu);
  std::map<std::string, std::pair<int, double>> acc;
  for (const Pending& p : g_pending) {
    float ms = 0.f;
    if (cudaEventSynchronize(p.b) == cudaSuccess && cudaEventElapsedTime(&ms, p.a, p.b) == cudaSuccess) {
      auto& e = acc[p.name];
      e.first += 1;
      e.second += ms;
    }
    g_free.push_back(p.a);
    g_free.push_back(p.b);
  }
  g_pending.clear();
  int n = 0;
  for (const auto& kv : acc) {
    if (out && n < max_entries) {
      std::memset(out[n].name, 0, sizeof(out[n].name));
      std::strncpy(out[n].name, kv.first.c_str(), sizeof(out[n].name) - 1);
      out[n].launches = kv.second.first;
      out[n].ms = kv.second.second;
    }
    ++n;
  }
  return n;
}

}  // extern "C"
