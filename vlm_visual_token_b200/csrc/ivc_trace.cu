// ivc_trace.cu — optional per-kernel timing of the library's launches.
//
// When tracing is on (ivc_trace_enable(1)), every kernel launch of the hot
// path is bracketed by two CUDA events on its stream and filed under its
// role ("mlp1.fc1", "pool.kv", "pool.attention", ...). ivc_trace_report()
// waits for the recorded events and returns, per role, the launch count and
// the summed device time. Off by default; when off a launch costs one branch.
#include <cuda_runtime.h>

#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "ivc_internal.h"

namespace ivc {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t a, b;
};

struct TraceState {
  std::mutex mu;
  bool on = false;
  std::vector<cudaEvent_t> pool;  // reusable events
  std::vector<Rec> recs;
  size_t used = 0;                // events handed out from `pool`
};

TraceState& st() {
  static TraceState s;
  return s;
}

cudaEvent_t take_event(TraceState& s) {
  if (s.used == s.pool.size()) {
    cudaEvent_t e;
    if (cudaEventCreate(&e) != cudaSuccess) return nullptr;
    s.pool.push_back(e);
  }
  return s.pool[s.used++];
}

}  // namespace

TraceScope::TraceScope(const char* name, cudaStream_t s) : stream_(s), active_(false) {
  TraceState& t = st();
  if (!t.on) return;
  std::lock_guard<std::mutex> g(t.mu);
  cudaEvent_t a = take_event(t), b = take_event(t);
  if (!a || !b) return;
  t.recs.push_back({name, a, b});
  idx_ = t.recs.size() - 1;
  cudaEventRecord(a, s);
  active_ = true;
}

TraceScope::~TraceScope() {
  if (!active_) return;
  TraceState& t = st();
  std::lock_guard<std::mutex> g(t.mu);
  cudaEventRecord(t.recs[idx_].b, stream_);
}

}  // namespace ivc

extern "C" {

int ivc_trace_enable(int on) {
  ivc::TraceState& t = ivc::st();
  std::lock_guard<std::mutex> g(t.mu);
  t.on = on != 0;
  return IVC_OK;
}

int ivc_trace_reset(void) {
  ivc::TraceState& t = ivc::st();
  std::lock_guard<std::mutex> g(t.mu);
  t.recs.clear();
  t.used = 0;
  return IVC_OK;
}

int ivc_trace_report(char* buf, size_t n) {
  ivc::TraceState& t = ivc::st();
  std::lock_guard<std::mutex> g(t.mu);
  std::map<std::string, std::pair<long long, double>> agg;
  std::vector<std::string> order;
  for (const auto& r : t.recs) {
    if (cudaEventSynchronize(r.b) != cudaSuccess) return IVC_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, r.a, r.b) != cudaSuccess) return IVC_ECUDA;
    auto it = agg.find(r.name);
    if (it == agg.end()) {
      order.push_back(r.name);
      agg[r.name] = {1, ms};
    } else {
      it->second.first += 1;
      it->second.second += ms;
    }
  }
  std::string out = "{";
  char tmp[256];
  for (size_t i = 0; i < order.size(); ++i) {
    const auto& v = agg[order[i]];
    std::snprintf(tmp, sizeof(tmp), "%s\"%s\": {\"launches\": %lld, \"ms\": %.6f}",
                  i ? ", " : "", order[i].c_str(), v.first, v.second);
    out += tmp;
  }
  out += "}";
  if (!buf || n < out.size() + 1) return IVC_EINVAL;
  std::memcpy(buf, out.c_str(), out.size() + 1);
  return IVC_OK;
}

}  // extern "C"
