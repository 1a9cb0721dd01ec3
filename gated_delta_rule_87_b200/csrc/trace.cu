// Per-kernel device timing on the launching stream (optional).
//
// When enabled with kda_trace_enable(1), every kernel the library launches is
// bracketed by two CUDA events recorded on the caller's stream; the
// durations are read back by kda_trace_read().  Disabled (the default), the
// launch path records nothing.
#include <stdio.h>
#include <string.h>

#include <mutex>
#include <vector>

#include "gated_delta.h"
#include "internal.h"

namespace gdr {
namespace {

struct Record {
  const char *name;
  cudaEvent_t start, stop;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Record> g_records;
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

TraceScope::TraceScope(const char *name, cudaStream_t s) : name_(name), stream_(s) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  start_ = take_event();
  stop_ = take_event();
  if (start_ && stop_) cudaEventRecord(static_cast<cudaEvent_t>(start_), s);
  else start_ = stop_ = nullptr;
}

TraceScope::~TraceScope() {
  if (!start_ || !stop_) return;
  cudaEventRecord(static_cast<cudaEvent_t>(stop_), stream_);
  std::lock_guard<std::mutex> lk(g_mu);
  g_records.push_back({name_, static_cast<cudaEvent_t>(start_), static_cast<cudaEvent_t>(stop_)});
}

}  // namespace gdr

extern "C" {

kda_status_t kda_trace_enable(int32_t on) {
  std::lock_guard<std::mutex> lk(gdr::g_mu);
  gdr::g_on = (on != 0);
  return KDA_OK;
}

int32_t kda_trace_read(char *names, int32_t name_stride, float *ms, int32_t capacity) {
  std::vector<gdr::Record> recs;
  {
    std::lock_guard<std::mutex> lk(gdr::g_mu);
    recs.swap(gdr::g_records);
  }
  int32_t n = 0;
  for (const auto &r : recs) {
    float t = -1.f;
    if (cudaEventSynchronize(r.stop) == cudaSuccess) cudaEventElapsedTime(&t, r.start, r.stop);
    if (n < capacity) {
      if (names && name_stride > 0) {
        strncpy(names + (size_t)n * name_stride, r.name, (size_t)name_stride - 1);
        names[(size_t)n * name_stride + name_stride - 1] = '\0';
      }
      if (ms) ms[n] = t;
      ++n;
    }
  }
  std::lock_guard<std::mutex> lk(gdr::g_mu);
  for (const auto &r : recs) {
    gdr::g_free.push_back(r.start);
    gdr::g_free.push_back(r.stop);
  }
  return n;
}

}  // extern "C"
