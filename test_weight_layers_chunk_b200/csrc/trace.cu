// Launch tracing (see trace.h) and its C ABI.
#include <stdio.h>

#include <map>
#include <mutex>
#include <string>
#include <vector>

#include "../../include/e2ttt.h"
#include "trace.h"

namespace e2ttt {
namespace {

struct Rec {
  const char* name;
  cudaEvent_t beg, end;
};

std::mutex g_mu;
bool g_on = false;
std::vector<Rec> g_recs;          // recorded since the last reset
std::vector<cudaEvent_t> g_pool;  // events free for reuse
std::string g_summary;

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

void recycle_all() {
  for (Rec& r : g_recs) {
    if (r.beg) g_pool.push_back(r.beg);
    if (r.end) g_pool.push_back(r.end);
  }
  g_recs.clear();
}

}  // namespace

void trace_begin(const char* name, cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on) return;
  Rec r{name, take_event(), nullptr};
  if (r.beg) cudaEventRecord(r.beg, st);
  g_recs.push_back(r);
}

void trace_end(cudaStream_t st) {
  std::lock_guard<std::mutex> lk(g_mu);
  if (!g_on || g_recs.empty() || g_recs.back().end) return;
  Rec& r = g_recs.back();
  r.end = take_event();
  if (r.end) cudaEventRecord(r.end, st);
}

}  // namespace e2ttt

using namespace e2ttt;

extern "C" {

void e2ttt_trace_enable(int on) {
  std::lock_guard<std::mutex> lk(g_mu);
  g_on = on != 0;
  recycle_all();
}

const char* e2ttt_trace_summary(void) {
  std::lock_guard<std::mutex> lk(g_mu);
  std::map<std::string, std::pair<long, double>> agg;
  long launches = 0;
  for (const Rec& r : g_recs) {
    float ms = 0.f;
    if (r.beg && r.end && cudaEventSynchronize(r.end) == cudaSuccess &&
        cudaEventElapsedTime(&ms, r.beg, r.end) == cudaSuccess) {
      auto& a = agg[r.name];
      a.first += 1;
      a.second += ms;
      ++launches;
    }
  }
  std::string s = "{\"launches\": " + std::to_string(launches) + ", \"kernels\": {";
  bool first = true;
  for (auto& kv : agg) {
    char buf[256];
    snprintf(buf, sizeof(buf), "%s\"%s\": {\"launches\": %ld, \"total_ms\": %.6f}",
             first ? "" : ", ", kv.first.c_str(), kv.second.first, kv.second.second);
    s += buf;
    first = false;
  }
  s += "}}";
  g_summary = s;
  recycle_all();
  return g_summary.c_str();
}

}  // extern "C"
