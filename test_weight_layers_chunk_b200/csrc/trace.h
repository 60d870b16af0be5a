// Opt-in launch tracing: a CUDA event pair around every kernel the library
// launches, recorded on the launch stream, summarised per kernel name.
#pragma once
#include <cuda_runtime.h>

namespace e2ttt {

void trace_begin(const char* name, cudaStream_t st);
void trace_end(cudaStream_t st);

struct TraceScope {
  cudaStream_t st;
  TraceScope(const char* name, cudaStream_t s) : st(s) { trace_begin(name, s); }
  ~TraceScope() { trace_end(st); }
};

}  // namespace e2ttt

#define E2TTT_TRACE(name, st) ::e2ttt::TraceScope _e2ttt_trace_scope_(name, st)
