// Per-kernel tracing hooks (see trace.cu).
#pragma once
#include <cuda_runtime.h>

namespace hstu {
bool trace_on();
int trace_begin(const char* name, cudaStream_t st);
void trace_end(int handle, cudaStream_t st);

struct TraceScope {
  int h;
  cudaStream_t st;
  TraceScope(const char* name, cudaStream_t s) : h(trace_on() ? trace_begin(name, s) : -1), st(s) {}
  ~TraceScope() { trace_end(h, st); }
};
}  // namespace hstu
