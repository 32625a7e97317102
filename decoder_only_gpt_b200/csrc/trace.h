// RAII launch tracing used by the step orchestration (see gpt_trace_* in gpt.h).
#pragma once

#include "gpt.h"

namespace gpt {

// Records an event pair around its scope when a trace is attached to the
// calling thread; does nothing otherwise.
class TraceScope {
 public:
  TraceScope(int cls, int nkernels, double flops, double bytes, void* stream);
  ~TraceScope();
  TraceScope(const TraceScope&) = delete;
  TraceScope& operator=(const TraceScope&) = delete;

 private:
  void* stream_;
  int slot_;
};

}  // namespace gpt
