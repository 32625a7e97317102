// Optional per-launch tracing: CUDA event pairs around each launcher call,
// tagged with a kernel class and the launch's algorithmic FLOPs / bytes.
#include <cuda_runtime.h>

#include <vector>

#include "trace.h"

struct gpt_trace {
  struct Rec {
    int cls;
    int nk;
    double flops, bytes;
  };
  std::vector<cudaEvent_t> ev;  // 2 per record
  std::vector<Rec> rec;
  int capacity = 0;
  int used = 0;
  int dropped = 0;
  int device = 0;
};

namespace gpt {

static thread_local gpt_trace* t_trace = nullptr;

TraceScope::TraceScope(int cls, int nkernels, double flops, double bytes, void* stream)
    : stream_(stream), slot_(-1) {
  gpt_trace* t = t_trace;
  if (!t) return;
  if (t->used >= t->capacity) {
    t->dropped++;
    return;
  }
  slot_ = t->used++;
  t->rec[slot_] = {cls, nkernels, flops, bytes};
  cudaEventRecord(t->ev[2 * slot_], static_cast<cudaStream_t>(stream_));
}

TraceScope::~TraceScope() {
  gpt_trace* t = t_trace;
  if (!t || slot_ < 0) return;
  cudaEventRecord(t->ev[2 * slot_ + 1], static_cast<cudaStream_t>(stream_));
}

}  // namespace gpt

extern "C" {

int gpt_trace_create(gpt_trace** out, int capacity) {
  if (!out || capacity <= 0) return GPT_EINVAL;
  gpt_trace* t = new gpt_trace();
  t->capacity = capacity;
  t->rec.resize(capacity);
  t->ev.resize(2 * size_t(capacity));
  cudaGetDevice(&t->device);
  for (auto& e : t->ev) {
    if (cudaEventCreate(&e) != cudaSuccess) {
      gpt_trace_destroy(t);
      return GPT_ECUDA;
    }
  }
  *out = t;
  return GPT_OK;
}

int gpt_trace_attach(gpt_trace* t) {
  gpt::t_trace = t;
  return GPT_OK;
}

int gpt_trace_reset(gpt_trace* t) {
  if (!t) return GPT_EINVAL;
  t->used = 0;
  t->dropped = 0;
  return GPT_OK;
}

int gpt_trace_summary(gpt_trace* t, gpt_trace_stat* stats, int32_t* dropped) {
  if (!t || !stats) return GPT_EINVAL;
  for (int c = 0; c < GPT_K_COUNT; ++c) stats[c] = gpt_trace_stat{0, 0, 0.0, 0.0, 0.0};
  for (int i = 0; i < t->used; ++i) {
    if (cudaEventSynchronize(t->ev[2 * i + 1]) != cudaSuccess) return GPT_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t->ev[2 * i], t->ev[2 * i + 1]) != cudaSuccess)
      return GPT_ECUDA;
    const auto& r = t->rec[i];
    gpt_trace_stat& s = stats[r.cls];
    s.launches += 1;
    s.kernels += r.nk;
    s.ms += ms;
    s.flops += r.flops;
    s.bytes += r.bytes;
  }
  if (dropped) *dropped = t->dropped;
  return GPT_OK;
}

int gpt_trace_records(gpt_trace* t, gpt_trace_record* out, int capacity, int32_t* count) {
  if (!t || (!out && capacity > 0) || !count) return GPT_EINVAL;
  int n = 0;
  for (int i = 0; i < t->used && n < capacity; ++i, ++n) {
    if (cudaEventSynchronize(t->ev[2 * i + 1]) != cudaSuccess) return GPT_ECUDA;
    float ms = 0.f;
    if (cudaEventElapsedTime(&ms, t->ev[2 * i], t->ev[2 * i + 1]) != cudaSuccess) return GPT_ECUDA;
    const auto& r = t->rec[i];
    out[n] = gpt_trace_record{r.cls, r.nk, ms, r.flops, r.bytes};
  }
  *count = n;
  return GPT_OK;
}

int gpt_trace_destroy(gpt_trace* t) {
  if (!t) return GPT_EINVAL;
  if (gpt::t_trace == t) gpt::t_trace = nullptr;
  for (auto& e : t->ev)
    if (e) cudaEventDestroy(e);
  delete t;
  return GPT_OK;
}

}  // extern "C"
