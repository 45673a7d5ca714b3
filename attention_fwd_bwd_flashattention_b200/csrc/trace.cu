// Tracing of the library's kernel launches: an NVTX range around each launch (visible
// to any NVTX-aware profiler, free when none is attached) and, for callers that ask for
// it, a pair of CUDA events recorded on the launch stream around each kernel, so that
// one kernel of a pass can be timed on the device without a profiler.  The events are
// the caller's; the registration is per host thread, so calls made from other threads
// are not traced and no state is shared between threads.
#include <string.h>

#include <cuda_runtime.h>
#include <nvtx3/nvToolsExt.h>

#include "relpos_attn.h"
#include "kernels.h"

namespace rp {

static thread_local relpos_trace_t *t_trace = nullptr;

void trace_pre(const char *name, cudaStream_t st) {
  nvtxRangePushA(name);
  relpos_trace_t *t = t_trace;
  if (!t || (t->only && strcmp(t->only, name) != 0)) return;
  if (t->count >= t->capacity) {
    ++t->dropped;
    return;
  }
  t->names[t->count] = name;
  cudaEventRecord((cudaEvent_t)t->events[2 * t->count], st);
}

void trace_post(cudaStream_t st) {
  nvtxRangePop();
  relpos_trace_t *t = t_trace;
  // the kernel just launched was recorded by trace_pre iff its slot holds a name
  if (!t || t->count >= t->capacity || t->names[t->count] == nullptr) return;
  cudaEventRecord((cudaEvent_t)t->events[2 * t->count + 1], st);
  ++t->count;
}

}  // namespace rp

extern "C" int relpos_trace_begin(relpos_trace_t *trace) {
  if (!trace || !trace->events || trace->capacity < 1 || trace->capacity > RELPOS_TRACE_MAX) return RELPOS_ERR_INVALID_ARG;
  for (int k = 0; k < 2 * trace->capacity; ++k)
    if (!trace->events[k]) return RELPOS_ERR_INVALID_ARG;
  trace->count = 0;
  trace->dropped = 0;
  for (int k = 0; k < RELPOS_TRACE_MAX; ++k) trace->names[k] = nullptr;
  rp::t_trace = trace;
  return RELPOS_OK;
}

extern "C" int relpos_trace_end(void) {
  rp::t_trace = nullptr;
  return RELPOS_OK;
}
