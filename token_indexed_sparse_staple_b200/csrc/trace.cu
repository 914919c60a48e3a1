// Per-kernel timing for a context: when enabled, every kernel the library
// launches on behalf of an entry point is bracketed by a pair of CUDA events
// recorded on the launch stream; staple_trace_read turns them into
// (kernel name, milliseconds) records.  Off by default: no events, no cost.
#include <cuda_runtime.h>

#include <cstring>
#include <mutex>
#include <vector>

#include "internal.h"

namespace stp {

struct Tracer {
  std::mutex mu;
  bool enabled = false;
  int device = 0;
  std::vector<cudaEvent_t> ev;       // 2 per record
  std::vector<const char*> names;
  int used = 0;                      // records in use
  int dropped = 0;
};

static thread_local Tracer* t_current = nullptr;

// Inside stream capture an event must be recorded as an external node to be
// recorded (and timed) on every replay of the graph; outside capture a plain
// record is used.
static cudaError_t record(cudaEvent_t e, cudaStream_t st) {
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  if (cudaStreamIsCapturing(st, &cap) != cudaSuccess) return cudaErrorUnknown;
  return cap == cudaStreamCaptureStatusActive
             ? cudaEventRecordWithFlags(e, st, cudaEventRecordExternal)
             : cudaEventRecord(e, st);
}

Tracer* tracer_create(int device) {
  Tracer* t = new Tracer();
  t->device = device;
  return t;
}

void tracer_destroy(Tracer* t) {
  if (!t) return;
  for (cudaEvent_t e : t->ev) cudaEventDestroy(e);
  delete t;
}

bool tracer_enable(Tracer* t, bool on) {
  std::lock_guard<std::mutex> g(t->mu);
  if (on && t->ev.empty()) {
    t->ev.resize(2 * kTraceCapacity);
    t->names.resize(kTraceCapacity);
    for (auto& e : t->ev)
      if (cudaEventCreate(&e) != cudaSuccess) return false;
  }
  t->enabled = on;
  t->used = 0;
  t->dropped = 0;
  return true;
}

TraceScope::TraceScope(Tracer* t) : prev(t_current) { t_current = t; }
TraceScope::~TraceScope() { t_current = prev; }

int trace_begin(const char* name, cudaStream_t st) {
  Tracer* t = t_current;
  if (!t || !t->enabled) return -1;
  std::lock_guard<std::mutex> g(t->mu);
  if (t->used >= kTraceCapacity) {
    ++t->dropped;
    return -1;
  }
  const int i = t->used++;
  t->names[i] = name;
  if (record(t->ev[2 * i], st) != cudaSuccess) {
    cudaGetLastError();
    t->names[i] = nullptr;
  }
  return i;
}

void trace_end(int slot, cudaStream_t st) {
  Tracer* t = t_current;
  if (!t || slot < 0) return;
  if (record(t->ev[2 * slot + 1], st) != cudaSuccess) {
    cudaGetLastError();
    t->names[slot] = nullptr;
  }
}

int tracer_read(Tracer* t, staple_trace_record* out, int cap, int* dropped) {
  std::lock_guard<std::mutex> g(t->mu);
  const int n = t->used < cap ? t->used : cap;
  for (int i = 0; i < n; ++i) {
    float ms = -1.0f;
    if (t->names[i] == nullptr ||
        cudaEventSynchronize(t->ev[2 * i + 1]) != cudaSuccess ||
        cudaEventElapsedTime(&ms, t->ev[2 * i], t->ev[2 * i + 1]) != cudaSuccess) {
      cudaGetLastError();  // leave no stale error behind for the next launch check
      ms = -1.0f;
    }
    std::memset(out[i].kernel, 0, sizeof(out[i].kernel));
    std::strncpy(out[i].kernel, t->names[i] ? t->names[i] : "?", sizeof(out[i].kernel) - 1);
    out[i].ms = ms;
  }
  if (dropped) *dropped = t->dropped + (t->used - n);
  t->used = 0;
  t->dropped = 0;
  return n;
}

}  // namespace stp
