// Launchers shared between the translation units of libstaple (not part of
// the public ABI).
#pragma once

#include <cuda_runtime.h>
#include <stdint.h>

#include "../../include/staple.h"

namespace stp {

constexpr int kMaxDedupT = 32768;  // one-block dedup keeps the batch in shared memory
constexpr int kSegChunk = 64;      // sorted positions per block in the dE reduction
// Kernel waits: default and largest bound (staple_set_wait_limit), in ns.
constexpr uint64_t kWaitLimitNs = 4000000000ull;
constexpr int64_t kMaxWaitLimitNs = 60000000000ll;

struct DeviceInfo {
  int device;
  int num_sms;
  uint64_t wait_ns;   // bound of every kernel wait (staple_set_wait_limit)
  int sm_reserve;     // SMs the persistent GEMMs leave free (staple_set_sm_reserve)
};

// trace.cu: optional per-kernel CUDA-event timing of a context
constexpr int kTraceCapacity = 1 << 16;
struct Tracer;
Tracer* tracer_create(int device);
void tracer_destroy(Tracer* t);
bool tracer_enable(Tracer* t, bool on);
int tracer_read(Tracer* t, staple_trace_record* out, int cap, int* dropped);
int trace_begin(const char* name, cudaStream_t st);   // -1 when tracing is off
void trace_end(int slot, cudaStream_t st);
struct TraceScope {                                   // makes a tracer current for one API call
  explicit TraceScope(Tracer* t);
  ~TraceScope();
  Tracer* prev;
};
#define STP_LAUNCH(name, st, ...)                     \
  do {                                                \
    const int _slot = ::stp::trace_begin(name, st);   \
    __VA_ARGS__;                                      \
    ::stp::trace_end(_slot, st);                      \
  } while (0)

// retrieval.cu
staple_status launch_dedup(const int32_t* ids, int T, int64_t V, int32_t* unique,
                           int32_t* inverse, int32_t* seg_off, int32_t* sorted_pos,
                           int32_t* U_dev, int32_t* err, cudaStream_t st);
staple_status launch_probe(const int32_t* unique, const int32_t* U_dev, const int32_t* hkeys,
                           const int32_t* hvals, uint32_t hmask, int32_t* slot,
                           int32_t* miss_list, int32_t* miss_count, cudaStream_t st);
staple_status launch_gather_hits(const void* cache_rows, int64_t row_bytes, const int32_t* U_dev,
                                 const int32_t* slot, void* rows, int num_sms, cudaStream_t st);
staple_status launch_gather_misses(const void* table_dev, int64_t table_pitch_bytes,
                                   int64_t row_bytes, const int32_t* unique,
                                   const int32_t* miss_list, const int32_t* miss_count,
                                   void* rows, int num_sms, bool host_table, cudaStream_t st);
staple_status launch_cache_fill(const int32_t* hot, int K, int32_t* hkeys, int32_t* hvals,
                                uint32_t hmask, cudaStream_t st);
staple_status launch_scatter_misses(const void* staging, int64_t row_bytes,
                                    const int32_t* miss_list, const int32_t* miss_count,
                                    void* rows, int num_sms, cudaStream_t st);
staple_status launch_cache_refresh(const void* table_dev, int64_t table_pitch_bytes,
                                   int64_t row_bytes, const int32_t* unique, const int32_t* slot,
                                   const int32_t* U_dev, void* cache_rows, int num_sms,
                                   cudaStream_t st);
staple_status launch_copy_rows(const void* table_dev, int64_t table_pitch_bytes,
                               int64_t row_bytes, const int32_t* ids, const int32_t* count_dev,
                               void* dst, int num_sms, cudaStream_t st);

// embed_grad.cu
// k8 scratch: the partial pieces (seg_reduce_workspace bytes, after the
// workspace's counter head) and the crossing-segment counters
// (seg_counter_bytes, in the counter head after the decode flags; zero before
// the first call and zero again after every call)
size_t seg_reduce_workspace(int T, int F);
size_t seg_counter_bytes(int T, int F);
staple_status launch_seg_reduce(bool bf16, const void* dh, int64_t ld, const int32_t* sorted_pos,
                                const int32_t* inverse, const int32_t* seg_off,
                                const int32_t* U_dev, int T, int F, float* dE, float* part,
                                int32_t* counters, cudaStream_t st);
staple_status launch_grad_to_host(const float* dE, const int32_t* unique, const int32_t* U_dev,
                                  int F, int cap, float* host_dE, int32_t* host_unique,
                                  int32_t* host_U, int num_sms, cudaStream_t st);

// ffn_tc.cu (bf16, tcgen05)
staple_status tc_ffn_fwd(const DeviceInfo& di, int T, int D, int F, const void* x,
                         const staple_embed* e, const void* wg, const void* wu, const void* wd,
                         void* z, void* y, void* g_save, void* h_save, int32_t* err,
                         cudaStream_t st);
staple_status tc_dz(const DeviceInfo& di, int T, int D, int F, const void* dy, const void* g_save,
                    const void* h_save, const void* wd, void* dgh, int32_t* err, cudaStream_t st);
staple_status tc_ffn_bwd(const DeviceInfo& di, int T, int D, int F, const void* dy,
                         const void* x, const void* z, const void* dgh, const void* wg,
                         const void* wu, void* dx, float* dwg, float* dwu, float* dwd,
                         int32_t* err, cudaStream_t st);

// decode path (ffn_tc.cu): 1 <= T <= kMaxDecodeT tokens, bf16
constexpr int kMaxDecodeT = 256;
constexpr int kMaxDecodeGrid = 160;   // blocks of the persistent decode kernel (<= one per SM)
// Workspace layout: [decode counters, decode_counter_bytes(D, F), zero-filled
// once by the caller and left at zero by every call][shared scratch].
// The workspace's counter head: the decode kernel's flags
// (decode_flag_bytes), then the table-gradient counters for up to kMaxDedupT
// tokens.  Left untouched by everything else.
size_t decode_flag_bytes(int D, int F);
size_t decode_counter_bytes(int D, int F);
size_t decode_scratch_bytes(int T, int D, int F);
staple_status tc_decode_fwd(const DeviceInfo& di, int T, int D, int F, const void* x,
                            const staple_embed* e, const void* wg, const void* wu, const void* wd,
                            void* z, void* y, void* g_save, void* h_save, void* ws,
                            int32_t* err, cudaStream_t st);

// simt_f32.cu (fp32 on CUDA cores)
staple_status f32_ffn_fwd(int T, int D, int F, const float* x, const staple_embed* e,
                          const float* wg, const float* wu, const float* wd, float* z, float* y,
                          float* g_save, float* h_save, int32_t* err, cudaStream_t st);
staple_status f32_dz(int T, int D, int F, const float* dy, const float* g_save,
                     const float* h_save, const float* wd, float* dgh, cudaStream_t st);
staple_status f32_ffn_bwd(int T, int D, int F, const float* dy, const float* x, const float* z,
                          const float* dgh, const float* wg, const float* wu, float* dx,
                          float* dwg, float* dwu, float* dwd, cudaStream_t st);

}  // namespace stp
