// The extern "C" entry points of libstaple: argument checks, host-side
// bookkeeping (contexts, registered tables, the hot-row cache) and the
// stream orchestration around the kernels.  Every compute step runs in the
// CUDA kernels of the other translation units.
#include <cuda_runtime.h>
#include <thread>

#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstring>
#include <new>
#include <vector>

#include "../../include/staple.h"
#include "internal.h"

struct staple_context {
  stp::DeviceInfo di;
  int32_t* d_err;          // device error word
  cudaEvent_t ev_main;     // main -> side ordering
  cudaEvent_t ev_side;     // side -> main ordering
  stp::Tracer* tracer;     // optional per-kernel timing
};

struct staple_table {
  void* base;              // caller's pointer (host or device)
  const uint8_t* dev;      // device-visible address of the first row
  size_t bytes;
  int64_t V;
  int32_t F;
  int32_t groups;
  staple_dtype dtype;
  uint32_t flags;
  bool registered;         // we called cudaHostRegister
};

struct staple_cache {
  int device;
  int32_t K;
  int32_t cap;             // hash capacity (power of two)
  int64_t row_bytes;       // groups * F * element size
  void* rows;              // [K][groups * F]
  int32_t* hkeys;          // [cap], -1 = empty
  int32_t* hvals;          // [cap]
  int32_t* hot_dev;        // [K] ids in slot order, followed by K itself
  std::vector<int32_t> hot;
};

namespace {

inline size_t esize(staple_dtype d) { return d == STAPLE_BF16 ? 2 : 4; }
inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
inline cudaStream_t cs(staple_stream s) { return reinterpret_cast<cudaStream_t>(s); }

staple_status set_device(const staple_context* ctx) {
  return cudaSetDevice(ctx->di.device) == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

#define STP_TRY(expr)                              \
  do {                                             \
    staple_status _s = (expr);                     \
    if (_s != STAPLE_OK) return _s;                \
  } while (0)
#define STP_CUDA(expr)                                        \
  do {                                                        \
    if ((expr) != cudaSuccess) return STAPLE_ECUDA;           \
  } while (0)

inline bool replaces_up(const staple_embed* e) {
  return e && (e->flags & STAPLE_EMBED_REPLACE_UP);
}

staple_status check_embed(const staple_embed* e, staple_dtype dt, int F) {
  if (e && (e->flags & ~uint32_t(STAPLE_EMBED_REPLACE_UP))) return STAPLE_EINVAL;
  if (replaces_up(e) && e->mode == STAPLE_EMBED_NONE) return STAPLE_EINVAL;
  if (!e || e->mode == STAPLE_EMBED_NONE) return STAPLE_OK;
  if (e->mode != STAPLE_EMBED_TABLE && e->mode != STAPLE_EMBED_ROWS) return STAPLE_EINVAL;
  if (!e->base || !e->index || e->n_rows <= 0 || e->row_pitch < F) return STAPLE_EINVAL;
  if (dt == STAPLE_BF16 && (!aligned16(e->base) || (e->row_pitch % 8) != 0)) return STAPLE_EINVAL;
  return STAPLE_OK;
}

staple_status check_dims(staple_dtype dt, int32_t T, int32_t D, int32_t F) {
  if (dt != STAPLE_BF16 && dt != STAPLE_F32) return STAPLE_EINVAL;
  if (T < 0 || D <= 0 || F <= 0) return STAPLE_EINVAL;
  if (dt == STAPLE_BF16 && ((D % 64) != 0 || (F % 64) != 0)) return STAPLE_EINVAL;
  if (dt == STAPLE_F32 && (F % 8) != 0) return STAPLE_EINVAL;
  if (int64_t(T) * 2 * F > (int64_t(1) << 31) * 4) return STAPLE_EUNSUPPORTED;
  return STAPLE_OK;
}

// The table-gradient counters in the workspace's counter head.
int32_t* k8_counters(void* workspace, int D, int F) {
  return reinterpret_cast<int32_t*>(static_cast<uint8_t*>(workspace) +
                                    stp::decode_flag_bytes(D, F));
}

bool ptrs_ok(staple_dtype dt, std::initializer_list<const void*> ps) {
  for (const void* p : ps) {
    if (!p) return false;
    if (dt == STAPLE_BF16 && !aligned16(p)) return false;
  }
  return true;
}

}  // namespace

extern "C" {

int staple_abi_version(void) { return STAPLE_ABI_VERSION; }

const char* staple_status_string(staple_status s) {
  switch (s) {
    case STAPLE_OK: return "STAPLE_OK";
    case STAPLE_EINVAL: return "STAPLE_EINVAL: invalid argument";
    case STAPLE_EIDRANGE: return "STAPLE_EIDRANGE: token id outside [0, V)";
    case STAPLE_ECUDA: return "STAPLE_ECUDA: CUDA runtime error";
    case STAPLE_ENOMEM: return "STAPLE_ENOMEM: allocation failed";
    case STAPLE_ETIMEOUT: return "STAPLE_ETIMEOUT: a bounded kernel wait ran out";
    case STAPLE_EUNSUPPORTED: return "STAPLE_EUNSUPPORTED: not supported by this build";
    case STAPLE_ENODEV: return "STAPLE_ENODEV: no sm_100 device";
  }
  return "STAPLE_UNKNOWN";
}

// Every device allocation the library makes goes through here (none happens
// in a per-step call).  Fault injection for tests, on the host: with
// STAPLE_FAIL_ALLOC set to an allocation's site name ("context_err",
// "cache_rows", "cache_hash", "cache_hot") or to "all", that allocation
// fails as if the device were out of memory.
static cudaError_t lib_malloc(void** p, size_t bytes, const char* site) {
  if (const char* e = std::getenv("STAPLE_FAIL_ALLOC")) {
    if (!std::strcmp(e, site) || !std::strcmp(e, "all")) {
      *p = nullptr;
      return cudaErrorMemoryAllocation;
    }
  }
  return cudaMalloc(p, bytes);
}

staple_status staple_context_create(int device, staple_context** out) {
  if (!out) return STAPLE_EINVAL;
  *out = nullptr;
  int n = 0;
  if (cudaGetDeviceCount(&n) != cudaSuccess || device < 0 || device >= n) return STAPLE_ENODEV;
  cudaDeviceProp prop;
  STP_CUDA(cudaGetDeviceProperties(&prop, device));
  if (prop.major != 10) return STAPLE_ENODEV;
  STP_CUDA(cudaSetDevice(device));
  staple_context* c = new (std::nothrow) staple_context();
  if (!c) return STAPLE_ENOMEM;
  c->di.device = device;
  c->di.num_sms = prop.multiProcessorCount;
  c->di.wait_ns = stp::kWaitLimitNs;
  c->di.sm_reserve = 0;
  if (lib_malloc(reinterpret_cast<void**>(&c->d_err), sizeof(int32_t), "context_err") !=
      cudaSuccess) {
    cudaGetLastError();
    delete c;
    return STAPLE_ENOMEM;
  }
  if (cudaMemset(c->d_err, 0, sizeof(int32_t)) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_main, cudaEventDisableTiming) != cudaSuccess ||
      cudaEventCreateWithFlags(&c->ev_side, cudaEventDisableTiming) != cudaSuccess) {
    cudaFree(c->d_err);
    delete c;
    return STAPLE_ECUDA;
  }
  c->tracer = stp::tracer_create(device);
  *out = c;
  return STAPLE_OK;
}

staple_status staple_set_wait_limit(staple_context* ctx, int64_t limit_ns) {
  if (!ctx || limit_ns < 1 || limit_ns > stp::kMaxWaitLimitNs) return STAPLE_EINVAL;
  ctx->di.wait_ns = uint64_t(limit_ns);
  return STAPLE_OK;
}

staple_status staple_set_sm_reserve(staple_context* ctx, int32_t sms) {
  if (!ctx || sms < 0 || sms > ctx->di.num_sms / 4) return STAPLE_EINVAL;
  ctx->di.sm_reserve = sms;
  return STAPLE_OK;
}

staple_status staple_trace_enable(staple_context* ctx, int enable) {
  if (!ctx) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  return stp::tracer_enable(ctx->tracer, enable != 0) ? STAPLE_OK : STAPLE_ECUDA;
}

staple_status staple_trace_read(staple_context* ctx, staple_trace_record* out, int32_t capacity,
                                int32_t* count) {
  if (!ctx || !count || capacity < 0 || (capacity > 0 && !out)) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  *count = stp::tracer_read(ctx->tracer, out, capacity, nullptr);
  return STAPLE_OK;
}

staple_status staple_context_destroy(staple_context* ctx) {
  if (!ctx) return STAPLE_OK;
  cudaSetDevice(ctx->di.device);
  cudaEventDestroy(ctx->ev_main);
  cudaEventDestroy(ctx->ev_side);
  stp::tracer_destroy(ctx->tracer);
  cudaFree(ctx->d_err);
  delete ctx;
  return STAPLE_OK;
}

staple_status staple_get_error(staple_context* ctx, staple_stream stream, int32_t* device_error) {
  if (!ctx || !device_error) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  STP_CUDA(cudaStreamSynchronize(cs(stream)));
  int32_t h = 0;
  STP_CUDA(cudaMemcpy(&h, ctx->d_err, sizeof(h), cudaMemcpyDeviceToHost));
  STP_CUDA(cudaMemset(ctx->d_err, 0, sizeof(int32_t)));
  *device_error = h;
  return STAPLE_OK;
}

// ------------------------------------------------------------------ tables

staple_status staple_table_register(staple_context* ctx, void* base, size_t bytes, int64_t V,
                                    int32_t F, int32_t groups, staple_dtype dtype, uint32_t flags,
                                    staple_table** out) {
  if (!ctx || !base || !out || V <= 0 || F <= 0 || groups <= 0) return STAPLE_EINVAL;
  if (dtype != STAPLE_BF16 && dtype != STAPLE_F32) return STAPLE_EINVAL;
  const uint32_t loc = flags & (STAPLE_TABLE_DEVICE | STAPLE_TABLE_HOST_PINNED |
                                STAPLE_TABLE_HOST_REGISTER);
  if (loc != STAPLE_TABLE_DEVICE && loc != STAPLE_TABLE_HOST_PINNED &&
      loc != STAPLE_TABLE_HOST_REGISTER)
    return STAPLE_EINVAL;
  const size_t need = size_t(V) * size_t(groups) * size_t(F) * esize(dtype);
  if (bytes < need || !aligned16(base) || (size_t(F) * esize(dtype)) % 16 != 0) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  staple_table* t = new (std::nothrow) staple_table();
  if (!t) return STAPLE_ENOMEM;
  t->base = base;
  t->bytes = bytes;
  t->V = V;
  t->F = F;
  t->groups = groups;
  t->dtype = dtype;
  t->flags = loc;
  t->registered = false;
  if (loc == STAPLE_TABLE_DEVICE) {
    t->dev = static_cast<const uint8_t*>(base);
  } else {
    if (loc == STAPLE_TABLE_HOST_REGISTER) {
      if (cudaHostRegister(base, bytes, cudaHostRegisterMapped | cudaHostRegisterPortable) !=
          cudaSuccess) {
        cudaGetLastError();
        delete t;
        return STAPLE_ECUDA;
      }
      t->registered = true;
    }
    void* dp = nullptr;
    if (cudaHostGetDevicePointer(&dp, base, 0) != cudaSuccess) {
      cudaGetLastError();
      if (t->registered) cudaHostUnregister(base);
      delete t;
      return STAPLE_ECUDA;
    }
    t->dev = static_cast<const uint8_t*>(dp);
  }
  *out = t;
  return STAPLE_OK;
}

staple_status staple_table_unregister(staple_table* t) {
  if (!t) return STAPLE_OK;
  if (t->registered) cudaHostUnregister(t->base);
  delete t;
  return STAPLE_OK;
}

// ------------------------------------------------------------------- cache

staple_status staple_cache_build(staple_context* ctx, const staple_table* table,
                                 const int64_t* freq, double frac, staple_stream stream,
                                 staple_cache** out) {
  if (!ctx || !table || !freq || !out || !(frac >= 0.0 && frac <= 1.0)) return STAPLE_EINVAL;
  *out = nullptr;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  const int64_t V = table->V;
  if (V > INT32_MAX) return STAPLE_EUNSUPPORTED;
  int64_t K = frac > 0 ? int64_t(std::ceil(frac * double(V) - 1e-9)) : 0;
  K = std::min<int64_t>(std::max<int64_t>(K, 0), V);
  std::vector<int32_t> order(V);
  for (int64_t i = 0; i < V; ++i) order[i] = int32_t(i);
  std::partial_sort(order.begin(), order.begin() + K, order.end(), [&](int32_t a, int32_t b) {
    return freq[a] > freq[b] || (freq[a] == freq[b] && a < b);
  });
  staple_cache* c = new (std::nothrow) staple_cache();
  if (!c) return STAPLE_ENOMEM;
  c->device = ctx->di.device;
  c->K = int32_t(K);
  int32_t cap = 16;
  while (cap < 2 * K) cap <<= 1;
  c->cap = cap;
  c->row_bytes = int64_t(table->groups) * table->F * int64_t(esize(table->dtype));
  c->hot.assign(order.begin(), order.begin() + K);
  cudaStream_t st = cs(stream);
  bool ok = lib_malloc(reinterpret_cast<void**>(&c->rows),
                       size_t(std::max<int64_t>(K, 1)) * c->row_bytes, "cache_rows") == cudaSuccess &&
            lib_malloc(reinterpret_cast<void**>(&c->hkeys), size_t(cap) * 4, "cache_hash") ==
                cudaSuccess &&
            lib_malloc(reinterpret_cast<void**>(&c->hvals), size_t(cap) * 4, "cache_hash") ==
                cudaSuccess &&
            lib_malloc(reinterpret_cast<void**>(&c->hot_dev), size_t(K + 1) * 4, "cache_hot") ==
                cudaSuccess;
  if (!ok) {
    cudaGetLastError();
    staple_cache_free(c);
    return STAPLE_ENOMEM;
  }
  std::vector<int32_t> hk(c->hot);
  hk.push_back(int32_t(K));
  ok = cudaMemsetAsync(c->hkeys, 0xFF, size_t(cap) * 4, st) == cudaSuccess &&
       cudaMemcpyAsync(c->hot_dev, hk.data(), hk.size() * 4, cudaMemcpyHostToDevice, st) ==
           cudaSuccess &&
       stp::launch_cache_fill(c->hot_dev, int(K), c->hkeys, c->hvals, uint32_t(cap - 1), st) ==
           STAPLE_OK &&
       stp::launch_copy_rows(table->dev, c->row_bytes, c->row_bytes, c->hot_dev,
                             c->hot_dev + K, c->rows, ctx->di.num_sms, st) == STAPLE_OK &&
       cudaStreamSynchronize(st) == cudaSuccess;
  if (!ok) {
    staple_cache_free(c);
    return STAPLE_ECUDA;
  }
  *out = c;
  return STAPLE_OK;
}

staple_status staple_cache_info(const staple_cache* c, int32_t* K, int32_t* cap) {
  if (!c) return STAPLE_EINVAL;
  if (K) *K = c->K;
  if (cap) *cap = c->cap;
  return STAPLE_OK;
}

staple_status staple_cache_hot_ids(const staple_cache* c, int32_t* hot_ids) {
  if (!c || (!hot_ids && c->K > 0)) return STAPLE_EINVAL;
  if (c->K > 0) std::memcpy(hot_ids, c->hot.data(), size_t(c->K) * 4);
  return STAPLE_OK;
}

staple_status staple_cache_rows(const staple_cache* c, const void** rows) {
  if (!c || !rows) return STAPLE_EINVAL;
  *rows = c->rows;
  return STAPLE_OK;
}

staple_status staple_cache_free(staple_cache* c) {
  if (!c) return STAPLE_OK;
  cudaSetDevice(c->device);
  if (c->rows) cudaFree(c->rows);
  if (c->hkeys) cudaFree(c->hkeys);
  if (c->hvals) cudaFree(c->hvals);
  if (c->hot_dev) cudaFree(c->hot_dev);
  delete c;
  return STAPLE_OK;
}

// --------------------------------------------------------------- workspace

size_t staple_workspace_bytes(int32_t T, int32_t D, int32_t F, uint32_t flags) {
  (void)flags;
  if (T < 0 || F <= 0 || D <= 0) return 0;
  const size_t b = std::max(stp::seg_reduce_workspace(T, F), stp::decode_scratch_bytes(T, D, F));
  return stp::decode_counter_bytes(D, F) + ((b + 255) & ~size_t(255));
}

// --------------------------------------------------------------- retrieval

staple_status staple_dedup(staple_context* ctx, const int32_t* ids, int32_t T, int64_t V,
                           int32_t* unique, int32_t* inverse, int32_t* seg_off,
                           int32_t* sorted_pos, int32_t* U_dev, staple_stream stream) {
  if (!ctx || T < 0 || V <= 0 || V > INT32_MAX || !seg_off || !U_dev) return STAPLE_EINVAL;
  if (T > 0 && (!ids || !unique || !inverse || !sorted_pos)) return STAPLE_EINVAL;
  if (T > stp::kMaxDedupT) return STAPLE_EUNSUPPORTED;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  return stp::launch_dedup(ids, T, V, unique, inverse, seg_off, sorted_pos, U_dev, ctx->d_err,
                           cs(stream));
}

staple_status staple_gather_unique_rows(staple_context* ctx, const staple_cache* cache,
                                        const staple_table* table, const int32_t* unique,
                                        const int32_t* U_dev, int32_t T, int32_t* slot,
                                        int32_t* miss_list, int32_t* miss_count, void* rows,
                                        staple_stream stream, staple_stream side) {
  if (!ctx || !table || !U_dev || !slot || !miss_list || !miss_count || T < 0) return STAPLE_EINVAL;
  if (T > 0 && (!unique || !rows)) return STAPLE_EINVAL;
  if (!aligned16(rows)) return STAPLE_EINVAL;
  const int64_t row_bytes = int64_t(table->groups) * table->F * int64_t(esize(table->dtype));
  if (cache && cache->row_bytes != row_bytes) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  cudaStream_t st = cs(stream);
  cudaStream_t sd = cs(side);
  STP_TRY(stp::launch_probe(unique, U_dev, cache && cache->K > 0 ? cache->hkeys : nullptr,
                            cache ? cache->hvals : nullptr,
                            cache ? uint32_t(cache->cap - 1) : 0u, slot, miss_list, miss_count,
                            st));
  const bool split = sd != st;
  if (split) {
    STP_CUDA(cudaEventRecord(ctx->ev_main, st));
    STP_CUDA(cudaStreamWaitEvent(sd, ctx->ev_main, 0));
  }
  STP_TRY(stp::launch_gather_misses(table->dev, row_bytes, row_bytes, unique, miss_list,
                                    miss_count, rows, ctx->di.num_sms,
                                    table->flags != STAPLE_TABLE_DEVICE, split ? sd : st));
  if (cache && cache->K > 0)
    STP_TRY(stp::launch_gather_hits(cache->rows, row_bytes, U_dev, slot, rows, ctx->di.num_sms, st));
  if (split) {
    STP_CUDA(cudaEventRecord(ctx->ev_side, sd));
    STP_CUDA(cudaStreamWaitEvent(st, ctx->ev_side, 0));
  }
  return STAPLE_OK;
}

staple_status staple_gather_unique_rows_bulk(staple_context* ctx, const staple_cache* cache,
                                             const staple_table* table, const int32_t* unique,
                                             const int32_t* U_dev, int32_t T, int32_t* slot,
                                             int32_t* miss_list, int32_t* miss_count, void* rows,
                                             void* staging_host, void* staging_dev,
                                             int32_t* list_host, int32_t chunk_rows,
                                             int32_t threads, staple_stream stream) {
  if (!ctx || !table || !U_dev || !slot || !miss_list || !miss_count || T < 0) return STAPLE_EINVAL;
  if (T > 0 && (!unique || !rows || !staging_host || !staging_dev || !list_host)) return STAPLE_EINVAL;
  if (!aligned16(rows) || !aligned16(staging_dev) || chunk_rows < 1) return STAPLE_EINVAL;
  if (!(table->flags & (STAPLE_TABLE_HOST_PINNED | STAPLE_TABLE_HOST_REGISTER))) return STAPLE_EINVAL;
  const int64_t row_bytes = int64_t(table->groups) * table->F * int64_t(esize(table->dtype));
  if (cache && cache->row_bytes != row_bytes) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  cudaStream_t st = cs(stream);
  cudaStreamCaptureStatus cap = cudaStreamCaptureStatusNone;
  STP_CUDA(cudaStreamIsCapturing(st, &cap));
  if (cap != cudaStreamCaptureStatusNone) return STAPLE_EINVAL;  // the host must wait below
  stp::TraceScope trace_scope(ctx->tracer);
  if (T == 0) return STAPLE_OK;
  STP_TRY(stp::launch_probe(unique, U_dev, cache && cache->K > 0 ? cache->hkeys : nullptr,
                            cache ? cache->hvals : nullptr,
                            cache ? uint32_t(cache->cap - 1) : 0u, slot, miss_list, miss_count,
                            st));
  // the miss ids to the host: count, miss list, unique ids (list_host: [1 + 2T])
  STP_CUDA(cudaMemcpyAsync(list_host, miss_count, sizeof(int32_t), cudaMemcpyDeviceToHost, st));
  STP_CUDA(cudaMemcpyAsync(list_host + 1, miss_list, size_t(T) * sizeof(int32_t),
                           cudaMemcpyDeviceToHost, st));
  STP_CUDA(cudaMemcpyAsync(list_host + 1 + T, unique, size_t(T) * sizeof(int32_t),
                           cudaMemcpyDeviceToHost, st));
  STP_CUDA(cudaEventRecord(ctx->ev_main, st));
  if (cache && cache->K > 0)
    STP_TRY(stp::launch_gather_hits(cache->rows, row_bytes, U_dev, slot, rows, ctx->di.num_sms, st));
  STP_CUDA(cudaEventSynchronize(ctx->ev_main));
  // pack the miss rows from the host table in miss order, chunk by chunk;
  // each chunk's copy to the device starts as soon as it is packed
  const int32_t n = std::max(0, std::min(list_host[0], T));
  const int32_t* ml = list_host + 1;
  const int32_t* uq = list_host + 1 + T;
  const uint8_t* src = static_cast<const uint8_t*>(table->base);
  uint8_t* hs = static_cast<uint8_t*>(staging_host);
  uint8_t* ds = static_cast<uint8_t*>(staging_dev);
  // a chunk never exceeds the batch, so the chunk arithmetic below stays in
  // range for any chunk_rows >= 1
  const int32_t crows = std::max<int32_t>(1, std::min<int32_t>(chunk_rows, std::max(n, 1)));
  const int32_t nchunks = int32_t((int64_t(n) + crows - 1) / crows);
  int nt = threads > 0 ? threads : int(std::thread::hardware_concurrency());
  nt = std::max(1, std::min(nt, nchunks));
  // one pool per call: workers claim chunks and mark each one packed; this
  // thread issues the chunks' copies in order as they become ready
  std::atomic<int32_t> next{0};
  std::atomic<bool> bad_id{false};
  std::vector<std::atomic<int>> packed(size_t(std::max(nchunks, 1)));
  for (auto& a : packed) a.store(0, std::memory_order_relaxed);
  auto worker = [&]() {
    for (int32_t c; (c = next.fetch_add(1)) < nchunks;) {
      const int32_t c1 = int32_t(std::min<int64_t>(n, (int64_t(c) + 1) * crows));
      for (int32_t i = c * crows; i < c1; ++i) {
        // the host reads its own memory here: an id outside the table (the
        // dedup reports it, it does not clamp) must not steer the read
        const int32_t pos = ml[i];
        const int64_t id = pos >= 0 && pos < T ? int64_t(uq[pos]) : -1;
        uint8_t* dst = hs + int64_t(i) * row_bytes;
        if (id < 0 || id >= table->V) {
          std::memset(dst, 0, size_t(row_bytes));
          bad_id.store(true, std::memory_order_relaxed);
          continue;
        }
        std::memcpy(dst, src + id * row_bytes, size_t(row_bytes));
      }
      packed[size_t(c)].store(1, std::memory_order_release);
    }
  };
  std::vector<std::thread> pool;
  for (int t = 0; t < nt; ++t) pool.emplace_back(worker);
  cudaError_t ce = cudaSuccess;
  for (int32_t c = 0; c < nchunks; ++c) {
    while (!packed[size_t(c)].load(std::memory_order_acquire)) std::this_thread::yield();
    const int32_t c0 = c * crows, c1 = int32_t(std::min<int64_t>(n, int64_t(c0) + crows));
    if (ce == cudaSuccess)
      ce = cudaMemcpyAsync(ds + int64_t(c0) * row_bytes, hs + int64_t(c0) * row_bytes,
                           size_t(c1 - c0) * size_t(row_bytes), cudaMemcpyHostToDevice, st);
  }
  for (auto& th : pool) th.join();
  if (ce != cudaSuccess) return STAPLE_ECUDA;
  STP_TRY(stp::launch_scatter_misses(staging_dev, row_bytes, miss_list, miss_count, rows,
                                     ctx->di.num_sms, st));
  return bad_id.load() ? STAPLE_EIDRANGE : STAPLE_OK;
}

staple_status staple_cache_refresh(staple_context* ctx, staple_cache* cache,
                                   const staple_table* table, const int32_t* unique,
                                   const int32_t* slot, const int32_t* U_dev,
                                   staple_stream stream) {
  if (!ctx || !cache || !table || !unique || !slot || !U_dev) return STAPLE_EINVAL;
  if (cache->device != ctx->di.device ||
      cache->row_bytes != int64_t(table->groups) * table->F * int64_t(esize(table->dtype)))
    return STAPLE_EINVAL;
  if (cache->K == 0) return STAPLE_OK;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  return stp::launch_cache_refresh(table->dev, cache->row_bytes, cache->row_bytes, unique, slot,
                                   U_dev, cache->rows, ctx->di.num_sms, cs(stream));
}

staple_status staple_gather_rows(staple_context* ctx, const staple_cache* cache,
                                 const staple_table* table, const int32_t* ids, int32_t T,
                                 int32_t* unique, int32_t* inverse, int32_t* seg_off,
                                 int32_t* sorted_pos, int32_t* U_dev, int32_t* slot,
                                 int32_t* miss_list, int32_t* miss_count, void* rows,
                                 staple_stream stream, staple_stream side) {
  if (!table) return STAPLE_EINVAL;
  STP_TRY(staple_dedup(ctx, ids, T, table->V, unique, inverse, seg_off, sorted_pos, U_dev,
                       stream));
  return staple_gather_unique_rows(ctx, cache, table, unique, U_dev, T, slot, miss_list,
                                   miss_count, rows, stream, side);
}

// ------------------------------------------------------------ FFN forward

staple_status staple_ffn_fwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                             int32_t F, const void* x, const staple_embed* embed,
                             const void* w_gate, const void* w_up, const void* w_down, void* z,
                             void* y, void* g_save, void* h_save, void* workspace,
                             size_t workspace_bytes, staple_stream stream) {
  if (!ctx) return STAPLE_EINVAL;
  STP_TRY(check_dims(dtype, T, D, F));
  STP_TRY(check_embed(embed, dtype, F));
  const bool decode = dtype == STAPLE_BF16 && T >= 1 && T <= stp::kMaxDecodeT;
  if (decode && (!workspace || !aligned16(workspace) ||
                 workspace_bytes < stp::decode_counter_bytes(D, F) +
                                       stp::decode_scratch_bytes(T, D, F)))
    return STAPLE_EINVAL;
  if (!ptrs_ok(dtype, {w_gate, w_down})) return STAPLE_EINVAL;
  if (!replaces_up(embed) && !ptrs_ok(dtype, {w_up})) return STAPLE_EINVAL;
  if (T > 0 && !ptrs_ok(dtype, {x, z, y})) return STAPLE_EINVAL;
  if ((g_save && !ptrs_ok(dtype, {g_save})) || (h_save && !ptrs_ok(dtype, {h_save})))
    return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  if (decode) {
    // the decode kernel refuses (before launching anything) a STEM layer
    // whose d_ff is not a multiple of its 128-feature gate tiles, or a device
    // that cannot hold its whole grid at once; the tiled kernels then compute
    // the same layer
    const staple_status s = stp::tc_decode_fwd(ctx->di, T, D, F, x, embed, w_gate, w_up, w_down, z,
                                               y, g_save, h_save, workspace, ctx->d_err, cs(stream));
    if (s != STAPLE_EUNSUPPORTED) return s;
  }
  if (dtype == STAPLE_BF16)
    return stp::tc_ffn_fwd(ctx->di, T, D, F, x, embed, w_gate, w_up, w_down, z, y, g_save, h_save,
                           ctx->d_err, cs(stream));
  return stp::f32_ffn_fwd(T, D, F, static_cast<const float*>(x), embed,
                          static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
                          static_cast<const float*>(w_down), static_cast<float*>(z),
                          static_cast<float*>(y), static_cast<float*>(g_save),
                          static_cast<float*>(h_save), ctx->d_err, cs(stream));
}

// ----------------------------------------------------------- FFN backward

staple_status staple_embed_bwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                               int32_t F, const void* dy, const void* g_save, const void* h_save,
                               const void* w_down, const int32_t* sorted_pos,
                               const int32_t* inverse, const int32_t* seg_off,
                               const int32_t* U_dev, void* dgh, float* dE, void* workspace,
                               size_t workspace_bytes, staple_stream stream) {
  if (!ctx) return STAPLE_EINVAL;
  STP_TRY(check_dims(dtype, T, D, F));
  if (!ptrs_ok(dtype, {w_down})) return STAPLE_EINVAL;
  if (T > 0 && !ptrs_ok(dtype, {dy, g_save, h_save, dgh})) return STAPLE_EINVAL;
  const size_t head = stp::decode_counter_bytes(D, F);  // left untouched
  if (dE) {
    if (!sorted_pos || !inverse || !seg_off || !U_dev || !aligned16(dE)) return STAPLE_EINVAL;
    if (T > stp::kMaxDedupT) return STAPLE_EUNSUPPORTED;   // more than one dedup holds
    const size_t need = head + stp::seg_reduce_workspace(T, F);
    if (T > 0 && (!workspace || workspace_bytes < need || !aligned16(workspace)))
      return STAPLE_EINVAL;
  }
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  cudaStream_t st = cs(stream);
  if (dtype == STAPLE_BF16)
    STP_TRY(stp::tc_dz(ctx->di, T, D, F, dy, g_save, h_save, w_down, dgh, ctx->d_err, st));
  else
    STP_TRY(stp::f32_dz(T, D, F, static_cast<const float*>(dy), static_cast<const float*>(g_save),
                        static_cast<const float*>(h_save), static_cast<const float*>(w_down),
                        static_cast<float*>(dgh), st));
  if (!dE) return STAPLE_OK;
  const size_t es = esize(dtype);
  const void* dh = static_cast<const uint8_t*>(dgh) + size_t(F) * es;
  return stp::launch_seg_reduce(dtype == STAPLE_BF16, dh, 2 * int64_t(F), sorted_pos, inverse,
                                seg_off, U_dev, T, F, dE,
                                reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + head),
                                k8_counters(workspace, D, F), st);
}

staple_status staple_embed_grad(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                                int32_t F, const void* dh, int64_t ld, const int32_t* sorted_pos,
                                const int32_t* inverse, const int32_t* seg_off,
                                const int32_t* U_dev, float* dE, void* workspace,
                                size_t workspace_bytes, staple_stream stream) {
  if (!ctx) return STAPLE_EINVAL;
  STP_TRY(check_dims(dtype, T, D, F));
  if (T == 0) return STAPLE_OK;
  if (!dh || ld < F || !sorted_pos || !inverse || !seg_off || !U_dev || !dE || !aligned16(dE) ||
      !aligned16(dh) || (ld * int64_t(esize(dtype))) % 16)
    return STAPLE_EINVAL;
  if (T > stp::kMaxDedupT) return STAPLE_EUNSUPPORTED;   // more than one dedup holds
  const size_t head = stp::decode_counter_bytes(D, F);  // left untouched
  if (!workspace || workspace_bytes < head + stp::seg_reduce_workspace(T, F) ||
      !aligned16(workspace))
    return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  return stp::launch_seg_reduce(dtype == STAPLE_BF16, dh, ld, sorted_pos, inverse, seg_off, U_dev,
                                T, F, dE,
                                reinterpret_cast<float*>(static_cast<uint8_t*>(workspace) + head),
                                k8_counters(workspace, D, F), cs(stream));
}

staple_status staple_embed_grad_to_host(staple_context* ctx, int32_t F, int32_t capacity,
                                        const float* dE, const int32_t* unique,
                                        const int32_t* U_dev, float* host_dE,
                                        int32_t* host_unique, int32_t* host_U,
                                        staple_stream stream) {
  if (!ctx || F <= 0 || F % 4 || capacity < 0) return STAPLE_EINVAL;
  if (capacity == 0) return STAPLE_OK;
  if (!dE || !unique || !U_dev || !host_dE || !host_unique || !host_U || !aligned16(dE) ||
      !aligned16(host_dE))
    return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  // the host buffers must be page-locked and mapped: their device-side
  // addresses are what the kernel stores to
  void* d_rows = nullptr;
  void* d_ids = nullptr;
  void* d_u = nullptr;
  if (cudaHostGetDevicePointer(&d_rows, host_dE, 0) != cudaSuccess ||
      cudaHostGetDevicePointer(&d_ids, host_unique, 0) != cudaSuccess ||
      cudaHostGetDevicePointer(&d_u, host_U, 0) != cudaSuccess) {
    cudaGetLastError();
    return STAPLE_EINVAL;
  }
  if (!aligned16(d_rows)) return STAPLE_EINVAL;
  stp::TraceScope trace_scope(ctx->tracer);
  return stp::launch_grad_to_host(dE, unique, U_dev, F, capacity, static_cast<float*>(d_rows),
                                  static_cast<int32_t*>(d_ids), static_cast<int32_t*>(d_u),
                                  ctx->di.num_sms, cs(stream));
}

staple_status staple_ffn_bwd(staple_context* ctx, staple_dtype dtype, int32_t T, int32_t D,
                             int32_t F, const void* dy, const void* x, const void* z,
                             const void* dgh, const void* w_gate, const void* w_up, void* dx,
                             float* dw_gate, float* dw_up, float* dw_down, void* workspace,
                             size_t workspace_bytes, staple_stream stream) {
  (void)workspace;
  (void)workspace_bytes;
  if (!ctx) return STAPLE_EINVAL;
  STP_TRY(check_dims(dtype, T, D, F));
  if (T > 0 && !ptrs_ok(dtype, {dy, x, z, dgh})) return STAPLE_EINVAL;
  if (dx && !ptrs_ok(dtype, {dx, w_gate})) return STAPLE_EINVAL;
  if (w_up && !ptrs_ok(dtype, {w_up})) return STAPLE_EINVAL;
  if (!w_up && dw_up) return STAPLE_EINVAL;   // no up-projection (STEM): no dW_up
  for (const float* p : {dw_gate, dw_up, dw_down})
    if (p && !aligned16(p)) return STAPLE_EINVAL;
  STP_TRY(set_device(ctx));
  stp::TraceScope trace_scope(ctx->tracer);
  if (dtype == STAPLE_BF16)
    return stp::tc_ffn_bwd(ctx->di, T, D, F, dy, x, z, dgh, w_gate, w_up, dx, dw_gate, dw_up,
                           dw_down, ctx->d_err, cs(stream));
  if (T == 0) {
    cudaStream_t st = cs(stream);
    if (dw_gate) STP_CUDA(cudaMemsetAsync(dw_gate, 0, size_t(F) * D * 4, st));
    if (dw_up) STP_CUDA(cudaMemsetAsync(dw_up, 0, size_t(F) * D * 4, st));
    if (dw_down) STP_CUDA(cudaMemsetAsync(dw_down, 0, size_t(F) * D * 4, st));
    return STAPLE_OK;
  }
  return stp::f32_ffn_bwd(T, D, F, static_cast<const float*>(dy), static_cast<const float*>(x),
                          static_cast<const float*>(z), static_cast<const float*>(dgh),
                          static_cast<const float*>(w_gate), static_cast<const float*>(w_up),
                          static_cast<float*>(dx), dw_gate, dw_up, dw_down, cs(stream));
}

}  // extern "C"
