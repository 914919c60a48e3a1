// Allocation-free variant of the table-gradient reduction (dE from dh).
//
// staple_embed_bwd takes its partial-sum scratch from a workspace the caller
// allocates.  Some callers cannot allocate device memory at all: a serving
// process whose device memory is entirely owned by another allocator, code
// that must not call cudaMalloc because it synchronizes the device, or a
// plug-in host that only hands over its input and output buffers.  This entry
// point keeps the scratch in a file-scope device array instead, so neither the
// caller nor the library allocates anything when it runs.
//
// The array is part of the library's device image: every GPU that loads the
// library holds kStaticScratchBytes until the process exits.  Host code may
// not use the array's name as a device address (on the host it names a
// stand-in object), so its device address is looked up with
// cudaGetSymbolAddress, with the device current, on the first call in each
// CUDA context of a device and kept for later calls in that context.  A new
// context on the device (after cudaDeviceReset, for instance) loads the
// library's device image again, possibly elsewhere, so the address is looked
// up again there.  Every call shares the one array: calls that overlap on the
// GPU (on different streams without ordering) race on it.  Nothing in it
// needs to start at zero: each call writes every partial slot it later reads.
// A second, small array holds the reduction's crossing-segment counters; it
// is zero when the image is loaded, and every call leaves it at zero.
#include <cuda.h>
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/staple.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_seg_scratch[kStaticScratchBytes / sizeof(float)];
// The reduction's crossing-segment counters: zero when the library's device
// image is loaded, and every call leaves them at zero.  A call the size check
// admits has ceil(T / 64) * ceil(F / 2048) of them: at most 1024 + 512.
constexpr int kStaticCounters = 2048;
static __device__ __align__(256) int32_t g_seg_counters[kStaticCounters];

using CtxGetCurrent = CUresult (*)(CUcontext*);

std::mutex g_addr_mu;
float* g_addr[kMaxDevices] = {};
int32_t* g_cnt_addr[kMaxDevices] = {};
CUcontext g_addr_ctx[kMaxDevices] = {};

// The current CUDA context of the calling thread, through the driver entry
// point (the runtime has made it current by the time this runs).
CUcontext current_context() {
  static CtxGetCurrent fn = [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess)
      return CtxGetCurrent(nullptr);
    return reinterpret_cast<CtxGetCurrent>(f);
  }();
  CUcontext c = nullptr;
  if (!fn || fn(&c) != CUDA_SUCCESS) return nullptr;
  return c;
}

// Device addresses of g_seg_scratch and g_seg_counters on `device` (which
// must be current), looked up once per context of that device.
staple_status scratch_address(int device, float** out, int32_t** counters) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (device < 0 || device >= kMaxDevices) return STAPLE_EUNSUPPORTED;
  const CUcontext ctx = current_context();
  if (!g_addr[device] || ctx == nullptr || ctx != g_addr_ctx[device]) {
    void* p = nullptr;
    void* c = nullptr;
    if (cudaGetSymbolAddress(&p, g_seg_scratch) != cudaSuccess || p == nullptr ||
        cudaGetSymbolAddress(&c, g_seg_counters) != cudaSuccess || c == nullptr) {
      cudaGetLastError();
      g_addr[device] = nullptr;
      g_cnt_addr[device] = nullptr;
      return STAPLE_ECUDA;
    }
    g_addr[device] = static_cast<float*>(p);
    g_cnt_addr[device] = static_cast<int32_t*>(c);
    g_addr_ctx[device] = ctx;
  }
  *out = g_addr[device];
  *counters = g_cnt_addr[device];
  return STAPLE_OK;
}

inline bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

}  // namespace

extern "C" staple_status staple_embed_grad_static(staple_dtype dtype, int32_t T, int32_t F,
                                                  const void* dh, int64_t ld,
                                                  const int32_t* sorted_pos,
                                                  const int32_t* inverse, const int32_t* seg_off,
                                                  float* dE, staple_stream stream) {
  if (dtype != STAPLE_BF16 && dtype != STAPLE_F32) return STAPLE_EINVAL;
  if (T < 0 || F <= 0 || (F % 8) != 0 || ld < F) return STAPLE_EINVAL;
  // Sizes are checked before the pointers: a request the built-in scratch
  // cannot hold (or longer than a dedup can produce) is refused as such.
  if (T > stp::kMaxDedupT || stp::seg_reduce_workspace(T, F) > kStaticScratchBytes ||
      stp::seg_counter_bytes(T, F) > sizeof(int32_t) * kStaticCounters)
    return STAPLE_EUNSUPPORTED;
  if (T == 0) return STAPLE_OK;
  if (!dh || !sorted_pos || !inverse || !seg_off || !dE) return STAPLE_EINVAL;
  const size_t esz = dtype == STAPLE_BF16 ? 2 : 4;
  if (!aligned16(dh) || !aligned16(dE) || (size_t(ld) * esz) % 16 != 0) return STAPLE_EINVAL;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return STAPLE_ECUDA;
  float* part = nullptr;
  int32_t* counters = nullptr;
  const staple_status s = scratch_address(device, &part, &counters);
  if (s != STAPLE_OK) return s;
  return stp::launch_seg_reduce(dtype == STAPLE_BF16, dh, ld, sorted_pos, inverse, seg_off,
                                nullptr, T, F, dE, part, counters,
                                reinterpret_cast<cudaStream_t>(stream));
}
