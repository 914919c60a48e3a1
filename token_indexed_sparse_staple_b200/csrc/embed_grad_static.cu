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
// stand-in object), so its device address is looked up once per device with
// cudaGetSymbolAddress, with that device current, on the first call.  Every
// call shares the one array: calls that overlap on the GPU (on different
// streams without ordering) race on it.  Nothing in it needs to start at zero:
// each call writes every partial slot it later reads.
#include <cuda_runtime.h>

#include <mutex>

#include "../../include/staple.h"
#include "internal.h"

namespace {

constexpr size_t kStaticScratchBytes = size_t(16) << 20;  // 16 MiB
constexpr int kMaxDevices = 64;

static __device__ __align__(256) float g_seg_scratch[kStaticScratchBytes / sizeof(float)];

std::mutex g_addr_mu;
float* g_addr[kMaxDevices] = {};

// Device address of g_seg_scratch on `device` (which must be current).
staple_status scratch_address(int device, float** out) {
  std::lock_guard<std::mutex> lock(g_addr_mu);
  if (device < 0 || device >= kMaxDevices) return STAPLE_EUNSUPPORTED;
  if (!g_addr[device]) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_seg_scratch) != cudaSuccess || p == nullptr) {
      cudaGetLastError();
      return STAPLE_ECUDA;
    }
    g_addr[device] = static_cast<float*>(p);
  }
  *out = g_addr[device];
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
  if (T == 0) return STAPLE_OK;
  if (!dh || !sorted_pos || !inverse || !seg_off || !dE) return STAPLE_EINVAL;
  const size_t esz = dtype == STAPLE_BF16 ? 2 : 4;
  if (!aligned16(dh) || !aligned16(dE) || (size_t(ld) * esz) % 16 != 0) return STAPLE_EINVAL;
  if (stp::seg_reduce_workspace(T, F) > kStaticScratchBytes) return STAPLE_EINVAL;
  int device = 0;
  if (cudaGetDevice(&device) != cudaSuccess) return STAPLE_ECUDA;
  float* part = nullptr;
  const staple_status s = scratch_address(device, &part);
  if (s != STAPLE_OK) return s;
  return stp::launch_seg_reduce(dtype == STAPLE_BF16, dh, ld, sorted_pos, inverse, seg_off,
                                nullptr, T, F, dE, part, reinterpret_cast<cudaStream_t>(stream));
}
