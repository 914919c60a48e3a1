// K8: the table gradient of the U distinct rows of a batch.
//
//   dE[j][f] = sum of dh[i][f] over the tokens i whose id is unique[j]
//
// (AI Radio episode, paper summary: during training only the U x d_ff active
// rows exist on the GPU, as an autograd leaf, so the gradient is one row per
// distinct id.)  The dedup's sorted_pos lists each segment's tokens in
// ascending position.  The sorted order is cut into chunks of kSegChunk
// positions; one block per (chunk, 2048-feature slice) sums each segment
// piece in order with fp32 accumulators.  A segment that lies inside one
// chunk is written to dE directly; a piece of a segment that crosses a chunk
// boundary goes to a partial buffer (at most two pieces per chunk).  Each
// block then counts its crossing pieces on a per-(segment, slice) counter,
// and the block that brings the count to the segment's number of pieces adds
// them in chunk order and writes the row; it also sets the counter back to
// zero, so the counters are zero again after every call.  No float atomics,
// and the order of the adds does not depend on which block finishes last:
// the result is deterministic.
#include "common.cuh"
#include "internal.h"

namespace stp {

constexpr int kSegThreads = 256;
constexpr int kSegVec = 8;                           // features per thread
constexpr int kSegSlice = kSegThreads * kSegVec;     // features per block

template <bool BF16>
__device__ __forceinline__ void load8(const void* base, int64_t off, float* v) {
  if constexpr (BF16) {
    const uint4 w = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(base) + off));
    v[0] = bf_lo(w.x); v[1] = bf_hi(w.x); v[2] = bf_lo(w.y); v[3] = bf_hi(w.y);
    v[4] = bf_lo(w.z); v[5] = bf_hi(w.z); v[6] = bf_lo(w.w); v[7] = bf_hi(w.w);
  } else {
    const float4* p = reinterpret_cast<const float4*>(static_cast<const float*>(base) + off);
    const float4 a = __ldg(p), b = __ldg(p + 1);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
}

__device__ __forceinline__ void store8(float* dst, const float* v) {
  float4* d = reinterpret_cast<float4*>(dst);
  d[0] = make_float4(v[0], v[1], v[2], v[3]);
  d[1] = make_float4(v[4], v[5], v[6], v[7]);
}

// Pieces of chunk c: part[(2c + side) * F + f]; side 0 = the chunk's first
// segment (it started before the chunk), side 1 = its last segment (it
// continues after the chunk).
// cnt[c0 * slices + slice]: pieces written so far of the crossing segment
// that starts in chunk c0 (a chunk starts at most one segment that continues
// past it).
template <bool BF16>
__global__ void __launch_bounds__(kSegThreads)
    seg_reduce_kernel(const void* __restrict__ dh, int64_t ld, const int32_t* __restrict__ sorted_pos,
                      const int32_t* __restrict__ inverse, const int32_t* __restrict__ seg_off,
                      int T, int F, float* __restrict__ dE, float* __restrict__ part,
                      int32_t* __restrict__ cnt) {
  __shared__ int32_t s_pos[kSegChunk];
  __shared__ int32_t s_seg[kSegChunk];
  __shared__ int32_t s_fin[2];
  const int c = blockIdx.x;
  const int p0 = c * kSegChunk;
  const int p1 = min(T, p0 + kSegChunk);
  const int n = p1 - p0;
  if (threadIdx.x < n) {
    const int pos = sorted_pos[p0 + threadIdx.x];
    s_pos[threadIdx.x] = pos;
    s_seg[threadIdx.x] = inverse[pos];
  }
  __syncthreads();
  const int f = (blockIdx.y * kSegThreads + threadIdx.x) * kSegVec;
  const bool active = f < F;   // every thread stays for the block barriers below
  const int first_seg = s_seg[0];
  float acc[kSegVec];
#pragma unroll
  for (int i = 0; i < kSegVec; ++i) acc[i] = 0.0f;
  int cur = first_seg;
  auto flush = [&](int j) {
    const int s0 = seg_off[j], s1 = seg_off[j + 1];
    if (s0 >= p0 && s1 <= p1) {
      store8(dE + int64_t(j) * F + f, acc);
    } else {
      const int side = (j == first_seg) ? 0 : 1;
      store8(part + (int64_t(2 * c + side)) * F + f, acc);
    }
  };
  // One row at a time, in position order.  Many blocks are resident per SM,
  // which keeps enough loads in flight; loading several rows ahead per thread
  // measured slower (more registers, fewer resident blocks).
  for (int q = 0; q < n && active; ++q) {
    const int j = s_seg[q];
    if (j != cur) {
      flush(cur);
      cur = j;
#pragma unroll
      for (int i = 0; i < kSegVec; ++i) acc[i] = 0.0f;
    }
    float v[kSegVec];
    load8<BF16>(dh, int64_t(s_pos[q]) * ld + f, v);
#pragma unroll
    for (int i = 0; i < kSegVec; ++i) acc[i] += v[i];
  }
  if (n > 0 && active) flush(cur);
  __threadfence();   // this thread's pieces before the block's count below
  // Crossing segments: the chunk's first one (if it started earlier or goes
  // on past the chunk) and its last one (if it goes on past the chunk).
  __syncthreads();   // this block's pieces are stored
  if (threadIdx.x < 2) {
    int fin = -1;
    const int j = threadIdx.x == 0 ? first_seg : s_seg[n - 1];
    const int s0 = seg_off[j], s1 = seg_off[j + 1];
    const bool crossing = !(s0 >= p0 && s1 <= p1);
    if (crossing && (threadIdx.x == 0 || j != first_seg)) {
      const int c0 = s0 / kSegChunk, c1 = (s1 - 1) / kSegChunk;
      __threadfence();   // the pieces before the count
      int32_t* k = cnt + int64_t(c0) * gridDim.y + blockIdx.y;
      if (atomicAdd(k, 1) == c1 - c0) {
        fin = j;
        *k = 0;          // every piece has arrived: nobody counts on it again
      }
    }
    s_fin[threadIdx.x] = fin;
  }
  __syncthreads();
#pragma unroll 1
  for (int w = 0; w < 2; ++w) {
    const int j = s_fin[w];
    if (j < 0 || !active) continue;
    __threadfence();     // the other blocks' pieces, seen through the count
    const int s0 = seg_off[j], s1 = seg_off[j + 1];
    const int c0 = s0 / kSegChunk, c1 = (s1 - 1) / kSegChunk;
    // chunk c0's piece is its last segment (side 1) unless the segment starts
    // the chunk (side 0); every later chunk's piece is its first (side 0)
    const int side = (s0 == c0 * kSegChunk) ? 0 : 1;
    float v[kSegVec];
    const float4* a = reinterpret_cast<const float4*>(part + int64_t(2 * c0 + side) * F + f);
    float4 x = __ldcg(a), y = __ldcg(a + 1);
    v[0] = x.x; v[1] = x.y; v[2] = x.z; v[3] = x.w;
    v[4] = y.x; v[5] = y.y; v[6] = y.z; v[7] = y.w;
    for (int cc = c0 + 1; cc <= c1; ++cc) {
      a = reinterpret_cast<const float4*>(part + int64_t(2 * cc) * F + f);
      x = __ldcg(a);
      y = __ldcg(a + 1);
      v[0] += x.x; v[1] += x.y; v[2] += x.z; v[3] += x.w;
      v[4] += y.x; v[5] += y.y; v[6] += y.z; v[7] += y.w;
    }
    store8(dE + int64_t(j) * F + f, v);
  }
}

size_t seg_reduce_workspace(int T, int F) {
  const int64_t chunks = (int64_t(T) + kSegChunk - 1) / kSegChunk;
  return size_t(chunks) * 2 * size_t(F) * sizeof(float);
}

size_t seg_counter_bytes(int T, int F) {
  const int64_t chunks = (int64_t(T) + kSegChunk - 1) / kSegChunk;
  const int64_t slices = (int64_t(F) + kSegSlice - 1) / kSegSlice;
  return (size_t(chunks * slices) * sizeof(int32_t) + 255) & ~size_t(255);
}

staple_status launch_seg_reduce(bool bf16, const void* dh, int64_t ld, const int32_t* sorted_pos,
                                const int32_t* inverse, const int32_t* seg_off,
                                const int32_t* U_dev, int T, int F, float* dE, float* part,
                                int32_t* counters, cudaStream_t st) {
  (void)U_dev;
  if (T == 0) return STAPLE_OK;
  const int chunks = (T + kSegChunk - 1) / kSegChunk;
  const dim3 grid(chunks, (F + kSegSlice - 1) / kSegSlice);
  if (bf16)
    STP_LAUNCH("k8_seg_reduce", st,
               seg_reduce_kernel<true><<<grid, kSegThreads, 0, st>>>(
                   dh, ld, sorted_pos, inverse, seg_off, T, F, dE, part, counters));
  else
    STP_LAUNCH("k8_seg_reduce", st,
               seg_reduce_kernel<false><<<grid, kSegThreads, 0, st>>>(
                   dh, ld, sorted_pos, inverse, seg_off, T, F, dE, part, counters));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// ---------------------------------------------------------------------------
// Table-gradient return to host memory: the U rows only, U read on the device
// ---------------------------------------------------------------------------

// Rows [0, U) of dE (fp32, F floats per row) to mapped host memory with
// 16-byte loads and stores.  Stores to host memory are posted writes over the
// host link, so a grid that keeps many in flight runs at the link's rate.
// Block 0 also writes the U ids and U itself.
__global__ void __launch_bounds__(256)
    grad_to_host_kernel(const float* __restrict__ dE, const int32_t* __restrict__ unique,
                        const int32_t* __restrict__ U_dev, int F, int cap, float* host_dE,
                        int32_t* host_unique, int32_t* host_U) {
  const int U = min(*U_dev, cap);
  const int64_t vecs = int64_t(U) * (F / 4);
  const float4* src = reinterpret_cast<const float4*>(dE);
  float4* dst = reinterpret_cast<float4*>(host_dE);
  for (int64_t v = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; v < vecs;
       v += int64_t(gridDim.x) * blockDim.x)
    dst[v] = __ldcs(src + v);
  if (blockIdx.x == 0) {
    for (int j = threadIdx.x; j < U; j += blockDim.x) host_unique[j] = unique[j];
    if (threadIdx.x == 0) *host_U = U;
  }
}

staple_status launch_grad_to_host(const float* dE, const int32_t* unique, const int32_t* U_dev,
                                  int F, int cap, float* host_dE, int32_t* host_unique,
                                  int32_t* host_U, int num_sms, cudaStream_t st) {
  if (cap == 0) return STAPLE_OK;
  STP_LAUNCH("k12_grad_to_host", st,
             grad_to_host_kernel<<<2 * num_sms, 256, 0, st>>>(dE, unique, U_dev, F, cap, host_dE,
                                                              host_unique, host_U));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

}  // namespace stp
