// Retrieval path of the STAPLE layer on sm_100a: token dedup (K1), cache
// probe (K2), hit gather from the HBM cache (K3), miss gather straight from
// mapped host memory (K4), and the cache build's hash fill.
//
// Paper: thelatestinai listing of arXiv 2610.12599, retrieval-path table
// (dedup the batch once and reuse the inverse map in every augmented layer;
// probe the GPU cache; on a miss read the row from CUDA-registered host
// memory with no CPU gather); AI Radio episode, paper summary (only the U
// active rows are materialised on the GPU).
#include <atomic>

#include "common.cuh"
#include "internal.h"

namespace stp {

// ---------------------------------------------------------------------------
// K1: dedup.  One block of 1024 threads.
//
// Each token becomes one word (id << pos_bits) | position.  A stable LSD
// radix sort over the id bits (8-bit digits) leaves the words ordered by
// (id, position).  Each warp owns a contiguous chunk of the array; digits are
// ranked inside a warp with __match_any_sync, and per-warp digit counts give
// every warp its scatter offsets, so the order is deterministic.  Runs of
// equal ids are then found with warp ballots and a block scan.
// ---------------------------------------------------------------------------
constexpr int kDedupThreads = 1024;
constexpr int kDedupWarps = kDedupThreads / 32;
constexpr int kRadix = 256;

template <typename W, int IPL>
__global__ void __launch_bounds__(kDedupThreads, 1)
    dedup_kernel(const int32_t* __restrict__ ids, int T, int64_t V, int key_bits, int pos_bits,
                 int32_t* __restrict__ unique, int32_t* __restrict__ inverse,
                 int32_t* __restrict__ seg_off, int32_t* __restrict__ sorted_pos,
                 int32_t* __restrict__ U_dev, int32_t* err) {
  extern __shared__ uint8_t smem_raw[];
  int32_t* hist = reinterpret_cast<int32_t*>(smem_raw);              // [warps][256]
  int32_t* wsum = hist + kDedupWarps * kRadix;                        // [32]
  W* buf = reinterpret_cast<W*>(smem_raw + (kDedupWarps * kRadix + 64) * sizeof(int32_t));

  const int tid = threadIdx.x;
  const int warp = tid >> 5;
  const int lane = tid & 31;
  const uint32_t lt_mask = (1u << lane) - 1u;
  const int chunk = IPL * 32;   // elements per warp
  const int wbase = warp * chunk;

  for (int i = tid; i < T; i += kDedupThreads) {
    int64_t id = ids[i];
    if (id < 0 || id >= V) {
      report(err, STAPLE_EIDRANGE);
      id = 0;
    }
    buf[i] = (W(id) << pos_bits) | W(i);
  }
  __syncthreads();

  for (int shift = 0; shift < key_bits; shift += 8) {
    const int sh = pos_bits + shift;
    W r[IPL];
#pragma unroll
    for (int it = 0; it < IPL; ++it) {
      const int idx = wbase + it * 32 + lane;
      r[it] = idx < T ? buf[idx] : W(0);
    }
    for (int d = lane; d < kRadix; d += 32) hist[warp * kRadix + d] = 0;
    __syncwarp();
#pragma unroll
    for (int it = 0; it < IPL; ++it) {
      const int idx = wbase + it * 32 + lane;
      const bool valid = idx < T;
      const uint32_t d = valid ? uint32_t((r[it] >> sh) & 0xFF) : 0x100u;
      const uint32_t peers = __match_any_sync(0xffffffffu, d);
      if (valid && lane == __ffs(peers) - 1) atomicAdd(&hist[warp * kRadix + d], __popc(peers));
    }
    __syncthreads();
    // Digit offsets: exclusive over warps within a digit (column scan), plus
    // the exclusive scan of the digit totals over the 256 digits.
    int dtotal = 0, dincl = 0;
    if (tid < kRadix) {
      for (int w = 0; w < kDedupWarps; ++w) {
        const int c = hist[w * kRadix + tid];
        hist[w * kRadix + tid] = dtotal;
        dtotal += c;
      }
      dincl = dtotal;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, dincl, o);
        if (lane >= o) dincl += n;
      }
      if (lane == 31) wsum[warp] = dincl;
    }
    __syncthreads();
    if (tid < kRadix) {
      int dbase = dincl - dtotal;
      for (int w = 0; w < warp; ++w) dbase += wsum[w];
      for (int w = 0; w < kDedupWarps; ++w) hist[w * kRadix + tid] += dbase;
    }
    __syncthreads();
#pragma unroll
    for (int it = 0; it < IPL; ++it) {
      const int idx = wbase + it * 32 + lane;
      const bool valid = idx < T;
      const uint32_t d = valid ? uint32_t((r[it] >> sh) & 0xFF) : 0x100u;
      const uint32_t peers = __match_any_sync(0xffffffffu, d);
      if (valid) {
        const int dest = hist[warp * kRadix + d] + __popc(peers & lt_mask);
        buf[dest] = r[it];
      }
      __syncwarp();
      if (valid && lane == __ffs(peers) - 1) hist[warp * kRadix + d] += __popc(peers);
      __syncwarp();
    }
    __syncthreads();
  }

  // Run detection: flag[i] = id(i) != id(i-1); unique index = inclusive count - 1.
  const W pos_mask = (W(1) << pos_bits) - 1;
  int wcount = 0;
#pragma unroll
  for (int it = 0; it < IPL; ++it) {
    const int idx = wbase + it * 32 + lane;
    bool flag = false;
    if (idx < T) flag = idx == 0 || (buf[idx] >> pos_bits) != (buf[idx - 1] >> pos_bits);
    wcount += __popc(__ballot_sync(0xffffffffu, flag));
  }
  if (lane == 0) wsum[warp] = wcount;
  __syncthreads();
  int run = 0;
  for (int w = 0; w < warp; ++w) run += wsum[w];
#pragma unroll
  for (int it = 0; it < IPL; ++it) {
    const int idx = wbase + it * 32 + lane;
    bool flag = false;
    W e = 0;
    if (idx < T) {
      e = buf[idx];
      flag = idx == 0 || (e >> pos_bits) != (buf[idx - 1] >> pos_bits);
    }
    const uint32_t b = __ballot_sync(0xffffffffu, flag);
    if (idx < T) {
      const int u = run + __popc(b & (lt_mask | (1u << lane))) - 1;
      const int pos = int(e & pos_mask);
      sorted_pos[idx] = pos;
      inverse[pos] = u;
      if (flag) {
        unique[u] = int32_t(e >> pos_bits);
        seg_off[u] = idx;
      }
    }
    run += __popc(b);
  }
  if (tid == 0) {
    int U = 0;
    for (int w = 0; w < kDedupWarps; ++w) U += wsum[w];
    *U_dev = U;
    seg_off[U] = T;
  }
}

static int bits_for(int64_t n) {  // bits needed to represent values in [0, n)
  int b = 0;
  while ((int64_t(1) << b) < n) ++b;
  return b;
}

template <typename W, int IPL>
static cudaError_t launch_dedup_t(const int32_t* ids, int T, int64_t V, int key_bits,
                                  int pos_bits, int32_t* unique, int32_t* inverse,
                                  int32_t* seg_off, int32_t* sorted_pos, int32_t* U_dev,
                                  int32_t* err, cudaStream_t st) {
  const size_t smem = (kDedupWarps * kRadix + 64) * sizeof(int32_t) + size_t(T) * sizeof(W);
  auto k = dedup_kernel<W, IPL>;
  // opt in to the largest shared-memory size once per device and instantiation
  static std::atomic<uint64_t> attr_done{0};
  int dev = 0;
  cudaGetDevice(&dev);
  const uint64_t bit = uint64_t(1) << (dev & 63);
  if (!(attr_done.load() & bit)) {
    const int max_smem = (kDedupWarps * kRadix + 64) * int(sizeof(int32_t)) + kMaxDedupT * int(sizeof(W));
    cudaError_t e = cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         max_smem < 227 * 1024 ? max_smem : 227 * 1024);
    if (e != cudaSuccess) return e;
    attr_done.fetch_or(bit);
  }
  STP_LAUNCH("k1_dedup", st,
             k<<<1, kDedupThreads, smem, st>>>(ids, T, V, key_bits, pos_bits, unique, inverse,
                                                seg_off, sorted_pos, U_dev, err));
  return cudaGetLastError();
}

staple_status launch_dedup(const int32_t* ids, int T, int64_t V, int32_t* unique,
                           int32_t* inverse, int32_t* seg_off, int32_t* sorted_pos,
                           int32_t* U_dev, int32_t* err, cudaStream_t st) {
  if (T > kMaxDedupT) return STAPLE_EUNSUPPORTED;
  const int key_bits = bits_for(V);
  const int pos_bits = bits_for(T > 1 ? T : 2);
  const int ipl_needed = (T + kDedupThreads - 1) / kDedupThreads;
  cudaError_t e;
  const bool narrow = key_bits + pos_bits <= 32;
  if (!narrow && T > 16384) return STAPLE_EUNSUPPORTED;
#define STP_DEDUP(IPL)                                                                        \
  (narrow ? launch_dedup_t<uint32_t, IPL>(ids, T, V, key_bits, pos_bits, unique, inverse,     \
                                          seg_off, sorted_pos, U_dev, err, st)                \
          : launch_dedup_t<uint64_t, IPL>(ids, T, V, key_bits, pos_bits, unique, inverse,     \
                                          seg_off, sorted_pos, U_dev, err, st))
  if (ipl_needed <= 1)
    e = STP_DEDUP(1);
  else if (ipl_needed <= 4)
    e = STP_DEDUP(4);
  else if (ipl_needed <= 16)
    e = STP_DEDUP(16);
  else
    e = STP_DEDUP(32);
#undef STP_DEDUP
  return e == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// ---------------------------------------------------------------------------
// K2: cache probe.  One block; slot[j] for every distinct id, and the miss
// list in `unique` order (a block-wide ballot scan keeps it deterministic).
// Hash: open addressing, linear probing, capacity a power of two.
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t hash_id(int32_t id, uint32_t mask) {
  return (uint32_t(id) * 2654435761u) & mask;
}

__global__ void __launch_bounds__(1024)
    probe_kernel(const int32_t* __restrict__ unique, const int32_t* __restrict__ U_dev,
                 const int32_t* __restrict__ hkeys, const int32_t* __restrict__ hvals,
                 uint32_t hmask, int32_t* __restrict__ slot, int32_t* __restrict__ miss_list,
                 int32_t* __restrict__ miss_count) {
  __shared__ int32_t wtot[32];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int U = *U_dev;
  int run = 0;
  for (int base = 0; base < U; base += 1024) {
    const int j = base + tid;
    int32_t s = -1;
    if (j < U && hkeys != nullptr) {
      const int32_t id = unique[j];
      uint32_t h = hash_id(id, hmask);
      for (uint32_t probes = 0; probes <= hmask; ++probes) {
        const int32_t k = hkeys[h];
        if (k == id) {
          s = hvals[h];
          break;
        }
        if (k < 0) break;
        h = (h + 1) & hmask;
      }
    }
    if (j < U) slot[j] = s;
    const bool miss = j < U && s < 0;
    const uint32_t b = __ballot_sync(0xffffffffu, miss);
    if (lane == 0) wtot[warp] = __popc(b);
    __syncthreads();
    int before = run;
    int total = 0;
    for (int w = 0; w < 32; ++w) {
      if (w < warp) before += wtot[w];
      total += wtot[w];
    }
    if (miss) miss_list[before + __popc(b & ((1u << lane) - 1u))] = j;
    run += total;
    __syncthreads();
  }
  if (tid == 0) *miss_count = run;
}

// ---------------------------------------------------------------------------
// K3 / K4: row copies.  One warp per row, 16-byte vector loads, several in
// flight per thread.  K3 copies hit rows from the cache; K4 reads miss rows
// from the table (mapped host memory, or HBM for a device table).
// ---------------------------------------------------------------------------
enum GatherMode { G_HITS = 0, G_MISSES = 1, G_LIST = 2, G_REFRESH = 3, G_SCATTER = 4 };

// A warp copies a row, or, when there are fewer rows than warps, a 2 KB
// chunk of one (its four 16-byte loads per lane), in row-major order: with a
// few long rows (a decode step's misses, 88 KB each for four grouped 7B
// layers) every warp of the grid then has one in flight, where one warp per
// row would leave most of them idle and walk each row one round trip at a
// time.  With many rows (a training batch's misses) each warp keeps its own
// row: over the host link many rows in flight at once read faster than the
// same bytes a few rows at a time.
constexpr int kChunkVecs = 128;

template <int MODE>
__global__ void __launch_bounds__(256)
    gather_kernel(const uint8_t* __restrict__ src, int64_t src_pitch,
                  const int32_t* __restrict__ ids, const int32_t* __restrict__ count_dev,
                  const int32_t* __restrict__ slot, const int32_t* __restrict__ miss_list,
                  uint8_t* __restrict__ rows, int64_t row_bytes) {
  const int lane = threadIdx.x & 31;
  const int gw = (blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int nw = (gridDim.x * blockDim.x) >> 5;
  const int n = *count_dev;
  const int64_t vecs = row_bytes / 16;
  const int64_t cv = n < nw ? kChunkVecs : vecs;   // 16-byte vectors per work item
  const int64_t cpr = (vecs + cv - 1) / cv;        // work items per row
  const int64_t items = int64_t(n) * cpr;
  for (int64_t it = gw; it < items; it += nw) {
    const int i = int(it / cpr);
    const int64_t c0 = (it - int64_t(i) * cpr) * cv;
    int j;
    int64_t srow;
    if (MODE == G_HITS) {          // rows[j] = cache[slot[j]] for hits
      j = i;
      srow = slot[j];
      if (srow < 0) continue;
    } else if (MODE == G_MISSES) { // rows[j] = table[unique[j]], j from the miss list
      j = miss_list[i];
      srow = ids[j];
    } else if (MODE == G_SCATTER) { // rows[miss_list[i]] = staging[i]
      j = miss_list[i];
      srow = i;
    } else if (MODE == G_REFRESH) { // cache[slot[j]] = table[ids[j]] for cached ids
      if (slot[i] < 0) continue;
      j = slot[i];
      srow = ids[i];
    } else {                       // rows[i] = table[ids[i]]
      j = i;
      srow = ids[i];
    }
    const uint4* sp = reinterpret_cast<const uint4*>(src + srow * src_pitch);
    uint4* dp = reinterpret_cast<uint4*>(rows + int64_t(j) * row_bytes);
    const int64_t vend = c0 + cv < vecs ? c0 + cv : vecs;
    int64_t v = c0 + lane;
    for (; v + 96 < vend; v += 128) {
      const uint4 a0 = sp[v], a1 = sp[v + 32], a2 = sp[v + 64], a3 = sp[v + 96];
      dp[v] = a0;
      dp[v + 32] = a1;
      dp[v + 64] = a2;
      dp[v + 96] = a3;
    }
    for (; v < vend; v += 32) dp[v] = sp[v];
  }
}

staple_status launch_probe(const int32_t* unique, const int32_t* U_dev, const int32_t* hkeys,
                           const int32_t* hvals, uint32_t hmask, int32_t* slot,
                           int32_t* miss_list, int32_t* miss_count, cudaStream_t st) {
  STP_LAUNCH("k2_probe", st,
             probe_kernel<<<1, 1024, 0, st>>>(unique, U_dev, hkeys, hvals, hmask, slot, miss_list,
                                              miss_count));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

staple_status launch_gather_hits(const void* cache_rows, int64_t row_bytes, const int32_t* U_dev,
                                 const int32_t* slot, void* rows, int num_sms, cudaStream_t st) {
  STP_LAUNCH("k3_gather_hits", st,
             gather_kernel<G_HITS><<<num_sms * 2, 256, 0, st>>>(
                 static_cast<const uint8_t*>(cache_rows), row_bytes, nullptr, U_dev, slot,
                 nullptr, static_cast<uint8_t*>(rows), row_bytes));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

staple_status launch_gather_misses(const void* table_dev, int64_t table_pitch_bytes,
                                   int64_t row_bytes, const int32_t* unique,
                                   const int32_t* miss_list, const int32_t* miss_count,
                                   void* rows, int num_sms, bool host_table, cudaStream_t st) {
  // Over the host link a quarter of the SMs' worth of warps (each with 2 KB
  // of loads in flight) already keeps far more in flight than the link's
  // bandwidth-delay product; more only takes thread slots from kernels that
  // run beside the gather.  A table in HBM gets every SM.
  const int grid = host_table ? (num_sms + 3) / 4 : num_sms;
  STP_LAUNCH("k4_gather_misses", st,
             gather_kernel<G_MISSES><<<grid, 256, 0, st>>>(
                 static_cast<const uint8_t*>(table_dev), table_pitch_bytes, unique, miss_count,
                 nullptr, miss_list, static_cast<uint8_t*>(rows), row_bytes));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// Miss rows that arrived packed in miss order (bulk path): staging row i goes
// to rows[miss_list[i]].
staple_status launch_scatter_misses(const void* staging, int64_t row_bytes,
                                    const int32_t* miss_list, const int32_t* miss_count,
                                    void* rows, int num_sms, cudaStream_t st) {
  STP_LAUNCH("k4b_scatter_misses", st,
             gather_kernel<G_SCATTER><<<num_sms * 2, 256, 0, st>>>(
                 static_cast<const uint8_t*>(staging), row_bytes, nullptr, miss_count, nullptr,
                 miss_list, static_cast<uint8_t*>(rows), row_bytes));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// Cache write-back after a table update: the cached copies of the listed
// distinct ids (slot from the probe, -1 when not cached) are read again from
// the table.
staple_status launch_cache_refresh(const void* table_dev, int64_t table_pitch_bytes,
                                   int64_t row_bytes, const int32_t* unique, const int32_t* slot,
                                   const int32_t* U_dev, void* cache_rows, int num_sms,
                                   cudaStream_t st) {
  STP_LAUNCH("k14_cache_refresh", st,
             gather_kernel<G_REFRESH><<<num_sms, 256, 0, st>>>(
                 static_cast<const uint8_t*>(table_dev), table_pitch_bytes, unique, U_dev, slot,
                 nullptr, static_cast<uint8_t*>(cache_rows), row_bytes));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// Cache build: copy the K hot rows (ids in slot order) into the cache and
// insert id -> slot into the hash (keys start at -1).
__global__ void cache_fill_kernel(const int32_t* __restrict__ hot, int K, int32_t* hkeys,
                                  int32_t* hvals, uint32_t hmask) {
  const int k = blockIdx.x * blockDim.x + threadIdx.x;
  if (k >= K) return;
  const int32_t id = hot[k];
  uint32_t h = hash_id(id, hmask);
  for (uint32_t probes = 0; probes <= hmask; ++probes) {
    const int32_t prev = atomicCAS(&hkeys[h], -1, id);
    if (prev == -1 || prev == id) {
      hvals[h] = k;
      return;
    }
    h = (h + 1) & hmask;
  }
}

staple_status launch_cache_fill(const int32_t* hot, int K, int32_t* hkeys, int32_t* hvals,
                                uint32_t hmask, cudaStream_t st) {
  if (K > 0) cache_fill_kernel<<<(K + 255) / 256, 256, 0, st>>>(hot, K, hkeys, hvals, hmask);
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

// Row copy for the cache build (rows of the table in slot order).
staple_status launch_copy_rows(const void* table_dev, int64_t table_pitch_bytes,
                               int64_t row_bytes, const int32_t* ids, const int32_t* count_dev,
                               void* dst, int num_sms, cudaStream_t st) {
  gather_kernel<G_LIST><<<num_sms, 256, 0, st>>>(
      static_cast<const uint8_t*>(table_dev), table_pitch_bytes, ids, count_dev, nullptr,
      nullptr, static_cast<uint8_t*>(dst), row_bytes);
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

}  // namespace stp
