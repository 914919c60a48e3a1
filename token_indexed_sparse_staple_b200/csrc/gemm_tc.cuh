// Persistent, warp-specialised tcgen05 GEMM for sm_100a with the STAPLE
// epilogues fused in.
//
//   C[M][N] = sum_k A(m, k) * B(n, k)        bf16 operands, fp32 accumulators
//
// A and B are read by TMA into 128-byte-swizzled shared-memory stages.  Each
// operand may be K-major (k contiguous in global memory) or MN-major (m or n
// contiguous), which covers every contraction of the layer's forward and
// backward pass without transposing anything in memory.  The B operand may
// come from two tensors: stacked along N (the gate and up projections share
// one 256-wide tile: columns [0,128) are W_gate rows, [128,256) the matching
// W_up rows) or concatenated along K (dx = dg W_gate + dh W_up).
//
// Block = 6 warps: warp 0 issues TMA, warp 1 allocates tensor memory and
// issues the MMAs (one thread), warps 2..5 drain the accumulators (each warp
// may only touch its 32-lane quarter of tensor memory) and run the epilogue.
// Two 128x256 fp32 accumulators in tensor memory (all 512 columns) let the
// epilogue of one tile overlap the main loop of the next.  Every wait is
// bounded (see mbar_wait): on a timeout the block records STAPLE_ETIMEOUT,
// drains its outstanding copies and releases tensor memory before exiting.
#pragma once

#include "common.cuh"

namespace stp {
namespace tc {

constexpr int BM = 128;
constexpr int BN = 256;
constexpr int BK = 64;
constexpr int STAGES = 4;
constexpr int kThreads = 192;
constexpr int A_STAGE = BM * BK * 2;  // 16 KiB
constexpr int B_STAGE = BN * BK * 2;  // 32 KiB
constexpr int STAGE_BYTES = A_STAGE + B_STAGE;
constexpr int kTmemCols = 512;
constexpr int kSmemBytes = STAGES * STAGE_BYTES + 1024 /*align*/ + 256 /*barriers*/;

enum BSrc { B_ONE = 0, B_NHALF = 1, B_KSPLIT = 2 };
// EPI_GATE_E: the STEM variant of EPI_GATEUP (the row replaces the
// up-projection): the tile is 256 W_gate rows, h = E[row], z = SiLU(g) h.
enum Epi { EPI_BF16 = 0, EPI_F32 = 1, EPI_GATEUP = 2, EPI_DZ = 3, EPI_GATE_E = 4 };

// The heavy epilogues stage every 32-row x 32-column output block of a warp
// in shared memory (64-byte swizzle) and write it with one TMA store: a
// thread holds one accumulator row, so its own stores would each touch a
// different row.  2 KB per block: z, g, h for EPI_GATEUP; for EPI_DZ two
// buffers of two blocks, which take the g and h blocks in (by TMA) and then
// the dg and dh blocks out.
constexpr int kOutBox = 32 * 32 * 2;
template <int EPI>
constexpr int out_blocks() {
  return (EPI == EPI_GATEUP || EPI == EPI_GATE_E) ? 3 : (EPI == EPI_DZ ? 4 : 0);
}
template <int EPI>
constexpr int smem_bytes() { return kSmemBytes + 4 * out_blocks<EPI>() * kOutBox; }

struct Params {
  int32_t M, N, K;            // output rows, output columns (features for GATEUP / DZ), K
  int32_t tiles_m, tiles_n, k_blocks;
  // EPI_F32: the last nsplit tiles (raster order) run as two work items each,
  // k blocks [0, kb_split) and [kb_split, k_blocks), which both add their sums
  // (red.add) onto an output the launcher zeroed: the last, partial round of
  // tiles then takes half as long.  0: every tile is one item.
  int32_t nsplit, kb_split;
  int32_t ksplit;             // B_KSPLIT: first k served by the second B tensor
  int32_t group_m;            // tile raster: group_m M-blocks per sweep over N
  // EPI_BF16 / EPI_F32: out[m * ldo + n]; rows m >= m_split go to out2[(m - m_split) * ldo + n]
  void* out;
  void* out2;
  int64_t ldo;
  int32_t m_split;
  // EPI_GATEUP
  uint16_t* z;
  uint16_t* g_save;
  uint16_t* h_save;
  int64_t ldf;                // row pitch of z / g / h (= F)
  const uint16_t* e_base;
  int64_t e_pitch;
  const int32_t* e_index;
  int64_t e_rows;
  int32_t e_mode;             // staple_embed_mode
  // EPI_DZ
  const uint16_t* g_in;
  const uint16_t* h_in;
  uint16_t* dgh;              // [M][2 * ldf]: dg in [0, F), dh in [F, 2F)
  int32_t* err;
  uint64_t wait_ns;           // bound of every wait (STAPLE_ETIMEOUT past it)
};

// Work item t: its tile and k-block range [kb0, kb1); add: a split tile's half.
__device__ __forceinline__ int item_tile(int t, const Params& p, int& kb0, int& kb1, bool& add) {
  const int nfull = p.tiles_m * p.tiles_n - p.nsplit;
  if (t < nfull) {
    kb0 = 0;
    kb1 = p.k_blocks;
    add = false;
    return t;
  }
  const int h = (t - nfull) & 1;
  kb0 = h ? p.kb_split : 0;
  kb1 = h ? p.k_blocks : p.kb_split;
  add = true;
  return nfull + ((t - nfull) >> 1);
}

__device__ __forceinline__ void red_add4(float* a, float x, float y, float z, float w) {
  asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};" ::"l"(a), "f"(x), "f"(y), "f"(z),
               "f"(w)
               : "memory");
}

__device__ __forceinline__ void tile_coords(int t, const Params& p, int& mb, int& nb) {
  const int per_group = p.group_m * p.tiles_n;
  const int g = t / per_group;
  const int first_m = g * p.group_m;
  const int rows = min(p.group_m, p.tiles_m - first_m);
  const int r = t - g * per_group;
  mb = first_m + r % rows;
  nb = r / rows;
}

// --------------------------------------------------------------------------
// Epilogue helpers (one thread = one accumulator row, 32 columns per load)
// --------------------------------------------------------------------------
__device__ __forceinline__ void store_bf16x32(uint16_t* dst, const float* v) {
  uint4* d = reinterpret_cast<uint4*>(dst);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    uint4 w;
    w.x = pack_bf2(v[8 * i + 0], v[8 * i + 1]);
    w.y = pack_bf2(v[8 * i + 2], v[8 * i + 3]);
    w.z = pack_bf2(v[8 * i + 4], v[8 * i + 5]);
    w.w = pack_bf2(v[8 * i + 6], v[8 * i + 7]);
    d[i] = w;
  }
}

// 32 bf16 values as four 16-byte words: the loads are issued here and only
// waited for where the words are first used, so a chunk's loads can be in
// flight while the previous chunk is computed.
__device__ __forceinline__ void load_raw32(const uint16_t* src, uint4 (&w)[4]) {
  const uint4* s = reinterpret_cast<const uint4*>(src);
#pragma unroll
  for (int i = 0; i < 4; ++i) w[i] = __ldg(s + i);
}
__device__ __forceinline__ void unpack32(const uint4 (&w)[4], float* v) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    v[8 * i + 0] = bf_lo(w[i].x);
    v[8 * i + 1] = bf_hi(w[i].x);
    v[8 * i + 2] = bf_lo(w[i].y);
    v[8 * i + 3] = bf_hi(w[i].y);
    v[8 * i + 4] = bf_lo(w[i].z);
    v[8 * i + 5] = bf_hi(w[i].z);
    v[8 * i + 6] = bf_lo(w[i].w);
    v[8 * i + 7] = bf_hi(w[i].w);
  }
}

// Row r (32 bf16 values) of a 32 x 32 block in the 64-byte-swizzled layout
// the TMA store reads: 16-byte chunk k of row r sits at chunk k ^ ((r/2) % 4).
__device__ __forceinline__ void write_row_sw64(uint8_t* box, int r, const float* v) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    uint4 w;
    w.x = pack_bf2(v[8 * k + 0], v[8 * k + 1]);
    w.y = pack_bf2(v[8 * k + 2], v[8 * k + 3]);
    w.z = pack_bf2(v[8 * k + 4], v[8 * k + 5]);
    w.w = pack_bf2(v[8 * k + 6], v[8 * k + 7]);
    *reinterpret_cast<uint4*>(box + r * 64 + ((k ^ ((r >> 1) & 3)) << 4)) = w;
  }
}

// Row r of a 32 x 32 block in the same layout, as 32 floats.
__device__ __forceinline__ void read_row_sw64(const uint8_t* box, int r, float* v) {
#pragma unroll
  for (int k = 0; k < 4; ++k) {
    const uint4 w = *reinterpret_cast<const uint4*>(box + r * 64 + ((k ^ ((r >> 1) & 3)) << 4));
    v[8 * k + 0] = bf_lo(w.x);
    v[8 * k + 1] = bf_hi(w.x);
    v[8 * k + 2] = bf_lo(w.y);
    v[8 * k + 3] = bf_hi(w.y);
    v[8 * k + 4] = bf_lo(w.z);
    v[8 * k + 5] = bf_hi(w.z);
    v[8 * k + 6] = bf_lo(w.w);
    v[8 * k + 7] = bf_hi(w.w);
  }
}

// Tensor maps of the staged blocks (box 32 x 32): the outputs (EPI_GATEUP:
// z, g, h; EPI_DZ: dg, dh) and, for EPI_DZ, the inputs g and h in m[2], m[3].
struct OutMaps {
  const CUtensorMap* m[4];
};

// EPI_DZ input stream of one epilogue warp: chunk k (counted over all of the
// warp's tiles) lands in buffer k & 1, on bar[k & 1].
struct DzIn {
  uint64_t* bar;          // [2]
  volatile int* abort;    // the block's abort flag
  uint32_t next;          // chunks issued so far
  uint32_t done;          // chunks consumed so far
  bool ok;                // false once a wait gave up
};

// Lane 0 waits until the warp's previous block stores have read the staging
// buffer; then the whole warp may write it again.
__device__ __forceinline__ void stage_begin(int lane) {
  if (lane == 0) bulk_wait_read0();
  __syncwarp();
}
// Make the staged rows visible to TMA, then lane 0 stores the n blocks.
__device__ __forceinline__ void stage_store(int lane, uint8_t* stg, const OutMaps& om,
                                            const bool (&use)[3], int col, int row0) {
  fence_async_smem();
  __syncwarp();
  if (lane == 0) {
#pragma unroll
    for (int b = 0; b < 3; ++b)
      if (use[b]) tma_store_2d(om.m[b], stg + b * kOutBox, col, row0);
    bulk_commit();
  }
}

// m = this thread's accumulator row; lane = m % 32; stg = the warp's staging
// blocks (EPI_GATEUP, EPI_DZ).
// EPI_DZ: lane 0 issues the g and h blocks of chunk c (columns f, rows from
// row0) of a tile into the warp's next input buffer.
__device__ __forceinline__ void dz_load(DzIn& in, uint8_t* stg, const OutMaps& om, int f,
                                        int row0) {
  const int b = int(in.next & 1u);
  uint8_t* buf = stg + b * 2 * kOutBox;
  mbar_arrive_expect_tx(&in.bar[b], 2 * kOutBox);
  tma_load_2d(om.m[2], &in.bar[b], buf, f, row0);
  tma_load_2d(om.m[3], &in.bar[b], buf + kOutBox, f, row0);
  ++in.next;
}

// Chunks of 32 features of tile column nb with f < N.
__device__ __forceinline__ int dz_chunks(const Params& p, int nb) {
  return min(BN / 32, (p.N - nb * BN + 31) / 32);
}


// nxt_nb / nxt_row0: the warp's next tile (nxt_nb < 0: none), whose first
// input chunk an EPI_DZ warp requests during this tile's last chunk.
template <int EPI>
__device__ __forceinline__ void epilogue_tile(const Params& p, uint32_t tacc, int m, int nb,
                                              int lane, uint8_t* stg, const OutMaps& om,
                                              DzIn& in, int nxt_nb, int nxt_row0, bool add) {
  const bool row_ok = m < p.M;
  const int m0w = m - lane;   // the warp's first row
  if constexpr (EPI == EPI_BF16 || EPI == EPI_F32) {
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint32_t r[32];
      tmem_ld32(tacc + c * 32, r);
      tmem_ld_wait(r);
      const int n = nb * BN + c * 32;
      if (row_ok && n < p.N) {
        float v[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
        if constexpr (EPI == EPI_BF16) {
          store_bf16x32(static_cast<uint16_t*>(p.out) + int64_t(m) * p.ldo + n, v);
        } else {
          float* base = m < p.m_split
                            ? static_cast<float*>(p.out) + int64_t(m) * p.ldo
                            : static_cast<float*>(p.out2) + int64_t(m - p.m_split) * p.ldo;
          if (add) {
#pragma unroll
            for (int i = 0; i < 8; ++i)
              red_add4(base + n + 4 * i, v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          } else {
            float4* d = reinterpret_cast<float4*>(base + n);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              d[i] = make_float4(v[4 * i], v[4 * i + 1], v[4 * i + 2], v[4 * i + 3]);
          }
        }
      }
    }
  } else if constexpr (EPI == EPI_GATEUP) {
    // Accumulator columns [0,128): g for features f0..f0+127; [128,256): u.
    const uint16_t* erow = nullptr;
    if (row_ok && p.e_mode != STAPLE_EMBED_NONE) {
      const int64_t idx = p.e_index[m];
      if (idx < 0 || idx >= p.e_rows) {
        report(p.err, STAPLE_EIDRANGE);
      } else {
        erow = p.e_base + idx * p.e_pitch;
      }
    }
    const int f0 = nb * (BN / 2);
    // the E row's chunk c+1 is loaded while chunk c is computed
    uint4 ew[4] = {};
    if (erow && row_ok && f0 < p.N) load_raw32(erow + f0, ew);
#pragma unroll 1
    for (int c = 0; c < BN / 64; ++c) {
      uint4 ec[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ec[i] = ew[i];
      const int f = f0 + c * 32;
      if (erow && row_ok && c + 1 < BN / 64 && f + 32 < p.N) load_raw32(erow + f + 32, ew);
      uint32_t rg[32], ru[32];
      tmem_ld32(tacc + c * 32, rg);
      tmem_ld32(tacc + BN / 2 + c * 32, ru);
      tmem_ld_wait(rg);
      reg_fence(ru);
      if (f < p.N) {   // the same for the whole warp
        // rows past M are staged too; the TMA store leaves them out
        float e[32];
        unpack32(ec, e);   // zeros when the layer has no table
        float g[32], h[32], z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          g[i] = __uint_as_float(rg[i]);
          h[i] = __uint_as_float(ru[i]) + e[i];
          z[i] = g[i] * sigmoid_f(g[i]) * h[i];
        }
        const bool use[3] = {true, p.g_save != nullptr, p.h_save != nullptr};
        stage_begin(lane);
        write_row_sw64(stg, lane, z);
        if (use[1]) write_row_sw64(stg + kOutBox, lane, g);
        if (use[2]) write_row_sw64(stg + 2 * kOutBox, lane, h);
        stage_store(lane, stg, om, use, f, m0w);
      }
    }
  } else if constexpr (EPI == EPI_GATE_E) {
    // Accumulator columns [0,256): g for features f0..f0+255; h is the row.
    const uint16_t* erow = nullptr;
    if (row_ok && p.e_mode != STAPLE_EMBED_NONE) {
      const int64_t idx = p.e_index[m];
      if (idx < 0 || idx >= p.e_rows) {
        report(p.err, STAPLE_EIDRANGE);
      } else {
        erow = p.e_base + idx * p.e_pitch;
      }
    }
    const int f0 = nb * BN;
    // the row's chunk c+1 is loaded while chunk c is computed
    uint4 ew[4] = {};
    if (erow && f0 < p.N) load_raw32(erow + f0, ew);
#pragma unroll 1
    for (int c = 0; c < BN / 32; ++c) {
      uint4 ec[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) ec[i] = ew[i];
      const int f = f0 + c * 32;
      if (erow && c + 1 < BN / 32 && f + 32 < p.N) load_raw32(erow + f + 32, ew);
      uint32_t rg[32];
      tmem_ld32(tacc + c * 32, rg);
      tmem_ld_wait(rg);
      if (f < p.N) {   // the same for the whole warp
        float e[32];
        unpack32(ec, e);
        float g[32], z[32];
#pragma unroll
        for (int i = 0; i < 32; ++i) {
          g[i] = __uint_as_float(rg[i]);
          z[i] = g[i] * sigmoid_f(g[i]) * e[i];
        }
        const bool use[3] = {true, p.g_save != nullptr, p.h_save != nullptr};
        stage_begin(lane);
        write_row_sw64(stg, lane, z);
        if (use[1]) write_row_sw64(stg + kOutBox, lane, g);
        if (use[2]) write_row_sw64(stg + 2 * kOutBox, lane, e);
        stage_store(lane, stg, om, use, f, m0w);
      }
    }
  } else {  // EPI_DZ: accumulator = dz for features [nb*256, nb*256 + 256)
    // g and h arrive as 32 x 32 blocks by TMA (rows past M zero-filled) into
    // two buffers: chunk c+1's (or the next tile's first chunk) is requested
    // while chunk c is computed.  dg and dh are then staged in the buffer
    // chunk c came in (each lane reads and writes only its own row) and
    // stored by TMA.  Before a buffer is loaded again, lane 0 waits until the
    // stores of the chunk it last held have read it.  (Sending the next
    // tile's blocks to L2 ahead of time, or the current tile's at its start,
    // measured slower.)
    (void)m;
    const int nch = dz_chunks(p, nb);
#pragma unroll 1
    for (int c = 0; c < nch; ++c) {
      const int f = nb * BN + c * 32;
      const int b = int(in.done & 1u);
      uint8_t* buf = stg + b * 2 * kOutBox;
      const bool ok = mbar_wait(&in.bar[b], (in.done >> 1) & 1u, in.abort, p.err, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) {
        in.ok = false;
        return;
      }
      ++in.done;
      float g[32], h[32];
      read_row_sw64(buf, lane, g);
      read_row_sw64(buf + kOutBox, lane, h);
      uint32_t r[32];
      tmem_ld32(tacc + c * 32, r);
      tmem_ld_wait(r);
      float dg[32], dh[32];
#pragma unroll
      for (int i = 0; i < 32; ++i) {
        const float dz = __uint_as_float(r[i]);
        const float s = sigmoid_f(g[i]);
        dh[i] = dz * g[i] * s;
        dg[i] = dz * h[i] * (s * (1.0f + g[i] * (1.0f - s)));
      }
      if (lane == 0) {
        bulk_wait_read0();   // the other buffer's last stores have read it
        if (c + 1 < nch) dz_load(in, stg, om, f + 32, m0w);
        else if (nxt_nb >= 0) dz_load(in, stg, om, nxt_nb * BN, nxt_row0);
      }
      write_row_sw64(buf, lane, dg);
      write_row_sw64(buf + kOutBox, lane, dh);
      const bool use[3] = {true, true, false};
      stage_store(lane, buf, om, use, f, m0w);
    }
  }
}

// --------------------------------------------------------------------------
// The kernel
// --------------------------------------------------------------------------
template <bool A_MN, bool B_MN, int BSRC, int EPI>
__global__ void __launch_bounds__(kThreads, 1)
    gemm_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB0,
                const __grid_constant__ CUtensorMap tmB1, const __grid_constant__ CUtensorMap tmO0,
                const __grid_constant__ CUtensorMap tmO1, const __grid_constant__ CUtensorMap tmO2,
                const __grid_constant__ CUtensorMap tmO3, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  uint8_t* sA = smem;
  uint8_t* sB = smem + STAGES * A_STAGE;
  uint8_t* s_out = sB + STAGES * B_STAGE;  // [4 warps][out_blocks][32][32] bf16, swizzled
  uint64_t* full = reinterpret_cast<uint64_t*>(s_out + 4 * out_blocks<EPI>() * kOutBox);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;
  uint64_t* tempty = tfull + 2;
  uint64_t* dbar = tempty + 2;   // MMA drain before tensor memory is freed
  uint64_t* in_bar = dbar + 1;   // [4 warps][2]: EPI_DZ input blocks landed
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(in_bar + 8);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
#pragma unroll
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(&tfull[0], 1);
    mbar_init(&tfull[1], 1);
    mbar_init(&tempty[0], 4);
    mbar_init(&tempty[1], 4);
    mbar_init(dbar, 1);
    if (EPI == EPI_DZ)
      for (int i = 0; i < 8; ++i) mbar_init(&in_bar[i], 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB0);
    if (BSRC != B_ONE) tma_prefetch_desc(&tmB1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  const int ntiles = p.tiles_m * p.tiles_n;
  const int nitems = ntiles + p.nsplit;   // work items (a split tile is two)

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      int issued = 0;
      for (int t = blockIdx.x; t < nitems && ok; t += gridDim.x) {
        int mb, nb, kb0, kb1;
        bool add;
        tile_coords(item_tile(t, p, kb0, kb1, add), p, mb, nb);
        const int m0 = mb * BM;
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          uint64_t* bar = &full[stage];
          mbar_arrive_expect_tx(bar, STAGE_BYTES);
          uint8_t* a = sA + stage * A_STAGE;
          uint8_t* b = sB + stage * B_STAGE;
          const int k0 = kb * BK;
          if (A_MN) {
            tma_load_2d(&tmA, bar, a, m0, k0);
            tma_load_2d(&tmA, bar, a + A_STAGE / 2, m0 + 64, k0);
          } else {
            tma_load_2d(&tmA, bar, a, k0, m0);
          }
          if (BSRC == B_NHALF) {
            const int n0 = nb * (BN / 2);
            tma_load_2d(&tmB0, bar, b, k0, n0);
            tma_load_2d(&tmB1, bar, b + B_STAGE / 2, k0, n0);
          } else {
            const CUtensorMap* mp = &tmB0;
            int kk = k0;
            if (BSRC == B_KSPLIT && k0 >= p.ksplit) {
              mp = &tmB1;
              kk = k0 - p.ksplit;
            }
            const int n0 = nb * BN;
            if (B_MN) {
#pragma unroll
              for (int i = 0; i < 4; ++i) tma_load_2d(mp, bar, b + i * (B_STAGE / 4), n0 + 64 * i, kk);
            } else {
              tma_load_2d(mp, bar, b, kk, n0);
              tma_load_2d(mp, bar, b + B_STAGE / 2, kk, n0 + 128);
            }
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
      }
      // Let the copies still in flight land before the block goes away (on
      // the normal path every fill was consumed and this returns at once).
      drain_ring(full, STAGES, stage, phase, issued);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, BN, A_MN, B_MN);
      int stage = 0;
      uint32_t phase = 0;
      int iter = 0;
      bool ok = true;
      for (int t = blockIdx.x; t < nitems && ok; t += gridDim.x, ++iter) {
        const int buf = iter & 1;
        const uint32_t use = uint32_t(iter >> 1);
        if (!mbar_wait(&tempty[buf], (use & 1) ^ 1, abort_flag, p.err, p.wait_ns)) break;
        tc_fence_after();
        const uint32_t dacc = tmem_base + uint32_t(buf * BN);
        int kb0, kb1;
        bool add;
        item_tile(t, p, kb0, kb1, add);
        for (int kb = kb0; kb < kb1; ++kb) {
          if (!mbar_wait(&full[stage], phase, abort_flag, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a_addr = smem_u32(sA + stage * A_STAGE);
          const uint32_t b_addr = smem_u32(sB + stage * B_STAGE);
#pragma unroll
          for (int k = 0; k < BK / 16; ++k) {
            const uint64_t ad = A_MN ? sw128_desc(a_addr + k * 2048, A_STAGE / 2, 1024)
                                     : sw128_desc(a_addr + k * 32, 16, 1024);
            const uint64_t bd = B_MN ? sw128_desc(b_addr + k * 2048, B_STAGE / 4, 1024)
                                     : sw128_desc(b_addr + k * 32, 16, 1024);
            umma_bf16(dacc, ad, bd, idesc, (kb != kb0 || k != 0) ? 1u : 0u);
          }
          umma_commit(&empty[stage]);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1;
          }
        }
        if (ok) umma_commit(&tfull[buf]);
      }
      // Every MMA this thread issued completes before tensor memory and the
      // operand stages are released (after an abort some may still run).
      umma_commit(dbar);
      mbar_drain(dbar, 0);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    uint8_t* stg = s_out + q * out_blocks<EPI>() * kOutBox;
    const OutMaps om{{&tmO0, &tmO1, &tmO2, &tmO3}};
    DzIn in{in_bar + 2 * q, abort_flag, 0u, 0u, true};
    if (EPI == EPI_DZ && lane == 0 && int(blockIdx.x) < ntiles) {
      int mb, nb;
      tile_coords(blockIdx.x, p, mb, nb);
      dz_load(in, stg, om, nb * BN, mb * BM + q * 32);   // the first tile's first chunk
    }
    int iter = 0;
    for (int t = blockIdx.x; t < nitems; t += gridDim.x, ++iter) {
      const int buf = iter & 1;
      const uint32_t use = uint32_t(iter >> 1);
      int mb, nb, kb0, kb1;
      bool add;
      tile_coords(item_tile(t, p, kb0, kb1, add), p, mb, nb);
      int nxt_nb = -1, nxt_row0 = 0;
      if (t + int(gridDim.x) < ntiles) {   // (EPI_DZ: no split tiles, items are tiles)
        int mb2;
        tile_coords(t + gridDim.x, p, mb2, nxt_nb);
        nxt_row0 = mb2 * BM + q * 32;
      }
      const bool ok = mbar_wait(&tfull[buf], use & 1, abort_flag, p.err, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf * BN);
      epilogue_tile<EPI>(p, tacc, mb * BM + row, nb, lane, stg, om, in, nxt_nb, nxt_row0, add);
      if (!in.ok) break;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
    // input blocks still in flight (after an abort) land before the shared
    // memory goes away, and so do the block's last staged stores
    if (EPI == EPI_DZ && lane == 0)
      for (uint32_t k = in.done; k < in.next; ++k) mbar_drain(&in.bar[k & 1u], (k >> 1) & 1u);
    if (out_blocks<EPI>() > 0 && lane == 0) bulk_wait0();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, kTmemCols);
  }
}

// Zero the output of the split tiles (EPI_F32), which both halves then add
// onto: block i takes rows 16 (i % 8) .. +15 of split tile i / 8 (256 fp32
// columns), four float4 stores per thread.
constexpr int kZeroRows = 16;
__global__ void __launch_bounds__(256) zero_split_tiles_kernel(const Params p) {
  const int t = p.tiles_m * p.tiles_n - p.nsplit + int(blockIdx.x) / (BM / kZeroRows);
  const int r0 = (int(blockIdx.x) % (BM / kZeroRows)) * kZeroRows;
  int mb, nb;
  tile_coords(t, p, mb, nb);
  for (int i = threadIdx.x; i < kZeroRows * (BN / 4); i += 256) {
    const int m = mb * BM + r0 + i / (BN / 4), n = nb * BN + (i % (BN / 4)) * 4;
    if (m >= p.M || n >= p.N) continue;
    float* base = m < p.m_split ? static_cast<float*>(p.out) + int64_t(m) * p.ldo
                                : static_cast<float*>(p.out2) + int64_t(m - p.m_split) * p.ldo;
    *reinterpret_cast<float4*>(base + n) = make_float4(0.f, 0.f, 0.f, 0.f);
  }
}

}  // namespace tc
}  // namespace stp
