// Decode-shaped tcgen05 GEMMs for the STAPLE layer (few tokens, T <= 256).
//
// With a handful of tokens the layer streams its weights once per step and
// is bound by HBM bandwidth.  The weights therefore take the MMA's M side
// (128 rows per tile) and the tokens its N side (T rounded up to 16), so the
// tensor core works on full tiles and every SM streams its own slice:
//
//   gate/up: C[128][N] = [W_gate rows f0..f0+63 ; W_up rows f0..f0+63] . x^T
//            (one tile = 64 features, g in accumulator lanes 0..63, u in
//            64..127, the whole K; F/64 blocks).  Epilogue: u passes through
//            shared memory to the g lanes, h = u + E[id_t][f],
//            z[t][f] = SiLU(g) h, g and h saved when asked.
//   down:    C[128][N] = W_down rows d0..d0+127 . z^T with K split over the
//            `splits` blocks of a thread-block cluster.  Each block leaves
//            its fp32 partial tile in its own shared memory; after a cluster
//            barrier, block r sums rows [r*128/splits, (r+1)*128/splits) of
//            all partials in rank order through distributed shared memory
//            (deterministic, no global scratch) and writes y[t][d] in bf16.
//
// Each pipeline stage carries `sub` consecutive 64-wide k blocks, so every
// weight row is read in runs of sub * 128 bytes: short runs per row leave
// HBM far below its bandwidth.  Every block walks its k steps from its own
// starting point, so the blocks do not all ask L2 for the same activation
// tile at the same moment.  The gate/up epilogue warps fetch the block's E
// rows into shared memory while the main loop runs.
//
// Both kernels are launched as programmatic dependents: before
// griddepcontrol.wait they allocate tensor memory and fill the shared-memory
// ring with weight tiles (which no earlier kernel writes); activations and
// outputs are touched only after the wait.
//
// Warp roles as in gemm_tc.cuh: warp 0 TMA, warp 1 MMA (+ tensor memory),
// warps 2..5 epilogue.  Every mbarrier wait is bounded; every thread reaches
// both cluster barriers on every path.
#pragma once

#include "common.cuh"

namespace stp {
namespace dec {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kMaxStages = 8;
constexpr int kThreads = 192;
constexpr int A_BLOCK = BM * BK * 2;        // one 64-wide k block of 128 weight rows: 16 KiB
constexpr int kMaxN = 256;
constexpr int kMaxSplits = 8;               // portable cluster size
constexpr int kTail = 256 + kMaxN * 4 + kMaxN * 64 * 2;  // barriers, flags, token ids, E tile

enum Mode { GATEUP = 0, DOWN = 1 };

struct Params {
  int32_t T;          // tokens
  int32_t N;          // T rounded up to a multiple of 16 (MMA N)
  int32_t M;          // rows of the weight side: F (gate/up) or D (down)
  int32_t K;          // D (gate/up) or F (down)
  int32_t k_blocks;   // K / BK
  int32_t kb_per;     // k blocks per split (a multiple of sub)
  int32_t splits;     // down: splits of K = cluster size; gate/up: 1
  int32_t sub;        // k blocks per pipeline stage
  int32_t stages;     // depth of the shared-memory ring (<= kMaxStages)
  // gate/up epilogue
  uint16_t* z;        // [T][F]
  uint16_t* g_save;
  uint16_t* h_save;
  int64_t ldf;
  const uint16_t* e_base;
  int64_t e_pitch;
  const int32_t* e_index;
  int64_t e_rows;
  int32_t e_mode;
  // down epilogue
  uint16_t* y;        // [T][D]
  int32_t* err;
};

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() {  // the four epilogue warps
  asm volatile("bar.sync 1, 128;" ::: "memory");
}
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::
                   : "memory");
}
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t map_shared(uint32_t addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(addr), "r"(rank));
  return r;
}
__device__ __forceinline__ float ld_cluster_f32(uint32_t addr) {
  float v;
  asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(addr) : "memory");
  return v;
}

template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
    decode_kernel(const __grid_constant__ CUtensorMap tmA0, const __grid_constant__ CUtensorMap tmA1,
                  const __grid_constant__ CUtensorMap tmB, const Params p) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~uintptr_t(1023));
  const int b_block = p.N * BK * 2;           // one k block of activations: a multiple of 2 KiB
  const int a_stage = p.sub * A_BLOCK;
  const int b_stage = p.sub * b_block;
  const int stage_bytes = a_stage + b_stage;
  const int S = p.stages;
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * a_stage;
  uint64_t* full = reinterpret_cast<uint64_t*>(sB + S * b_stage);
  uint64_t* empty = full + kMaxStages;
  uint64_t* tfull = empty + kMaxStages;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tfull + 1);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int32_t* s_ids = reinterpret_cast<int32_t*>(full) + 64;           // [kMaxN]
  uint16_t* s_e = reinterpret_cast<uint16_t*>(s_ids + kMaxN);       // [T][64] E rows of the tile
  // After the accumulator is complete every copy has landed and been consumed,
  // so the ring is free: gate/up passes u through it ([64][ustride] fp32),
  // down keeps its partial tile in it ([128][pstride] fp32).
  float* s_x = reinterpret_cast<float*>(smem);
  const int nround = (p.N + 31) & ~31;
  const int ustride = nround + 1;
  const int pstride = nround + 1;

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int tile = MODE == GATEUP ? blockIdx.x : blockIdx.x / p.splits;
  const int split = MODE == GATEUP ? 0 : blockIdx.x % p.splits;
  const int kb0 = split * p.kb_per;
  const int kb1 = min(p.k_blocks, kb0 + p.kb_per);
  const int nsteps = kb1 > kb0 ? (kb1 - kb0 + p.sub - 1) / p.sub : 0;
  const int rot = nsteps > 0 ? (tile * 5) % nsteps : 0;   // this block's first k step
  const uint32_t tmem_cols = p.N <= 32 ? 32 : (p.N <= 64 ? 64 : (p.N <= 128 ? 128 : 256));

  if (threadIdx.x == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    mbar_init(tfull, 1);
    *abort_flag = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tmA0);
    tma_prefetch_desc(&tmB);
    if (MODE == GATEUP) tma_prefetch_desc(&tmA1);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // let the next kernel in the stream start its own prologue on free SMs
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      const int m0 = tile * BM;
      auto load_a = [&](int i, int s) {
        const int step = (i + rot) % nsteps;
        uint8_t* a = sA + s * a_stage;
        for (int j = 0; j < p.sub; ++j) {
          const int k0 = (kb0 + step * p.sub + j) * BK;
          if (MODE == GATEUP) {
            const int f0 = tile * (BM / 2);
            tma_load_2d(&tmA0, &full[s], a + j * A_BLOCK, k0, f0);
            tma_load_2d(&tmA1, &full[s], a + j * A_BLOCK + A_BLOCK / 2, k0, f0);
          } else {
            tma_load_2d(&tmA0, &full[s], a + j * A_BLOCK, k0, m0);
          }
        }
      };
      auto load_b = [&](int i, int s) {
        const int step = (i + rot) % nsteps;
        for (int j = 0; j < p.sub; ++j)
          tma_load_2d(&tmB, &full[s], sB + s * b_stage + j * b_block,
                      (kb0 + step * p.sub + j) * BK, 0);
      };
      // weights first: they do not depend on the previous kernel
      const int pre = min(S, nsteps);
      for (int i = 0; i < pre; ++i) {
        mbar_arrive_expect_tx(&full[i], stage_bytes);
        load_a(i, i);
      }
      grid_dep_wait();
      for (int i = 0; i < pre; ++i) load_b(i, i);
      int stage = pre % S;
      uint32_t phase = pre == S ? 1 : 0;
      for (int i = pre; i < nsteps; ++i) {
        if (!mbar_wait(&empty[stage], phase ^ 1, abort_flag, p.err)) break;
        mbar_arrive_expect_tx(&full[stage], stage_bytes);
        load_a(i, stage);
        load_b(i, stage);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      const uint32_t idesc = idesc_bf16_f32(BM, p.N, false, false);
      int stage = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int i = 0; i < nsteps; ++i) {
        if (!mbar_wait(&full[stage], phase, abort_flag, p.err)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t a_addr = smem_u32(sA + stage * a_stage);
        const uint32_t b_addr = smem_u32(sB + stage * b_stage);
        for (int j = 0; j < p.sub; ++j) {
#pragma unroll
          for (int k = 0; k < BK / 16; ++k)
            umma_bf16(tmem_base, sw128_desc(a_addr + j * A_BLOCK + k * 32, 16, 1024),
                      sw128_desc(b_addr + j * b_block + k * 32, 16, 1024), idesc,
                      (i | j | k) != 0 ? 1u : 0u);
        }
        umma_commit(&empty[stage]);
        if (++stage == S) {
          stage = 0;
          phase ^= 1;
        }
      }
      if (ok) umma_commit(tfull);
    }
  } else {
    // -------------------------------------------------------------- epilogue
    const int q = warp & 3;                 // tensor-memory lane quarter
    const int row = q * 32 + lane;          // accumulator row
    const int et = threadIdx.x - 64;        // 0..127 among epilogue threads
    grid_dep_wait();
    if (MODE == GATEUP && p.e_mode != STAPLE_EMBED_NONE) {
      for (int t = et; t < p.T; t += 128) {
        const int64_t idx = p.e_index[t];
        const bool bad = idx < 0 || idx >= p.e_rows;
        if (bad) report(p.err, STAPLE_EIDRANGE);
        s_ids[t] = bad ? -1 : int32_t(idx);
      }
      epi_bar();
      // E[id_t][f0 .. f0+63] for every token: 128 bytes per row, 16-byte loads,
      // issued while the main loop is still streaming weights
      const int f0 = tile * (BM / 2);
      for (int v = et; v < p.T * 8; v += 128) {
        const int t = v >> 3, part = v & 7;
        const int id = s_ids[t];
        uint4 w = make_uint4(0u, 0u, 0u, 0u);
        if (id >= 0 && f0 + part * 8 < p.M)
          w = __ldg(reinterpret_cast<const uint4*>(p.e_base + int64_t(id) * p.e_pitch + f0) + part);
        reinterpret_cast<uint4*>(s_e)[t * 8 + part] = w;
      }
    }
    const bool ok = nsteps > 0 && mbar_wait(tfull, 0, abort_flag, p.err);
    const bool all_ok = __all_sync(0xffffffffu, ok);
    tc_fence_after();
    const uint32_t tacc = tmem_base + (uint32_t(q * 32) << 16);
    if (MODE == GATEUP) {
      const int f = tile * (BM / 2) + (row & 63);
      // u rows (lanes 64..127) hand their values to the g rows through smem
      if (row >= 64 && all_ok) {
        for (int c = 0; c < p.N; c += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + c, r);
          tmem_ld_wait(r);
#pragma unroll
          for (int j = 0; j < 32; ++j) s_x[(row - 64) * ustride + c + j] = __uint_as_float(r[j]);
        }
      }
      epi_bar();
      if (row < 64 && all_ok) {
        for (int c = 0; c < p.N; c += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + c, r);
          tmem_ld_wait(r);
          if (f < p.M) {
            const int tn = min(32, p.T - c);
            for (int j = 0; j < tn; ++j) {
              const int t = c + j;
              const float g = __uint_as_float(r[j]);
              float h = s_x[row * ustride + t];
              if (p.e_mode != STAPLE_EMBED_NONE) h += bf2f(s_e[t * 64 + row]);
              const float zf = g * sigmoid_f(g) * h;
              const int64_t off = int64_t(t) * p.ldf + f;
              p.z[off] = __bfloat16_as_ushort(__float2bfloat16_rn(zf));
              if (p.g_save) p.g_save[off] = __bfloat16_as_ushort(__float2bfloat16_rn(g));
              if (p.h_save) p.h_save[off] = __bfloat16_as_ushort(__float2bfloat16_rn(h));
            }
          }
        }
      }
    } else {
      const int d = tile * BM + row;
      if (p.splits == 1) {
        for (int c = 0; c < p.N && all_ok; c += 32) {
          uint32_t r[32];
          tmem_ld32(tacc + c, r);
          tmem_ld_wait(r);
          if (d < p.M)
            for (int j = 0; j < 32 && c + j < p.T; ++j)
              p.y[int64_t(c + j) * p.M + d] =
                  __bfloat16_as_ushort(__float2bfloat16_rn(__uint_as_float(r[j])));
        }
      } else {
        // partial tile -> own shared memory (zeros if this block failed)
        for (int c = 0; c < p.N; c += 32) {
          uint32_t r[32];
          if (all_ok) {
            tmem_ld32(tacc + c, r);
            tmem_ld_wait(r);
          } else {
#pragma unroll
            for (int j = 0; j < 32; ++j) r[j] = 0u;
          }
#pragma unroll
          for (int j = 0; j < 32; ++j) s_x[row * pstride + c + j] = __uint_as_float(r[j]);
        }
      }
    }
  }

  if (MODE == DOWN && p.splits > 1) {
    // every thread of every block of the cluster passes both barriers, with
    // each warp converged (the producer and MMA lanes finish their loops first)
    __syncthreads();
    __syncwarp();
    cluster_sync_all();
    if (warp >= 2) {
      const int et = threadIdx.x - 64;
      const int rows_per = (BM + p.splits - 1) / p.splits;
      const int r0 = int(cluster_rank()) * rows_per;
      const int nrows = max(0, min(rows_per, BM - r0));
      // the partial tiles of all blocks sit at the same offset in each block
      uint32_t peer[kMaxSplits];
#pragma unroll
      for (int s = 0; s < kMaxSplits; ++s)
        peer[s] = map_shared(smem_u32(s_x), uint32_t(s < p.splits ? s : 0));
      for (int e = et; e < nrows * p.T; e += 128) {
        const int rr = r0 + e % nrows;       // consecutive threads: consecutive d
        const int t = e / nrows;
        const int d = tile * BM + rr;
        const uint32_t off = uint32_t((rr * pstride + t) * 4);
        float v[kMaxSplits];
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)   // all loads in flight before the sum
          v[s] = s < p.splits ? ld_cluster_f32(peer[s] + off) : 0.0f;
        float acc = 0.0f;
#pragma unroll
        for (int s = 0; s < kMaxSplits; ++s)   // rank order: deterministic
          if (s < p.splits) acc += v[s];
        if (d < p.M) p.y[int64_t(t) * p.M + d] = __bfloat16_as_ushort(__float2bfloat16_rn(acc));
      }
    }
    __syncwarp();
    cluster_sync_all();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// Ring depth and dynamic shared memory for N tokens (N a multiple of 16) and
// `sub` k blocks per stage.
inline int ring_stages(int N, int sub) {
  const int budget = 227 * 1024 - 1024 - kTail;
  int s = budget / (sub * (A_BLOCK + N * BK * 2));
  return s > kMaxStages ? kMaxStages : s;
}
inline int smem_bytes(int N, int sub) {
  return 1024 + ring_stages(N, sub) * sub * (A_BLOCK + N * BK * 2) + kTail;
}

}  // namespace dec
}  // namespace stp
