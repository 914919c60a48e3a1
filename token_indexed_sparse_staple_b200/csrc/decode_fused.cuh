// The STAPLE layer at decode sizes (T <= 256 tokens): one persistent tcgen05
// kernel for gate/up (with the fused E-row add and SiLU gating) and the down
// projection's split-k pieces.  The pieces are summed either by a small
// kernel launched right behind it (two-launch path) or, when the layer has
// enough down tiles, inside the same launch by clusters of blocks through
// distributed shared memory (cluster path).
//
// With a handful of tokens the layer streams its weights once per step and
// is bound by HBM bandwidth, so the kernel is organised around that stream:
//
//  * The weights take the MMA's M side (128 rows per tile) and the tokens its
//    N side (T rounded up to 16).  A gate/up tile stacks 64 W_gate and the
//    matching 64 W_up rows (64 features); a down tile is 128 W_down rows.
//    Every stage carries `sub` 64-wide k blocks, so each weight row is read
//    in runs of sub * 128 bytes (short runs per row leave HBM far below its
//    bandwidth).  Weights and activations have separate rings: the weight
//    ring is deep (HBM latency), the activation ring shallow (it hits L2).
//    Weights depend on nothing earlier, so the first ring fills are issued
//    before the block's set-up barrier.
//  * Phase 1, gate/up: whole tiles are spread over the blocks.  A block
//    finishes a tile straight from tensor memory, 16 tokens at a time: g and
//    u rows go to shared memory, then each of the 128 epilogue threads
//    computes 8 consecutive features of one token, h = u + E[id_t][f] (E rows
//    prefetched into shared memory during the main loop) and z = SiLU(g) h
//    (g and h saved when asked), written 16 bytes at a time; then one thread
//    publishes the tile with a release store of its ready flag.
//  * Phase 2, down: the down units (tile x `sub` k blocks) are split evenly
//    over the blocks (stream-K), so every SM streams the same share of
//    W_down.  The first units' weights are copied from the ring into the
//    tensor-memory columns the accumulators leave free as soon as they land,
//    which frees the ring for the next units: W_down streams while the
//    gate/up phase is still finishing.  The activation loads wait (bounded
//    spin, all flags of the block polled at once by one warp) on the ready
//    flags of the gate/up tiles that produced the block's z columns; weight
//    loads do not wait.  Each block's piece of a tile leaves an fp32 partial
//    [N][128] in the workspace (L2-resident; a warp writes 128 contiguous
//    bytes per token), and the block is done.
//  * Two-launch path: the split-k sums run in decode_reduce_kernel, launched
//    right behind as a programmatic dependent (see there), which also clears
//    the ready flags.
//  * Cluster path (kClu): the grid is one cluster of kCluster blocks per down
//    tile, and the tile's units are split over the cluster's blocks.  At the
//    end each block pushes its accumulator rows into the shared memory of the
//    block that sums them (block r of the cluster sums rows 32r .. 32r+31),
//    and after a cluster barrier each block adds the cluster's pieces in
//    block order and writes its rows of y.  No partial leaves the SMs, and
//    the next call's activations are ready as soon as this launch completes.
//    The last block to finish polling clears the ready flags.
//  * Every block finishes its gate/up tiles before it needs anybody's z, so
//    all waits end while all blocks are resident (one block per SM; the
//    launcher checks the grid against the blocks, or clusters, the device
//    holds at once).  The ready flags live in the first bytes
//    of the workspace and are zero again after every call, so a zero-filled
//    workspace stays valid across calls and graph replays.
//
// The STEM variant (kStem: the row replaces the up-projection) streams no
// W_up: a gate tile is 128 W_gate rows (128 features) and h = E[id_t].
//
// Warps: 0 weight (A) loads, 1 MMA issue + tensor memory, 2 activation (B)
// loads, 3..6 epilogue (each owns one 32-lane quarter of tensor memory).
// Every mbarrier wait and flag spin is bounded (STAPLE_ETIMEOUT); after a
// timeout each role lets its issued copies and MMAs finish before the block
// exits.  The kernel is launched as a programmatic dependent: weights stream
// before griddepcontrol.wait; activations, outputs and flags only after it.
#pragma once

#include "common.cuh"

namespace stp {
namespace fused {

constexpr int BM = 128;
constexpr int BK = 64;
constexpr int kMaxStages = 8;
constexpr int kThreads = 224;
constexpr int A_BLOCK = BM * BK * 2;  // 128 weight rows x 64 k: 16 KiB
constexpr int kMaxN = 256;
constexpr int kStagesB = 3;
constexpr int kChunkRows = 16;        // rows of a down tile per reduction chunk
constexpr int kXStride = 17;          // fp32 words per row of the g/u exchange chunk
constexpr int kCluster = 4;           // blocks per cluster (cluster path)
constexpr int kRowsPer = BM / kCluster;  // rows of a down tile each cluster block sums
// shared memory after the rings: barriers + flags (512 B), token ids,
// g/u exchange chunk [128][17] fp32; then the E tile [N][features per tile] bf16
constexpr int kTailFixed = 512 + kMaxN * 4 + 128 * kXStride * 4;
// features per gate/up tile: 64 W_gate over the matching 64 W_up rows, or
// (STEM) 128 W_gate rows
template <bool kStem>
constexpr int tile_features() { return kStem ? 128 : 64; }

struct Params {
  int32_t T, N, D, F;
  int32_t sub;         // k blocks per unit (and per pipeline stage)
  int32_t stages;      // depth of the weight ring
  int32_t stages_b;    // depth of the activation ring
  int32_t G;           // gate/up tiles (F / features per tile)
  int32_t Dt;          // down tiles (ceil(D / 128))
  int32_t ug, ud;      // units per gate/up tile, per down tile
  int32_t Ud;          // down units (Dt * ud)
  int32_t maxp_d;      // partial slots per down tile
  int32_t stage_tmem;  // stage down-unit weights in spare tensor memory
  // activations / outputs
  uint16_t* z;
  uint16_t* g_save;
  uint16_t* h_save;
  uint16_t* y;
  const uint16_t* e_base;
  int64_t e_pitch;
  const int32_t* e_index;
  int64_t e_rows;
  int32_t e_mode;
  // workspace
  uint32_t* ready;     // [G] gate/up tile finished (reset after every call)
  float* part;         // two-launch path: [Dt * maxp_d][N][128] fp32 partial sums, summed
                       // by the next kernel
  int32_t* err;
  uint64_t wait_ns;    // bound of every wait and flag spin (STAPLE_ETIMEOUT past it)
  uint32_t* fin;       // cluster path: blocks whose z poll is over; the last one clears `ready`
};

__host__ __device__ inline int range_start(int c, int U, int grid) {
  return int((int64_t(c) * U) / grid);
}
// The block whose range holds unit x.
__host__ __device__ inline int owner(int x, int U, int grid) {
  int c = int((int64_t(x) * grid) / U);
  while (c + 1 < grid && range_start(c + 1, U, grid) <= x) ++c;
  while (c > 0 && range_start(c, U, grid) > x) --c;
  return c;
}

// Gate/up tiles of block b: [gate_start(b), gate_start(b + 1)).  With no
// more tiles than blocks, tile b goes to block b, so the blocks with the
// highest indices, which are the last to get an SM when launches follow one
// another (each SM takes the next block as the previous launch's block on it
// exits), make no gate/up tile that every block then waits for; otherwise
// the tiles are spread evenly.
__host__ __device__ inline int gate_start(int b, int G, int grid) {
  return G <= grid ? min(b, G) : range_start(b, G, grid);
}
// The block that makes gate/up tile t.
__host__ __device__ inline int gate_owner(int t, int G, int grid) {
  return G <= grid ? t : owner(t, G, grid);
}

// A block finishes its gate/up tiles one after the other, so a tile's ready
// flag rises later the further it sits in its block's range.  The lateness of
// down unit x is the largest such position among the tiles that make the z
// columns x reads (0 when each is its block's first tile).
template <int FT>
__device__ inline int unit_lateness(int x, const Params& p, int grid) {
  const int f_lo = (x % p.ud) * p.sub * BK, f_hi = min(p.F, f_lo + p.sub * BK);
  int late = 0;
  for (int t = f_lo / FT; t <= (f_hi - 1) / FT; ++t)
    late = max(late, t - gate_start(gate_owner(t, p.G, grid), p.G, grid));
  return late;
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
__device__ __forceinline__ uint32_t cluster_id() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%clusterid.x;" : "=r"(r));
  return r;
}
// Every thread of every block of the cluster; stores before it (shared
// memory of any block of the cluster included) are seen after it.
__device__ __forceinline__ void cluster_sync() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" :::
                   "memory");
}
// The address of this block's shared-memory word `a` in block `rank` of the cluster.
__device__ __forceinline__ uint32_t map_peer(uint32_t a, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(a), "r"(rank));
  return r;
}
__device__ __forceinline__ void st_peer4(uint32_t a, uint32_t x, uint32_t y, uint32_t z, uint32_t w) {
  asm volatile("st.shared::cluster.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(a), "r"(x), "r"(y), "r"(z),
               "r"(w)
               : "memory");
}
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* a, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ uint32_t atom_add_acq_rel(uint32_t* a, uint32_t v) {
  uint32_t old;
  asm volatile("atom.acq_rel.gpu.global.add.u32 %0, [%1], %2;" : "=r"(old) : "l"(a), "r"(v) : "memory");
  return old;
}
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ void add4(float4& a, const float4 b) {
  a.x += b.x;
  a.y += b.y;
  a.z += b.z;
  a.w += b.w;
}
// Bounded spin until *a >= want (acquire).  False (and *abort set, the
// error word written) after limit_ns.
__device__ __forceinline__ bool spin_until(const uint32_t* a, uint32_t want, volatile int* abort,
                                           int32_t* err, uint64_t limit_ns) {
  if (ld_acquire(a) >= want) return true;
  const uint64_t t0 = globaltimer();
  while (ld_acquire(a) < want) {
    __nanosleep(64);
    if (*abort) return false;
    if (globaltimer() - t0 > limit_ns) {
      *abort = 1;
      report(err, STAPLE_ETIMEOUT);
      return false;
    }
  }
  return true;
}

// kOrder: blocks order their down steps by lateness.  Only useful when
// some block makes two or more gate/up tiles (more tiles than blocks); with
// kOrder false that code is compiled out, which keeps the kernel body small
// (the gate/up epilogue runs while the memory queues are full, where extra
// code shows up as instruction-fetch stalls).
// kClu: the cluster path (launched in clusters of kCluster blocks, see the
// end of the kernel): the split-k sum is done inside the launch.
template <bool kOrder, bool kStem, bool kClu>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_wg,
                        const __grid_constant__ CUtensorMap tm_wu,
                        const __grid_constant__ CUtensorMap tm_wd,
                        const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_z,
                        const Params p) {
  constexpr int FT = tile_features<kStem>();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = align_smem_1024(smem_raw);
  const int b_block = p.N * BK * 2;
  const int a_stage = p.sub * A_BLOCK;
  const int b_stage = p.sub * b_block;
  const int S = p.stages;
  const int SB = p.stages_b;
  uint8_t* sA = smem;
  uint8_t* sB = smem + S * a_stage;
  uint8_t* tail = sB + SB * b_stage;
  uint64_t* fullA = reinterpret_cast<uint64_t*>(tail);
  uint64_t* fullB = fullA + kMaxStages;
  uint64_t* emptyA = fullB + kMaxStages;
  uint64_t* emptyB = emptyA + kMaxStages;
  uint64_t* tfull = emptyB + kMaxStages;  // [2]
  uint64_t* tempty = tfull + 2;           // [2]
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(tempty + 2);
  volatile int* abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  int* s_flag = const_cast<int*>(abort_flag + 1);
  // set by an epilogue warp whose wait failed, read by all four after a
  // barrier, so every epilogue warp takes the same path through bar.sync
  int* s_epi_fail = s_flag + 1;
  uint64_t* obar = reinterpret_cast<uint64_t*>(tail + 328);  // down-step order written
  uint64_t* dbar = reinterpret_cast<uint64_t*>(tail + 336);  // MMA drain before TMEM is freed
  // Down-step order (blocks with at most kMaxOrder down units): within each
  // piece, the units whose z is ready first (lateness 0) come first.  The
  // weight loader, the activation loader and the MMA thread all follow it.
  constexpr int kMaxOrder = 64;
  uint8_t* s_late = tail + 384;   // [kMaxOrder] lateness (capped) of unit d0 + k
  uint8_t* s_order = tail + 448;  // [kMaxOrder] down step k -> unit d0 + s_order[k]
  int32_t* s_ids = reinterpret_cast<int32_t*>(tail + 512);            // [kMaxN]
  float* s_x = reinterpret_cast<float*>(s_ids + kMaxN);               // [128][kXStride]
  uint16_t* s_e = reinterpret_cast<uint16_t*>(s_x + 128 * kXStride);  // [N][FT]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grid = gridDim.x;
  // this block's work: gate/up tiles [t0, t1) (ug units each), then down
  // units [d0, d1); local step i < ngs is gate/up, the rest down
  const int t0 = gate_start(blockIdx.x, p.G, grid), t1 = gate_start(blockIdx.x + 1, p.G, grid);
  // Cluster path: cluster c takes down tile c, its blocks split the tile's
  // units (one piece per block).
  const uint32_t crank = kClu ? cluster_rank() : 0u;
  const int ctile = kClu ? int(cluster_id()) : 0;
  const int d0 = kClu ? ctile * p.ud + range_start(int(crank), p.ud, kCluster)
                      : range_start(blockIdx.x, p.Ud, grid);
  const int d1 = kClu ? ctile * p.ud + range_start(int(crank) + 1, p.ud, kCluster)
                      : range_start(blockIdx.x + 1, p.Ud, grid);
  const int ngs = (t1 - t0) * p.ug;
  const int nsteps = ngs + (d1 - d0);
  const int nd = d1 - d0;
  // With no more gate/up tiles than blocks, every tile is its block's first,
  // every lateness is 0 and the order is the identity: skip it.
  const bool reorder = kOrder && nd <= kMaxOrder && p.G > grid;
  const uint32_t ncols = p.N <= 32 ? 32 : (p.N <= 64 ? 64 : (p.N <= 128 ? 128 : 256));
  // Tensor memory: two accumulators of ncols columns, then (p.stage_tmem) as
  // many down-unit weight slots as fit in the 512 columns; a slot holds one
  // unit's 128 rows x sub*64 bf16 (two k values per column).
  const uint32_t slot_cols = uint32_t(p.sub) * (BK / 2);
  const int nslots = p.stage_tmem ? int((512 - 2 * ncols) / slot_cols) : 0;
  const uint32_t tmem_cols = nslots > 0 ? 512 : 2 * ncols;

  // cluster path: the accumulator that holds the block's down piece, once
  // the epilogue has seen it complete (-1: none, or the block gave up)
  int acc_buf = -1;

  // the unit of the block's k-th down step
  auto unit = [&](int k) { return d0 + (reorder ? int(s_order[k]) : k); };
  const bool ordered = reorder && nd > 0;
  // The weights of local step i into ring stage s (bytes counted on fullA[s]).
  auto issue_weights = [&](int i, int s, uint64_t once) {
    mbar_arrive_expect_tx(&fullA[s], a_stage);
    uint8_t* a = sA + s * a_stage;
    if (i < ngs) {
      const int tile = t0 + i / p.ug, u = i % p.ug;
      for (int j = 0; j < p.sub; ++j) {
        const int k0 = (u * p.sub + j) * BK;
        if (kStem) {   // 128 W_gate rows (the map's box is 128 rows)
          tma_load_2d_hint(&tm_wg, &fullA[s], a + j * A_BLOCK, k0, tile * FT, once);
        } else {       // 64 W_gate rows over the matching 64 W_up rows
          tma_load_2d_hint(&tm_wg, &fullA[s], a + j * A_BLOCK, k0, tile * FT, once);
          tma_load_2d_hint(&tm_wu, &fullA[s], a + j * A_BLOCK + A_BLOCK / 2, k0, tile * FT, once);
        }
      }
    } else {
      // one 3-D copy brings all `sub` k blocks of the unit
      const int x = unit(i - ngs), tile = x / p.ud, u = x % p.ud;
      tma_load_3d_hint(&tm_wd, &fullA[s], a, 0, tile * BM, u * p.sub, once);
    }
  };
  // Weights depend on no earlier kernel and on nothing else of the set-up,
  // so the weight loader (thread 0) fills the whole ring before the block
  // barrier, while tensor memory is being allocated (the down steps of a
  // block that orders them wait for the order, worked out after the barrier).
  const int early = min(S, ordered ? ngs : nsteps);
  if (threadIdx.x == 0) {
    tma_prefetch_desc(&tm_wg);
    tma_prefetch_desc(kStem ? &tm_wd : &tm_wu);
    for (int s = 0; s < S; ++s) {
      mbar_init(&fullA[s], 1);
      mbar_init(&emptyA[s], 1);
    }
    for (int s = 0; s < SB; ++s) {
      mbar_init(&fullB[s], 1);
      mbar_init(&emptyB[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&tfull[b], 1);
      mbar_init(&tempty[b], 4);
    }
    mbar_init(obar, 1);
    mbar_init(dbar, 1);
    *abort_flag = 0;
    *s_epi_fail = 0;
    fence_barrier_init();
    const uint64_t once = l2_policy_evict_first();
    for (int i = 0; i < early; ++i) issue_weights(i, i, once);
    tma_prefetch_desc(&tm_wd);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_z);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // The step order is worked out by an epilogue warp (idle until the first
  // gate/up tile is done), off the path of the first weight loads; the
  // loaders wait for it on obar before their first down step.
  if (warp == 3 && ordered) {
    for (int k = lane; k < nd; k += 32)
      s_late[k] = uint8_t(min(255, unit_lateness<FT>(d0 + k, p, grid)));
    __syncwarp();
    if (lane == 0) {
      int pos = 0;
      for (int xb = d0; xb < d1;) {
        const int xe = min(d1, (xb / p.ud + 1) * p.ud);  // one piece: one down tile
        for (int pass = 0; pass < 2; ++pass)
          for (int x = xb; x < xe; ++x)
            if ((s_late[x - d0] == 0) == (pass == 0)) s_order[pos++] = uint8_t(x - d0);
        xb = xe;
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(obar);
  }
  grid_dep_launch();

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------------- weight (A) loads
      const uint64_t once = l2_policy_evict_first();  // weights are read once per call
      // the first `early` steps went out before the block barrier
      int s = early % S;
      uint32_t ph = early == S ? 1u : 0u;
      int issued = early;
      for (int i = early; i < nsteps; ++i) {
        if (i == ngs && ordered && !mbar_wait(obar, 0, abort_flag, p.err, p.wait_ns)) break;
        if (!mbar_wait(&emptyA[s], ph ^ 1, abort_flag, p.err, p.wait_ns)) break;
        issue_weights(i, s, once);
        ++issued;
        if (++s == S) {
          s = 0;
          ph ^= 1;
        }
      }
      // after an abort, copies still in flight land before the block exits
      drain_ring(fullA, S, s, ph, issued);
    }
  } else if (warp == 2) {
    // ---------------------------------------------------- activation (B) loads
    grid_dep_wait();
    int s = 0;
    uint32_t ph = 0;
    int issued = 0;   // lane 0's fills
    bool ok = true;
    // x for the gate/up steps
    if (lane == 0) {
      for (int i = 0; i < ngs && ok; ++i) {
        ok = mbar_wait(&emptyB[s], ph ^ 1, abort_flag, p.err, p.wait_ns);
        if (!ok) break;
        const int u = i % p.ug;
        uint8_t* b = sB + s * b_stage;
        mbar_arrive_expect_tx(&fullB[s], b_stage);
        tma_load_3d(&tm_x, &fullB[s], b, 0, 0, u * p.sub);
        ++issued;
        if (++s == SB) {
          s = 0;
          ph ^= 1;
        }
      }
    }
    ok = __shfl_sync(0xffffffffu, ok, 0);
    // z for the down steps, in two rounds: first the units of lateness 0,
    // then the rest.  Before a round the whole warp polls every ready flag
    // the round needs at once (checked one unit at a time, each check would
    // put an L2 round trip on the issue path of every unit); lane 0 then
    // issues the round's z loads in step order.
    auto poll = [&](bool late_round) {
      bool mine = true;
      for (int k = lane; k < nd && mine; k += 32) {
        if (reorder && ((s_late[k] != 0) != late_round)) continue;
        // unit d0 + k reads z columns [f_lo, f_hi), made by tiles f_lo/FT .. (f_hi-1)/FT
        const int f_lo = ((d0 + k) % p.ud) * p.sub * BK;
        const int f_hi = min(p.F, f_lo + p.sub * BK);
        for (int t = f_lo / FT; t <= (f_hi - 1) / FT && mine; ++t)
          mine = spin_until(&p.ready[t], 1u, abort_flag, p.err, p.wait_ns);
      }
      return __all_sync(0xffffffffu, mine);
    };
    int k = 0;  // next down step to issue (lane 0)
    auto issue = [&](bool stop_at_late) {
      fence_async_global();
      for (; k < nd; ++k) {
        const int x = unit(k);
        if (stop_at_late && reorder && s_late[x - d0] != 0) break;
        if (!mbar_wait(&emptyB[s], ph ^ 1, abort_flag, p.err, p.wait_ns)) return false;
        uint8_t* b = sB + s * b_stage;
        mbar_arrive_expect_tx(&fullB[s], b_stage);
        tma_load_3d(&tm_z, &fullB[s], b, 0, 0, (x % p.ud) * p.sub);
        ++issued;
        if (++s == SB) {
          s = 0;
          ph ^= 1;
        }
      }
      return true;
    };
    if (ok && ordered)
      ok = __all_sync(0xffffffffu, mbar_wait(obar, 0, abort_flag, p.err, p.wait_ns));
    if (ok && nd > 0) {
      ok = poll(false);
      if (lane == 0 && ok) ok = issue(true);
      if (kOrder) {
        ok = __shfl_sync(0xffffffffu, ok, 0);
        const int k1 = __shfl_sync(0xffffffffu, k, 0);
        if (ok && k1 < nd) {
          ok = poll(true);
          if (lane == 0 && ok) issue(false);
        }
      }
    }
    if (kClu) {
      // The block's last look at the ready flags is behind it (every lane's
      // poll, ordered by the warp barrier and the release).  Every tile is
      // polled by some block after it was published, so once every block has
      // counted itself here the last one clears the flags for the next call
      // (which reads them only after this launch completes).
      __syncwarp();
      if (lane == 0 && atom_add_acq_rel(p.fin, 1u) == uint32_t(grid - 1)) {
        for (int t = 0; t < p.G; ++t) p.ready[t] = 0u;
        *p.fin = 0u;
      }
    }
    if (lane == 0) drain_ring(fullB, SB, s, ph, issued);
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------------- MMA
      const uint32_t idesc = idesc_bf16_f32(BM, p.N, false, false);
      const uint32_t slot0 = tmem_base + 2 * ncols;  // first tensor-memory staging column
      const int n_stage = min(d1 - d0, nslots);
      int sa = 0, sb = 0;
      uint32_t pha = 0, phb = 0;
      int piece = 0;
      bool ok = true;
      for (int i0 = 0; i0 < nsteps && ok; ++piece) {
        if (i0 == ngs && n_stage > 0) {
          // The first n_stage down units' weights move to tensor memory as
          // they land; each copy's commit frees its ring stage for the next
          // unit's weights, so W_down streams while z is still being made.
          for (int k = 0; k < n_stage; ++k) {
            if (!mbar_wait(&fullA[sa], pha, abort_flag, p.err, p.wait_ns)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t a_addr = smem_u32(sA + sa * a_stage);
            const uint32_t dst = slot0 + uint32_t(k) * slot_cols;
            for (int j = 0; j < p.sub; ++j) {
#pragma unroll
              for (int kk = 0; kk < BK / 16; ++kk)
                tmem_cp_128x256b(dst + uint32_t(j * (BK / 16) + kk) * 8,
                                 sw128_desc(a_addr + j * A_BLOCK + kk * 32, 16, 1024));
            }
            umma_commit(&emptyA[sa]);
            if (++sa == S) {
              sa = 0;
              pha ^= 1;
            }
          }
          if (!ok) break;
        }
        int nunits;
        if (i0 < ngs) {
          nunits = p.ug;
        } else {
          const int x = d0 + i0 - ngs;
          nunits = min(d1, (x / p.ud + 1) * p.ud) - x;
        }
        const int buf = piece & 1;
        if (!mbar_wait(&tempty[buf], ((piece >> 1) & 1) ^ 1, abort_flag, p.err, p.wait_ns))
          break;
        tc_fence_after();
        const uint32_t dacc = tmem_base + uint32_t(buf) * ncols;
        for (int i = 0; i < nunits; ++i) {
          const int du = i0 + i - ngs;  // down unit index (negative for gate/up)
          const bool staged = du >= 0 && du < n_stage;
          if ((!staged && !mbar_wait(&fullA[sa], pha, abort_flag, p.err, p.wait_ns)) ||
              !mbar_wait(&fullB[sb], phb, abort_flag, p.err, p.wait_ns)) {
            ok = false;
            break;
          }
          tc_fence_after();
          // Descriptors are built once per unit; a k step of 32 bytes adds 2
          // to the start-address field (shared addresses stay below 2^18, so
          // the field never carries).  At decode sizes each MMA is small and
          // the issuing thread's own instructions set the pace.
          const uint64_t bd = sw128_desc(smem_u32(sB + sb * b_stage), 16, 1024);
          const uint32_t acc0 = i != 0 ? 1u : 0u;
          if (staged) {
            const uint32_t a_t = slot0 + uint32_t(du) * slot_cols;
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (j < p.sub) {
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                  umma_bf16_ta(dacc, a_t + uint32_t(j * (BK / 16) + k) * 8,
                               bd + uint64_t((j * b_block + k * 32) >> 4), idesc,
                               (j | k) != 0 ? 1u : acc0);
              }
            }
          } else {
            const uint64_t ad = sw128_desc(smem_u32(sA + sa * a_stage), 16, 1024);
#pragma unroll
            for (int j = 0; j < 2; ++j) {
              if (j < p.sub) {
#pragma unroll
                for (int k = 0; k < BK / 16; ++k)
                  umma_bf16(dacc, ad + uint64_t((j * A_BLOCK + k * 32) >> 4),
                            bd + uint64_t((j * b_block + k * 32) >> 4), idesc,
                            (j | k) != 0 ? 1u : acc0);
              }
            }
            umma_commit(&emptyA[sa]);
            if (++sa == S) {
              sa = 0;
              pha ^= 1;
            }
          }
          umma_commit(&emptyB[sb]);
          if (++sb == SB) {
            sb = 0;
            phb ^= 1;
          }
        }
        i0 += nunits;
        if (ok) umma_commit(&tfull[buf]);
      }
      // every MMA and tensor-memory copy issued here completes before tensor
      // memory and the ring are released (after an abort some may still run)
      umma_commit(dbar);
      mbar_drain(dbar, 0);
    }
  } else {
    // ----------------------------------------------------------- epilogue
    const int q = warp & 3;
    const int row = q * 32 + lane;
    const int et = threadIdx.x - 96;  // 0..127
    grid_dep_wait();
    for (int t = et; t < p.T; t += 128) {
      int32_t id = -1;
      if (p.e_mode != STAPLE_EMBED_NONE) {
        const int64_t v = p.e_index[t];
        if (v < 0 || v >= p.e_rows) report(p.err, STAPLE_EIDRANGE);
        else id = int32_t(v);
      }
      s_ids[t] = id;
    }
    epi_bar();
    int piece = 0;
    bool alive = true;
    // ---- phase 1: whole gate/up tiles, finished from tensor memory
    constexpr int kVecs = FT / 8;   // 16-byte pieces of a token's E row slice
    for (int tile = t0; tile < t1 && alive; ++tile, ++piece) {
      const int f0 = tile * FT;
      // E[id_t][f0 .. f0+FT) for every token, 16-byte loads issued while the
      // tile's main loop is still streaming.  Up to 8 loads per thread are
      // put in flight before any of them is stored (behind a saturated weight
      // stream each round trip is long).
      for (int vb = et; vb < p.T * kVecs; vb += 8 * 128) {
        uint4 w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = vb + k * 128;
          w[k] = make_uint4(0u, 0u, 0u, 0u);
          if (v < p.T * kVecs) {
            const int id = s_ids[v / kVecs];
            if (id >= 0)
              w[k] = __ldg(reinterpret_cast<const uint4*>(p.e_base + int64_t(id) * p.e_pitch + f0) +
                           (v % kVecs));
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = vb + k * 128;
          if (v < p.T * kVecs) reinterpret_cast<uint4*>(s_e)[v] = w[k];
        }
      }
      const int buf = piece & 1;
      const bool ok = mbar_wait(&tfull[buf], (piece >> 1) & 1, abort_flag, p.err, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok) && lane == 0) *s_epi_fail = 1;
      epi_bar();
      if (*s_epi_fail) {
        alive = false;
        break;
      }
      tc_fence_after();
      const uint32_t tacc = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf) * ncols;
      for (int c = 0; c < p.N; c += 16) {
        uint32_t r[16];
        tmem_ld16(tacc + c, r);
        tmem_ld_wait16(r);
#pragma unroll
        for (int j = 0; j < 16; ++j) s_x[row * kXStride + j] = __uint_as_float(r[j]);
        epi_bar();
        // thread -> token c + et / 8, features FT/8 (et % 8) .. +FT/8-1, in
        // 16-byte stores (the memory system is saturated by the weight stream
        // here, so the number of stores is what costs).  Rows f and 64 + f of
        // the chunk are g and u of feature f; for STEM all 128 rows are g.
        const int j = et >> 3, t = c + j;
        if (t < p.T) {
#pragma unroll
          for (int half = 0; half < FT / 64; ++half) {
            const int fl0 = (et & 7) * (FT / 8) + half * 8;
            const uint4 ev = *reinterpret_cast<const uint4*>(s_e + t * FT + fl0);
            const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
            uint32_t zw[4], gw[4], hw[4];
#pragma unroll
            for (int k = 0; k < 4; ++k) {
              const int f = fl0 + 2 * k;
              const float g0 = s_x[f * kXStride + j], g1 = s_x[(f + 1) * kXStride + j];
              const float h0 = kStem ? bf_lo(ew[k]) : s_x[(64 + f) * kXStride + j] + bf_lo(ew[k]);
              const float h1 = kStem ? bf_hi(ew[k]) : s_x[(65 + f) * kXStride + j] + bf_hi(ew[k]);
              zw[k] = pack_bf2(g0 * sigmoid_f(g0) * h0, g1 * sigmoid_f(g1) * h1);
              gw[k] = pack_bf2(g0, g1);
              hw[k] = pack_bf2(h0, h1);
            }
            const int64_t off = int64_t(t) * p.F + f0 + fl0;
            *reinterpret_cast<uint4*>(p.z + off) = make_uint4(zw[0], zw[1], zw[2], zw[3]);
            if (p.g_save)
              *reinterpret_cast<uint4*>(p.g_save + off) = make_uint4(gw[0], gw[1], gw[2], gw[3]);
            if (p.h_save)
              *reinterpret_cast<uint4*>(p.h_save + off) = make_uint4(hw[0], hw[1], hw[2], hw[3]);
          }
        }
        epi_bar();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      // The last epi_bar ordered every thread's z stores before this point
      // (CTA scope); one thread's release store then publishes all of them (a
      // release is cumulative), and the consumers' TMA loads of z follow
      // their acquire of the flag and an async-proxy fence.
      if (et == 0) {
        fence_async_global();
        st_release(&p.ready[tile], 1u);
      }
    }
    // ---- phase 2: down pieces -> fp32 partial slots (cluster path: the one
    // piece stays in tensor memory for the cluster's sum at the end)
    for (int x = d0; x < d1 && alive; ++piece) {
      const int tile = x / p.ud;
      const int x_end = min(d1, (tile + 1) * p.ud);
      x = x_end;
      const int buf = piece & 1;
      const bool ok = mbar_wait(&tfull[buf], (piece >> 1) & 1, abort_flag, p.err, p.wait_ns);
      if (!__all_sync(0xffffffffu, ok) && lane == 0) *s_epi_fail = 1;
      epi_bar();
      if (*s_epi_fail) {
        alive = false;
        break;
      }
      tc_fence_after();
      if (kClu) {
        acc_buf = buf;
        break;
      }
      const int idx = blockIdx.x - owner(tile * p.ud, p.Ud, grid);
      float* mine = p.part + int64_t(tile * p.maxp_d + idx) * p.N * BM;
      const uint32_t tacc = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(buf) * ncols;
      for (int c = 0; c < p.N; c += 32) {
        uint32_t r[32];
        tmem_ld32(tacc + c, r);
        tmem_ld_wait(r);
        const int cn = min(32, p.N - c);  // the slot holds N token rows
#pragma unroll
        for (int j = 0; j < 32; ++j)
          if (j < cn) mine[(c + j) * BM + row] = __uint_as_float(r[j]);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
    }
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (kClu) {
    // ---- the split-k sum of the cluster path.  (1) After this barrier every
    // block of the cluster is done with its rings (copies landed, MMAs
    // drained), and the weight ring takes the pushed accumulator rows:
    // recv[source block][kRowsPer][N + 4] fp32.  Epilogue warp q holds rows
    // 32q .. 32q+31 of the block's piece, which block q of the cluster sums.
    static_assert(kRowsPer == 32, "one epilogue warp's rows per cluster block");
    cluster_sync();
    float* recv = reinterpret_cast<float*>(sA);
    const int rs = p.N + 4;   // padded row: the pushes of a warp's 32 rows spread over the banks
    if (warp >= 3 && acc_buf >= 0) {
      const int q = warp & 3;
      const uint32_t tacc = tmem_base + (uint32_t(q * 32) << 16) + uint32_t(acc_buf) * ncols;
      const uint32_t dst =
          map_peer(smem_u32(recv + (int(crank) * kRowsPer + lane) * rs), uint32_t(q));
      for (int c = 0; c < p.N; c += 32) {
        uint32_t r[32];
        tmem_ld32(tacc + c, r);
        tmem_ld_wait(r);
        const int cn = min(32, p.N - c);
#pragma unroll
        for (int j = 0; j < 32; j += 4)
          if (j < cn) st_peer4(dst + uint32_t(c + j) * 4u, r[j], r[j + 1], r[j + 2], r[j + 3]);
      }
    }
    tc_fence_before();
    cluster_sync();   // (2) every push has landed
    tc_fence_after();
    if (warp >= 3) {
      // This block's slice: rows row0 .. row0+31 of y, for every token.  A
      // thread takes 8 rows of one token (lanes: consecutive tokens) and adds
      // the cluster's pieces in block order.
      const int et = threadIdx.x - 96;
      const int row0 = ctile * BM + int(crank) * kRowsPer;
      const int nitems = (kRowsPer / 8) * p.N;
      for (int it = et; it < nitems; it += 128) {
        const int t = it % p.N, rg = it / p.N;
        const int d = row0 + rg * 8;
        if (t >= p.T || d >= p.D) continue;   // D % 64 == 0: 8 rows all in or all out
        float a[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) a[k] = recv[(rg * 8 + k) * rs + t];
#pragma unroll
        for (int src = 1; src < kCluster; ++src)
#pragma unroll
          for (int k = 0; k < 8; ++k) a[k] += recv[(src * kRowsPer + rg * 8 + k) * rs + t];
        *reinterpret_cast<uint4*>(p.y + int64_t(t) * p.D + d) =
            make_uint4(pack_bf2(a[0], a[1]), pack_bf2(a[2], a[3]), pack_bf2(a[4], a[5]),
                       pack_bf2(a[6], a[7]));
      }
    }
  }
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// ---------------------------------------------------------------------------
// The split-k sum of the down projection, a kernel of its own.  It is
// launched as a programmatic dependent of the decode kernel, right behind it:
// its blocks (small, no shared memory) start early and release the next
// kernel in the stream at once, then wait for the decode kernel to complete,
// so every partial slot is written and visible and nothing needs to be
// counted or polled; meanwhile the next decode kernel's blocks take the SMs
// the decode kernel left and start streaming their weights.  Block b sums
// 16-row chunk b % 8 of down tile b / 8 over the tile's pieces, in piece
// order (deterministic), and writes y = bf16(sum); block 0 also clears the
// gate/up ready flags for the next call.
// ---------------------------------------------------------------------------
constexpr int kReduceThreads = 256;

struct ReduceParams {
  int32_t T, N, D;
  int32_t G;           // ready flags to clear
  int32_t ud, Ud;      // down units per tile, in all
  int32_t grid;        // the decode kernel's grid (its stream-K ranges)
  int32_t maxp_d;      // partial slots per down tile
  const float* part;   // [Dt * maxp_d][N][128]
  uint16_t* y;
  uint32_t* ready;
};

__global__ void __launch_bounds__(kReduceThreads)
    decode_reduce_kernel(const ReduceParams r) {
  grid_dep_launch();
  grid_dep_wait();
  if (blockIdx.x == 0)
    for (int k = threadIdx.x; k < r.G; k += kReduceThreads) r.ready[k] = 0u;
  const int tile = blockIdx.x / (BM / kChunkRows);
  const int r0 = (blockIdx.x % (BM / kChunkRows)) * kChunkRows;
  if (tile * BM + r0 >= r.D) return;
  const int first = owner(tile * r.ud, r.Ud, r.grid);
  const int np = owner((tile + 1) * r.ud - 1, r.Ud, r.grid) - first + 1;
  const float* base = r.part + int64_t(tile) * r.maxp_d * r.N * BM;
  // thread -> float4 groups g = tid + kReduceThreads m: token g / kGpt, rows
  // 4 (g % kGpt) .. +3 of the chunk; pieces go in batches whose loads are all
  // in flight at once
  constexpr int kBatch = 8;
  constexpr int kGpt = kChunkRows / 4;   // float4 groups per token
  const int ngroups = r.T * kGpt;
  for (int g = threadIdx.x; g < ngroups; g += kReduceThreads) {
    const int t = g / kGpt;
    const int64_t off = int64_t(t) * BM + r0 + (g % kGpt) * 4;
    float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int i0 = 0; i0 < np; i0 += kBatch) {
      float4 v[kBatch];
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        if (i0 + i < np)
          v[i] = __ldcg(reinterpret_cast<const float4*>(base + int64_t(i0 + i) * r.N * BM + off));
#pragma unroll
      for (int i = 0; i < kBatch; ++i)
        if (i0 + i < np) add4(acc, v[i]);
    }
    const int d = tile * BM + r0 + (g % kGpt) * 4;
    uint16_t* dst = r.y + int64_t(t) * r.D + d;
    if (d + 3 < r.D) {
      uint2 w;
      w.x = pack_bf2(acc.x, acc.y);
      w.y = pack_bf2(acc.z, acc.w);
      *reinterpret_cast<uint2*>(dst) = w;
    } else {
      const float a[4] = {acc.x, acc.y, acc.z, acc.w};
      for (int k = 0; k < 4 && d + k < r.D; ++k)
        dst[k] = __bfloat16_as_ushort(__float2bfloat16_rn(a[k]));
    }
  }
}

// Shared memory after the rings for N tokens and FT features per gate/up tile.
inline int tail_bytes(int N, int FT) { return kTailFixed + N * FT * 2; }
// Ring depths: the activation ring keeps kStagesB stages (it is fed from
// L2), the weight ring takes the rest of shared memory.
// A block with many down units (each one a z load from L2 behind a ready
// flag) gets one activation stage more, at the cost of a weight stage: the 7B
// layer's blocks (T = 64), 21-22 units each, run 1.8 % faster with four; the
// 1B layer's, eight units each, are faster with three.  (Larger N keep three:
// their stages are bigger and the weight ring would drop to three.)
constexpr int kManyDownUnits = 16;
inline int stages_b(int N, int sub, int down_units = 0) {
  (void)sub;
  return down_units >= kManyDownUnits && N <= 64 ? kStagesB + 1 : kStagesB;
}
inline int ring_stages(int N, int sub, int FT, int down_units = 0) {
  const int budget = 227 * 1024 - 1024 - tail_bytes(N, FT) -
                     stages_b(N, sub, down_units) * sub * N * BK * 2;
  const int s = budget / (sub * A_BLOCK);
  return s > kMaxStages ? kMaxStages : s;
}
inline int smem_bytes(int N, int sub, int FT, int down_units = 0) {
  return 1024 + ring_stages(N, sub, FT, down_units) * sub * A_BLOCK +
         stages_b(N, sub, down_units) * sub * N * BK * 2 + tail_bytes(N, FT);
}

}  // namespace fused
}  // namespace stp
