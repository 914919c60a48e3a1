// One persistent tcgen05 kernel for the STAPLE layer at decode sizes
// (T <= 256 tokens): gate/up with the fused E-row add and SiLU gating, then
// the down projection, in a single launch.
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
//  * Phase 1, gate/up: whole tiles are spread over the blocks.  A block
//    finishes a tile straight from tensor memory, 16 tokens at a time: g and
//    u rows go to shared memory, then each of the 128 epilogue threads
//    computes 8 consecutive features of one token, h = u + E[id_t][f] (E rows
//    prefetched into shared memory during the main loop) and z = SiLU(g) h
//    (g and h saved when asked), written 16 bytes at a time; then the
//    tile's ready flag goes up.
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
//    bytes per token) and bumps the tile's counter.
//  * The down sums are spread over all blocks: once a block has finished its
//    own pieces, its epilogue warps take 16-row chunks from an atomic work
//    queue, wait (bounded) until the chunk's tile is complete, bring every
//    piece's 16 x N slice into the (then idle) ring memory with TMA loads
//    that are all in flight at once, sum them in piece order
//    (deterministic) and write y = bf16(sum).
//  * Every block finishes its gate/up tiles before it needs anybody's z, so
//    all waits end while all blocks are resident (grid <= SMs, one block
//    per SM).  Counters, flags and queue counters live in the first bytes of
//    the workspace; the last event of a call resets them, so a zero-filled
//    workspace stays valid across calls and graph replays.
//
// Warps: 0 weight (A) loads, 1 MMA issue + tensor memory, 2 activation (B)
// loads, 3..6 epilogue (each owns one 32-lane quarter of tensor memory).
// Every mbarrier wait and flag spin is bounded (STAPLE_ETIMEOUT).  The
// kernel is launched as a programmatic dependent: weights stream before
// griddepcontrol.wait; activations, outputs and counters only after it.
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
// shared memory after the rings: barriers + flags (512 B), token ids,
// g/u exchange chunk [128][17] fp32; then the E tile [N][64] bf16
constexpr int kTailFixed = 512 + kMaxN * 4 + 128 * kXStride * 4;

struct Params {
  int32_t T, N, D, F;
  int32_t sub;         // k blocks per unit (and per pipeline stage)
  int32_t stages;      // depth of the weight ring
  int32_t stages_b;    // depth of the activation ring
  int32_t G;           // gate/up tiles (F / 64)
  int32_t Dt;          // down tiles (ceil(D / 128))
  int32_t ug, ud;      // units per gate/up tile, per down tile
  int32_t Ud;          // down units (Dt * ud)
  int32_t maxp_d;      // partial slots per down tile
  int32_t rcap;        // partial slices per reduction batch (ring memory / slice)
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
  uint32_t* cnt;       // [Dt] pieces finished per down tile
  uint32_t* ready;     // [G] gate/up tile finished
  uint32_t* queue;     // [2]: next chunk to reduce, events seen
  float* part;         // [Dt * maxp_d][N][128]
  int32_t* err;
  uint64_t wait_ns;    // bound of every wait and flag spin (STAPLE_ETIMEOUT past it)
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

// A block finishes its gate/up tiles one after the other, so a tile's ready
// flag rises later the further it sits in its block's range.  The lateness of
// down unit x is the largest such position among the tiles that make the z
// columns x reads (0 when each is its block's first tile).
__device__ inline int unit_lateness(int x, const Params& p, int grid) {
  const int u = x % p.ud;
  int late = 0;
  for (int j = 0; j < p.sub; ++j) {
    const int t = u * p.sub + j;  // gate/up tile: 64 features = one 64-wide k block of z
    if (t >= p.G) break;
    late = max(late, t - range_start(owner(t, p.G, grid), p.G, grid));
  }
  return late;
}

__device__ __forceinline__ void grid_dep_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void grid_dep_launch() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}
__device__ __forceinline__ void epi_bar() { asm volatile("bar.sync 1, 128;" ::: "memory"); }
__device__ __forceinline__ uint32_t ld_acquire(const uint32_t* a) {
  uint32_t v;
  asm volatile("ld.acquire.gpu.global.u32 %0, [%1];" : "=r"(v) : "l"(a) : "memory");
  return v;
}
__device__ __forceinline__ void st_release(uint32_t* a, uint32_t v) {
  asm volatile("st.release.gpu.global.u32 [%0], %1;" ::"l"(a), "r"(v) : "memory");
}
__device__ __forceinline__ void fence_async_global() {
  asm volatile("fence.proxy.async.global;" ::: "memory");
}
__device__ __forceinline__ float4 ldcg4(const float* a) {
  return __ldcg(reinterpret_cast<const float4*>(a));
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
template <bool kOrder>
__global__ void __launch_bounds__(kThreads, 1)
    decode_fused_kernel(const __grid_constant__ CUtensorMap tm_wg,
                        const __grid_constant__ CUtensorMap tm_wu,
                        const __grid_constant__ CUtensorMap tm_wd,
                        const __grid_constant__ CUtensorMap tm_x,
                        const __grid_constant__ CUtensorMap tm_z,
                        const __grid_constant__ CUtensorMap tm_part, const Params p) {
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
  uint64_t* rbar = reinterpret_cast<uint64_t*>(tail + 320);  // partial slices landed
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
  uint16_t* s_e = reinterpret_cast<uint16_t*>(s_x + 128 * kXStride);  // [N][64]

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const int grid = gridDim.x;
  // this block's work: gate/up tiles [t0, t1) (ug units each), then down
  // units [d0, d1); local step i < ngs is gate/up, the rest down
  const int t0 = range_start(blockIdx.x, p.G, grid), t1 = range_start(blockIdx.x + 1, p.G, grid);
  const int d0 = range_start(blockIdx.x, p.Ud, grid), d1 = range_start(blockIdx.x + 1, p.Ud, grid);
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

  if (threadIdx.x == 0) {
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
    mbar_init(rbar, 1);
    mbar_init(obar, 1);
    mbar_init(dbar, 1);
    *abort_flag = 0;
    *s_epi_fail = 0;
    fence_barrier_init();
    tma_prefetch_desc(&tm_wg);
    tma_prefetch_desc(&tm_wu);
    tma_prefetch_desc(&tm_wd);
    tma_prefetch_desc(&tm_x);
    tma_prefetch_desc(&tm_z);
    tma_prefetch_desc(&tm_part);
  }
  if (warp == 1) {
    tmem_alloc(tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *tmem_slot;
  // the unit of the block's k-th down step
  auto unit = [&](int k) { return d0 + (reorder ? int(s_order[k]) : k); };
  // The step order is worked out by an epilogue warp (idle until the first
  // gate/up tile is done), off the path of the first weight loads; the
  // loaders wait for it on obar before their first down step.
  const bool ordered = reorder && nd > 0;
  if (warp == 3 && ordered) {
    for (int k = lane; k < nd; k += 32)
      s_late[k] = uint8_t(min(255, unit_lateness(d0 + k, p, grid)));
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
      int s = 0;
      uint32_t ph = 0;
      int issued = 0;
      for (int i = 0; i < nsteps; ++i) {
        if (i == ngs && ordered && !mbar_wait(obar, 0, abort_flag, p.err, p.wait_ns)) break;
        if (!mbar_wait(&emptyA[s], ph ^ 1, abort_flag, p.err, p.wait_ns)) break;
        mbar_arrive_expect_tx(&fullA[s], a_stage);
        uint8_t* a = sA + s * a_stage;
        for (int j = 0; j < p.sub; ++j) {
          if (i < ngs) {
            const int tile = t0 + i / p.ug, u = i % p.ug;
            const int k0 = (u * p.sub + j) * BK;
            tma_load_2d_hint(&tm_wg, &fullA[s], a + j * A_BLOCK, k0, tile * 64, once);
            tma_load_2d_hint(&tm_wu, &fullA[s], a + j * A_BLOCK + A_BLOCK / 2, k0, tile * 64, once);
          } else if (j == 0) {
            // one 3-D copy brings all `sub` k blocks of the unit
            const int x = unit(i - ngs), tile = x / p.ud, u = x % p.ud;
            tma_load_3d_hint(&tm_wd, &fullA[s], a, 0, tile * BM, u * p.sub, once);
          }
        }
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
        // unit d0 + k reads z columns [f_lo, f_hi), made by tiles f_lo/64 .. (f_hi-1)/64
        const int f_lo = ((d0 + k) % p.ud) * p.sub * BK;
        const int f_hi = min(p.F, f_lo + p.sub * BK);
        for (int t = f_lo / 64; t <= (f_hi - 1) / 64 && mine; ++t)
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
    for (int tile = t0; tile < t1 && alive; ++tile, ++piece) {
      const int f0 = tile * 64;
      // E[id_t][f0 .. f0+63] for every token: 128 bytes per row, 16-byte loads
      // issued while the tile's main loop is still streaming.  Up to 8 loads
      // per thread are put in flight before any of them is stored (behind a
      // saturated weight stream each round trip is long).
      for (int vb = et; vb < p.T * 8; vb += 8 * 128) {
        uint4 w[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = vb + k * 128;
          w[k] = make_uint4(0u, 0u, 0u, 0u);
          if (v < p.T * 8) {
            const int id = s_ids[v >> 3];
            if (id >= 0)
              w[k] = __ldg(reinterpret_cast<const uint4*>(p.e_base + int64_t(id) * p.e_pitch + f0) +
                           (v & 7));
          }
        }
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          const int v = vb + k * 128;
          if (v < p.T * 8) reinterpret_cast<uint4*>(s_e)[v] = w[k];
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
        // thread -> token c + et / 8, features 8 (et % 8) .. +7: one 16-byte
        // store per output row piece (the memory system is saturated by the
        // weight stream here, so the number of stores is what costs)
        const int j = et >> 3, fl0 = (et & 7) * 8, t = c + j;
        if (t < p.T) {
          const uint4 ev = *reinterpret_cast<const uint4*>(s_e + t * 64 + fl0);
          const uint32_t ew[4] = {ev.x, ev.y, ev.z, ev.w};
          uint32_t zw[4], gw[4], hw[4];
#pragma unroll
          for (int k = 0; k < 4; ++k) {
            const int f = fl0 + 2 * k;
            const float g0 = s_x[f * kXStride + j], g1 = s_x[(f + 1) * kXStride + j];
            const float h0 = s_x[(64 + f) * kXStride + j] + bf_lo(ew[k]);
            const float h1 = s_x[(65 + f) * kXStride + j] + bf_hi(ew[k]);
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
        epi_bar();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&tempty[buf]);
      __threadfence();
      fence_async_global();
      epi_bar();
      if (et == 0) st_release(&p.ready[tile], 1u);
    }
    // ---- phase 2: down pieces -> fp32 partial slots
    for (int x = d0; x < d1 && alive; ++piece) {
      const int tile = x / p.ud;
      const int x_end = min(d1, (tile + 1) * p.ud);
      const int idx = blockIdx.x - owner(tile * p.ud, p.Ud, grid);
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
      __threadfence();
      epi_bar();
      if (et == 0) atomicAdd(&p.cnt[tile], 1u);
    }

    // ---- down sums: 16-row chunks from the shared work queue.  queue[0]
    // hands out chunks; queue[1] counts events: each reduced chunk and each
    // block's final fetch past the end.  The event that completes the count
    // (nchunks + grid) is the last use of any counter or flag of this call,
    // so that thread resets them all for the next call.
    const int chunks_per_tile = BM / kChunkRows;
    const uint32_t nchunks = uint32_t(p.Dt * chunks_per_tile);
    const uint32_t nevents = nchunks + uint32_t(grid);
    // slices land in the ring memory, idle once this block's MMAs are done
    uint8_t* rbuf = sA;
    const int slice = p.N * kChunkRows * 4;   // bytes of one piece's [N][16] fp32 slice
    uint32_t rph = 0;
    // thread et == 0 issues the slice loads; a batch it issued and has not
    // seen land (after an abort) is waited for before the block exits
    bool r_pending = false;
    uint32_t r_phase = 0;
    auto event = [&]() {
      if (atomicAdd(&p.queue[1], 1u) == nevents - 1) {
        for (int k = 0; k < p.Dt; ++k) p.cnt[k] = 0u;
        for (int k = 0; k < p.G; ++k) p.ready[k] = 0u;
        p.queue[0] = 0u;
        p.queue[1] = 0u;
        __threadfence();
      }
    };
    // thread et owns the float4 groups g = et + 128 m (token g / 4, rows
    // 4 (g % 4) .. +3 of the chunk); kMaxN * 4 groups at most
    constexpr int kGroups = kMaxN * (kChunkRows / 4) / 128;
    while (alive) {
      // one thread takes a chunk, waits for its tile and puts the first batch
      // of slice loads in flight; all follow its verdict
      epi_bar();
      if (et == 0) {
        int code = int(atomicAdd(&p.queue[0], 1u));
        if (code < int(nchunks)) {
          const int tl = code / chunks_per_tile;
          const int first = owner(tl * p.ud, p.Ud, grid);
          const int np = owner((tl + 1) * p.ud - 1, p.Ud, grid) - first + 1;
          if (!spin_until(&p.cnt[tl], uint32_t(np), abort_flag, p.err, p.wait_ns)) {
            code = -1;
          } else {
            fence_async_global();
            const int nb = min(np, p.rcap);
            const int r0 = (code % chunks_per_tile) * kChunkRows;
            r_pending = true;
            r_phase = rph;
            mbar_arrive_expect_tx(rbar, uint32_t(nb * slice));
            for (int i = 0; i < nb; ++i)
              tma_load_2d(&tm_part, rbar, rbuf + i * slice, r0, (tl * p.maxp_d + i) * p.N);
          }
        }
        *s_flag = code;
      }
      epi_bar();
      const int code = *s_flag;
      if (code < 0) break;
      const uint32_t c = uint32_t(code);
      if (c >= nchunks) {
        if (et == 0) event();
        break;
      }
      const int tile = int(c) / chunks_per_tile;
      const int r0 = (int(c) % chunks_per_tile) * kChunkRows;
      const int o0 = owner(tile * p.ud, p.Ud, grid);
      const int npieces = owner((tile + 1) * p.ud - 1, p.Ud, grid) - o0 + 1;
      const int ngroups = p.T * (kChunkRows / 4);
      float4 acc[kGroups];
#pragma unroll
      for (int m = 0; m < kGroups; ++m) acc[m] = make_float4(0.f, 0.f, 0.f, 0.f);
      bool ok = true;
      for (int i0 = 0; i0 < npieces; i0 += p.rcap) {
        const int nb = min(npieces - i0, p.rcap);
        if (i0 > 0) {
          epi_bar();  // the previous batch has been read
          if (et == 0) {
            r_pending = true;
            r_phase = rph;
            mbar_arrive_expect_tx(rbar, uint32_t(nb * slice));
            for (int i = 0; i < nb; ++i)
              tma_load_2d(&tm_part, rbar, rbuf + i * slice, r0,
                          (tile * p.maxp_d + i0 + i) * p.N);
          }
        }
        ok = mbar_wait(rbar, rph, abort_flag, p.err, p.wait_ns);
        if (ok && et == 0) r_pending = false;
        rph ^= 1u;
        if (!__all_sync(0xffffffffu, ok) && lane == 0) *s_epi_fail = 1;
        epi_bar();
        if (*s_epi_fail) {
          ok = false;
          break;
        }
        for (int i = 0; i < nb; ++i) {
          const float4* sl = reinterpret_cast<const float4*>(rbuf + i * slice);
#pragma unroll
          for (int m = 0; m < kGroups; ++m) {
            const int gi = et + 128 * m;
            if (gi < ngroups) add4(acc[m], sl[gi]);
          }
        }
      }
      if (!ok) break;
#pragma unroll
      for (int m = 0; m < kGroups; ++m) {
        const int gi = et + 128 * m;
        if (gi >= ngroups) continue;
        const int t = gi >> 2, d = tile * BM + r0 + (gi & 3) * 4;
        uint16_t* dst = p.y + int64_t(t) * p.D + d;
        if (d + 3 < p.D) {
          uint2 w;
          w.x = pack_bf2(acc[m].x, acc[m].y);
          w.y = pack_bf2(acc[m].z, acc[m].w);
          *reinterpret_cast<uint2*>(dst) = w;
        } else {
          const float a[4] = {acc[m].x, acc[m].y, acc[m].z, acc[m].w};
          for (int k = 0; k < 4 && d + k < p.D; ++k)
            dst[k] = __bfloat16_as_ushort(__float2bfloat16_rn(a[k]));
        }
      }
      if (et == 0) event();
    }
    if (et == 0 && r_pending) mbar_drain(rbar, r_phase);
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) {
    __syncwarp();
    tmem_dealloc(tmem_base, tmem_cols);
  }
}

// Shared memory after the rings for N tokens.
inline int tail_bytes(int N) { return kTailFixed + N * 64 * 2; }
// Ring depths: the activation ring keeps kStagesB stages (it is fed from
// L2), the weight ring takes the rest of shared memory.
inline int stages_b(int N, int sub) { (void)N; (void)sub; return kStagesB; }
inline int ring_stages(int N, int sub) {
  const int budget = 227 * 1024 - 1024 - tail_bytes(N) - stages_b(N, sub) * sub * N * BK * 2;
  const int s = budget / (sub * A_BLOCK);
  return s > kMaxStages ? kMaxStages : s;
}
// Partial slices (one piece's [N][16] fp32) that fit in the two rings.
inline int reduce_slices(int N, int sub) {
  const int ring = ring_stages(N, sub) * sub * A_BLOCK + stages_b(N, sub) * sub * N * BK * 2;
  return ring / (N * kChunkRows * 4);
}
inline int smem_bytes(int N, int sub) {
  return 1024 + ring_stages(N, sub) * sub * A_BLOCK + stages_b(N, sub) * sub * N * BK * 2 +
         tail_bytes(N);
}

}  // namespace fused
}  // namespace stp
