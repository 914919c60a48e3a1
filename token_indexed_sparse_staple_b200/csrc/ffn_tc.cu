// Host side of the bf16 tcgen05 path: TMA tensor maps and the launches of
// the six contractions of the layer (K5, K6, K7, K9, K10), each with its
// epilogue fused into the GEMM kernel of gemm_tc.cuh.
//
//   K5  [g | u] = x W_gate^T | x W_up^T, epilogue h = u + E[row], z = SiLU(g) h
//   K6  y       = z W_down^T
//   K7  dz      = dY W_down,  epilogue dh = dz SiLU(g), dg = dz h SiLU'(g)
//   K9  dx      = dg W_gate + dh W_up                  (K concatenated)
//   K10 dW_gate | dW_up = [dg | dh]^T x,  dW_down = dY^T z
#include <cudaTypedefs.h>

#include <algorithm>
#include <atomic>
#include <map>
#include <mutex>
#include <tuple>

#include "decode_fused.cuh"
#include "gemm_tc.cuh"
#include "internal.h"

namespace stp {

namespace {

PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;
std::once_flag g_encode_once;

PFN_cuTensorMapEncodeTiled_v12000 encoder() {
  std::call_once(g_encode_once, [] {
    void* fn = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
  });
  return g_encode;
}

// 2-D bf16 tensor map over a row-major matrix with `rows` rows of `cols`
// elements (leading dimension ld), box = box_cols x box_rows, 128-byte swizzle.
bool make_map(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
              uint32_t box_cols, uint32_t box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 2};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D fp32 tensor map without swizzle: `rows` rows of `cols` floats
// (leading dimension ld floats), box = box_cols x box_rows.
bool make_map_f32(CUtensorMap* m, const void* base, uint64_t cols, uint64_t rows, uint64_t ld,
                  uint32_t box_cols, uint32_t box_rows) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {ld * 4};
  cuuint32_t box[2] = {box_cols, box_rows};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_NONE,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major bf16 operand [rows][k] seen as 3-D: (k within a 64-wide block,
// row, block).  A box of `depth` blocks lands in shared memory as `depth`
// consecutive [box_rows][64] 128-byte-swizzled tiles, so one copy fetches
// what `depth` 2-D copies would.
bool kmajor_blocks(CUtensorMap* m, const void* base, int rows, int k, int64_t ld, int box_rows,
                   int depth) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {uint64_t(tc::BK), uint64_t(rows), uint64_t(k / tc::BK)};
  cuuint64_t strides[2] = {uint64_t(ld) * 2, uint64_t(tc::BK) * 2};
  cuuint32_t box[3] = {uint32_t(tc::BK), uint32_t(box_rows), uint32_t(depth)};
  cuuint32_t estr[3] = {1, 1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// K-major operand [rows][k]: box 64 (k) x 128 (rows).
bool kmajor(CUtensorMap* m, const void* base, int rows, int k, int64_t ld) {
  return make_map(m, base, uint64_t(k), uint64_t(rows), uint64_t(ld), tc::BK, 128);
}
// MN-major operand stored [k][mn]: box 64 (mn) x 64 (k).
bool mnmajor(CUtensorMap* m, const void* base, int k, int mn, int64_t ld) {
  return make_map(m, base, uint64_t(mn), uint64_t(k), uint64_t(ld), 64, tc::BK);
}

// Output map for the staged epilogue stores: bf16 [rows][cols] with leading
// dimension ld, box 32 x 32, 64-byte swizzle (the layout write_row_sw64
// stages).
bool out_map(CUtensorMap* m, const void* base, int rows, int cols, int64_t ld) {
  auto enc = encoder();
  if (!enc) return false;
  cuuint64_t dims[2] = {uint64_t(cols), uint64_t(rows)};
  cuuint64_t strides[1] = {uint64_t(ld) * 2};
  cuuint32_t box[2] = {32, 32};
  cuuint32_t estr[2] = {1, 1};
  return enc(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
             estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_64B,
             CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// o: the maps of a staged epilogue (EPI_GATEUP: z, g, h; EPI_DZ: dg, dh, then
// the inputs g, h), NULL for the other epilogues.
template <bool A_MN, bool B_MN, int BSRC, int EPI>
staple_status launch(const char* name, const DeviceInfo& di, const CUtensorMap& a,
                     const CUtensorMap& b0, const CUtensorMap& b1, tc::Params p, cudaStream_t st,
                     const CUtensorMap* o = nullptr) {
  p.k_blocks = (p.K + tc::BK - 1) / tc::BK;
  p.wait_ns = di.wait_ns;
  const int ntiles = p.tiles_m * p.tiles_n;
  if (ntiles == 0) return STAPLE_OK;
  if (p.group_m <= 0) p.group_m = 16;
  auto kern = tc::gemm_kernel<A_MN, B_MN, BSRC, EPI>;
  // the shared-memory opt-in is set once per device and instantiation, so
  // that no runtime attribute call happens while a stream is being captured
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t bit = uint64_t(1) << (di.device & 63);
  if (!(attr_done.load() & bit)) {
    if (cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             tc::smem_bytes<EPI>()) != cudaSuccess)
      return STAPLE_ECUDA;
    attr_done.fetch_or(bit);
  }
  const int avail = std::max(1, di.num_sms - di.sm_reserve);
  // fp32 outputs (the weight gradients): when the tiles of the last, partial
  // round, taken twice, still fit in one round, each of them runs as two
  // halves of its k range that add onto a zeroed output.  That round then
  // takes half as long (dW_down, 512 tiles on 148 SMs: 3.5 rounds of work
  // instead of 4).  Both halves add onto zero, so the sum (0 + a) + b is the
  // same whichever lands first.
  p.nsplit = 0;
  p.kb_split = 0;
  if (EPI == tc::EPI_F32 && p.k_blocks >= 2) {
    const int rem = ntiles % avail;
    if (rem > 0 && 2 * rem <= avail) {
      p.nsplit = rem;
      p.kb_split = p.k_blocks / 2;
    }
  }
  int grid;
  if (p.nsplit > 0) {
    grid = std::min(avail, ntiles + p.nsplit);
  } else {
    // The fewest blocks that take the same largest number of tiles each
    // (1024 tiles on 148 SMs: 147 blocks of seven), leaving the rest of the
    // SMs to kernels on other streams.
    const int per_block = (ntiles + avail - 1) / avail;
    grid = (ntiles + per_block - 1) / per_block;
  }
  const CUtensorMap& o0 = o ? o[0] : a;
  const CUtensorMap& o1 = o ? o[1] : a;
  const CUtensorMap& o2 = o ? o[2] : a;
  const CUtensorMap& o3 = (o && EPI == tc::EPI_DZ) ? o[3] : a;
  if (p.nsplit > 0) {
    STP_LAUNCH("gemm_split_zero", st,
               tc::zero_split_tiles_kernel<<<p.nsplit * (tc::BM / tc::kZeroRows), 256, 0, st>>>(p));
    if (cudaGetLastError() != cudaSuccess) return STAPLE_ECUDA;
  }
  STP_LAUNCH(name, st,
             kern<<<grid, tc::kThreads, tc::smem_bytes<EPI>(), st>>>(a, b0, b1, o0, o1, o2, o3,
                                                                      p));
  return cudaGetLastError() == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

inline int cdiv(int a, int b) { return (a + b - 1) / b; }

// K-major operand with a box of `rows` rows (weights: 64 or 128; tokens: N).
bool kmajor_rows(CUtensorMap* m, const void* base, int rows, int k, int64_t ld, int box_rows) {
  return make_map(m, base, uint64_t(k), uint64_t(rows), uint64_t(ld), tc::BK, uint32_t(box_rows));
}

}  // namespace

// ---------------------------------------------------------------- decode
namespace {

struct DecodePlan {
  int N, sub, G, Dt, ug, ud, Ud, grid, maxp_d;
  size_t counter_bytes, part_bytes;
};

// Partial slots per down tile for every grid up to kMaxDecodeGrid: a block's
// range holds at least floor(Ud / kMaxDecodeGrid) units, so a tile of `units`
// units meets at most (units - 1) / that + 2 ranges.  (The exact count is not
// monotone in the grid size, so the bound is what sizes the workspace and
// strides the slots.)
int piece_bound(int units, int U) {
  const int minlen = std::max(1, U / kMaxDecodeGrid);
  return std::min(kMaxDecodeGrid, (units - 1) / minlen + 2);
}

// FT: features per gate/up tile (64: W_gate over W_up rows; 128: STEM, W_gate alone)
DecodePlan plan_decode(int T, int D, int F, int FT, int num_sms) {
  DecodePlan pl{};
  pl.N = cdiv(T, 16) * 16;
  pl.sub = ((D / 64) % 2 == 0 && (F / 64) % 2 == 0 && fused::ring_stages(pl.N, 2, FT) >= 3) ? 2 : 1;
  pl.G = F / FT;
  pl.Dt = cdiv(D, fused::BM);
  pl.ug = (D / 64) / pl.sub;
  pl.ud = (F / 64) / pl.sub;
  pl.Ud = pl.Dt * pl.ud;
  // every block needs at least one down unit (so the blocks covering a down
  // tile are consecutive and each writes its partial slot)
  pl.grid = std::max(1, std::min(std::min(num_sms, kMaxDecodeGrid), pl.Ud));
  // Prefer the largest grid that divides the down units, if it keeps at
  // least 3/4 of the SMs: every block then streams the same share of W_down,
  // a down tile's pieces are whole blocks' ranges, and the SMs left over
  // take the split-k sum kernel's blocks at once (1024 units: 128 blocks of
  // eight instead of 148 of six or seven).
  for (int g = pl.grid; 4 * g >= 3 * pl.grid; --g)
    if (pl.Ud % g == 0) {
      pl.grid = g;
      break;
    }
  // With more gate/up tiles than blocks, use the fewest blocks that take the
  // same largest number of tiles each, so that no block makes more tiles
  // than the others (172 tiles: 86 blocks of two instead of 148 of one or two).
  if (pl.G > pl.grid) {
    const int per = cdiv(pl.G, pl.grid);
    pl.grid = std::max(1, std::min(pl.grid, cdiv(pl.G, per)));
  }
  pl.maxp_d = piece_bound(pl.ud, pl.Ud);
  pl.counter_bytes = decode_counter_bytes(D, F);
  pl.part_bytes = size_t(pl.Dt * pl.maxp_d) * pl.N * fused::BM * sizeof(float);
  return pl;
}

}  // namespace

size_t decode_flag_bytes(int D, int F) {
  (void)D;
  // ready flags and the cluster path's count of blocks past their z poll
  const size_t words = size_t((F / 64) + 2);
  return (words * sizeof(uint32_t) + 255) & ~size_t(255);
}

size_t decode_counter_bytes(int D, int F) {
  return decode_flag_bytes(D, F) + seg_counter_bytes(kMaxDedupT, F);
}

size_t decode_scratch_bytes(int T, int D, int F) {
  if (T < 1 || T > kMaxDecodeT || D % 64 || F % 64) return 0;
  // the largest grid the launcher may use gives the most pieces per tile (the
  // partial slots do not depend on the gate/up tiling)
  const DecodePlan pl = plan_decode(T, D, F, 64, kMaxDecodeGrid);
  return pl.part_bytes;
}

staple_status tc_decode_fwd(const DeviceInfo& di, int T, int D, int F, const void* x,
                            const staple_embed* e, const void* wg, const void* wu, const void* wd,
                            void* z, void* y, void* g_save, void* h_save, void* ws,
                            int32_t* err, cudaStream_t st) {
  const bool stem = e && (e->flags & STAPLE_EMBED_REPLACE_UP);
  const int FT = stem ? 128 : 64;
  if (F % FT) return STAPLE_EUNSUPPORTED;
  const DecodePlan pl = plan_decode(T, D, F, FT, di.num_sms);
  void* part = static_cast<uint8_t*>(ws) + pl.counter_bytes;
  CUtensorMap mg, mu, md, mx, mz;
  if (!kmajor_rows(&mg, wg, F, D, D, FT) || !kmajor_rows(&mu, stem ? wg : wu, F, D, D, 64) ||
      !kmajor_blocks(&md, wd, D, F, F, fused::BM, pl.sub) ||
      !kmajor_blocks(&mx, x, T, D, D, pl.N, pl.sub) || !kmajor_blocks(&mz, z, T, F, F, pl.N, pl.sub))
    return STAPLE_ECUDA;
  fused::Params p{};
  p.T = T;
  p.N = pl.N;
  p.D = D;
  p.F = F;
  p.sub = pl.sub;
  p.stages = fused::ring_stages(pl.N, pl.sub, FT);
  p.stages_b = fused::stages_b(pl.N, pl.sub);
  p.G = pl.G;
  p.Dt = pl.Dt;
  p.ug = pl.ug;
  p.ud = pl.ud;
  p.Ud = pl.Ud;
  p.maxp_d = pl.maxp_d;
  p.stage_tmem = 1;
  p.z = static_cast<uint16_t*>(z);
  p.g_save = static_cast<uint16_t*>(g_save);
  p.h_save = static_cast<uint16_t*>(h_save);
  p.y = static_cast<uint16_t*>(y);
  p.e_mode = e ? e->mode : STAPLE_EMBED_NONE;
  if (e && e->mode != STAPLE_EMBED_NONE) {
    p.e_base = static_cast<const uint16_t*>(e->base);
    p.e_pitch = e->row_pitch;
    p.e_index = e->index;
    p.e_rows = e->n_rows;
  }
  uint32_t* words = static_cast<uint32_t*>(ws);
  p.ready = words;
  p.part = static_cast<float*>(part);
  p.err = err;
  p.wait_ns = di.wait_ns;
  p.fin = words + F / 64;

  using Kern = void (*)(CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap, CUtensorMap,
                        fused::Params);
  // [cluster][order][stem]
  const Kern kerns[2][2][2] = {{{fused::decode_fused_kernel<false, false, false>,
                                 fused::decode_fused_kernel<false, true, false>},
                                {fused::decode_fused_kernel<true, false, false>,
                                 fused::decode_fused_kernel<true, true, false>}},
                               {{fused::decode_fused_kernel<false, false, true>,
                                 fused::decode_fused_kernel<false, true, true>},
                                {fused::decode_fused_kernel<true, false, true>,
                                 fused::decode_fused_kernel<true, true, true>}}};
  int smem = fused::smem_bytes(pl.N, pl.sub, FT);   // (the path's own rings: below)
  static std::atomic<uint64_t> attr_done{0};
  const uint64_t bit = uint64_t(1) << (di.device & 63);
  if (!(attr_done.load() & bit)) {
    for (const auto& a : kerns)
      for (const auto& row : a)
        for (Kern k : row)
          if (cudaFuncSetAttribute(k, cudaFuncAttributeMaxDynamicSharedMemorySize, 227 * 1024) !=
              cudaSuccess)
            return STAPLE_ECUDA;
    attr_done.fetch_or(bit);
  }
  // Blocks wait (bounded) on flags other blocks raise, so the whole grid must
  // be resident at once.  Checked per device, kernel, shared-memory size and
  // cluster size (queried outside any stream capture on first use): the
  // grid may not exceed what the device can hold at once, in blocks or in
  // clusters.
  auto resident = [&](Kern k, int cluster) -> int {
    static std::mutex mu;
    static std::map<std::tuple<const void*, int, int, int>, int> known;
    std::lock_guard<std::mutex> lock(mu);
    const auto key = std::make_tuple(reinterpret_cast<const void*>(k), di.device, smem, cluster);
    auto it = known.find(key);
    if (it != known.end()) return it->second;
    int n = 0;
    if (cluster == 1) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&n, k, fused::kThreads, smem) != cudaSuccess)
        return -1;
      n *= di.num_sms;
    } else {
      cudaLaunchConfig_t q = {};
      q.gridDim = dim3(cluster);
      q.blockDim = dim3(fused::kThreads);
      q.dynamicSmemBytes = smem;
      cudaLaunchAttribute ca[1];
      ca[0].id = cudaLaunchAttributeClusterDimension;
      ca[0].val.clusterDim.x = cluster;
      ca[0].val.clusterDim.y = 1;
      ca[0].val.clusterDim.z = 1;
      q.attrs = ca;
      q.numAttrs = 1;
      if (cudaOccupancyMaxActiveClusters(&n, k, &q) != cudaSuccess) return -1;
    }
    known.emplace(key, n);
    return n;
  };
  // The cluster path (the split-k sum inside the launch, see the kernel):
  // one cluster of kCluster blocks per down tile, all resident at once, at
  // least one down unit per block, the pushed accumulator rows within the
  // rings, and at least as many blocks as the two-launch path would stream
  // with (7B layer: 32 tiles, 128 blocks instead of 86).  With fewer tiles
  // than that (1B layer: 16), a tile would need several clusters whose
  // partials meet in global memory at the end of the launch, which measured
  // slower than the sum kernel; those shapes take the two-launch path.
  int clu = 0;
  {
    const int maxcl = resident(kerns[1][0][stem ? 1 : 0], fused::kCluster);
    if (maxcl < 0) return STAPLE_ECUDA;
    const size_t rings = size_t(p.stages) * pl.sub * fused::A_BLOCK +
                         size_t(p.stages_b) * pl.sub * pl.N * fused::BK * 2;
    const size_t recv = size_t(fused::BM) * (pl.N + 4) * sizeof(float);
    clu = (maxcl >= pl.Dt && pl.ud >= fused::kCluster && recv <= rings &&
           pl.Dt * fused::kCluster >= pl.grid) ? 1 : 0;
  }
  const int grid = clu ? pl.Dt * fused::kCluster : pl.grid;
  // the rings for the path taken: the most down units a block gets sets the
  // activation ring's depth
  {
    const int upb = clu ? cdiv(pl.ud, fused::kCluster) : cdiv(pl.Ud, grid);
    p.stages = fused::ring_stages(pl.N, pl.sub, FT, upb);
    p.stages_b = fused::stages_b(pl.N, pl.sub, upb);
    smem = fused::smem_bytes(pl.N, pl.sub, FT, upb);
  }
  // down-step ordering only where some block makes two or more gate/up tiles
  const int order = pl.G > grid ? 1 : 0;
  const Kern kern = kerns[clu][order][stem ? 1 : 0];
  if (!clu) {
    const int n = resident(kern, 1);
    if (n < 0) return STAPLE_ECUDA;
    if (grid > n) return STAPLE_EUNSUPPORTED;
  }
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(grid);
  cfg.blockDim = dim3(fused::kThreads);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = fused::kCluster;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = clu ? 2 : 1;
  cudaError_t ce = cudaSuccess;
  STP_LAUNCH(stem ? "k5k6_decode_fused_stem" : "k5k6_decode_fused", st,
             ce = cudaLaunchKernelEx(&cfg, kern, mg, mu, md, mx, mz, p));
  if (ce != cudaSuccess) return STAPLE_ECUDA;
  if (clu) return STAPLE_OK;
  // the split-k sums, right behind (programmatic dependent, see the kernel)
  fused::ReduceParams r{};
  r.T = T;
  r.N = pl.N;
  r.D = D;
  r.G = pl.G;
  r.ud = pl.ud;
  r.Ud = pl.Ud;
  r.grid = pl.grid;
  r.maxp_d = pl.maxp_d;
  r.part = p.part;
  r.y = p.y;
  r.ready = p.ready;
  cudaLaunchConfig_t rcfg = cfg;
  rcfg.gridDim = dim3(pl.Dt * (fused::BM / fused::kChunkRows));
  rcfg.blockDim = dim3(fused::kReduceThreads);
  rcfg.dynamicSmemBytes = 0;
  STP_LAUNCH("k6r_decode_reduce", st,
             ce = cudaLaunchKernelEx(&rcfg, fused::decode_reduce_kernel, r));
  return ce == cudaSuccess ? STAPLE_OK : STAPLE_ECUDA;
}

staple_status tc_ffn_fwd(const DeviceInfo& di, int T, int D, int F, const void* x,
                         const staple_embed* e, const void* wg, const void* wu, const void* wd,
                         void* z, void* y, void* g_save, void* h_save, int32_t* err,
                         cudaStream_t st) {
  if (T == 0) return STAPLE_OK;
  CUtensorMap mx, mg, mu, mz, md;
  if (!kmajor(&mx, x, T, D, D) || !kmajor(&mg, wg, F, D, D) ||
      !kmajor(&mu, wu ? wu : wg, F, D, D) || !kmajor(&mz, z, T, F, F) ||
      !kmajor(&md, wd, D, F, F))
    return STAPLE_ECUDA;
  {
    tc::Params p{};
    p.M = T;
    p.N = F;
    p.K = D;
    p.tiles_m = cdiv(T, tc::BM);
    p.tiles_n = cdiv(F, tc::BN / 2);
    p.z = static_cast<uint16_t*>(z);
    p.g_save = static_cast<uint16_t*>(g_save);
    p.h_save = static_cast<uint16_t*>(h_save);
    p.ldf = F;
    p.e_mode = e ? e->mode : STAPLE_EMBED_NONE;
    if (e && e->mode != STAPLE_EMBED_NONE) {
      p.e_base = static_cast<const uint16_t*>(e->base);
      p.e_pitch = e->row_pitch;
      p.e_index = e->index;
      p.e_rows = e->n_rows;
    }
    p.err = err;
    CUtensorMap mo[3];
    if (!out_map(&mo[0], z, T, F, F) || !out_map(&mo[1], g_save ? g_save : z, T, F, F) ||
        !out_map(&mo[2], h_save ? h_save : z, T, F, F))
      return STAPLE_ECUDA;
    staple_status s;
    if (e && (e->flags & STAPLE_EMBED_REPLACE_UP)) {
      // STEM: the gate projection alone, 256 features per tile
      p.tiles_n = cdiv(F, tc::BN);
      s = launch<false, false, tc::B_ONE, tc::EPI_GATE_E>("k5_gate_stem", di, mx, mg, mg, p, st,
                                                            mo);
    } else {
      s = launch<false, false, tc::B_NHALF, tc::EPI_GATEUP>("k5_gateup", di, mx, mg, mu, p, st,
                                                            mo);
    }
    if (s != STAPLE_OK) return s;
  }
  tc::Params q{};
  q.M = T;
  q.N = D;
  q.K = F;
  q.tiles_m = cdiv(T, tc::BM);
  q.tiles_n = cdiv(D, tc::BN);
  q.out = y;
  q.ldo = D;
  q.m_split = T;
  q.err = err;
  return launch<false, false, tc::B_ONE, tc::EPI_BF16>("k6_down", di, mz, md, md, q, st);
}

staple_status tc_dz(const DeviceInfo& di, int T, int D, int F, const void* dy, const void* g_save,
                    const void* h_save, const void* wd, void* dgh, int32_t* err, cudaStream_t st) {
  if (T == 0) return STAPLE_OK;
  CUtensorMap mdy, mwd;
  // A = dY [T][D] (K-major over d); B(n = f, k = d) = W_down[d][f]: MN-major
  if (!kmajor(&mdy, dy, T, D, D) || !mnmajor(&mwd, wd, D, F, F)) return STAPLE_ECUDA;
  tc::Params p{};
  p.M = T;
  p.N = F;
  p.K = D;
  p.tiles_m = cdiv(T, tc::BM);
  p.tiles_n = cdiv(F, tc::BN);
  p.ldf = F;
  p.g_in = static_cast<const uint16_t*>(g_save);
  p.h_in = static_cast<const uint16_t*>(h_save);
  p.dgh = static_cast<uint16_t*>(dgh);
  p.err = err;
  // dg = columns [0, F) of dgh, dh = [F, 2F): two maps of F columns, row pitch 2F
  // inputs g and h: [T][F] with row pitch F, the same 32 x 32 box
  CUtensorMap mo[4];
  if (!out_map(&mo[0], dgh, T, F, 2 * int64_t(F)) ||
      !out_map(&mo[1], static_cast<uint16_t*>(dgh) + F, T, F, 2 * int64_t(F)) ||
      !out_map(&mo[2], g_save, T, F, F) || !out_map(&mo[3], h_save, T, F, F))
    return STAPLE_ECUDA;
  return launch<false, true, tc::B_ONE, tc::EPI_DZ>("k7_dz", di, mdy, mwd, mwd, p, st, mo);
}

staple_status tc_ffn_bwd(const DeviceInfo& di, int T, int D, int F, const void* dy,
                         const void* x, const void* z, const void* dgh, const void* wg,
                         const void* wu, void* dx, float* dwg, float* dwu, float* dwd,
                         int32_t* err, cudaStream_t st) {
  staple_status s;
  const uint16_t* dgh16 = static_cast<const uint16_t*>(dgh);
  if (T == 0) {
    if (dwg && cudaMemsetAsync(dwg, 0, size_t(F) * D * 4, st) != cudaSuccess) return STAPLE_ECUDA;
    if (dwu && cudaMemsetAsync(dwu, 0, size_t(F) * D * 4, st) != cudaSuccess) return STAPLE_ECUDA;
    if (dwd && cudaMemsetAsync(dwd, 0, size_t(F) * D * 4, st) != cudaSuccess) return STAPLE_ECUDA;
    return STAPLE_OK;
  }
  if (dx && !wu) {
    // K9 of the STEM layer (no up-projection): dx = dg W_gate, A = the dg
    // half of dgh (K = F, row pitch 2F), B(n = d, k = f) = W_gate[f][d]
    CUtensorMap ma, mb0;
    if (!kmajor(&ma, dgh, T, F, 2 * F) || !mnmajor(&mb0, wg, F, D, D)) return STAPLE_ECUDA;
    tc::Params p{};
    p.M = T;
    p.N = D;
    p.K = F;
    p.tiles_m = cdiv(T, tc::BM);
    p.tiles_n = cdiv(D, tc::BN);
    p.out = dx;
    p.ldo = D;
    p.m_split = T;
    p.err = err;
    if ((s = launch<false, true, tc::B_ONE, tc::EPI_BF16>("k9_dx", di, ma, mb0, mb0, p, st)) !=
        STAPLE_OK)
      return s;
  } else if (dx) {
    // K9: A = dgh [T][2F] K-major; B(n = d, k = f') = W_gate[f'][d] | W_up[f' - F][d]: MN-major
    CUtensorMap ma, mb0, mb1;
    if (!kmajor(&ma, dgh, T, 2 * F, 2 * F) || !mnmajor(&mb0, wg, F, D, D) ||
        !mnmajor(&mb1, wu, F, D, D))
      return STAPLE_ECUDA;
    tc::Params p{};
    p.M = T;
    p.N = D;
    p.K = 2 * F;
    p.ksplit = F;
    p.tiles_m = cdiv(T, tc::BM);
    p.tiles_n = cdiv(D, tc::BN);
    p.out = dx;
    p.ldo = D;
    p.m_split = T;
    p.err = err;
    if ((s = launch<false, true, tc::B_KSPLIT, tc::EPI_BF16>("k9_dx", di, ma, mb0, mb1, p, st)) !=
        STAPLE_OK)
      return s;
  }
  if (dwg || dwu) {
    // K10a: C[m = f'][n = d] = sum_t dgh[t][f'] x[t][d]; A and B MN-major
    const bool both = dwg && dwu;
    const int M = both ? 2 * F : F;
    CUtensorMap ma, mb;
    if (!mnmajor(&ma, dwg ? dgh16 : dgh16 + F, T, M, 2 * F) || !mnmajor(&mb, x, T, D, D))
      return STAPLE_ECUDA;
    tc::Params p{};
    p.M = M;
    p.N = D;
    p.K = T;
    p.tiles_m = cdiv(M, tc::BM);
    p.tiles_n = cdiv(D, tc::BN);
    p.out = dwg ? dwg : dwu;
    p.out2 = dwu;
    p.ldo = D;
    p.m_split = both ? F : M;
    p.err = err;
    if ((s = launch<true, true, tc::B_ONE, tc::EPI_F32>("k10_dw_gate_up", di, ma, mb, mb, p, st)) != STAPLE_OK)
      return s;
  }
  if (dwd) {
    // K10b: C[m = d][n = f] = sum_t dY[t][d] z[t][f]; A and B MN-major
    CUtensorMap ma, mb;
    if (!mnmajor(&ma, dy, T, D, D) || !mnmajor(&mb, z, T, F, F)) return STAPLE_ECUDA;
    tc::Params p{};
    p.M = D;
    p.N = F;
    p.K = T;
    p.tiles_m = cdiv(D, tc::BM);
    p.tiles_n = cdiv(F, tc::BN);
    p.out = dwd;
    p.ldo = F;
    p.m_split = D;
    p.err = err;
    if ((s = launch<true, true, tc::B_ONE, tc::EPI_F32>("k10_dw_down", di, ma, mb, mb, p, st)) != STAPLE_OK)
      return s;
  }
  return STAPLE_OK;
}

}  // namespace stp
