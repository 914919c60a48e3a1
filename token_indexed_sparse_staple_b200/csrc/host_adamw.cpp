// Host-side AdamW on the rows of a table that a step touched: the tables and
// their fp32 moments live in host memory (the pages keep the 12 tables and
// their AdamW moments in host DRAM: 91.9 GiB with moments, Table 4's caption
// and the ai4snews summary), and only the U rows whose gradient came back
// from the GPU are updated.  Plain host C++ (compiled by the host compiler,
// no CUDA), split over std::threads.
//
// AdamW with decoupled weight decay (Loshchilov & Hutter, "Decoupled Weight
// Decay Regularization"):
//   m = b1 m + (1 - b1) g,   v = b2 v + (1 - b2) g^2
//   w = w - lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd w)
// in fp32; bf16 tables are rounded to nearest, ties to even.
//
// With one scalar square root and division per element the update is bound
// by arithmetic (about 6 GB/s of table + moment traffic per core), so it runs
// on x86 vector units when the CPU has them: 16 lanes (AVX-512F) or 8
// (AVX2), picked at run time.  Every path performs the same IEEE operations
// in the same order, without fused multiply-adds (this file is built with
// -ffp-contract=off), so all paths give the same bits.  STAPLE_ADAMW_ISA =
// "scalar" | "avx2" | "avx512" in the environment caps the path (for tests).
#include <algorithm>
#include <cmath>
#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <thread>
#include <vector>

#if defined(__x86_64__)
#include <immintrin.h>
#define STP_X86 1
#else
#define STP_X86 0
#endif

#include "staple.h"

namespace {

inline float bf16_to_f32(uint16_t b) {
  const uint32_t u = uint32_t(b) << 16;
  float f;
  std::memcpy(&f, &u, 4);
  return f;
}

// Round to nearest even on the fp32 bit pattern (finite inputs; a NaN stays
// a NaN).
inline uint16_t f32_to_bf16(float f) {
  uint32_t u;
  std::memcpy(&u, &f, 4);
  if ((u & 0x7f800000u) == 0x7f800000u && (u & 0x007fffffu)) return uint16_t((u >> 16) | 0x40);
  u += 0x7fffu + ((u >> 16) & 1u);
  return uint16_t(u >> 16);
}

struct Job {
  uint8_t* table;
  int64_t table_pitch;  // elements
  bool bf16;
  int F;
  const int32_t* ids;
  const float* grad;
  int64_t grad_pitch;
  float* m;
  float* v;
  int64_t moment_pitch;
  float lr, b1, b2, eps, wd;
  float omb1, omb2;     // 1 - b1, 1 - b2
  float c1, c2;         // 1 / (1 - b1^t), 1 / (1 - b2^t)
};

// One element; the vector paths below follow exactly these operations.
inline float update(const Job& j, float g, float& m, float& v, float w) {
  const float mf = j.b1 * m + j.omb1 * g;
  const float vf = j.b2 * v + (j.omb2 * g) * g;
  m = mf;
  v = vf;
  return w - j.lr * ((mf * j.c1) / (std::sqrt(vf * j.c2) + j.eps) + j.wd * w);
}

// Elements [f0, F) of row r (the scalar path, and the vector paths' tails).
inline void row_tail(const Job& j, int r, int f0) {
  const int64_t id = j.ids[r];
  const float* g = j.grad + int64_t(r) * j.grad_pitch;
  float* m = j.m + id * j.moment_pitch;
  float* v = j.v + id * j.moment_pitch;
  if (j.bf16) {
    uint16_t* w = reinterpret_cast<uint16_t*>(j.table) + id * j.table_pitch;
    for (int f = f0; f < j.F; ++f) w[f] = f32_to_bf16(update(j, g[f], m[f], v[f], bf16_to_f32(w[f])));
  } else {
    float* w = reinterpret_cast<float*>(j.table) + id * j.table_pitch;
    for (int f = f0; f < j.F; ++f) w[f] = update(j, g[f], m[f], v[f], w[f]);
  }
}

void rows_scalar(const Job& j, int r0, int r1) {
  for (int r = r0; r < r1; ++r) row_tail(j, r, 0);
}

#if STP_X86
__attribute__((target("avx512f"))) void rows_avx512(const Job& j, int r0, int r1) {
  const __m512 b1 = _mm512_set1_ps(j.b1), b2 = _mm512_set1_ps(j.b2);
  const __m512 omb1 = _mm512_set1_ps(j.omb1), omb2 = _mm512_set1_ps(j.omb2);
  const __m512 c1 = _mm512_set1_ps(j.c1), c2 = _mm512_set1_ps(j.c2);
  const __m512 eps = _mm512_set1_ps(j.eps), wd = _mm512_set1_ps(j.wd), lr = _mm512_set1_ps(j.lr);
  const __m512i rnd = _mm512_set1_epi32(0x7fff), one = _mm512_set1_epi32(1);
  const __m512i quiet = _mm512_set1_epi32(0x40);
  const int F16 = j.F & ~15;
  for (int r = r0; r < r1; ++r) {
    const int64_t id = j.ids[r];
    const float* g = j.grad + int64_t(r) * j.grad_pitch;
    float* m = j.m + id * j.moment_pitch;
    float* v = j.v + id * j.moment_pitch;
    for (int f = 0; f < F16; f += 16) {
      const __m512 gf = _mm512_loadu_ps(g + f);
      const __m512 mf = _mm512_add_ps(_mm512_mul_ps(b1, _mm512_loadu_ps(m + f)), _mm512_mul_ps(omb1, gf));
      const __m512 vf = _mm512_add_ps(_mm512_mul_ps(b2, _mm512_loadu_ps(v + f)),
                                      _mm512_mul_ps(_mm512_mul_ps(omb2, gf), gf));
      _mm512_storeu_ps(m + f, mf);
      _mm512_storeu_ps(v + f, vf);
      __m512 w;
      uint16_t* wb = nullptr;
      float* wf = nullptr;
      if (j.bf16) {
        wb = reinterpret_cast<uint16_t*>(j.table) + id * j.table_pitch + f;
        const __m512i u = _mm512_cvtepu16_epi32(_mm256_loadu_si256(reinterpret_cast<const __m256i*>(wb)));
        w = _mm512_castsi512_ps(_mm512_slli_epi32(u, 16));
      } else {
        wf = reinterpret_cast<float*>(j.table) + id * j.table_pitch + f;
        w = _mm512_loadu_ps(wf);
      }
      const __m512 q = _mm512_div_ps(_mm512_mul_ps(mf, c1),
                                     _mm512_add_ps(_mm512_sqrt_ps(_mm512_mul_ps(vf, c2)), eps));
      const __m512 nw = _mm512_sub_ps(w, _mm512_mul_ps(lr, _mm512_add_ps(q, _mm512_mul_ps(wd, w))));
      if (j.bf16) {
        const __m512i u = _mm512_castps_si512(nw);
        const __m512i hi = _mm512_srli_epi32(u, 16);
        __m512i o = _mm512_srli_epi32(_mm512_add_epi32(_mm512_add_epi32(u, rnd), _mm512_and_si512(hi, one)), 16);
        const __mmask16 nan = _mm512_cmp_ps_mask(nw, nw, _CMP_UNORD_Q);
        o = _mm512_mask_blend_epi32(nan, o, _mm512_or_si512(hi, quiet));
        _mm256_storeu_si256(reinterpret_cast<__m256i*>(wb), _mm512_cvtepi32_epi16(o));
      } else {
        _mm512_storeu_ps(wf, nw);
      }
    }
    row_tail(j, r, F16);
  }
}

__attribute__((target("avx2"))) void rows_avx2(const Job& j, int r0, int r1) {
  const __m256 b1 = _mm256_set1_ps(j.b1), b2 = _mm256_set1_ps(j.b2);
  const __m256 omb1 = _mm256_set1_ps(j.omb1), omb2 = _mm256_set1_ps(j.omb2);
  const __m256 c1 = _mm256_set1_ps(j.c1), c2 = _mm256_set1_ps(j.c2);
  const __m256 eps = _mm256_set1_ps(j.eps), wd = _mm256_set1_ps(j.wd), lr = _mm256_set1_ps(j.lr);
  const __m256i rnd = _mm256_set1_epi32(0x7fff), one = _mm256_set1_epi32(1);
  const __m256i quiet = _mm256_set1_epi32(0x40);
  const int F8 = j.F & ~7;
  for (int r = r0; r < r1; ++r) {
    const int64_t id = j.ids[r];
    const float* g = j.grad + int64_t(r) * j.grad_pitch;
    float* m = j.m + id * j.moment_pitch;
    float* v = j.v + id * j.moment_pitch;
    for (int f = 0; f < F8; f += 8) {
      const __m256 gf = _mm256_loadu_ps(g + f);
      const __m256 mf = _mm256_add_ps(_mm256_mul_ps(b1, _mm256_loadu_ps(m + f)), _mm256_mul_ps(omb1, gf));
      const __m256 vf = _mm256_add_ps(_mm256_mul_ps(b2, _mm256_loadu_ps(v + f)),
                                      _mm256_mul_ps(_mm256_mul_ps(omb2, gf), gf));
      _mm256_storeu_ps(m + f, mf);
      _mm256_storeu_ps(v + f, vf);
      __m256 w;
      uint16_t* wb = nullptr;
      float* wf = nullptr;
      if (j.bf16) {
        wb = reinterpret_cast<uint16_t*>(j.table) + id * j.table_pitch + f;
        const __m256i u = _mm256_cvtepu16_epi32(_mm_loadu_si128(reinterpret_cast<const __m128i*>(wb)));
        w = _mm256_castsi256_ps(_mm256_slli_epi32(u, 16));
      } else {
        wf = reinterpret_cast<float*>(j.table) + id * j.table_pitch + f;
        w = _mm256_loadu_ps(wf);
      }
      const __m256 q = _mm256_div_ps(_mm256_mul_ps(mf, c1),
                                     _mm256_add_ps(_mm256_sqrt_ps(_mm256_mul_ps(vf, c2)), eps));
      const __m256 nw = _mm256_sub_ps(w, _mm256_mul_ps(lr, _mm256_add_ps(q, _mm256_mul_ps(wd, w))));
      if (j.bf16) {
        const __m256i u = _mm256_castps_si256(nw);
        const __m256i hi = _mm256_srli_epi32(u, 16);
        __m256i o = _mm256_srli_epi32(_mm256_add_epi32(_mm256_add_epi32(u, rnd), _mm256_and_si256(hi, one)), 16);
        const __m256i nan = _mm256_castps_si256(_mm256_cmp_ps(nw, nw, _CMP_UNORD_Q));
        o = _mm256_blendv_epi8(o, _mm256_or_si256(hi, quiet), nan);
        // every lane is <= 0xffff, so the unsigned-saturating pack is exact
        const __m128i packed = _mm_packus_epi32(_mm256_castsi256_si128(o), _mm256_extracti128_si256(o, 1));
        _mm_storeu_si128(reinterpret_cast<__m128i*>(wb), packed);
      } else {
        _mm256_storeu_ps(wf, nw);
      }
    }
    row_tail(j, r, F8);
  }
}
#endif  // STP_X86

using RowsFn = void (*)(const Job&, int, int);

// The widest path the CPU runs, capped by STAPLE_ADAMW_ISA.
RowsFn pick_rows() {
  int cap = 2;  // 0 scalar, 1 avx2, 2 avx512
  if (const char* e = std::getenv("STAPLE_ADAMW_ISA")) {
    if (!std::strcmp(e, "scalar")) cap = 0;
    else if (!std::strcmp(e, "avx2")) cap = 1;
  }
#if STP_X86
  __builtin_cpu_init();
  if (cap >= 2 && __builtin_cpu_supports("avx512f")) return rows_avx512;
  if (cap >= 1 && __builtin_cpu_supports("avx2")) return rows_avx2;
#else
  (void)cap;
#endif
  return rows_scalar;
}

}  // namespace

extern "C" staple_status staple_adamw_rows(void* table, int64_t table_pitch, staple_dtype dtype,
                                           int32_t F, const int32_t* ids, int32_t U,
                                           const float* grad, int64_t grad_pitch, float* m,
                                           float* v, int64_t moment_pitch,
                                           const staple_adamw* hp, int32_t threads) {
  if (U == 0) return STAPLE_OK;
  if (!table || !ids || !grad || !m || !v || !hp || U < 0 || F <= 0 || table_pitch < F ||
      grad_pitch < F || moment_pitch < F || hp->step < 1 ||
      (dtype != STAPLE_BF16 && dtype != STAPLE_F32))
    return STAPLE_EINVAL;
  // ids index host memory directly: reject a negative one before any update
  for (int32_t r = 0; r < U; ++r)
    if (ids[r] < 0) return STAPLE_EINVAL;
  Job j;
  j.table = static_cast<uint8_t*>(table);
  j.table_pitch = table_pitch;
  j.bf16 = dtype == STAPLE_BF16;
  j.F = F;
  j.ids = ids;
  j.grad = grad;
  j.grad_pitch = grad_pitch;
  j.m = m;
  j.v = v;
  j.moment_pitch = moment_pitch;
  j.lr = hp->lr;
  j.b1 = hp->beta1;
  j.b2 = hp->beta2;
  j.eps = hp->eps;
  j.wd = hp->weight_decay;
  j.omb1 = 1.0f - hp->beta1;
  j.omb2 = 1.0f - hp->beta2;
  j.c1 = float(1.0 / (1.0 - std::pow(double(hp->beta1), double(hp->step))));
  j.c2 = float(1.0 / (1.0 - std::pow(double(hp->beta2), double(hp->step))));
  const RowsFn rows = pick_rows();
  int n = threads > 0 ? threads : int(std::thread::hardware_concurrency());
  n = std::max(1, std::min(n, U));
  if (n == 1) {
    rows(j, 0, U);
    return STAPLE_OK;
  }
  std::vector<std::thread> pool;
  pool.reserve(n);
  for (int t = 0; t < n; ++t) {
    const int r0 = int(int64_t(U) * t / n), r1 = int(int64_t(U) * (t + 1) / n);
    pool.emplace_back(rows, std::cref(j), r0, r1);
  }
  for (auto& th : pool) th.join();
  return STAPLE_OK;
}
