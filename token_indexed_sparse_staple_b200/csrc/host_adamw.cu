// Host-side AdamW on the rows of a table that a step touched: the tables and
// their fp32 moments live in host memory (the pages keep the 12 tables and
// their AdamW moments in host DRAM: 91.9 GiB with moments, Table 4's caption
// and the ai4snews summary), and only the U rows whose gradient came back
// from the GPU are updated.  Plain host code, split over std::threads.
//
// AdamW with decoupled weight decay (Loshchilov & Hutter, "Decoupled Weight
// Decay Regularization"):
//   m = b1 m + (1 - b1) g,   v = b2 v + (1 - b2) g^2
//   w = w - lr (m / (1 - b1^t) / (sqrt(v / (1 - b2^t)) + eps) + wd w)
// in fp32; bf16 tables are rounded to nearest, ties to even.
#include <cmath>
#include <cstring>
#include <thread>
#include <vector>

#include "internal.h"

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
  float c1, c2;         // 1 / (1 - b1^t), 1 / (1 - b2^t)
};

void update_rows(const Job& j, int r0, int r1) {
  for (int r = r0; r < r1; ++r) {
    const int64_t id = j.ids[r];
    const float* g = j.grad + int64_t(r) * j.grad_pitch;
    float* m = j.m + id * j.moment_pitch;
    float* v = j.v + id * j.moment_pitch;
    if (j.bf16) {
      uint16_t* w = reinterpret_cast<uint16_t*>(j.table) + id * j.table_pitch;
      for (int f = 0; f < j.F; ++f) {
        const float mf = j.b1 * m[f] + (1.0f - j.b1) * g[f];
        const float vf = j.b2 * v[f] + (1.0f - j.b2) * g[f] * g[f];
        m[f] = mf;
        v[f] = vf;
        const float wf = bf16_to_f32(w[f]);
        w[f] = f32_to_bf16(wf - j.lr * (mf * j.c1 / (std::sqrt(vf * j.c2) + j.eps) + j.wd * wf));
      }
    } else {
      float* w = reinterpret_cast<float*>(j.table) + id * j.table_pitch;
      for (int f = 0; f < j.F; ++f) {
        const float mf = j.b1 * m[f] + (1.0f - j.b1) * g[f];
        const float vf = j.b2 * v[f] + (1.0f - j.b2) * g[f] * g[f];
        m[f] = mf;
        v[f] = vf;
        w[f] = w[f] - j.lr * (mf * j.c1 / (std::sqrt(vf * j.c2) + j.eps) + j.wd * w[f]);
      }
    }
  }
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
  j.c1 = float(1.0 / (1.0 - std::pow(double(hp->beta1), double(hp->step))));
  j.c2 = float(1.0 / (1.0 - std::pow(double(hp->beta2), double(hp->step))));
  int n = threads > 0 ? threads : int(std::thread::hardware_concurrency());
  n = std::max(1, std::min(n, U));
  if (n == 1) {
    update_rows(j, 0, U);
    return STAPLE_OK;
  }
  std::vector<std::thread> pool;
  pool.reserve(n);
  for (int t = 0; t < n; ++t) {
    const int r0 = int(int64_t(U) * t / n), r1 = int(int64_t(U) * (t + 1) / n);
    pool.emplace_back(update_rows, std::cref(j), r0, r1);
  }
  for (auto& th : pool) th.join();
  return STAPLE_OK;
}
