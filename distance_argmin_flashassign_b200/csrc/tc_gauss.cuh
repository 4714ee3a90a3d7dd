// tc_gauss.cuh -- the Gaussian-sum epilogue of the tensor-core engine
// ("Fast Gauss Sums via Flash Attention", abstract: the sum over centroids
// kept as a running log-sum-exp, as the softmax of flash attention keeps it).
#pragma once
#include "tc_argmin.cuh"

namespace fk {

// With the bias of centroid k set to -|c_k|^2/2 + ln(w_k)/(2 beta), the
// accumulator holds s'_k = <x, c_k> - |c_k|^2/2 + ln(w_k)/(2 beta), and
// w_k exp(-beta |x - c_k|^2) = exp(-beta |x|^2) exp(2 beta s'_k).  A row keeps
// the largest s' seen (M) and S = sum of 2^(a (s'_k - M)), a = 2 beta log2(e),
// rescaled whenever M grows, as the softmax of flash attention does; the sum
// is exp(-beta |x|^2) 2^(a M) S.
struct GaussAcc {
  float M;  // largest score seen
  float S;  // sum of 2^(a (s' - M)) over the columns seen
};

__device__ __forceinline__ float ex2_approx(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}
__device__ __forceinline__ float lg2_approx(float x) {
  float y;
  asm("lg2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void gauss_fold(GaussAcc &g, const uint32_t (&v)[32], float a) {
  const float m = max32(v);
  if (m > g.M) {  // 2^(a (-inf)) = 0 clears S on the first finite chunk
    g.S *= ex2_approx((g.M - m) * a);
    g.M = m;
  }
  if (g.M == __int_as_float(0xff800000)) return;  // nothing but padding so far
  const float nb = -g.M * a;
  float t0 = 0.f, t1 = 0.f, t2 = 0.f, t3 = 0.f;
#pragma unroll
  for (int j = 0; j < 32; j += 4) {
    t0 += ex2_approx(fmaf(__uint_as_float(v[j]), a, nb));
    t1 += ex2_approx(fmaf(__uint_as_float(v[j + 1]), a, nb));
    t2 += ex2_approx(fmaf(__uint_as_float(v[j + 2]), a, nb));
    t3 += ex2_approx(fmaf(__uint_as_float(v[j + 3]), a, nb));
  }
  g.S += (t0 + t1) + (t2 + t3);
}

// (M, S) of two column halves of a row, merged.
__device__ __forceinline__ GaussAcc gauss_merge(GaussAcc x, GaussAcc y, float a) {
  const float M = fmaxf(x.M, y.M);
  if (M == __int_as_float(0xff800000)) return x;
  return GaussAcc{M, x.S * ex2_approx((x.M - M) * a) + y.S * ex2_approx((y.M - M) * a)};
}


}  // namespace fk
