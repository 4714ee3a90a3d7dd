// prep.cu -- centroid preparation for the assignment stage.
//
// The tensor-core assignment ranks centroids by the score
// s_k = <x, c_k> - |c_k|^2 / 2, which orders them exactly as the squared
// distance |x|^2 + |c_k|^2 - 2<x, c_k> does (Flash-KMeans abstract: the
// distance is computed on the fly and fed to an online arg-min).  The bias
// -|c_k|^2 / 2 is computed once per assignment in fp32 from the centroids as
// the tensor cores see them (already rounded to the input type) and padded
// with -inf up to a multiple of the 256-centroid tile, so padded columns
// never win.
//
// The tensor cores add the bias themselves (one tf32 MMA step against a
// block of ones starts every tile), so each centroid's bias is stored as
// kBiasTerms floats: three terms that tf32 represents exactly and whose sum
// is the fp32 bias, then zeros.
#include "fk_internal.h"

namespace fk {

// Keep the 11 leading significand bits (sign, exponent and 10 fraction bits):
// the value a tf32 operand holds exactly.
__device__ __forceinline__ float tf32_head(float x) { return __uint_as_float(__float_as_uint(x) & 0xffffe000u); }

// Terms of the bias s at dst[0..kBiasTerms): hi + mid + lo == s exactly.
// hi keeps s's top 11 significand bits; s - hi is exact (same sign and
// binade) and has at most 13 significant bits, of which mid keeps the top 11
// and lo = (s - hi) - mid the last 2, again exactly.
__device__ __forceinline__ void store_bias_terms(float *dst, float s) {
  const float hi = tf32_head(s);
  const float r1 = s - hi;
  const float mid = tf32_head(r1);
  dst[0] = hi;
  dst[1] = mid;
  dst[2] = r1 - mid;
#pragma unroll
  for (int i = 3; i < kBiasTerms; ++i) dst[i] = 0.f;
}
__device__ __forceinline__ void store_bias_padding(float *dst) {
  dst[0] = __int_as_float(0xff800000);  // -inf: a padded column never wins
#pragma unroll
  for (int i = 1; i < kBiasTerms; ++i) dst[i] = 0.f;
}

template <typename T>
__global__ void __launch_bounds__(256) bias_kernel(const T *__restrict__ C, int B, int K, int Kpad,
                                                    int D, float *__restrict__ bias) {
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * Kpad;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows;
       r += (long long)gridDim.x * 8) {
    const int b = (int)(r / Kpad), j = (int)(r % Kpad);
    if (j >= K) {
      if (lane == 0) store_bias_padding(bias + r * kBiasTerms);
      continue;
    }
    const T *c = C + ((size_t)b * K + j) * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      float v = to_f32<T>(c[d]);
      s = fmaf(v, v, s);
    }
    s = warp_sum(s);
    if (lane == 0) store_bias_terms(bias + r * kBiasTerms, -0.5f * s);
  }
}

template <typename T>
__global__ void __launch_bounds__(256) round_bias_kernel(const float *__restrict__ C32, int B, int K,
                                                          int Kpad, int D, T *__restrict__ Cdt,
                                                          float *__restrict__ bias) {
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * Kpad;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows;
       r += (long long)gridDim.x * 8) {
    const int b = (int)(r / Kpad), j = (int)(r % Kpad);
    if (j >= K) {
      if (lane == 0) store_bias_padding(bias + r * kBiasTerms);
      continue;
    }
    const size_t off = ((size_t)b * K + j) * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      T t = from_f32<T>(C32[off + d]);
      Cdt[off + d] = t;
      float v = to_f32<T>(t);
      s = fmaf(v, v, s);
    }
    s = warp_sum(s);
    if (lane == 0) store_bias_terms(bias + r * kBiasTerms, -0.5f * s);
  }
}

// Bias of the Gaussian-sum epilogue (assign_tc.cu): -|c_k|^2/2 +
// ln(w_k)/(2 beta) for the part of the weights of one sign (sign > 0: the
// positive part max(w, 0), sign < 0: the negative part max(-w, 0); w == null
// means every weight is 1).  A zero weight gets the -inf padding: its column
// adds nothing.
template <typename T>
__global__ void __launch_bounds__(256) gauss_bias_kernel(const T *__restrict__ C, int K, int Kpad, int D,
                                                         const float *__restrict__ w, int sign, float inv2beta,
                                                         float *__restrict__ bias) {
  const int lane = threadIdx.x & 31;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < Kpad; r += (long long)gridDim.x * 8) {
    const int j = (int)r;
    float wj = 0.f;
    if (j < K) wj = w ? (sign > 0 ? fmaxf(w[j], 0.f) : fmaxf(-w[j], 0.f)) : (sign > 0 ? 1.f : 0.f);
    if (!(wj > 0.f)) {
      if (lane == 0) store_bias_padding(bias + r * kBiasTerms);
      continue;
    }
    const T *c = C + (size_t)j * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      const float v = to_f32<T>(c[d]);
      s = fmaf(v, v, s);
    }
    s = warp_sum(s);
    if (lane == 0) store_bias_terms(bias + r * kBiasTerms, fmaf(logf(wj), inv2beta, -0.5f * s));
  }
}

cudaError_t launch_gauss_bias(DType dt, const void *C, int K, int Kpad, int D, const float *w, int sign, float beta,
                              float *bias, cudaStream_t s) {
  long long g = (Kpad + 7) / 8;
  g = g < 1 ? 1 : (g > 4096 ? 4096 : g);
  const float inv2beta = 0.5f / beta;
  switch (dt) {
    case kF32:
      gauss_bias_kernel<float><<<(int)g, 256, 0, s>>>((const float *)C, K, Kpad, D, w, sign, inv2beta, bias);
      break;
    case kF16:
      gauss_bias_kernel<__half><<<(int)g, 256, 0, s>>>((const __half *)C, K, Kpad, D, w, sign, inv2beta, bias);
      break;
    default:
      gauss_bias_kernel<__nv_bfloat16>
          <<<(int)g, 256, 0, s>>>((const __nv_bfloat16 *)C, K, Kpad, D, w, sign, inv2beta, bias);
  }
  count_launches(1);
  return cudaGetLastError();
}

// |x|^2 of every row of X (fp32 sums of the squares, which are exact for
// fp16/bf16 inputs): the row norms of the assignment stage, for its near-tie
// test and its squared distances.  One warp per row, 16-byte loads when rows
// are 16-byte multiples.
template <typename T>
__global__ void __launch_bounds__(256) point_norms_kernel(const T *__restrict__ X, long long rows, int D,
                                                          int vec, float *__restrict__ xnorm) {
  const int lane = threadIdx.x & 31;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows; r += (long long)gridDim.x * 8) {
    const T *x = X + (size_t)r * D;
    float s = 0.f;
    if (vec) {
      constexpr int E = 16 / sizeof(T);
      const uint4 *xv = reinterpret_cast<const uint4 *>(x);
      for (int v = lane; v < D / E; v += 32) {
        const uint4 w = __ldg(xv + v);
        const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
        for (int i = 0; i < E; ++i) {
          const float f = to_f32<T>(e[i]);
          s = fmaf(f, f, s);
        }
      }
    } else {
      for (int d = lane; d < D; d += 32) {
        const float f = to_f32<T>(x[d]);
        s = fmaf(f, f, s);
      }
    }
    s = warp_sum(s);
    if (lane == 0) xnorm[r] = s;
  }
}

static int grid_for_rows(long long rows) {
  long long g = (rows + 7) / 8;
  return (int)(g < 4096 ? (g < 1 ? 1 : g) : 4096);
}

cudaError_t launch_bias(DType dt, const void *C, int B, int K, int Kpad, int D, float *bias,
                         cudaStream_t s) {
  const int g = grid_for_rows((long long)B * Kpad);
  switch (dt) {
    case kF32: bias_kernel<float><<<g, 256, 0, s>>>((const float *)C, B, K, Kpad, D, bias); break;
    case kF16: bias_kernel<__half><<<g, 256, 0, s>>>((const __half *)C, B, K, Kpad, D, bias); break;
    default:
      bias_kernel<__nv_bfloat16><<<g, 256, 0, s>>>((const __nv_bfloat16 *)C, B, K, Kpad, D, bias);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_point_norms(DType dt, const void *X, long long rows, int D, float *xnorm, cudaStream_t s) {
  const int g = grid_for_rows(rows);
  const int vec = ((size_t)D * dtype_size(dt)) % 16 == 0 && (uintptr_t)X % 16 == 0;
  switch (dt) {
    case kF32: point_norms_kernel<float><<<g, 256, 0, s>>>((const float *)X, rows, D, vec, xnorm); break;
    case kF16: point_norms_kernel<__half><<<g, 256, 0, s>>>((const __half *)X, rows, D, vec, xnorm); break;
    default:
      point_norms_kernel<__nv_bfloat16><<<g, 256, 0, s>>>((const __nv_bfloat16 *)X, rows, D, vec, xnorm);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_round_bias(DType dt, const float *C32, int B, int K, int Kpad, int D, void *Cdt,
                               float *bias, cudaStream_t s) {
  const int g = grid_for_rows((long long)B * Kpad);
  switch (dt) {
    case kF32:
      round_bias_kernel<float><<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (float *)Cdt, bias);
      break;
    case kF16:
      round_bias_kernel<__half><<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (__half *)Cdt, bias);
      break;
    default:
      round_bias_kernel<__nv_bfloat16>
          <<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (__nv_bfloat16 *)Cdt, bias);
  }
  count_launches(1);
  return cudaGetLastError();
}

__global__ void __launch_bounds__(256) fill_f32_kernel(float *__restrict__ p, long long n, float v) {
  for (long long i = (long long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long long)gridDim.x * blockDim.x)
    p[i] = v;
}

cudaError_t launch_fill_f32(float *p, long long n, float v, cudaStream_t s) {
  if (n <= 0) return cudaSuccess;
  long long g = (n + 255) / 256;
  if (g > 4096) g = 4096;
  fill_f32_kernel<<<(int)g, 256, 0, s>>>(p, n, v);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk
