// gauss.cu -- weighted Gauss sums on CUDA cores, and the combination of the
// two sign parts of a signed-weight sum.
//
// "Fast Gauss Sums via Flash Attention" (abstract) evaluates
// G(x_i) = sum_k w_k exp(-beta |x_i - c_k|^2), with arbitrary signed weights,
// in fused tiles without storing the N x K kernel matrix; FlashDiffusion
// (Figure 4 caption) applies the same matrix-free Gaussian kernel to a vector
// (Kv, the case c = x).  The tensor-core path is the assignment kernel with
// its Gaussian-sum epilogue (assign_tc.cu).  This file holds the CUDA-core
// kernel for the inputs that path does not take (fp32, other shapes): one
// point per thread, centroids staged through shared memory, the direct
// difference |x - c|^2 in fp32, and a running log-sum-exp of
// ln(w_k) - beta |x - c_k|^2 over the centroids of one sign part.
#include "fk_internal.h"

namespace fk {

constexpr int kGsRows = 128;  // points per block
constexpr int kGsTile = 32;   // centroids per shared-memory tile

template <typename T>
__global__ void __launch_bounds__(kGsRows) gauss_simt_kernel(const T *__restrict__ X, const T *__restrict__ C, int N,
                                                             int D, int K, const float *__restrict__ w, int sign,
                                                             float beta, float *__restrict__ log_out,
                                                             float *__restrict__ val_out) {
  __shared__ float cs[kGsTile][65];
  __shared__ float lw[kGsTile];
  const int row = blockIdx.x * kGsRows + threadIdx.x;
  const bool valid = row < N;
  const T *xr = X + (size_t)(valid ? row : 0) * D;
  const float ninf = __int_as_float(0xff800000);
  float M = ninf, S = 0.f;  // running max of ln(w) - beta d, and sum of exp(. - M)
  for (int k0 = 0; k0 < K; k0 += kGsTile) {
    float acc[kGsTile];
#pragma unroll
    for (int t = 0; t < kGsTile; ++t) acc[t] = 0.f;
    __syncthreads();
    if (threadIdx.x < kGsTile) {
      const int k = k0 + threadIdx.x;
      float wk = 0.f;
      if (k < K) wk = w ? (sign > 0 ? fmaxf(w[k], 0.f) : fmaxf(-w[k], 0.f)) : (sign > 0 ? 1.f : 0.f);
      lw[threadIdx.x] = wk > 0.f ? logf(wk) : ninf;
    }
    for (int d0 = 0; d0 < D; d0 += 64) {
      __syncthreads();
      for (int e = threadIdx.x; e < kGsTile * 64; e += kGsRows) {
        const int kk = e / 64, dd = e % 64, k = k0 + kk, d = d0 + dd;
        cs[kk][dd] = (k < K && d < D) ? to_f32<T>(C[(size_t)k * D + d]) : 0.f;
      }
      __syncthreads();
      const int de = min(64, D - d0);
      for (int dd = 0; dd < de; ++dd) {
        const float xv = valid ? to_f32<T>(xr[d0 + dd]) : 0.f;
#pragma unroll
        for (int t = 0; t < kGsTile; ++t) {
          const float u = xv - cs[t][dd];
          acc[t] = fmaf(u, u, acc[t]);
        }
      }
    }
#pragma unroll
    for (int t = 0; t < kGsTile; ++t) {
      const float e = fmaf(-beta, acc[t], lw[t]);  // -inf for zero weights and past K
      if (e > M) {
        S = S * __expf(M - e) + 1.f;
        M = e;
      } else if (e != ninf) {
        S += __expf(e - M);
      }
    }
  }
  if (valid) {
    const float l = M + __logf(S);  // -inf when every weight of this part is zero
    if (log_out) log_out[row] = l;
    if (val_out) val_out[row] = __expf(l);
  }
}

cudaError_t launch_gauss_simt(DType dt, const void *X, const void *C, int N, int D, int K, const float *w, int sign,
                              float beta, float *log_out, float *val_out, cudaStream_t s) {
  const dim3 grid((N + kGsRows - 1) / kGsRows);
  switch (dt) {
    case kF32:
      gauss_simt_kernel<float><<<grid, kGsRows, 0, s>>>((const float *)X, (const float *)C, N, D, K, w, sign, beta,
                                                       log_out, val_out);
      break;
    case kF16:
      gauss_simt_kernel<__half><<<grid, kGsRows, 0, s>>>((const __half *)X, (const __half *)C, N, D, K, w, sign,
                                                        beta, log_out, val_out);
      break;
    default:
      gauss_simt_kernel<__nv_bfloat16><<<grid, kGsRows, 0, s>>>((const __nv_bfloat16 *)X, (const __nv_bfloat16 *)C,
                                                               N, D, K, w, sign, beta, log_out, val_out);
  }
  count_launches(1);
  return cudaGetLastError();
}

// G = e^lp - e^ln (the positive part less the negative part), ln G where
// G > 0 (NaN otherwise).
__global__ void __launch_bounds__(256) gauss_combine_kernel(const float *__restrict__ lp, const float *__restrict__ ln,
                                                            int N, float *__restrict__ log_out,
                                                            float *__restrict__ val_out) {
  for (int i = blockIdx.x * blockDim.x + threadIdx.x; i < N; i += gridDim.x * blockDim.x) {
    const float a = lp[i], b = ln[i];
    if (val_out) val_out[i] = __expf(a) - __expf(b);
    if (log_out) log_out[i] = a > b ? a + log1pf(-__expf(b - a)) : __int_as_float(0x7fc00000);
  }
}

cudaError_t launch_gauss_combine(const float *lp, const float *ln, int N, float *log_out, float *val_out,
                                 cudaStream_t s) {
  int g = (N + 255) / 256;
  g = g > 4096 ? 4096 : (g < 1 ? 1 : g);
  gauss_combine_kernel<<<g, 256, 0, s>>>(lp, ln, N, log_out, val_out);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk
