// prep.cu -- centroid preparation for the assignment stage.
//
// The expanded distance |x|^2 + |c|^2 - 2<x,c> (Flash-KMeans abstract:
// distances are computed on the fly and fed to an online argmin) needs the
// centroid norms |c_k|^2.  They are computed once per assignment, in fp32,
// from the centroids exactly as the tensor cores will see them (already
// rounded to the input type), and padded with +inf up to a multiple of the
// 256-centroid tile so padded columns never win the argmin.
#include "fk_internal.h"

namespace fk {

template <typename T>
__global__ void __launch_bounds__(256) norms_kernel(const T *__restrict__ C, int B, int K, int Kpad,
                                                    int D, float *__restrict__ cn) {
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * Kpad;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows;
       r += (long long)gridDim.x * 8) {
    const int b = (int)(r / Kpad), j = (int)(r % Kpad);
    if (j >= K) {
      if (lane == 0) cn[r] = __int_as_float(0x7f800000);
      continue;
    }
    const T *c = C + ((size_t)b * K + j) * D;
    float s = 0.f;
    for (int d = lane; d < D; d += 32) {
      float v = to_f32<T>(c[d]);
      s = fmaf(v, v, s);
    }
    s = warp_sum(s);
    if (lane == 0) cn[r] = s;
  }
}

template <typename T>
__global__ void __launch_bounds__(256) round_norms_kernel(const float *__restrict__ C32, int B, int K,
                                                          int Kpad, int D, T *__restrict__ Cdt,
                                                          float *__restrict__ cn) {
  const int lane = threadIdx.x & 31;
  const long long nrows = (long long)B * Kpad;
  for (long long r = (long long)blockIdx.x * 8 + (threadIdx.x >> 5); r < nrows;
       r += (long long)gridDim.x * 8) {
    const int b = (int)(r / Kpad), j = (int)(r % Kpad);
    if (j >= K) {
      if (lane == 0) cn[r] = __int_as_float(0x7f800000);
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
    if (lane == 0) cn[r] = s;
  }
}

static int grid_for_rows(long long rows) {
  long long g = (rows + 7) / 8;
  return (int)(g < 4096 ? (g < 1 ? 1 : g) : 4096);
}

cudaError_t launch_norms(DType dt, const void *C, int B, int K, int Kpad, int D, float *cn,
                         cudaStream_t s) {
  const int g = grid_for_rows((long long)B * Kpad);
  switch (dt) {
    case kF32: norms_kernel<float><<<g, 256, 0, s>>>((const float *)C, B, K, Kpad, D, cn); break;
    case kF16: norms_kernel<__half><<<g, 256, 0, s>>>((const __half *)C, B, K, Kpad, D, cn); break;
    default:
      norms_kernel<__nv_bfloat16><<<g, 256, 0, s>>>((const __nv_bfloat16 *)C, B, K, Kpad, D, cn);
  }
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_round_norms(DType dt, const float *C32, int B, int K, int Kpad, int D, void *Cdt,
                               float *cn, cudaStream_t s) {
  const int g = grid_for_rows((long long)B * Kpad);
  switch (dt) {
    case kF32:
      round_norms_kernel<float><<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (float *)Cdt, cn);
      break;
    case kF16:
      round_norms_kernel<__half><<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (__half *)Cdt, cn);
      break;
    default:
      round_norms_kernel<__nv_bfloat16>
          <<<g, 256, 0, s>>>(C32, B, K, Kpad, D, (__nv_bfloat16 *)Cdt, cn);
  }
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk
