// assign_simt.cu -- CUDA-core assignment stage (fused distance + argmin).
//
// Serves fp32 inputs and every shape the tensor-core kernel does not take.
// Like the tensor-core kernel it never writes the N x K distances to memory
// (FlashAssign, Flash-KMeans abstract): each thread owns one point, streams
// the centroids through shared memory in tiles of 32, keeps the 32 partial
// squared distances in registers and folds them into a running (min, argmin)
// in ascending centroid order, so ties go to the lowest index.  The distance
// is the direct difference sum_j (x_j - c_j)^2 in fp32.  Per tile of 32
// centroids (a chunk) the runner-up is tracked too: the smallest distance of
// the other chunks and its chunk, the second smallest of the other chunks,
// and the second smallest within the best chunk.  A point whose best and
// runner-up distances lie within the fp32 rounding bound of each other is
// listed for the exact re-decision (refine.cu) with the runner-up chunk, or
// with -2 (every chunk) when a third chunk is that close too.
#include "fk_internal.h"

namespace fk {

constexpr int kSimtRows = 128;  // points per block (one per thread)
constexpr int kSimtTileK = 32;  // centroids per shared-memory tile

template <typename T, int DCH>
__global__ void __launch_bounds__(kSimtRows) assign_simt_kernel(const T *__restrict__ X,
                                                                const T *__restrict__ C, int N,
                                                                int D, int K,
                                                                int32_t *__restrict__ labels,
                                                                float *__restrict__ mindist,
                                                                NearTies ties) {
  // every lane reads the same centroid value (a broadcast), so rows need no
  // padding, and 16-byte rows let a lane read four dimensions at once
  __shared__ __align__(16) float cs[kSimtTileK][DCH];
  const int b = blockIdx.y;
  const int row = blockIdx.x * kSimtRows + threadIdx.x;
  const bool valid = row < N;
  const T *xrow = X + ((size_t)b * N + (valid ? row : 0)) * D;
  const T *Cb = C + (size_t)b * K * D;

  const float inf = __int_as_float(0x7f800000);
  const int ex = (ties.excl != nullptr && valid) ? ties.excl[(size_t)b * N + row] : -1;  // left out, or -1
  float best = inf, s2 = inf, s3 = inf, s2in = inf;
  int bidx = 0, bbase = 0, base2 = -1;
  for (int k0 = 0; k0 < K; k0 += kSimtTileK) {
    float acc[kSimtTileK];
#pragma unroll
    for (int t = 0; t < kSimtTileK; ++t) acc[t] = 0.f;
    for (int d0 = 0; d0 < D; d0 += DCH) {
      __syncthreads();
      for (int e = threadIdx.x; e < kSimtTileK * DCH; e += kSimtRows) {
        const int kk = e / DCH, dd = e % DCH;
        const int k = k0 + kk, d = d0 + dd;
        cs[kk][dd] = (k < K && d < D) ? to_f32<T>(Cb[(size_t)k * D + d]) : 0.f;
      }
      __syncthreads();
      float xv[DCH];
#pragma unroll
      for (int dd = 0; dd < DCH; ++dd) xv[dd] = (valid && d0 + dd < D) ? to_f32<T>(xrow[d0 + dd]) : 0.f;
      // fully unrolled, so that acc[] stays in registers
#pragma unroll
      for (int t = 0; t < kSimtTileK; ++t) {
        float a = acc[t];
#pragma unroll
        for (int dd = 0; dd < DCH; dd += 4) {
          const float4 c4 = *reinterpret_cast<const float4 *>(&cs[t][dd]);
          const float u0 = xv[dd] - c4.x, u1 = xv[dd + 1] - c4.y, u2 = xv[dd + 2] - c4.z, u3 = xv[dd + 3] - c4.w;
          a = fmaf(u0, u0, a);
          a = fmaf(u1, u1, a);
          a = fmaf(u2, u2, a);
          a = fmaf(u3, u3, a);
        }
        acc[t] = a;
      }
    }
    // the chunk's smallest and second smallest distance, in centroid order
    float m = inf, m2 = inf;
    int mi = 0;
#pragma unroll
    for (int t = 0; t < kSimtTileK; ++t) {
      const float a = (k0 + t < K && k0 + t != ex) ? acc[t] : inf;
      if (a < m) {
        m2 = m;
        m = a;
        mi = t;
      } else if (a < m2) {
        m2 = a;
      }
    }
    const bool imp = m < best;  // strict: an earlier chunk keeps a tie
    const float lo = fmaxf(m, best);
    const int lob = imp ? bbase : k0;
    s3 = fminf(s3, fmaxf(lo, s2));
    const bool up = lo < s2;
    s2 = up ? lo : s2;
    base2 = up ? lob : base2;
    if (imp) {
      best = m;
      bidx = k0 + mi;
      bbase = k0;
      s2in = m2;
    }
  }
  const size_t g = (size_t)b * N + row;
  if (valid) {
    labels[g] = bidx;
    if (mindist) mindist[g] = best;
  }
  if (ties.list != nullptr) {
    const float second = fminf(s2, s2in);
    const bool near = valid && second < inf && (second - best) <= ties.tau * (best + second);
    const bool full = s3 < inf && (s3 - best) <= ties.tau * (best + s3);
    list_append(ties, near, full, (int)g, base2);
  }
}

template <typename T>
static cudaError_t launch_t(const void *X, const void *C, int B, int N, int D, int K, int32_t *labels,
                            float *mindist, NearTies ties, cudaStream_t s) {
  dim3 grid((N + kSimtRows - 1) / kSimtRows, B);
  if (D <= 32)
    assign_simt_kernel<T, 32><<<grid, kSimtRows, 0, s>>>((const T *)X, (const T *)C, N, D, K, labels,
                                                         mindist, ties);
  else
    assign_simt_kernel<T, 64><<<grid, kSimtRows, 0, s>>>((const T *)X, (const T *)C, N, D, K, labels,
                                                         mindist, ties);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_assign_simt(DType dt, const void *X, const void *C, int B, int N, int D, int K,
                               int32_t *labels, float *mindist, NearTies ties, cudaStream_t s) {
  switch (dt) {
    case kF32: return launch_t<float>(X, C, B, N, D, K, labels, mindist, ties, s);
    case kF16: return launch_t<__half>(X, C, B, N, D, K, labels, mindist, ties, s);
    default: return launch_t<__nv_bfloat16>(X, C, B, N, D, K, labels, mindist, ties, s);
  }
}

}  // namespace fk
