// refine.cu -- exact re-decision of the points the assignment kernels could
// not order with certainty.
//
// Flash-KMeans is exact k-means (arXiv 2603.09229, abstract; the Japanese
// Hacker News summary, results paragraph): the assignment must give the
// nearest centroid, ties to the lowest index.  The assignment kernels rank
// in fp32; a point whose best and second-best fp32 values lie within the
// rounding bound of the fp32 evaluation may be ordered wrongly, so those
// kernels list it (NearTies) with the two 32-centroid chunks holding its best
// and its runner-up values, or for a comparison with every centroid when a
// third chunk is that close too.  This kernel recomputes, for every listed
// point, the squared distance to each centroid it must compare as the plain
// definition states it, sum over j of (x_j - c_j)^2 in fp64 with j ascending
// and every operation rounded on its own (no fused multiply-add), takes the
// first minimum in ascending centroid order, and rewrites the label and the
// distance.  A point's excluded centroid (NearTies::excl) takes no part.
//
// Lane l of a warp owns centroid base + l of each chunk and reads its row
// with 16-byte loads (all of a round in flight) while x is read from shared
// memory.  Two-chunk points take one warp each; a full comparison takes all
// warps of a block, each over its share of the chunks, then the block picks
// the first minimum.  The last block to finish resets the counts for the next
// assignment.
#include "fk_internal.h"

namespace fk {

constexpr int kRefWarps = 8;

// Elements of T in one 16-byte vector, as fp32 (exact for fp32/fp16/bf16).
template <typename T>
__device__ __forceinline__ void unpack16(const uint4 &w, float (&f)[16 / sizeof(T)]) {
  const T *e = reinterpret_cast<const T *>(&w);
#pragma unroll
  for (int i = 0; i < (int)(16 / sizeof(T)); ++i) f[i] = to_f32<T>(e[i]);
}

// sa += (x - a)^2, sb += (x - b)^2 in fp64, each operation rounded.
__device__ __forceinline__ void acc2(double &sa, double &sb, float x, float a, float b) {
  const double xv = (double)x;
  const double ua = __dsub_rn(xv, (double)a);
  const double ub = __dsub_rn(xv, (double)b);
  sa = __dadd_rn(sa, __dmul_rn(ua, ua));
  sb = __dadd_rn(sb, __dmul_rn(ub, ub));
}

// Squared distances of x (xs: D floats in shared memory) to centroids
// ca + lane and cb + lane (rows at or beyond K give +inf, and are not read).
// vec: rows are 16-byte multiples at 16-byte aligned addresses.
template <typename T>
__device__ __forceinline__ void pair_distances(const T *__restrict__ Cb, int D, int K, int ca, int cb,
                                               const float *xs, bool vec, double &da, double &db) {
  const int lane = threadIdx.x & 31;
  const int ka = ca + lane, kb = cb + lane;
  const bool oka = ka < K, okb = kb < K;
  double sa = 0.0, sb = 0.0;
  if (vec) {
    constexpr int E = 16 / sizeof(T), NV = sizeof(T) == 4 ? 4 : 8;  // vectors per round
    const uint4 *ra = reinterpret_cast<const uint4 *>(Cb + (size_t)(oka ? ka : 0) * D);
    const uint4 *rb = reinterpret_cast<const uint4 *>(Cb + (size_t)(okb ? kb : 0) * D);
    const int nvec = D / E;
    for (int v0 = 0; v0 < nvec; v0 += NV) {
      uint4 A[NV], Bv[NV];
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        const bool in = v0 + v < nvec;
        A[v] = (in && oka) ? __ldg(ra + v0 + v) : make_uint4(0u, 0u, 0u, 0u);
        Bv[v] = (in && okb) ? __ldg(rb + v0 + v) : make_uint4(0u, 0u, 0u, 0u);
      }
#pragma unroll
      for (int v = 0; v < NV; ++v) {
        if (v0 + v < nvec) {
          float fa[E], fb[E];
          unpack16<T>(A[v], fa);
          unpack16<T>(Bv[v], fb);
#pragma unroll
          for (int e = 0; e < E; ++e) acc2(sa, sb, xs[(v0 + v) * E + e], fa[e], fb[e]);
        }
      }
    }
  } else {
    const T *ra = Cb + (size_t)(oka ? ka : 0) * D, *rb = Cb + (size_t)(okb ? kb : 0) * D;
    for (int j = 0; j < D; ++j)
      acc2(sa, sb, xs[j], oka ? to_f32<T>(ra[j]) : 0.f, okb ? to_f32<T>(rb[j]) : 0.f);
  }
  const double inf = __longlong_as_double(0x7ff0000000000000ll);
  da = oka ? sa : inf;
  db = okb ? sb : inf;
}

// (distance, index) minimum over the warp; the lower index wins a tie.
__device__ __forceinline__ void warp_argmin(double &d, int &k) {
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) {
    const double od = __shfl_xor_sync(0xffffffffu, d, off);
    const int ok = __shfl_xor_sync(0xffffffffu, k, off);
    if (od < d || (od == d && ok < k)) {
      d = od;
      k = ok;
    }
  }
}

// Fold the two chunks (ca < cb; lanes beyond K hold +inf) into (best, bk):
// candidates arrive in ascending centroid order, so a later one wins only
// when strictly closer.  Centroid `ex` (or none, -1) takes no part.
__device__ __forceinline__ void fold_pair(double da, double db, int ca, int cb, int K, int ex, double &best,
                                          int &bk) {
  const int lane = threadIdx.x & 31;
  const double inf = __longlong_as_double(0x7ff0000000000000ll);
  int ka = ca + lane < K && ca + lane != ex ? ca + lane : 0x7fffffff;
  int kb = cb + lane < K && cb + lane != ex ? cb + lane : 0x7fffffff;
  if (ka == 0x7fffffff) da = inf;
  if (kb == 0x7fffffff) db = inf;
  warp_argmin(da, ka);
  warp_argmin(db, kb);
  if (ka != 0x7fffffff && (da < best || bk == 0x7fffffff)) {
    best = da;
    bk = ka;
  }
  if (kb != 0x7fffffff && (db < best || bk == 0x7fffffff)) {
    best = db;
    bk = kb;
  }
}

template <typename T>
__global__ void __launch_bounds__(32 * kRefWarps, 2) refine_kernel(const T *__restrict__ X, const T *__restrict__ C,
                                                               int N, int D, int K, int vec, NearTies t,
                                                               int32_t *__restrict__ labels,
                                                               float *__restrict__ mindist) {
  // the assignment kernel that listed the points may still be running
  asm volatile("griddepcontrol.wait;" ::: "memory");
  __shared__ float xs[kRefWarps][kMaxD];
  __shared__ double wbest[kRefWarps];
  __shared__ int wk[kRefWarps];
  __shared__ int n_lo, n_hi;
  const int w = threadIdx.x >> 5, lane = threadIdx.x & 31;
  // one read of each count per block (every thread reading the one address
  // would queue on one L2 slice)
  if (threadIdx.x == 0) {
    const int lo = min(*(volatile int *)t.count, t.cap);
    n_lo = lo;
    n_hi = min(*(volatile int *)t.count_hi, t.cap - lo);
  }
  __syncthreads();
  const double inf = __longlong_as_double(0x7ff0000000000000ll);
  const int nchunks = (K + 31) / 32;

  // two-chunk points: one warp each
  for (int e = blockIdx.x * kRefWarps + w; e < n_lo; e += gridDim.x * kRefWarps) {
    const int2 ent = t.list[e];
    const int g = ent.x, b = g / N;
    const T *xr = X + (size_t)g * D;
    const T *Cb = C + (size_t)b * K * D;
    for (int j = lane; j < D; j += 32) xs[w][j] = to_f32<T>(xr[j]);
    __syncwarp();
    const int ca = labels[g] & ~31;
    const int cb = (ent.y < 0 || ent.y >= K) ? ca : ent.y;
    const int c0 = min(ca, cb), c1 = ca == cb ? K : max(ca, cb);  // c1 = K: nothing to read
    double d0, d1, best = inf;
    int bk = 0x7fffffff;
    const int ex = t.excl ? t.excl[g] : -1;
    pair_distances<T>(Cb, D, K, c0, c1, xs[w], vec, d0, d1);
    fold_pair(d0, d1, c0, c1, K, ex, best, bk);
    if (lane == 0 && bk != 0x7fffffff) {
      labels[g] = bk;
      if (mindist) mindist[g] = (float)best;
    }
    __syncwarp();
  }

  // full comparisons: a block each, warp w over chunk pairs w, w + 8, ...
  for (int f = blockIdx.x; f < n_hi; f += gridDim.x) {
    const int g = t.list[t.cap - 1 - f].x, b = g / N;
    const T *xr = X + (size_t)g * D;
    const T *Cb = C + (size_t)b * K * D;
    for (int j = lane; j < D; j += 32) xs[w][j] = to_f32<T>(xr[j]);
    __syncwarp();
    double best = inf;
    int bk = 0x7fffffff;
    const int ex = t.excl ? t.excl[g] : -1;
    for (int pr = w; 2 * pr < nchunks; pr += kRefWarps) {
      const int c0 = 64 * pr, c1 = c0 + 32 < K ? c0 + 32 : K;
      double d0, d1;
      pair_distances<T>(Cb, D, K, c0, c1, xs[w], vec, d0, d1);
      fold_pair(d0, d1, c0, c1, K, ex, best, bk);
    }
    if (lane == 0) {
      wbest[w] = best;
      wk[w] = bk;
    }
    __syncthreads();
    if (threadIdx.x == 0) {
      double bb = inf;
      int kk = 0x7fffffff;
      for (int i = 0; i < kRefWarps; ++i) {
        if (wk[i] != 0x7fffffff && (wbest[i] < bb || (wbest[i] == bb && wk[i] < kk) || kk == 0x7fffffff)) {
          bb = wbest[i];
          kk = wk[i];
        }
      }
      if (kk != 0x7fffffff) {
        labels[g] = kk;
        if (mindist) mindist[g] = (float)bb;
      }
    }
    __syncthreads();
  }

  // the last block to finish clears the counts for the next assignment
  __syncthreads();
  if (threadIdx.x == 0) {
    __threadfence();
    if (atomicAdd(t.done, 1) == (int)gridDim.x - 1) {
      *t.count = 0;
      *t.count_hi = 0;
      *t.done = 0;
      __threadfence();
    }
  }
}

template <typename T>
static cudaError_t launch_t(const void *X, const void *C, int N, int D, int K, NearTies t, int32_t *labels,
                            float *mindist, int num_sms, cudaStream_t s) {
  const int vec = ((size_t)D * sizeof(T)) % 16 == 0 && (uintptr_t)C % 16 == 0;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * (num_sms > 0 ? num_sms : 1));
  cfg.blockDim = dim3(32 * kRefWarps);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, refine_kernel<T>, (const T *)X, (const T *)C, N, D, K, vec, t, labels,
                                     mindist);
  count_launches(1);
  return e;
}

cudaError_t launch_refine(DType dt, const void *X, const void *C, int N, int D, int K, NearTies t,
                          int32_t *labels, float *mindist, int num_sms, cudaStream_t s) {
  switch (dt) {
    case kF32: return launch_t<float>(X, C, N, D, K, t, labels, mindist, num_sms, s);
    case kF16: return launch_t<__half>(X, C, N, D, K, t, labels, mindist, num_sms, s);
    default: return launch_t<__nv_bfloat16>(X, C, N, D, K, t, labels, mindist, num_sms, s);
  }
}

}  // namespace fk
