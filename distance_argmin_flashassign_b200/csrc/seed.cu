// seed.cu -- k-means++ seeding on the GPU.
//
// The Japanese Hacker News summary of Flash-KMeans (discussion section) notes
// that seeding (k-means++) lies outside the paper's target; this file builds
// it on the same distance step as the assignment: a running minimum, over
// the centres chosen so far, of each point's squared distance D2(x), then a
// draw of the next centre with probability proportional to D2 (Arthur and
// Vassilvitskii's k-means++).
//
// The draws are reproducible to the index.  D2 is the direct difference
// sum_j (x_j - c_j)^2 in fp64, j ascending, each operation rounded on its own
// (the same value the plain definition gives).  The weights are integers,
// q_i = floor(D2_i 2^s), with s fixed once after the first centre so that N
// times the largest D2 stays below 2^61 (D2 only decreases); their sums are
// exact in int64.  Round t draws r = floor(u_t T) from the caller's uniform
// u_t in [0, 1) and the total T, and takes the first point whose running
// weight exceeds r.  When every weight is zero (every point on a centre),
// round t takes point floor(u_t N).
//
// A round reads X once from HBM.  Each point is first screened in fp32 with a
// rigorous rounding margin: only where the new centre may be nearer than the
// current D2 is the fp64 sum taken, which after the first rounds is a small
// share of the points.
//
// Rows of a multiple of 16 bytes (16-byte aligned X) take one kernel per
// round, seed_round_kernel: warp-cooperative 16-byte loads, the update of D2,
// the blocks' weight sums and, in the last block to finish, the draw and the
// next centre's row.  The first round (which also finds the largest D2, and so s)
// adds seed_sample_kernel.  Other rows take seed_update_kernel +
// seed_sample_kernel every round.
#include "fk_internal.h"

namespace fk {

constexpr int kSeedThreads = 256;  // = rows per block in every seeding kernel

struct SeedCtl {
  unsigned long long maxbits;  // bits of the largest D2 after the first centre (>= 0 doubles order as integers)
  int done;                    // blocks of the current kernel that have finished
};

// The fp32 screen.  a, the fp32 value of |x - c|^2 (any summation order),
// carries at most D + 2 roundings of relative size 2^-24 each, plus at most
// 2^-150 of absolute error per rounding in the subnormal range; the exact
// fp64 sum is within D 2^-53 of |x - c|^2.  So when
// (a - (D + 4) 2^-148) (1 - (D + 8) 2^-23) exceeds the current D2, the new
// centre cannot lower it and the fp64 sum is skipped.  An infinite or NaN a
// rules out nothing.
__device__ __forceinline__ bool screen_rules_out(float a, double old, int D) {
  return a <= 3.4028234663852886e38f &&
         ((double)a - (D + 4) * 2.802596928649634e-45) * (1.0 - (D + 8) * 1.1920928955078125e-7) > old;
}

__device__ __forceinline__ long long weight_of(double d2, int s) { return (long long)floor(ldexp(d2, s)); }

// s from the largest D2 after the first centre: N max D2 2^s < 2^61, N <= 2^L.
__device__ __forceinline__ int weight_exponent(const SeedCtl *ctl, int L) {
  int e = 0;
  const double m = __longlong_as_double((long long)*(const volatile unsigned long long *)&ctl->maxbits);
  if (m > 0.0) frexp(m, &e);
  return m > 0.0 ? 61 - e - L : 0;
}

__device__ __forceinline__ long long block_sum(long long v, long long *ws) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  if (lane == 0) ws[w] = v;
  __syncthreads();
  long long b = 0;
  if (threadIdx.x == 0)
    for (int k = 0; k < kSeedThreads / 32; ++k) b += ws[k];
  return b;  // valid in thread 0
}

__device__ __forceinline__ void block_max_bits(unsigned long long b, unsigned long long *wm, SeedCtl *ctl) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    const unsigned long long ob = __shfl_xor_sync(0xffffffffu, b, o);
    b = ob > b ? ob : b;
  }
  if (lane == 0) wm[w] = b;
  __syncthreads();
  if (threadIdx.x == 0) {
    unsigned long long m = 0;
    for (int k = 0; k < kSeedThreads / 32; ++k) m = wm[k] > m ? wm[k] : m;
    atomicMax(&ctl->maxbits, m);
  }
}

struct DrawSmem {
  long long ws[kSeedThreads / 32];
  long long r;
  int blk, idx, last;
};

// Exclusive prefix of v over the block; *total gets the block's sum.
__device__ __forceinline__ long long block_exclusive_scan(long long v, long long *ws, long long *total) {
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  long long incl = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const long long n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) ws[w] = incl;
  __syncthreads();
  long long before = 0, tot = 0;
#pragma unroll
  for (int k = 0; k < kSeedThreads / 32; ++k) {
    const long long x = ws[k];
    before += k < w ? x : 0;
    tot += x;
  }
  __syncthreads();  // ws may be reused
  *total = tot;
  return before + incl - v;
}

// Thread 0 has published this block's weight sum in bsum; the block that
// finishes last draws round t: total T, r, the block whose running weight
// passes r, the point within it; then centers[t], the chosen row into crow,
// and the counter reset for the next kernel.  Other blocks return.
// Thread k of the last block sums the block totals [k P, k P + P) with
// independent loads; a block-wide exclusive scan places each range and gives
// T; the one thread whose range holds r walks it.  D2 and bsum written by
// other blocks of the same kernel are read through L2.
template <typename T>
__device__ void draw_if_last(DrawSmem &sm, const T *__restrict__ X, int N, int D, const double *d2,
                             const double *__restrict__ u, int t, const long long *bsum, int s, SeedCtl *ctl,
                             int32_t *__restrict__ centers, float *__restrict__ crow) {
  if (threadIdx.x == 0) {
    __threadfence();
    sm.last = atomicAdd(&ctl->done, 1) == (int)gridDim.x - 1;
  }
  __syncthreads();
  if (!sm.last) return;
  __threadfence();
  const int nb = (int)gridDim.x, P = (nb + kSeedThreads - 1) / kSeedThreads;
  const int b0 = min(nb, (int)threadIdx.x * P), b1 = min(nb, b0 + P);
  long long mine = 0;
  for (int b = b0; b < b1; b += 8) {
    long long v[8];
#pragma unroll
    for (int k = 0; k < 8; ++k) v[k] = b + k < b1 ? __ldcg(bsum + b + k) : 0;
#pragma unroll
    for (int k = 0; k < 8; ++k) mine += v[k];
  }
  long long total;
  const long long pre = block_exclusive_scan(mine, sm.ws, &total);
  if (total == 0) {
    if (threadIdx.x == 0) {
      const long long k = (long long)floor(u[t] * (double)N);
      sm.idx = (int)(k < N ? k : N - 1);
    }
  } else {
    long long r = (long long)floor(u[t] * (double)total);
    if (r >= total) r = total - 1;
    if (mine > 0 && pre <= r && r < pre + mine) {
      long long run = pre;
      int hit = b1 - 1;
      for (int b = b0; b < b1 && hit == b1 - 1; b += 8) {
        long long v[8];
#pragma unroll
        for (int k = 0; k < 8; ++k) v[k] = b + k < b1 ? __ldcg(bsum + b + k) : 0;
#pragma unroll
        for (int k = 0; k < 8; ++k) {
          if (hit == b1 - 1 && b + k < b1 - 1) {
            if (run + v[k] > r) hit = b + k;
            else run += v[k];
          }
        }
      }
      sm.blk = hit;
      sm.r = r - run;  // rank within block hit
      sm.idx = hit * kSeedThreads;
    }
    __syncthreads();
    // the first point of block blk whose running weight exceeds the rank
    const long long rank = sm.r;
    const int j = sm.blk * kSeedThreads + threadIdx.x;
    const long long qj = j < N ? weight_of(__ldcg(d2 + j), s) : 0;
    long long bt;
    const long long excl = block_exclusive_scan(qj, sm.ws, &bt);
    if (qj > 0 && excl <= rank && rank < excl + qj) sm.idx = j;  // the one point whose interval holds the rank
  }
  __syncthreads();
  const int idx = sm.idx;
  if (threadIdx.x == 0) {
    centers[t] = idx;
    ctl->done = 0;
  }
  const T *xr = X + (size_t)idx * D;
  for (int j = threadIdx.x; j < D; j += kSeedThreads) crow[j] = to_f32<T>(xr[j]);
}

template <typename T> struct Vec16;
template <> struct Vec16<float> {
  static constexpr int E = 4;
  __device__ static void unpack(const uint4 &q, float *x) {
    x[0] = __uint_as_float(q.x); x[1] = __uint_as_float(q.y); x[2] = __uint_as_float(q.z); x[3] = __uint_as_float(q.w);
  }
};
template <> struct Vec16<__half> {
  static constexpr int E = 8;
  __device__ static void unpack(const uint4 &q, float *x) {
    const __half2 *h = reinterpret_cast<const __half2 *>(&q);
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      const float2 f = __half22float2(h[k]);
      x[2 * k] = f.x;
      x[2 * k + 1] = f.y;
    }
  }
};
template <> struct Vec16<__nv_bfloat16> {
  static constexpr int E = 8;
  __device__ static void unpack(const uint4 &q, float *x) {
    const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      x[2 * k] = __uint_as_float(w[k] << 16);
      x[2 * k + 1] = __uint_as_float(w[k] & 0xffff0000u);
    }
  }
};

// One round on rows of NV 16-byte vectors.  A warp owns 32 consecutive rows;
// L lanes share a row (G = 32 / L rows per step), lane `sub` of a row reads
// its vectors sub, sub + L, ... (MV of them at most) and keeps the matching
// centre elements in registers.  The fp32 screen is summed per lane and over
// the row's L lanes; the rows it does not rule out are summed exactly in fp64
// by the lane that owns them, in dimension order.
template <typename T, int L, int MV>
__global__ void __launch_bounds__(kSeedThreads) seed_round_kernel(const T *__restrict__ X, int N, int D,
                                                                  float *__restrict__ crow, double *d2, int first,
                                                                  SeedCtl *ctl, long long *bsum,
                                                                  const double *__restrict__ u, int t,
                                                                  int32_t *__restrict__ centers, int Lg) {
  constexpr int G = 32 / L, E = Vec16<T>::E;
  __shared__ DrawSmem sm;
  __shared__ unsigned long long wm[kSeedThreads / 32];
  __shared__ int sh_s;
  const int NV = D / E;
  if (threadIdx.x == 0) sh_s = first ? 0 : weight_exponent(ctl, Lg);
  const int lane = threadIdx.x & 31, sub = lane % L, g = lane / L;
  // serpentine order: odd rounds walk the row blocks backwards, so the first
  // blocks to run read the rows the previous round read last (still in L2)
  const int rb = (t & 1) ? (int)gridDim.x - 1 - (int)blockIdx.x : (int)blockIdx.x;
  const int r0 = rb * kSeedThreads + (threadIdx.x & ~31);
  const int row_l = r0 + lane;  // the row this lane owns for the exact sum
  const uint4 *Xv = reinterpret_cast<const uint4 *>(X);
  double old = 0.0;
  if (!first && row_l < N) old = d2[row_l];
  unsigned mask = 0xffffffffu;
  if (!first) {
    float cr[MV][E];
#pragma unroll
    for (int m = 0; m < MV; ++m) {
      const int v = sub + L * m;
#pragma unroll
      for (int e = 0; e < E; ++e) cr[m][e] = v < NV ? crow[v * E + e] : 0.f;
    }
    unsigned mine = 0;
    // kU steps at a time: all their loads first, then the sums
    constexpr int kU = 8 / MV < L ? 8 / MV : L;
    for (int i0 = 0; i0 < L; i0 += kU) {
      uint4 q[kU][MV];
#pragma unroll
      for (int ii = 0; ii < kU; ++ii) {
        const int row = r0 + (i0 + ii) * G + g;
#pragma unroll
        for (int m = 0; m < MV; ++m) {
          const int v = sub + L * m;
          q[ii][m] = row < N && v < NV ? __ldg(Xv + (size_t)row * NV + v) : make_uint4(0u, 0u, 0u, 0u);
        }
      }
#pragma unroll
      for (int ii = 0; ii < kU; ++ii) {
        const int rr = (i0 + ii) * G + g, row = r0 + rr;
        float a = 0.f;
#pragma unroll
        for (int m = 0; m < MV; ++m) {
          float x[E];
          Vec16<T>::unpack(q[ii][m], x);
#pragma unroll
          for (int e = 0; e < E; ++e) {
            const float dlt = x[e] - cr[m][e];  // 0 past the row's end (cr = 0 there)
            a = fmaf(dlt, dlt, a);
          }
        }
#pragma unroll
        for (int o = L / 2; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
        const double o_old = __shfl_sync(0xffffffffu, old, rr);
        if (sub == 0 && row < N && !screen_rules_out(a, o_old, D)) mine |= 1u << rr;
      }
    }
    mask = __reduce_or_sync(0xffffffffu, mine);
  }
  __syncthreads();  // sh_s
  double dn = old;  // this lane's row's D2 after the round
  if (row_l < N && ((mask >> lane) & 1u)) {
    const uint4 *xr = Xv + (size_t)row_l * NV;
    double d = 0.0;
    for (int v = 0; v < NV; ++v) {
      float x[E];
      Vec16<T>::unpack(__ldg(xr + v), x);
#pragma unroll
      for (int e = 0; e < E; ++e) {
        const double dlt = __dsub_rn((double)x[e], (double)__ldg(crow + v * E + e));
        d = __dadd_rn(d, __dmul_rn(dlt, dlt));
      }
    }
    if (first || d < old) {
      d2[row_l] = d;
      dn = d;
    }
  }
  if (first) {
    block_max_bits(row_l < N ? (unsigned long long)__double_as_longlong(dn) : 0ull, wm, ctl);
    return;
  }
  const long long b = block_sum(row_l < N ? weight_of(dn, sh_s) : 0, sm.ws);
  if (threadIdx.x == 0) bsum[rb] = b;
  draw_if_last<T>(sm, X, N, D, d2, u, t, bsum, sh_s, ctl, centers, crow);
}

// Rows of any width: each thread updates the D2 of its own row.  Each warp
// first copies its 32 consecutive rows into shared memory with coalesced
// 4-byte loads (rows padded by 4 bytes, so that the lanes' reads of one
// dimension fall in different banks) where they fit; otherwise a thread reads
// its row from global memory.  The first round also takes the largest D2.
template <typename T>
__global__ void __launch_bounds__(kSeedThreads) seed_update_kernel(const T *__restrict__ X, int N, int D,
                                                                   const float *__restrict__ crow,
                                                                   double *__restrict__ d2, int first,
                                                                   SeedCtl *ctl, int staged) {
  extern __shared__ __align__(16) unsigned char seed_smem[];
  __shared__ unsigned long long wm[kSeedThreads / 32];
  double *cs = reinterpret_cast<double *>(seed_smem);                 // the centre, D doubles
  float *csf = reinterpret_cast<float *>(seed_smem + (size_t)D * 8);  // and as fp32
  const int rb = D * (int)sizeof(T), rs = rb + 4;                     // row bytes, padded row stride
  unsigned char *rows = seed_smem + (size_t)D * 12 + (size_t)(threadIdx.x >> 5) * 32 * rs;
  for (int j = threadIdx.x; j < D; j += kSeedThreads) {
    cs[j] = (double)crow[j];
    csf[j] = crow[j];
  }
  const int lane = threadIdx.x & 31;
  const int i0 = blockIdx.x * kSeedThreads + (threadIdx.x & ~31);  // the warp's first row
  const int nrows = min(32, N - i0);
  if (staged && nrows > 0) {
    const uint32_t *src = reinterpret_cast<const uint32_t *>(X + (size_t)i0 * D);
    const int words = rb / 4;
#pragma unroll 4
    for (int r = 0; r < nrows; ++r)
      for (int c = lane; c < words; c += 32)
        *reinterpret_cast<uint32_t *>(rows + r * rs + c * 4) = __ldg(src + (size_t)r * words + c);
  }
  __syncthreads();
  const int i = i0 + lane;
  double d = 0.0;
  if (lane < nrows) {
    const T *x = staged ? reinterpret_cast<const T *>(rows + lane * rs) : X + (size_t)i * D;
    const double old = first ? 0.0 : d2[i];
    bool need = first != 0;
    if (!first) {
      float a = 0.f;
      for (int j = 0; j < D; ++j) {
        const float dlt = to_f32<T>(x[j]) - csf[j];
        a = fmaf(dlt, dlt, a);
      }
      need = !screen_rules_out(a, old, D);
    }
    if (need) {
      for (int j = 0; j < D; ++j) {
        const double dlt = __dsub_rn((double)to_f32<T>(x[j]), cs[j]);
        d = __dadd_rn(d, __dmul_rn(dlt, dlt));
      }
      if (first || d < old) d2[i] = d;
    }
  }
  if (first) block_max_bits(lane < nrows ? (unsigned long long)__double_as_longlong(d) : 0ull, wm, ctl);
}

static size_t seed_update_smem(int D, size_t es) {
  return (size_t)D * 12 + (size_t)(kSeedThreads / 32) * 32 * (D * es + 4);
}

// Block sums of the weights of D2 as it stands; the last block draws.
template <typename T>
__global__ void __launch_bounds__(kSeedThreads) seed_sample_kernel(const T *__restrict__ X, int N, int D,
                                                                   const double *d2, const double *__restrict__ u,
                                                                   int t, long long *bsum, SeedCtl *ctl,
                                                                   int32_t *__restrict__ centers,
                                                                   float *__restrict__ crow, int L) {
  __shared__ DrawSmem sm;
  __shared__ int sh_s;
  if (threadIdx.x == 0) sh_s = weight_exponent(ctl, L);
  __syncthreads();
  const int i = blockIdx.x * kSeedThreads + threadIdx.x;
  const long long b = block_sum(i < N ? weight_of(d2[i], sh_s) : 0, sm.ws);
  if (threadIdx.x == 0) bsum[blockIdx.x] = b;
  draw_if_last<T>(sm, X, N, D, d2, u, t, bsum, sh_s, ctl, centers, crow);
}

// centers[0] = first, its row into crow.
template <typename T>
__global__ void seed_first_kernel(const T *__restrict__ X, int D, int first, int32_t *centers, float *crow,
                                  SeedCtl *ctl) {
  if (threadIdx.x == 0) {
    centers[0] = first;
    ctl->maxbits = 0ull;
    ctl->done = 0;
  }
  for (int j = threadIdx.x; j < D; j += blockDim.x) crow[j] = to_f32<T>(X[(size_t)first * D + j]);
}

size_t seed_workspace_bytes(int64_t N, int D, int K) {
  const size_t nb = (size_t)((N + kSeedThreads - 1) / kSeedThreads);
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return al(N * 8) + al(nb * 8) + al(sizeof(SeedCtl)) + al((size_t)D * 4) + al((size_t)K * 8);
}

template <typename T>
using RoundKernel = void (*)(const T *, int, int, float *, double *, int, SeedCtl *, long long *, const double *,
                             int, int32_t *, int);

// Lanes per row L: the smallest power of two >= NV up to 32; then MV vectors
// per lane.
template <typename T>
static RoundKernel<T> pick_round_kernel(int NV) {
  if (NV <= 1) return seed_round_kernel<T, 1, 1>;
  if (NV <= 2) return seed_round_kernel<T, 2, 1>;
  if (NV <= 4) return seed_round_kernel<T, 4, 1>;
  if (NV <= 8) return seed_round_kernel<T, 8, 1>;
  if (NV <= 16) return seed_round_kernel<T, 16, 1>;
  if (NV <= 32) return seed_round_kernel<T, 32, 1>;
  if (NV <= 64) return seed_round_kernel<T, 32, 2>;
  if (NV <= 128) return seed_round_kernel<T, 32, 4>;
  return seed_round_kernel<T, 32, 8>;
}

template <typename T>
static cudaError_t run_seed(const void *Xv, int N, int D, int K, const double *u_host, int32_t *centers, void *ws,
                            cudaStream_t s) {
  const T *X = (const T *)Xv;
  const int nb = (N + kSeedThreads - 1) / kSeedThreads;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  char *p = (char *)ws;
  double *d2 = (double *)p; p += al((size_t)N * 8);
  long long *bsum = (long long *)p; p += al((size_t)nb * 8);
  SeedCtl *ctl = (SeedCtl *)p; p += al(sizeof(SeedCtl));
  float *crow = (float *)p; p += al((size_t)D * 4);
  double *u = (double *)p;
  cudaError_t e = cudaMemcpyAsync(u, u_host, (size_t)K * 8, cudaMemcpyHostToDevice, s);
  if (e != cudaSuccess) return e;
  int L = 0;
  while ((1ll << L) < (long long)N) ++L;
  long long f = (long long)floor(u_host[0] * (double)N);
  const int first = (int)(f < N ? f : N - 1);
  seed_first_kernel<T><<<1, 256, 0, s>>>(X, D, first, centers, crow, ctl);
  int launches = 1;
  const bool vec = (D * sizeof(T)) % 16 == 0 && (uintptr_t)X % 16 == 0;
  if (vec) {
    const RoundKernel<T> k = pick_round_kernel<T>((int)(D * sizeof(T) / 16));
    for (int t = 1; t < K; ++t) {
      k<<<nb, kSeedThreads, 0, s>>>(X, N, D, crow, d2, t == 1, ctl, bsum, u, t, centers, L);
      ++launches;
      if (t == 1) {
        seed_sample_kernel<T><<<nb, kSeedThreads, 0, s>>>(X, N, D, d2, u, t, bsum, ctl, centers, crow, L);
        ++launches;
      }
      if ((t & 63) == 0 && (e = cudaGetLastError()) != cudaSuccess) break;
    }
  } else {
    const bool staged = seed_update_smem(D, sizeof(T)) <= 200 * 1024 && (D * sizeof(T)) % 4 == 0 &&
                        (uintptr_t)X % 4 == 0;
    const size_t smem = staged ? seed_update_smem(D, sizeof(T)) : (size_t)D * 12;
    if (smem > 48 * 1024) {
      e = cudaFuncSetAttribute(seed_update_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
      if (e != cudaSuccess) return e;
    }
    for (int t = 1; t < K; ++t) {
      seed_update_kernel<T><<<nb, kSeedThreads, smem, s>>>(X, N, D, crow, d2, t == 1, ctl, staged ? 1 : 0);
      seed_sample_kernel<T><<<nb, kSeedThreads, 0, s>>>(X, N, D, d2, u, t, bsum, ctl, centers, crow, L);
      launches += 2;
      if ((t & 63) == 0 && (e = cudaGetLastError()) != cudaSuccess) break;
    }
  }
  count_launches(launches);
  return e == cudaSuccess ? cudaGetLastError() : e;
}

cudaError_t launch_seed(DType dt, const void *X, int N, int D, int K, const double *u_host, int32_t *centers, void *ws,
                        cudaStream_t s) {
  switch (dt) {
    case kF32: return run_seed<float>(X, N, D, K, u_host, centers, ws, s);
    case kF16: return run_seed<__half>(X, N, D, K, u_host, centers, ws, s);
    default: return run_seed<__nv_bfloat16>(X, N, D, K, u_host, centers, ws, s);
  }
}

}  // namespace fk
