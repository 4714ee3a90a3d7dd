// fused.cu -- single-pass Lloyd iterations for problems whose centroids fit
// in shared memory.
//
// Flash-KMeans (abstract) runs an iteration as the assignment stage followed
// by the update stage, which reads X a second time.  When K x D fp32 values
// fit in a CTA's shared memory twice over (the centroids and the CTA's own
// partial sums), both stages can share one read of X: each CTA assigns its
// rows and immediately adds them into per-cluster partial sums, in a fixed
// order, without global atomics; a grid-wide barrier later, the CTAs combine
// the partial sums in CTA order and divide.  All iterations run in one
// cooperative launch (every CTA resident), so a small problem -- where the
// two-stage iteration is bound by its seven kernel launches -- pays one
// launch in total.
//
// Per iteration, per CTA:
//   1. the centroids C_t, rounded to the input type, into shared memory;
//   2. passes of 512 / S rows: S threads share a row (S grows for small N
//      so that every SM gets rows), thread s taking the centroids
//      k0 + t S + s of each block of 32 S, with the fp32 direct difference
//      (as the CUDA-core assignment kernel), keeping the best and
//      second-best distance; a row
//      whose two lie within the fp32 rounding bound of each other is
//      re-decided exactly by its warp, over every centroid, with the fp64
//      direct difference and the lowest index on ties -- so every label is
//      the exact one;
//   3. the pass's rows ordered by (label, row) in shared memory, then added
//      into the CTA's partial sums cluster by cluster in that order;
//   4. the partial sums and counts to global memory; grid barrier;
//   5. CTA j combines the (cluster, 32-dimension) slices j, j + G, ...: its
//      16 warps sum the CTAs w, w + 16, ... in order, then the 16 warp sums
//      are added in warp order; C_{t+1} = sum / count (an empty cluster keeps
//      its centroid); grid barrier.
// The summation order is fixed by the launch shape (one CTA per SM), so the
// result does not vary from run to run on a device.
#include "fk_internal.h"

namespace fk {

constexpr int kFzThreads = 512;  // rows per pass
constexpr int kFzWarps = kFzThreads / 32;
constexpr int kFzTileK = 32;     // centroids per register tile

struct FzArgs {
  const void *X;
  int N, D, K, Dp;  // Dp: D rounded up to a multiple of 4
  int xs_ok;        // the pass's rows fit in shared memory (staged for the sums)
  float *C;
  int32_t *labels;
  float *mindist;   // last iteration only, or null
  int32_t *counts;  // last iteration, or null
  float *part;      // [G][K][D] partial sums
  int *pcnt;        // [G][K] partial counts
  unsigned *bar;    // [0] arrivals, [1] generation, [2] abort; zero on entry
  int iters;
  int S;            // threads per row (a power of two, at most 16)
  float tau;
  DevCtl ctl;
};

// Grid-wide barrier, bounded: gives up after ctl.timeout_ns (recording
// kStTimeout and raising the abort word) or when another CTA has aborted.
__device__ bool fz_grid_sync(unsigned *bar, const DevCtl &ctl) {
  __shared__ int ok;
  __syncthreads();
  if (threadIdx.x == 0) {
    ok = 1;
    volatile unsigned *vb = bar;
    const unsigned gen = vb[1];
    __threadfence();
    if (atomicAdd(bar, 1u) == gridDim.x - 1) {
      atomicExch(bar, 0u);
      __threadfence();
      atomicAdd(bar + 1, 1u);
    } else {
      const uint64_t t0 = globaltimer();
      while (vb[1] == gen) {
        if (vb[2]) {
          ok = 0;
          break;
        }
        if (globaltimer() - t0 > ctl.timeout_ns) {
          atomicExch(bar + 2, 1u);
          record_status(ctl.status, kStTimeout);
          ok = 0;
          break;
        }
        __nanosleep(64);
      }
    }
    __threadfence();
  }
  __syncthreads();
  return ok != 0;
}

template <typename T> __device__ __forceinline__ float round_to(float v);
template <> __device__ __forceinline__ float round_to<float>(float v) { return v; }
template <> __device__ __forceinline__ float round_to<__half>(float v) { return __half2float(__float2half_rn(v)); }
template <> __device__ __forceinline__ float round_to<__nv_bfloat16>(float v) {
  return __bfloat162float(__float2bfloat16_rn(v));
}

template <typename T, int DCH>
__global__ void __launch_bounds__(kFzThreads) lloyd_fused_kernel(FzArgs a) {
  extern __shared__ __align__(16) float fz_smem[];
  const int D = a.D, K = a.K, Dp = a.Dp, N = a.N;
  // centroid rows Dp + 4 floats apart: the S threads of a row read S
  // consecutive centroids at once, which then fall in different banks
  const int Dr = Dp + 4;
  float *cs = fz_smem;                                   // [K][Dr] centroids of this iteration
  float *acc = cs + (size_t)K * Dr;                      // [K][D] this CTA's partial sums
  int *kcnt = reinterpret_cast<int *>(acc + (size_t)K * D);  // [K] its counts
  int *pc = kcnt + K;                                    // [K] counts of the pass
  int *cst = pc + K;                                     // [K] where each cluster's run starts
  int *lab = cst + K;                                    // [P] labels of the pass (-1: no row)
  int *srt = lab + kFzThreads;                           // [P] the pass's rows by (label, row)
  float *xs = reinterpret_cast<float *>(srt + kFzThreads);  // [P][D] the pass's rows, when xs_ok
  __shared__ float red[kFzWarps][32];
  __shared__ int wtot[kFzWarps];
  const T *X = (const T *)a.X;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int G = gridDim.x;
  const float inf = __int_as_float(0x7f800000);
  const int S = a.S, P = kFzThreads / S;  // rows per pass
  const int npass = (N + P * G - 1) / (P * G);
  // groups of D threads share a cluster's run: thread (g, d)
  const int ngrp = D <= kFzThreads ? kFzThreads / D : 1;
  const int grp = D <= kFzThreads ? tid / D : 0;
  for (int it = 0; it < a.iters; ++it) {
    const bool last_it = it == a.iters - 1;
    for (int i = tid; i < K * Dr; i += kFzThreads) {
      const int k = i / Dr, d = i % Dr;
      cs[i] = d < D ? round_to<T>(__ldcg(a.C + (size_t)k * D + d)) : 0.f;  // written by other CTAs: not from L1
    }
    for (int i = tid; i < K * D; i += kFzThreads) acc[i] = 0.f;
    for (int i = tid; i < K; i += kFzThreads) kcnt[i] = 0;
    __syncthreads();
    for (int p = 0; p < npass; ++p) {
      // S threads share a row (adjacent lanes); thread s of a row takes the
      // centroids k0 + t S + s (t < 32) of each block of 32 S centroids, so
      // the S threads read S consecutive centroid rows at once
      const int r0 = (p * G + blockIdx.x) * P;
      const int prow = tid / S, sub = tid % S;
      const int row = r0 + prow;
      const bool valid = row < N;
      const T *xrow = X + (size_t)(valid ? row : 0) * D;
      // ---- assignment of the row
      float best = inf, second = inf;
      int bidx = 0;
      // thread s of a row takes centroids k0 + t S + s of each block of 32 S
      for (int k0 = 0; k0 < K; k0 += S * kFzTileK) {
        float d2[kFzTileK];
#pragma unroll
        for (int t = 0; t < kFzTileK; ++t) d2[t] = 0.f;
        for (int d0 = 0; d0 < D; d0 += DCH) {
          float xv[DCH];
#pragma unroll
          for (int dd = 0; dd < DCH; ++dd) xv[dd] = (valid && d0 + dd < D) ? to_f32<T>(xrow[d0 + dd]) : 0.f;
#pragma unroll
          for (int t = 0; t < kFzTileK; ++t) {
            const int k = k0 + t * S + sub;
            const float *crow = cs + (size_t)(k < K ? k : 0) * Dr + d0;
            float sum = d2[t];
#pragma unroll
            for (int dd = 0; dd < DCH; dd += 4) {
              if (d0 + dd < Dp) {
                const float4 c4 = *reinterpret_cast<const float4 *>(crow + dd);
                const float u0 = xv[dd] - c4.x, u1 = xv[dd + 1] - c4.y, u2 = xv[dd + 2] - c4.z,
                            u3 = xv[dd + 3] - c4.w;
                sum = fmaf(u0, u0, sum);
                sum = fmaf(u1, u1, sum);
                sum = fmaf(u2, u2, sum);
                sum = fmaf(u3, u3, sum);
              }
            }
            d2[t] = sum;
          }
        }
#pragma unroll
        for (int t = 0; t < kFzTileK; ++t) {
          const int k = k0 + t * S + sub;
          const float v = k < K ? d2[t] : inf;
          if (v < best) {
            second = best;
            best = v;
            bidx = k;
          } else if (v < second) {
            second = v;
          }
        }
      }
      // merge the row's S partial results: smallest distance, lowest index
      // on equal distances; the second smallest over all the others
      for (int o = S / 2; o > 0; o >>= 1) {
        const float ob = __shfl_xor_sync(0xffffffffu, best, o), os = __shfl_xor_sync(0xffffffffu, second, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bidx, o);
        if (ob < best || (ob == best && oi < bidx)) {
          second = fminf(os, best);
          best = ob;
          bidx = oi;
        } else {
          second = fminf(second, ob);
        }
      }
      float md = best;
      // ---- rows too close to call in fp32: every centroid, exactly, by the
      // whole warp (lane j takes centroids j, j + 32, ...; fp64 direct
      // difference; the lowest index wins a tie)
      const bool near = valid && sub == 0 && second < inf && (second - best) <= a.tau * (best + second);
      unsigned todo = __ballot_sync(0xffffffffu, near);
      while (todo) {
        const int src = __ffs(todo) - 1;
        todo &= todo - 1;
        const int r = __shfl_sync(0xffffffffu, row, src);
        const T *xr = X + (size_t)r * D;
        double bb = 0.0;
        int bk = -1;
        for (int k = lane; k < K; k += 32) {
          const float *crow = cs + (size_t)k * Dr;
          double sum = 0.0;
          for (int d = 0; d < D; ++d) {
            const double u = __dsub_rn((double)to_f32<T>(xr[d]), (double)crow[d]);
            sum = __dadd_rn(sum, __dmul_rn(u, u));
          }
          if (bk < 0 || sum < bb) {
            bb = sum;
            bk = k;
          }
        }
        for (int o = 16; o > 0; o >>= 1) {
          const double ob = __shfl_xor_sync(0xffffffffu, bb, o);
          const int ok = __shfl_xor_sync(0xffffffffu, bk, o);
          if (ok >= 0 && (bk < 0 || ob < bb || (ob == bb && ok < bk))) {
            bb = ob;
            bk = ok;
          }
        }
        if (lane == src) {
          bidx = bk;
          md = (float)bb;
        }
      }
      const bool own = valid && sub == 0;
      if (own) {
        a.labels[row] = bidx;
        if (last_it && a.mindist) a.mindist[row] = md;
      }
      if (sub == 0) lab[prow] = valid ? bidx : -1;
      if (a.xs_ok && valid)
        for (int d = sub; d < D; d += S) xs[(size_t)prow * D + d] = to_f32<T>(xrow[d]);
      for (int i = tid; i < K; i += kFzThreads) pc[i] = 0;
      __syncthreads();
      // ---- the pass's rows ordered by (label, row): counts, starts, ranks
      int rank = 0;
      if (own) {
        atomicAdd(&pc[bidx], 1);
        for (int t = 0; t < prow; ++t) rank += lab[t] == bidx;
      }
      __syncthreads();
      {  // exclusive scan of pc over the clusters: thread i owns [i C, i C + C)
        const int per = (K + kFzThreads - 1) / kFzThreads;
        const int c0 = tid * per, c1 = min(K, c0 + per);
        int sum = 0;
        for (int c = c0; c < c1; ++c) sum += pc[c];
        int incl = sum;
#pragma unroll
        for (int o = 1; o < 32; o <<= 1) {
          const int n = __shfl_up_sync(0xffffffffu, incl, o);
          if (lane >= o) incl += n;
        }
        if (lane == 31) wtot[warp] = incl;
        __syncthreads();
        int run = incl - sum;
        for (int w = 0; w < warp; ++w) run += wtot[w];
        for (int c = c0; c < c1; ++c) {
          cst[c] = run;
          run += pc[c];
        }
      }
      __syncthreads();
      if (own) srt[cst[bidx] + rank] = prow;
      __syncthreads();
      // ---- add the rows into the partial sums, cluster by cluster in row order
      for (int k = grp < ngrp ? grp : K; k < K; k += ngrp) {
        const int n = pc[k];
        if (n == 0) continue;
        const int s0 = cst[k];
        for (int d = (D <= kFzThreads ? tid % D : tid); d < D; d += (D <= kFzThreads ? D : kFzThreads)) {
          float v = acc[(size_t)k * D + d];
          if (a.xs_ok)
            for (int j = 0; j < n; ++j) v += xs[(size_t)srt[s0 + j] * D + d];
          else
            for (int j = 0; j < n; ++j) v += to_f32<T>(X[(size_t)(r0 + srt[s0 + j]) * D + d]);
          acc[(size_t)k * D + d] = v;
        }
        if (tid % D == 0 || D > kFzThreads) {
          if (D <= kFzThreads || tid == 0) kcnt[k] += n;
        }
      }
      __syncthreads();
    }
    // ---- publish this CTA's partial sums; barrier; combine
    for (int i = tid; i < K * D; i += kFzThreads) a.part[(size_t)blockIdx.x * K * D + i] = acc[i];
    for (int i = tid; i < K; i += kFzThreads) a.pcnt[(size_t)blockIdx.x * K + i] = kcnt[i];
    if (!fz_grid_sync(a.bar, a.ctl)) return;
    const int dblk = (D + 31) / 32;
    for (int job = blockIdx.x; job < K * dblk; job += G) {
      const int k = job / dblk, d = (job % dblk) * 32 + lane;
      float s = 0.f;
      int n = 0;
      for (int b = warp; b < G; b += kFzWarps) {
        if (d < D) s += __ldcg(a.part + ((size_t)b * K + k) * D + d);
        n += __ldcg(a.pcnt + (size_t)b * K + k);
      }
      red[warp][lane] = s;
      if (lane == 0) wtot[warp] = n;
      __syncthreads();
      if (warp == 0) {
        float tot = 0.f;
        int cnt = 0;
        for (int w = 0; w < kFzWarps; ++w) {
          tot += red[w][lane];
          cnt += wtot[w];
        }
        if (cnt > 0 && d < D) a.C[(size_t)k * D + d] = tot / (float)cnt;
        if (last_it && a.counts && lane == 0 && job % dblk == 0) a.counts[k] = cnt;
      }
      __syncthreads();
    }
    if (!fz_grid_sync(a.bar, a.ctl)) return;
  }
}

size_t lloyd_fused_smem(int K, int D) {
  const int Dr = (D + 3) / 4 * 4 + 4;
  return ((size_t)K * Dr + (size_t)K * D) * 4 + (size_t)3 * K * 4 + (size_t)2 * kFzThreads * 4;
}

bool lloyd_fused_fits(int K, int D) { return D >= 1 && D <= 1024 && lloyd_fused_smem(K, D) <= 200 * 1024; }

size_t lloyd_fused_workspace_bytes(int K, int D, int num_sms) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return al((size_t)num_sms * K * D * 4) + al((size_t)num_sms * K * 4) + 256;
}

template <typename T, int DCH>
static cudaError_t run_fused(FzArgs a, int G, size_t smem, cudaStream_t s) {
  auto kern = lloyd_fused_kernel<T, DCH>;
  cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e != cudaSuccess) return e;
  int occ = 0;
  e = cudaOccupancyMaxActiveBlocksPerMultiprocessor(&occ, kern, kFzThreads, smem);
  if (e != cudaSuccess) return e;
  if (occ < 1) return cudaErrorNotSupported;
  void *args[] = {&a};
  e = cudaLaunchCooperativeKernel((const void *)kern, dim3(G), dim3(kFzThreads), args, smem, s);
  count_launches(1);
  return e;
}

cudaError_t launch_lloyd_fused(DType dt, const void *X, int N, int D, int K, float *C, int32_t *labels,
                               float *mindist, int32_t *counts, int iters, void *ws, DevCtl ctl, int num_sms,
                               cudaStream_t s) {
  if (!lloyd_fused_fits(K, D)) return cudaErrorNotSupported;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  // one CTA per SM (fewer for a small N): the combine reads G partial rows.
  // Threads per row S: the smallest power of two that gives every SM a
  // pass of rows, at most the number of 32-centroid tiles and 16.
  int S = 1;
  const int tiles = (K + kFzTileK - 1) / kFzTileK;
  while (S < 16 && 2 * S <= tiles && (long long)(kFzThreads / S) * num_sms > N) S *= 2;
  const int P = kFzThreads / S;
  const size_t xs_bytes = (size_t)P * D * 4;
  const bool xs_ok = lloyd_fused_smem(K, D) + xs_bytes <= 200 * 1024;
  int G = (N + P - 1) / P;
  if (G > num_sms) G = num_sms;
  if (G < 1) G = 1;
  FzArgs a{};
  a.X = X;
  a.N = N;
  a.D = D;
  a.K = K;
  a.Dp = (D + 3) / 4 * 4;
  a.C = C;
  a.labels = labels;
  a.mindist = mindist;
  a.counts = counts;
  char *p = (char *)ws;
  a.part = (float *)p;
  p += al((size_t)num_sms * K * D * 4);
  a.pcnt = (int *)p;
  p += al((size_t)num_sms * K * 4);
  a.bar = (unsigned *)p;
  a.iters = iters;
  a.S = S;
  a.xs_ok = xs_ok ? 1 : 0;
  a.tau = near_tie_tau_simt(D);
  a.ctl = ctl;
  cudaError_t e = cudaMemsetAsync(a.bar, 0, 16, s);
  if (e != cudaSuccess) return e;
  const size_t smem = lloyd_fused_smem(K, D) + (xs_ok ? xs_bytes : 0);
  const int DCH = D <= 8 ? 8 : D <= 16 ? 16 : 32;
  switch (dt) {
    case kF32:
      return DCH == 8 ? run_fused<float, 8>(a, G, smem, s) : DCH == 16 ? run_fused<float, 16>(a, G, smem, s)
                                                                       : run_fused<float, 32>(a, G, smem, s);
    case kF16:
      return DCH == 8 ? run_fused<__half, 8>(a, G, smem, s) : DCH == 16 ? run_fused<__half, 16>(a, G, smem, s)
                                                                        : run_fused<__half, 32>(a, G, smem, s);
    default:
      return DCH == 8 ? run_fused<__nv_bfloat16, 8>(a, G, smem, s)
                      : DCH == 16 ? run_fused<__nv_bfloat16, 16>(a, G, smem, s)
                                  : run_fused<__nv_bfloat16, 32>(a, G, smem, s);
  }
}

}  // namespace fk
