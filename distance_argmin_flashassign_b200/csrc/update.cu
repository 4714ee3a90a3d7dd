// update.cu -- sort-inverse centroid update.
//
// Flash-KMeans (arXiv 2603.09229, abstract) replaces the per-point atomic
// scatter of the update stage by an explicitly built inverse mapping and
// segment-level localized reductions.  Here:
//
//   1. stable LSD radix sort of the cluster ids (11-bit digits, one pass for
//      up to 2,048 clusters, two for up to 2^22; a batch of problems whose N
//      is whole 4096-key tiles takes one pass on the label per problem):
//      per-tile digit histograms, a per-digit scan over tiles, and a scatter
//      whose within-tile ranks come from shared-memory digit masks -- the
//      sorted point ids are the inverse map (cluster -> its points);
//   2. segmented sums: the sorted order is cut into equal chunks of R
//      positions, one worker per chunk (a half warp for 256-byte rows), so a
//      hot cluster (Zipf skew) is spread over many workers instead of
//      serialising on one address.  A worker gathers its rows (each row read
//      as one contiguous vector across its lanes), accumulates in fp32
//      registers and writes a segment that lies wholly inside its chunk
//      straight to the output; the two boundary segments of a chunk go to
//      partial slots.  The same workers write the segment offsets (first
//      sorted position of every cluster id);
//   3. finalize: per cluster, partials of chunk-crossing segments are summed
//      in a fixed order and divided by the count; empty clusters are left
//      untouched.  No global atomics anywhere, so results are deterministic.
//
// Batched problems are one problem over B*K clusters: point (b, i) gets key
// b*K + label.
#include "fk_internal.h"

namespace fk {

// Kernels of the update are launched with programmatic stream serialization:
// a kernel may start (set up shared memory, compute addresses) while the one
// before it drains, and waits here before its first read of that kernel's
// results.  The wait returns once the previous grid has completed and its
// writes are visible.
__device__ __forceinline__ void wait_prior_grid() { asm volatile("griddepcontrol.wait;" ::: "memory"); }

template <typename... KArgs, typename... Args>
static cudaError_t launch_chained(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                                  Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}

constexpr int kSortThreads = 256;
constexpr int kSortItems = 16;
constexpr int kSortTile = kSortThreads * kSortItems;  // 4096 keys per tile
constexpr int kSortWarps = kSortThreads / 32;
constexpr int kMaxDigitBits = 11;
constexpr int kMaxBins = 1 << kMaxDigitBits;

struct SortPlan {
  int npass;
  int shift[2], bits[2];
  int T;          // tiles
  int seg_tiles;  // > 0: one pass on the label digit, problems of seg_tiles whole tiles each
};

static int ceil_log2(long long v) {
  int b = 0;
  while ((1ll << b) < v) ++b;
  return b;
}

// A batch of B problems whose N is a whole number of tiles is sorted in one
// pass on the label alone when the key b*K + label would need two: the
// problems' points are already in problem order, and each tile belongs to
// one problem, so ranking a tile's points by label and placing problem b's
// runs at b*N gives the order of a stable sort by key.
static SortPlan plan_sort(long long Ntot, long long Ktot, int B) {
  SortPlan p{};
  int bits = ceil_log2(Ktot);
  if (bits < 1) bits = 1;
  p.npass = (bits + kMaxDigitBits - 1) / kMaxDigitBits;
  const int w = (bits + p.npass - 1) / p.npass;
  int sh = 0;
  for (int i = 0; i < p.npass; ++i) {
    p.shift[i] = sh;
    p.bits[i] = (bits - sh) < w ? (bits - sh) : w;
    sh += p.bits[i];
  }
  p.T = (int)((Ntot + kSortTile - 1) / kSortTile);
  if (B > 1 && p.npass > 1 && (Ntot / B) % kSortTile == 0 && ceil_log2(Ktot / B) <= kMaxDigitBits) {
    p.npass = 1;
    p.shift[0] = 0;
    p.bits[0] = ceil_log2(Ktot / B) < 1 ? 1 : ceil_log2(Ktot / B);
    p.seg_tiles = (int)(Ntot / B / kSortTile);
  }
  return p;
}

// Positions per segment-sum worker: enough workers for about one wave of a
// B200 (148 SMs x 48 resident half-warp workers), at least 128; two full
// waves once a chunk would exceed 512 positions (with long chunks the
// workers' uneven segment work leaves a tail that the second wave evens
// out: 640 -> 618 us on 8 M Zipf-labelled rows).  Depends on Ntot only, so
// the summation order (and the result) does not depend on the device.
static int chunk_rows_R(long long Ntot) {
  constexpr long long kWave = 7104;
  long long R = (Ntot + kWave - 1) / kWave;
  if (R > 512) R = (Ntot + 2 * kWave - 1) / (2 * kWave);
  R = (R + 31) / 32 * 32;
  return (int)(R < 128 ? 128 : R);
}

// --------------------------------------------------------------- sorting --
// Sort key of position pos from its label: b*K + label for problem b.  A
// label outside [0, K) counts as 0 and sets `bad`; the caller records it
// once, after all of its loads, so that no atomic sits between them.
__device__ __forceinline__ int key_of_label(int lab, int pos, int N, int K, int B, bool &bad) {
  if ((unsigned)lab >= (unsigned)K) {
    bad = true;
    lab = 0;
  }
  return B > 1 ? (pos / N) * K + lab : lab;
}

// SEG: one pass per problem (the digit is the label), see plan_sort.
template <bool FIRST, bool SEG>
__global__ void __launch_bounds__(kSortThreads) radix_hist_kernel(const int32_t *__restrict__ keys, int Ntot,
                                                                  int N, int K, int B, int shift, int nbins,
                                                                  int T, int *__restrict__ H,
                                                                  int *status, int seg_tiles) {
  __shared__ int hist[kMaxBins + 1];
  for (int i = threadIdx.x; i <= nbins; i += kSortThreads) hist[i] = 0;
  __syncthreads();
  wait_prior_grid();
  const int base = blockIdx.x * kSortTile;
  // all of the thread's keys are loaded before any is counted (16 loads in
  // flight), then counted with shared-memory atomics
  int v[kSortItems];
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int pos = base + it * kSortThreads + threadIdx.x;
    v[it] = pos < Ntot ? keys[pos] : 0;
  }
  bool bad = false;
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int pos = base + it * kSortThreads + threadIdx.x;
    int d = nbins;  // spare bin for positions past the end
    if (pos < Ntot) {
      const int key = FIRST ? key_of_label(v[it], pos, N, K, B, bad) : v[it];
      // one pass per problem: the digit is the label (each tile lies in one problem)
      d = SEG ? key - ((int)blockIdx.x / seg_tiles) * K : (key >> shift) & (nbins - 1);
    }
    atomicAdd(&hist[d], 1);
  }
  if (bad) record_status(status, kStBadLabel);
  __syncthreads();
  for (int i = threadIdx.x; i < nbins; i += kSortThreads) H[(size_t)i * T + blockIdx.x] = hist[i];
}

// In place: row d of H becomes the exclusive prefix over tiles; totals[d] = row sum.
__global__ void __launch_bounds__(256) scan_rows_kernel(int *__restrict__ H, int T, int nbins,
                                                        int *__restrict__ totals) {
  const int w = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  wait_prior_grid();
  if (w >= nbins) return;
  int *row = H + (size_t)w * T;
  int carry = 0;
  // 256 tiles per round: all of a lane's loads are issued before any is
  // scanned, so a round costs one memory round trip
  constexpr int kPerLane = 8;
  for (int t0 = 0; t0 < T; t0 += 32 * kPerLane) {
    int v[kPerLane];
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      const int tt = t0 + 32 * i + lane;
      v[i] = tt < T ? row[tt] : 0;
    }
#pragma unroll
    for (int i = 0; i < kPerLane; ++i) {
      int incl = v[i];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int n = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += n;
      }
      const int tt = t0 + 32 * i + lane;
      if (tt < T) row[tt] = carry + incl - v[i];
      carry += __shfl_sync(0xffffffffu, incl, 31);
    }
  }
  if (lane == 0) totals[w] = carry;
}

// ints of the region that holds the warps' digit masks while keys are
// ranked, then the tile's keys and values in sorted order
static __host__ __device__ int scatter_xbuf_ints(int nbins) {
  return 2 * kSortTile > kSortWarps * nbins ? 2 * kSortTile : kSortWarps * nbins;
}
static size_t scatter_smem_bytes(int nbins) {
  return (size_t)(2 * nbins + kSortWarps + scatter_xbuf_ints(nbins)) * 4 + (size_t)kSortWarps * (nbins + 1) * 4;
}

template <bool FIRST, bool SEG>
__global__ void __launch_bounds__(kSortThreads) radix_scatter_kernel(
    const int32_t *__restrict__ keys_in, const int32_t *__restrict__ vals_in, int32_t *__restrict__ keys_out,
    int32_t *__restrict__ vals_out, int Ntot, int N, int K, int B, int shift, int nbins, int T,
    const int *__restrict__ H, const int *__restrict__ totals, int *status, int seg_tiles) {
  extern __shared__ int sh[];
  const int stride = nbins + 1;
  int *dbase = sh;                                                   // [nbins]
  int *tstart = sh + nbins;                                          // [nbins]
  int *wsum = sh + 2 * nbins;                                        // [kSortWarps]
  int *keys_s = sh + 2 * nbins + kSortWarps;                         // [kSortTile]
  int *vals_s = keys_s + kSortTile;                                  // [kSortTile]
  unsigned *wmask = reinterpret_cast<unsigned *>(keys_s);            // [kSortWarps][nbins], same place
  int *wcnt = keys_s + scatter_xbuf_ints(nbins);                     // [kSortWarps][nbins + 1]
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  // one pass per problem (SEG): this tile's problem; the digit is the label
  // and the problem's runs start at pb * N
  const int pb = SEG ? (int)blockIdx.x / seg_tiles : 0;
  auto digit = [&](int key) { return SEG ? key - pb * K : (key >> shift) & (nbins - 1); };
  wait_prior_grid();
  // the warp's 512 consecutive keys and values are loaded first, so that
  // their latency overlaps the digit-base reads below
  int keyr[kSortItems], valr[kSortItems], locr[kSortItems];
  const int base = blockIdx.x * kSortTile + warp * (kSortItems * 32);
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int pos = base + it * 32 + lane;
    keyr[it] = pos < Ntot ? keys_in[pos] : 0;
    valr[it] = pos < Ntot ? (FIRST ? pos : vals_in[pos]) : 0;
  }

  // digit base of this tile = exclusive scan of digit totals + tile prefix;
  // both reads of a thread's digits are issued before either is used
  constexpr int kPer = kMaxBins / kSortThreads;  // digits per thread, at most
  const int per = (nbins + kSortThreads - 1) / kSortThreads;
  int tv[kPer], hv[kPer];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int d = tid * per + i;
    const bool ok = i < per && d < nbins;
    if (SEG) {
      // the problem's count of digit d and the count in its tiles before
      // this one, from the prefix over all tiles at the problem's bounds
      const int t0 = pb * seg_tiles, t1 = t0 + seg_tiles;
      const int p0 = ok ? H[(size_t)d * T + t0] : 0;
      const int p1 = ok ? (t1 < T ? H[(size_t)d * T + t1] : totals[d]) : 0;
      tv[i] = p1 - p0;
      hv[i] = (ok ? H[(size_t)d * T + blockIdx.x] : 0) - p0;
    } else {
      tv[i] = ok ? totals[d] : 0;
      hv[i] = ok ? H[(size_t)d * T + blockIdx.x] : 0;
    }
  }
  int s = 0;
#pragma unroll
  for (int i = 0; i < kPer; ++i) s += tv[i];
  int incl = s;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += n;
  }
  if (lane == 31) wsum[warp] = incl;
  for (int i = tid; i < kSortWarps * stride; i += kSortThreads) wcnt[i] = 0;
  for (int i = tid; i < kSortWarps * nbins; i += kSortThreads) wmask[i] = 0u;
  __syncthreads();
  int run = incl - s + pb * N;
  for (int w = 0; w < warp; ++w) run += wsum[w];
#pragma unroll
  for (int i = 0; i < kPer; ++i) {
    const int d = tid * per + i;
    if (i < per && d < nbins) dbase[d] = run + hv[i];
    run += tv[i];
  }

  // stable ranks within each warp's consecutive keys.  The lanes that hold
  // the same digit find each other through shared memory: each sets its bit
  // in the warp's mask word of its digit and reads the word back (on this
  // GPU much cheaper than a ballot per digit bit or match.any, whose cost
  // grows with the number of distinct digits).  The lowest of them clears
  // the word and adds the group's size to the warp's count of that digit;
  // the count before the add, broadcast after all of the warp's keys are
  // counted, is where the group starts.
  const unsigned lt_mask = (1u << lane) - 1u;
  int *mycnt = wcnt + warp * stride;
  unsigned *mymask = wmask + warp * nbins;
  unsigned peer[kSortItems];
  bool bad = false;
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int pos = base + it * 32 + lane;
    const bool valid = pos < Ntot;
    int d = 0;
    if (valid) {
      if (FIRST) keyr[it] = key_of_label(keyr[it], pos, N, K, B, bad);
      d = digit(keyr[it]);
    }
    if (valid) atomicOr(mymask + d, 1u << lane);
    __syncwarp();
    const unsigned peers = valid ? mymask[d] : 0u;
    __syncwarp();
    int c = 0;
    if (valid && lane == __ffs(peers) - 1) {
      mymask[d] = 0u;
      c = atomicAdd(mycnt + d, __popc(peers));
    }
    __syncwarp();  // the next key's mask and add come after these
    peer[it] = peers;
    locr[it] = c;
  }
#pragma unroll
  for (int it = 0; it < kSortItems; ++it)
    locr[it] = __shfl_sync(0xffffffffu, locr[it], (__ffs(peer[it]) - 1) & 31) + __popc(peer[it] & lt_mask);
  if (bad) record_status(status, kStBadLabel);
  __syncthreads();  // masks done: the region holds keys and values from here on
  // per digit: exclusive prefix over warps (in place) and the tile's count,
  // then the exclusive scan of the tile's counts over digits: where each
  // digit's run starts in the tile's sorted order
  int cnt[kPer];
  int tsum = 0;
  for (int i = 0; i < per; ++i) {
    const int d = tid * per + i;
    int r = 0;
    if (d < nbins)
      for (int w = 0; w < kSortWarps; ++w) {
        const int t = wcnt[w * stride + d];
        wcnt[w * stride + d] = r;
        r += t;
      }
    cnt[i] = r;
    tsum += r;
  }
  int tincl = tsum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int n = __shfl_up_sync(0xffffffffu, tincl, o);
    if (lane >= o) tincl += n;
  }
  __syncthreads();  // everyone is done reading wsum (digit bases above)
  if (lane == 31) wsum[warp] = tincl;
  __syncthreads();
  int trun = tincl - tsum;
  for (int w = 0; w < warp; ++w) trun += wsum[w];
  for (int i = 0; i < per; ++i) {
    const int d = tid * per + i;
    if (d < nbins) tstart[d] = trun;
    trun += cnt[i];
  }
  __syncthreads();
  // exchange through shared memory into the tile's sorted order ...
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int pos = base + it * 32 + lane;
    if (pos < Ntot) {
      const int d = digit(keyr[it]);
      const int lp = tstart[d] + mycnt[d] + locr[it];
      keys_s[lp] = keyr[it];
      vals_s[lp] = valr[it];
    }
  }
  __syncthreads();
  // ... and write it out in that order: consecutive threads store
  // consecutive positions of a digit's run
  const int nvalid = (Ntot - blockIdx.x * kSortTile) < kSortTile ? (Ntot - blockIdx.x * kSortTile) : kSortTile;
#pragma unroll
  for (int it = 0; it < kSortItems; ++it) {
    const int idx = it * kSortThreads + tid;
    if (idx < nvalid) {
      const int key = keys_s[idx];
      const int d = digit(key);
      const int o = dbase[d] + (idx - tstart[d]);
      keys_out[o] = key;
      vals_out[o] = vals_s[idx];
    }
  }
}

// Segment offsets are written by the segment-sum warps: at every position
// where the sorted key changes from kp to k, off[kp+1 .. k] = that position
// (empty clusters in between share it); the warp ending at Ntot writes
// off[k_last+1 .. Ktot] = Ntot.  Every entry is written exactly once.
__device__ __forceinline__ void write_offsets(int *__restrict__ off, int kp, int k, int pos, int lane) {
  for (int kk = kp + 1 + lane; kk <= k; kk += 32) off[kk] = pos;
}

__device__ __forceinline__ void cp_async16(void *smem_dst, const void *gsrc) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(smem_u32(smem_dst)), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N> __device__ __forceinline__ void cp_async_wait() {
  asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// ------------------------------------------------------- segmented sums --
template <typename T> struct Vec;
template <> struct Vec<float> {
  template <int N> __device__ static void load(const float *p, float *v) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        const float4 w = __ldg(reinterpret_cast<const float4 *>(p) + i);
        v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
      }
    } else if constexpr (N == 2) {
      const float2 w = __ldg(reinterpret_cast<const float2 *>(p));
      v[0] = w.x; v[1] = w.y;
    } else {
      v[0] = __ldg(p);
    }
  }
  template <int N> __device__ static void load_shared(const float *p, float *v) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int i = 0; i < N / 4; ++i) {
        const float4 w = reinterpret_cast<const float4 *>(p)[i];
        v[4 * i] = w.x; v[4 * i + 1] = w.y; v[4 * i + 2] = w.z; v[4 * i + 3] = w.w;
      }
    } else if constexpr (N == 2) {
      const float2 w = *reinterpret_cast<const float2 *>(p);
      v[0] = w.x; v[1] = w.y;
    } else {
      v[0] = p[0];
    }
  }
};
__device__ __forceinline__ void unpack_half2(uint32_t w, float *v) {
  const __half2 h = *reinterpret_cast<const __half2 *>(&w);
  v[0] = __low2float(h);
  v[1] = __high2float(h);
}
__device__ __forceinline__ void unpack_bf162(uint32_t w, float *v) {
  v[0] = __uint_as_float(w << 16);
  v[1] = __uint_as_float(w & 0xffff0000u);
}
template <typename T, bool BF> struct Vec16 {
  template <int N> __device__ static void load(const T *p, float *v) {
    auto up = [](uint32_t w, float *o) { if (BF) unpack_bf162(w, o); else unpack_half2(w, o); };
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        const uint4 w = __ldg(reinterpret_cast<const uint4 *>(p) + i);
        up(w.x, v + 8 * i); up(w.y, v + 8 * i + 2); up(w.z, v + 8 * i + 4); up(w.w, v + 8 * i + 6);
      }
    } else if constexpr (N == 4) {
      const uint2 w = __ldg(reinterpret_cast<const uint2 *>(p));
      up(w.x, v); up(w.y, v + 2);
    } else if constexpr (N == 2) {
      up(__ldg(reinterpret_cast<const unsigned int *>(p)), v);
    } else {
      v[0] = to_f32<T>(p[0]);
    }
  }
  template <int N> __device__ static void load_shared(const T *p, float *v) {
    auto up = [](uint32_t w, float *o) { if (BF) unpack_bf162(w, o); else unpack_half2(w, o); };
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int i = 0; i < N / 8; ++i) {
        const uint4 w = reinterpret_cast<const uint4 *>(p)[i];
        up(w.x, v + 8 * i); up(w.y, v + 8 * i + 2); up(w.z, v + 8 * i + 4); up(w.w, v + 8 * i + 6);
      }
    } else if constexpr (N == 4) {
      const uint2 w = *reinterpret_cast<const uint2 *>(p);
      up(w.x, v); up(w.y, v + 2);
    } else if constexpr (N == 2) {
      up(*reinterpret_cast<const unsigned int *>(p), v);
    } else {
      v[0] = to_f32<T>(p[0]);
    }
  }
};
template <> struct Vec<__half> : Vec16<__half, false> {};
template <> struct Vec<__nv_bfloat16> : Vec16<__nv_bfloat16, true> {};

// CONTIG: lane l owns dims [l*NACC, l*NACC + NACC) (D == 32*NACC, vector loads);
// otherwise lane l owns dims l + 32*a, a < NACC, masked by D.
template <typename T, int NACC, bool CONTIG, int MODE>
__global__ void __launch_bounds__(256) segsum_kernel(const T *__restrict__ X, int D,
                                                     const int32_t *__restrict__ perm,
                                                     const int32_t *__restrict__ skeys, int Ntot, int Ktot,
                                                     int R, float *__restrict__ C, double *__restrict__ acc,
                                                     float *__restrict__ parts, int *__restrict__ off) {
  constexpr int PF = NACC <= 4 ? 8 : (NACC <= 8 ? 4 : (NACC <= 16 ? 2 : 1));  // rows in flight
  const int lane = threadIdx.x & 31;
  wait_prior_grid();
  const long long wq = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const long long p0l = wq * R;
  if (p0l >= Ntot) return;
  const int p0 = (int)p0l;
  const int p1 = (Ntot - p0) < R ? Ntot : p0 + R;
  const int kfirst = skeys[p0];
  const int kprev = p0 > 0 ? skeys[p0 - 1] : -1;
  const bool split_start = kprev == kfirst;
  const bool split_end = p1 < Ntot && skeys[p1] == skeys[p1 - 1];
  write_offsets(off, kprev, kfirst, p0, lane);

  float a[NACC];
#pragma unroll
  for (int i = 0; i < NACC; ++i) a[i] = 0.f;
  int cur = kfirst, s = p0;

  auto dim_of = [&](int i) { return CONTIG ? lane * NACC + i : lane + 32 * i; };
  auto flush = [&](int k, int sb, int se) {
    const bool split = (sb == p0 && split_start) || (se == p1 && split_end);
    if (!split) {
      if (MODE == kMean) {
        const float fc = (float)(se - sb);
        float *dst = C + (size_t)k * D;
#pragma unroll
        for (int i = 0; i < NACC; ++i) {
          const int d = dim_of(i);
          if (CONTIG || d < D) dst[d] = a[i] / fc;
        }
      } else {
        double *dst = acc + (size_t)k * D;
#pragma unroll
        for (int i = 0; i < NACC; ++i) {
          const int d = dim_of(i);
          if (CONTIG || d < D) dst[d] += (double)a[i];
        }
      }
    } else {
      float *dst = parts + ((size_t)wq * 2 + (sb == p0 ? 0 : 1)) * D;
#pragma unroll
      for (int i = 0; i < NACC; ++i) {
        const int d = dim_of(i);
        if (CONTIG || d < D) dst[d] = a[i];
      }
    }
  };

  for (int b0 = p0; b0 < p1; b0 += 32) {
    const int n = (p1 - b0) < 32 ? (p1 - b0) : 32;
    const int mk = lane < n ? skeys[b0 + lane] : 0;
    const int mr = lane < n ? perm[b0 + lane] : 0;
    for (int t0 = 0; t0 < n; t0 += PF) {
      float v[PF][NACC];
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const int row = __shfl_sync(0xffffffffu, mr, (t0 + u) & 31);
        if (t0 + u < n) {
          const T *xr = X + (size_t)row * D;
          if (CONTIG) {
            Vec<T>::template load<NACC>(xr + lane * NACC, v[u]);
          } else {
#pragma unroll
            for (int i = 0; i < NACC; ++i) {
              const int d = lane + 32 * i;
              v[u][i] = d < D ? to_f32<T>(xr[d]) : 0.f;
            }
          }
        }
      }
#pragma unroll
      for (int u = 0; u < PF; ++u) {
        const int k = __shfl_sync(0xffffffffu, mk, (t0 + u) & 31);
        if (t0 + u < n) {
          if (k != cur) {
            flush(cur, s, b0 + t0 + u);
            write_offsets(off, cur, k, b0 + t0 + u, lane);
            cur = k;
            s = b0 + t0 + u;
#pragma unroll
            for (int i = 0; i < NACC; ++i) a[i] = 0.f;
          }
#pragma unroll
          for (int i = 0; i < NACC; ++i) a[i] += v[u][i];
        }
      }
    }
  }
  flush(cur, s, p1);
  if (p1 == Ntot) write_offsets(off, cur, Ktot, Ntot, lane);
}

// Staged variant for rows of 32*NACC elements whose byte size is a multiple
// of 16: every warp copies the rows of its next groups of 32 sorted
// positions into a shared-memory ring with cp.async (16 bytes per lane, no
// registers held), so about 16 KB per warp are in flight while it sums the
// group that has landed.
constexpr int kSegWarps = 4, kSegStages = 2;
template <typename T, int NACC, int MODE>
__global__ void __launch_bounds__(kSegWarps * 32) segsum_staged_kernel(
    const T *__restrict__ X, int D, const int32_t *__restrict__ perm, const int32_t *__restrict__ skeys, int Ntot,
    int Ktot, int R, float *__restrict__ C, double *__restrict__ acc, float *__restrict__ parts,
    int *__restrict__ off) {
  constexpr int RB = 32 * NACC * (int)sizeof(T);  // bytes per row
  constexpr int PIECES = RB / 16;
  constexpr int SLOT = 32 * RB;
  static_assert(RB % 16 == 0, "rows must be whole 16-byte pieces");
  extern __shared__ __align__(16) uint8_t seg_smem[];
  const int lane = threadIdx.x & 31, wib = threadIdx.x >> 5;
  wait_prior_grid();
  uint8_t *ring = seg_smem + wib * (kSegStages * SLOT);
  const long long wq = (long long)blockIdx.x * kSegWarps + wib;
  const long long p0l = wq * R;
  if (p0l >= Ntot) return;
  const int p0 = (int)p0l;
  const int p1 = (Ntot - p0) < R ? Ntot : p0 + R;
  const int kfirst = skeys[p0];
  const int kprev = p0 > 0 ? skeys[p0 - 1] : -1;
  const bool split_start = kprev == kfirst;
  const bool split_end = p1 < Ntot && skeys[p1] == skeys[p1 - 1];
  write_offsets(off, kprev, kfirst, p0, lane);
  const int ngroups = (p1 - p0 + 31) / 32;

  float a[NACC];
#pragma unroll
  for (int i = 0; i < NACC; ++i) a[i] = 0.f;
  int cur = kfirst, s = p0;
  auto flush = [&](int k, int sb, int se) {
    const bool split = (sb == p0 && split_start) || (se == p1 && split_end);
    float *dst;
    if (!split) {
      if (MODE == kMean) {
        const float fc = (float)(se - sb);
        dst = C + (size_t)k * D + lane * NACC;
#pragma unroll
        for (int i = 0; i < NACC; ++i) dst[i] = a[i] / fc;
      } else {
        double *dd = acc + (size_t)k * D + lane * NACC;
#pragma unroll
        for (int i = 0; i < NACC; ++i) dd[i] += (double)a[i];
      }
    } else {
      dst = parts + ((size_t)wq * 2 + (sb == p0 ? 0 : 1)) * D + lane * NACC;
#pragma unroll
      for (int i = 0; i < NACC; ++i) dst[i] = a[i];
    }
  };
  // copy the rows of group g into ring slot `slot`; returns (key, row) of lane
  auto issue = [&](int g, int slot, int &mk, int &mr) {
    const int base = p0 + g * 32;
    const int n = (p1 - base) < 32 ? (p1 - base) : 32;
    mk = lane < n ? skeys[base + lane] : 0;
    mr = lane < n ? perm[base + lane] : 0;
    uint8_t *dst = ring + slot * SLOT;
#pragma unroll
    for (int it = 0; it < PIECES; ++it) {
      const int q = it * 32 + lane;
      const int i = q / PIECES, pc = q % PIECES;
      const int row = __shfl_sync(0xffffffffu, mr, i);
      if (i < n) cp_async16(dst + q * 16, reinterpret_cast<const uint8_t *>(X) + (size_t)row * RB + pc * 16);
    }
    cp_async_commit();
  };
  auto consume = [&](int g, int slot, int mk) {
    const int base = p0 + g * 32;
    const int n = (p1 - base) < 32 ? (p1 - base) : 32;
    const T *src = reinterpret_cast<const T *>(ring + slot * SLOT) + lane * NACC;
    for (int t = 0; t < n; ++t) {
      const int k = __shfl_sync(0xffffffffu, mk, t);
      if (k != cur) {
        flush(cur, s, base + t);
        write_offsets(off, cur, k, base + t, lane);
        cur = k;
        s = base + t;
#pragma unroll
        for (int i = 0; i < NACC; ++i) a[i] = 0.f;
      }
      float v[NACC];
      Vec<T>::template load_shared<NACC>(src + t * (32 * NACC), v);
#pragma unroll
      for (int i = 0; i < NACC; ++i) a[i] += v[i];
    }
  };

  int k0 = 0, r0 = 0, k1 = 0, r1 = 0;
  issue(0, 0, k0, r0);
  if (ngroups > 1) issue(1, 1, k1, r1);
  for (int g = 0; g < ngroups; g += 2) {
    // slot 0 holds group g
    if (g + 1 < ngroups) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncwarp();
    consume(g, 0, k0);
    __syncwarp();
    if (g + 2 < ngroups) issue(g + 2, 0, k0, r0);
    if (g + 1 >= ngroups) break;
    // slot 1 holds group g + 1
    if (g + 2 < ngroups) cp_async_wait<1>(); else cp_async_wait<0>();
    __syncwarp();
    consume(g + 1, 1, k1);
    __syncwarp();
    if (g + 3 < ngroups) issue(g + 3, 1, k1, r1);
  }
  flush(cur, s, p1);
  if (p1 == Ntot) write_offsets(off, cur, Ktot, Ntot, lane);
}

// Gather workers of W lanes (W = row bytes / 16, 8 to 32): lane l of a
// worker owns the 16 bytes [16l, 16l + 16) of every row, and every worker
// sums the rows of its own chunk of R sorted positions, GATHER_ROWS of them
// in flight at a time (one 16-byte load per lane and row).  Small workers
// mean many independent gathers per SM, which is what HBM needs to serve
// random rows at full rate.  The segmentation (which segments are whole,
// which go to the two partial slots of the chunk) is the one of
// segsum_kernel, with worker index in place of warp index.
// 16 bytes of a row of X, read once: not kept in L1 (allocating L1 lines for
// the gathered rows cost the segment sums 7 % on the embedding workload).
__device__ __forceinline__ uint4 ld_row16(const void *p) {
  uint4 r;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(r.x), "=r"(r.y), "=r"(r.z), "=r"(r.w)
               : "l"(p));
  return r;
}
constexpr int kGatherRows = 8;
template <typename T, int W, int MODE>
__global__ void __launch_bounds__(256, 3) segsum_gather_kernel(const T *__restrict__ X, int D,
                                                            const int32_t *__restrict__ perm,
                                                            const int32_t *__restrict__ skeys, int Ntot, int Ktot,
                                                            int R, float *__restrict__ C, double *__restrict__ acc,
                                                            float *__restrict__ parts, int *__restrict__ off) {
  constexpr int EPL = 16 / (int)sizeof(T);  // elements per lane
  constexpr int U = kGatherRows;
  static_assert(W >= U && W <= 32 && (32 % W) == 0, "worker width");
  const int lw = threadIdx.x % W;
  const long long wq = ((long long)blockIdx.x * blockDim.x + threadIdx.x) / W;  // worker = chunk index
  wait_prior_grid();
  const long long p0l = wq * R;
  const bool live = p0l < Ntot;
  const int p0 = live ? (int)p0l : Ntot;
  const int p1 = (Ntot - p0) < R ? Ntot : p0 + R;
  int cur = 0, s = p0;
  bool split_start = false, split_end = false;
  // lanes 0 .. U-1 hold the sorted keys and point ids of a batch; those of
  // the next batch are loaded while this batch's rows are in flight, so a
  // batch costs one memory round trip, not two
  int mk_next = 0, mr_next = 0;
  auto batch_ids = [&](int bt) {
    const int b0 = p0 + bt * U;
    const bool in = lw < U && b0 + lw < p1;
    mk_next = in ? skeys[b0 + lw] : 0;
    mr_next = in ? perm[b0 + lw] : 0;
  };
  batch_ids(0);  // in flight together with the chunk-boundary keys below
  if (live) {
    const int kfirst = skeys[p0];
    const int kprev = p0 > 0 ? skeys[p0 - 1] : -1;
    split_start = kprev == kfirst;
    split_end = p1 < Ntot && skeys[p1] == skeys[p1 - 1];
    for (int kk = kprev + 1 + lw; kk <= kfirst; kk += W) off[kk] = p0;
    cur = kfirst;
  }
  float a[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) a[i] = 0.f;
  auto flush = [&](int k, int sb, int se) {
    const bool split = (sb == p0 && split_start) || (se == p1 && split_end);
    if (!split) {
      if (MODE == kMean) {
        const float inv = 1.f / (float)(se - sb);
        float *dst = C + (size_t)k * D + lw * EPL;
#pragma unroll
        for (int i = 0; i < EPL; i += 4)
          *reinterpret_cast<float4 *>(dst + i) = make_float4(a[i] * inv, a[i + 1] * inv, a[i + 2] * inv, a[i + 3] * inv);
      } else {
        double *dst = acc + (size_t)k * D + lw * EPL;
#pragma unroll
        for (int i = 0; i < EPL; ++i) dst[i] += (double)a[i];
      }
    } else {
      float *dst = parts + ((size_t)wq * 2 + (sb == p0 ? 0 : 1)) * D + lw * EPL;
#pragma unroll
      for (int i = 0; i < EPL; i += 4) *reinterpret_cast<float4 *>(dst + i) = make_float4(a[i], a[i + 1], a[i + 2], a[i + 3]);
    }
  };
  // every worker of the warp runs the same number of batches (shuffles stay
  // converged); positions past a worker's end are masked
  const int nb = (R + U - 1) / U;
  for (int bt = 0; bt < nb; ++bt) {
    const int b0 = p0 + bt * U;
    const int mk = mk_next, mr = mr_next;
    uint4 v[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int row = __shfl_sync(0xffffffffu, mr, u, W);
      v[u] = (b0 + u < p1) ? ld_row16(reinterpret_cast<const uint4 *>(X + (size_t)row * D) + lw) : make_uint4(0, 0, 0, 0);
    }
    if (bt + 1 < nb) batch_ids(bt + 1);
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int ku = __shfl_sync(0xffffffffu, mk, u, W);
      if (b0 + u < p1) {
        if (ku != cur) {
          flush(cur, s, b0 + u);
          for (int q = cur + 1 + lw; q <= ku; q += W) off[q] = b0 + u;
          cur = ku;
          s = b0 + u;
#pragma unroll
          for (int i = 0; i < EPL; ++i) a[i] = 0.f;
        }
        const uint32_t w[4] = {v[u].x, v[u].y, v[u].z, v[u].w};
        if constexpr (sizeof(T) == 4) {
#pragma unroll
          for (int i = 0; i < 4; ++i) a[i] += __uint_as_float(w[i]);
        } else {
#pragma unroll
          for (int i = 0; i < 4; ++i) {
            float f[2];
            if constexpr (std::is_same<T, __nv_bfloat16>::value) unpack_bf162(w[i], f);
            else unpack_half2(w[i], f);
            a[2 * i] += f[0];
            a[2 * i + 1] += f[1];
          }
        }
      }
    }
  }
  if (live) {
    flush(cur, s, p1);
    if (p1 == Ntot)
      for (int q = cur + 1 + lw; q <= Ktot; q += W) off[q] = Ntot;
  }
}

// Per cluster: the count and, for a segment that crosses chunk borders, the
// sum of its partial rows in a fixed order, divided by the count (segments
// inside one chunk were written by their segment-sum worker).  Block b of G
// owns the clusters b, b + G, b + 2G, ... (hot clusters of a skewed
// distribution are usually consecutive ids, so they land in different
// blocks) and takes them 1024 at a time.  Warp w handles the window's
// clusters w, w + 32, ...: a segment with at most kHotParts partial rows it
// sums itself (lanes over dimensions, rows in chunk order); longer ones are
// listed in shared memory and summed after the window by all 32 warps: warp
// w sums the partial rows w, w + 32, ..., then thread d adds the 32 warp sums
// of dimension d in warp order.
constexpr int kHotParts = 16;
template <int MODE>
__global__ void __launch_bounds__(1024) seg_finalize_kernel(const int *__restrict__ off, int Ktot, int D, int R,
                                                            const float *__restrict__ parts,
                                                            float *__restrict__ C, int32_t *__restrict__ counts,
                                                            double *__restrict__ acc, long long *__restrict__ cnt) {
  __shared__ float red[32][129];
  __shared__ int hot[1024];
  __shared__ int nhot;
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  wait_prior_grid();
  const long long G = gridDim.x;
  auto part_row = [&](int s, int q0, int i) {
    const size_t first = (size_t)q0 * 2 + (s == q0 * R ? 0 : 1);
    return parts + (i == 0 ? first : (size_t)(q0 + i) * 2) * D;
  };
  auto emit = [&](int k, int d, float sum, int n) {
    const size_t o = (size_t)k * D + d;
    if (MODE == kMean) C[o] = sum / (float)n;
    else acc[o] += (double)sum;
  };
  for (long long i0 = 0; blockIdx.x + G * i0 < Ktot; i0 += 1024) {
    if (threadIdx.x == 0) nhot = 0;
    __syncthreads();
    for (int j = w; j < 1024; j += 32) {
      const long long kl = blockIdx.x + G * (i0 + j);
      if (kl >= Ktot) break;
      const int k = (int)kl;
      const int s = off[k], e = off[k + 1], n = e - s;
      if (lane == 0) {
        if (MODE == kMean) {
          if (counts) counts[k] = n;
        } else {
          cnt[k] += n;
        }
      }
      if (n == 0) continue;
      const int q0 = s / R, q1 = (e - 1) / R;
      if (q0 == q1) continue;  // segment inside one chunk: already written
      const int np = q1 - q0 + 1;
      if (np > kHotParts) {
        if (lane == 0) hot[atomicAdd(&nhot, 1)] = k;
        continue;
      }
      // 4 dimensions per lane per pass; the partial rows are loaded 4 at a
      // time (in flight together), then added in chunk order
      for (int d0 = 0; d0 < D; d0 += 128) {
        float t[4] = {0.f, 0.f, 0.f, 0.f};
        for (int i0 = 0; i0 < np; i0 += 4) {
          float v[4][4];
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            const bool in = i0 + ii < np;
            const float *row = part_row(s, q0, in ? i0 + ii : 0) + d0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) v[ii][jj] = in && d0 + lane + 32 * jj < D ? row[lane + 32 * jj] : 0.f;
          }
#pragma unroll
          for (int ii = 0; ii < 4; ++ii)
            if (i0 + ii < np) {
#pragma unroll
              for (int jj = 0; jj < 4; ++jj) t[jj] += v[ii][jj];
            }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj)
          if (d0 + lane + 32 * jj < D) emit(k, d0 + lane + 32 * jj, t[jj], n);
      }
    }
    __syncthreads();
    const int nh = nhot;
    for (int h = 0; h < nh; ++h) {
      const int k = hot[h];
      const int s = off[k], e = off[k + 1], n = e - s;
      const int q0 = s / R, np = (e - 1) / R - q0 + 1;
      for (int d0 = 0; d0 < D; d0 += 128) {
        float t[4] = {0.f, 0.f, 0.f, 0.f};
        // rows w, w + 32, ... in that order, four loaded at a time
        for (int i0 = w; i0 < np; i0 += 4 * 32) {
          float v[4][4];
#pragma unroll
          for (int ii = 0; ii < 4; ++ii) {
            const int i = i0 + 32 * ii;
            const float *row = part_row(s, q0, i < np ? i : 0) + d0;
#pragma unroll
            for (int jj = 0; jj < 4; ++jj) v[ii][jj] = i < np && d0 + lane + 32 * jj < D ? row[lane + 32 * jj] : 0.f;
          }
#pragma unroll
          for (int ii = 0; ii < 4; ++ii)
            if (i0 + 32 * ii < np) {
#pragma unroll
              for (int jj = 0; jj < 4; ++jj)
                if (d0 + lane + 32 * jj < D) t[jj] += v[ii][jj];
            }
        }
#pragma unroll
        for (int jj = 0; jj < 4; ++jj) red[w][lane + 32 * jj] = t[jj];
        __syncthreads();
        if (threadIdx.x < 128 && d0 + threadIdx.x < D) {
          float tot = 0.f;
          for (int ww = 0; ww < 32; ++ww) tot += red[ww][threadIdx.x];
          emit(k, d0 + threadIdx.x, tot, n);
        }
        __syncthreads();
      }
    }
  }
}

__global__ void __launch_bounds__(256) divide_acc_kernel(const double *__restrict__ acc,
                                                         const long long *__restrict__ cnt, int Ktot, int D,
                                                         float *__restrict__ C, int32_t *__restrict__ counts) {
  const size_t total = (size_t)Ktot * D;
  wait_prior_grid();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < total; i += (size_t)gridDim.x * blockDim.x) {
    const int k = (int)(i / D);
    const long long n = cnt[k];
    if (n > 0) C[i] = (float)(acc[i] / (double)n);
    if (counts && i % D == 0) counts[k] = (int32_t)n;
  }
}

// ---------------------------------------------------------------- host ---
static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

struct UpdateWs {
  int32_t *kA, *vA, *kB, *vB;
  int *H, *totals, *off;
  float *parts;
  size_t bytes;
};

static UpdateWs carve(void *base, long long Ntot, long long Ktot, int D, int B) {
  const SortPlan sp = plan_sort(Ntot, Ktot, B);
  const int R = chunk_rows_R(Ntot);
  const long long nchunks = (Ntot + R - 1) / R;
  int maxbins = 0;
  for (int i = 0; i < sp.npass; ++i) maxbins = (1 << sp.bits[i]) > maxbins ? (1 << sp.bits[i]) : maxbins;
  UpdateWs w{};
  char *p = (char *)base;
  size_t o = 0;
  auto take = [&](size_t n) { char *r = p ? p + o : nullptr; o += al256(n); return r; };
  w.kA = (int32_t *)take((size_t)Ntot * 4);
  w.vA = (int32_t *)take((size_t)Ntot * 4);
  w.kB = (int32_t *)take((size_t)Ntot * 4);
  w.vB = (int32_t *)take((size_t)Ntot * 4);
  w.H = (int *)take((size_t)maxbins * sp.T * 4);
  w.totals = (int *)take((size_t)maxbins * 4);
  w.off = (int *)take((size_t)(Ktot + 1) * 4);
  w.parts = (float *)take((size_t)nchunks * 2 * D * 4);
  w.bytes = o;
  return w;
}

size_t update_workspace_bytes(int64_t Ntot, int64_t Ktot, int D, int B) {
  return carve(nullptr, Ntot, Ktot, D, B).bytes;
}

template <typename T, int MODE, int NACC>
static void launch_staged(const UpdateArgs &a, const int32_t *perm, const int32_t *skeys, int Ntot, int Ktot,
                          int R, float *parts, int *off, cudaStream_t s) {
  constexpr int smem = kSegWarps * kSegStages * 32 * 32 * NACC * (int)sizeof(T);
  static bool configured[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 64 && !configured[dev]) {
    cudaFuncSetAttribute(segsum_staged_kernel<T, NACC, MODE>, cudaFuncAttributeMaxDynamicSharedMemorySize, smem);
    configured[dev] = true;
  }
  const long long nchunks = ((long long)Ntot + R - 1) / R;
  const int grid = (int)((nchunks + kSegWarps - 1) / kSegWarps);
  launch_chained(segsum_staged_kernel<T, NACC, MODE>, dim3(grid), dim3(kSegWarps * 32), smem, s, (const T *)a.X, a.D, perm, skeys, Ntot,
                                                                        Ktot, R, a.C, a.acc, parts, off);
}

template <typename T, int MODE>
static void launch_segsum(const UpdateArgs &a, const int32_t *perm, const int32_t *skeys, int Ntot, int Ktot,
                          int R, float *parts, int *off, cudaStream_t s) {
  const T *X = (const T *)a.X;
  const int D = a.D;
  const bool aligned = ((uintptr_t)a.X % 16 == 0);
  const int nacc_c = D % 32 == 0 ? D / 32 : 0;
  const int rb = nacc_c * (int)sizeof(T) * 32;
  {
    const int W = D * (int)sizeof(T) / 16;
    const long long nworkers = ((long long)Ntot + R - 1) / R;
    if (aligned && (D * (int)sizeof(T)) % 16 == 0 && (W == 8 || W == 16 || W == 32)) {
      const int ggrid = (int)((nworkers * W + 255) / 256);
#define FK_GATHER(WW)                                                                                 \
  return (void)launch_chained(segsum_gather_kernel<T, WW, MODE>, dim3(ggrid), dim3(256), 0, s, X, D, perm, skeys, Ntot, Ktot, R, a.C, \
                                                                       a.acc, parts, off)
      if (W == 8) FK_GATHER(8);
      if (W == 16) FK_GATHER(16);
      FK_GATHER(32);
#undef FK_GATHER
    }
  }
  if (aligned && rb % 16 == 0 && rb > 0 && rb <= 512) {
    if (nacc_c == 1) return launch_staged<T, MODE, 1>(a, perm, skeys, Ntot, Ktot, R, parts, off, s);
    if (nacc_c == 2) return launch_staged<T, MODE, 2>(a, perm, skeys, Ntot, Ktot, R, parts, off, s);
    if (nacc_c == 4) return launch_staged<T, MODE, 4>(a, perm, skeys, Ntot, Ktot, R, parts, off, s);
    if (nacc_c == 8 && sizeof(T) == 2) return launch_staged<T, MODE, 8>(a, perm, skeys, Ntot, Ktot, R, parts, off, s);
  }
  const long long nchunks = ((long long)Ntot + R - 1) / R;
  const int grid = (int)((nchunks + 7) / 8);
  const bool contig_ok = D % 32 == 0 && aligned;
#define FK_SEG(NA, CG) \
  launch_chained(segsum_kernel<T, NA, CG, MODE>, dim3(grid), dim3(256), 0, s, X, D, perm, skeys, Ntot, Ktot, R, a.C, a.acc, parts, off)
  if (contig_ok && nacc_c == 1) FK_SEG(1, true);
  else if (contig_ok && nacc_c == 2) FK_SEG(2, true);
  else if (contig_ok && nacc_c == 4) FK_SEG(4, true);
  else if (contig_ok && nacc_c == 8) FK_SEG(8, true);
  else {
    const int need = (D + 31) / 32;
    if (need <= 1) FK_SEG(1, false);
    else if (need <= 2) FK_SEG(2, false);
    else if (need <= 4) FK_SEG(4, false);
    else if (need <= 8) FK_SEG(8, false);
    else if (need <= 16) FK_SEG(16, false);
    else FK_SEG(32, false);
  }
#undef FK_SEG
}

cudaError_t launch_update(const UpdateArgs &a, void *ws, size_t ws_bytes, DevCtl ctl, int num_sms,
                          cudaStream_t s) {
  const long long Ntot = (long long)a.B * a.N, Ktot = (long long)a.B * a.K;
  if (Ntot == 0) return cudaSuccess;
  const UpdateWs w = carve(ws, Ntot, Ktot, a.D, a.B);
  if (w.bytes > ws_bytes) return cudaErrorInvalidValue;
  const SortPlan sp = plan_sort(Ntot, Ktot, a.B);
  const int N = (int)Ntot;
  int nl = 0;

  {  // the scatter's tile exchange needs more than the default 48 KB of shared memory
    static bool configured[64] = {};
    int dev = 0;
    cudaGetDevice(&dev);
    if (dev < 64 && !configured[dev]) {
      const int most = (int)scatter_smem_bytes(kMaxBins);
      cudaFuncSetAttribute(radix_scatter_kernel<true, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      cudaFuncSetAttribute(radix_scatter_kernel<true, true>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      cudaFuncSetAttribute(radix_scatter_kernel<false, false>, cudaFuncAttributeMaxDynamicSharedMemorySize, most);
      configured[dev] = true;
    }
  }
  const int32_t *kin = a.labels, *vin = nullptr;
  int32_t *kout = w.kA, *vout = w.vA;
  for (int pass = 0; pass < sp.npass; ++pass) {
    const int nbins = 1 << sp.bits[pass];
    const bool seg = sp.seg_tiles > 0;  // one pass, so pass == 0
    const auto hist = pass > 0 ? radix_hist_kernel<false, false> : seg ? radix_hist_kernel<true, true>
                                                                          : radix_hist_kernel<true, false>;
    launch_chained(hist, dim3(sp.T), dim3(kSortThreads), 0, s, kin, N, a.N, a.K, a.B, sp.shift[pass], nbins, sp.T, w.H,
                   ctl.status, sp.seg_tiles);
    launch_chained(scan_rows_kernel, dim3((nbins + 7) / 8), dim3(256), 0, s, w.H, sp.T, nbins, w.totals);
    const auto scatter = pass > 0 ? radix_scatter_kernel<false, false>
                                  : seg ? radix_scatter_kernel<true, true> : radix_scatter_kernel<true, false>;
    launch_chained(scatter, dim3(sp.T), dim3(kSortThreads), scatter_smem_bytes(nbins), s, kin, vin, kout, vout, N, a.N,
                   a.K, a.B, sp.shift[pass], nbins, sp.T, w.H, w.totals, ctl.status, sp.seg_tiles);
    nl += 3;
    kin = kout;
    vin = vout;
    kout = (kout == w.kA) ? w.kB : w.kA;
    vout = (vout == w.vA) ? w.vB : w.vA;
  }
  const int32_t *skeys = kin, *perm = vin;
  const int R = chunk_rows_R(Ntot);
  const int KT = (int)Ktot;
  switch (a.dt) {
    case kF32:
      a.mode == kMean ? launch_segsum<float, kMean>(a, perm, skeys, N, KT, R, w.parts, w.off, s)
                      : launch_segsum<float, kAccumulate>(a, perm, skeys, N, KT, R, w.parts, w.off, s);
      break;
    case kF16:
      a.mode == kMean ? launch_segsum<__half, kMean>(a, perm, skeys, N, KT, R, w.parts, w.off, s)
                      : launch_segsum<__half, kAccumulate>(a, perm, skeys, N, KT, R, w.parts, w.off, s);
      break;
    default:
      a.mode == kMean ? launch_segsum<__nv_bfloat16, kMean>(a, perm, skeys, N, KT, R, w.parts, w.off, s)
                      : launch_segsum<__nv_bfloat16, kAccumulate>(a, perm, skeys, N, KT, R, w.parts, w.off, s);
  }
  // one block of 32 warps per 32 clusters, at most one per SM
  long long fgrid = (Ktot + 31) / 32;
  if (fgrid > num_sms) fgrid = num_sms;
  if (a.mode == kMean)
    launch_chained(seg_finalize_kernel<kMean>, dim3((int)fgrid), dim3(1024), 0, s, w.off, (int)Ktot, a.D, R, w.parts, a.C,
                   a.counts, nullptr, nullptr);
  else
    launch_chained(seg_finalize_kernel<kAccumulate>, dim3((int)fgrid), dim3(1024), 0, s, w.off, (int)Ktot, a.D, R, w.parts,
                   nullptr, nullptr, a.acc, a.cnt);
  nl += 2;
  count_launches(nl);
  return cudaGetLastError();
}

cudaError_t launch_divide_accumulated(double *acc, long long *cnt, int Ktot, int D, float *C,
                                      int32_t *counts, cudaStream_t s) {
  const size_t total = (size_t)Ktot * D;
  long long g = (long long)((total + 255) / 256);
  if (g > 8192) g = 8192;
  if (g < 1) g = 1;
  launch_chained(divide_acc_kernel, dim3((int)g), dim3(256), 0, s, acc, cnt, Ktot, D, C, counts);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk
