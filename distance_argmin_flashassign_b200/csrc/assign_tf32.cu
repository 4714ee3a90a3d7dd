// assign_tf32.cu -- fp32 assignment stage on the tcgen05 tensor cores.
//
// FlashAssign (Flash-KMeans, abstract) fuses the distance computation with
// the arg-min; for fp32 inputs the contraction <x, c> runs here as three tf32
// passes (the split-precision method of Ootomo and Yokota, 2022): every
// value v is split into hi = v rounded to tf32 (round to nearest, ties away)
// and lo = v - hi (exact in fp32), and
//     <x, c> ~ <x_hi, c_hi> + <x_hi, c_lo> + <x_lo, c_hi>,
// dropping <x_lo, c_lo> (below 2^-22 |x_j c_j| per term) and the bits of
// the lo parts beyond tf32 (below 2^-21 |x_j c_j| each).  As on the 16-bit
// path, the accumulator starts at -|c|^2/2 (three tf32-exact terms of the
// fp32 value, written by one tf32 MMA step against a block of ones), the
// epilogue keeps the running arg-max of s = <x, c> - |c|^2/2, and points
// whose best and runner-up scores lie within the error of this evaluation
// are listed for the exact fp64 re-decision (refine.cu), so the labels are
// those of the plain definition.
//
// Structure: one CTA per SM, 6 warps.  Warp 4 streams, for each (128-row
// unit, 128-centroid tile, 32-dimension k-block), the k-blocks of x_hi, x_lo,
// c_hi and c_lo (128 rows x 128 bytes each, 128-byte swizzle) and, with the
// first k-block, the tile's bias terms, into a ring of three 68 KB slots.
// One thread of warp 5 issues the MMAs (M = 128, N = 128, K = 8 per
// instruction; three per 32-byte step) into two 128-column TMEM accumulators
// that alternate over tiles.  Warps 0-3 (one point per thread, TMEM lane =
// row) fold each tile's four 32-column chunks into the running arg-max
// (tc_argmin.cuh) and write the label at the end of the unit.  Every wait is
// bounded (DevCtl).
#include <cuda.h>
#include <cudaTypedefs.h>

#include <mutex>

#include "fk_internal.h"
#include "tc_argmin.cuh"

namespace fk {

constexpr int kF32Rows = 128;                 // points per unit (MMA M)
constexpr int kF32TileN = 128;                // centroids per tile (MMA N)
constexpr int kF32Blk = 32;                   // fp32 elements per 128-byte k-block
constexpr int kF32Box = 128 * 128;            // one operand k-block, 16 KB
constexpr int kF32BiasBytes = kF32TileN * 32;  // bias terms of a tile, 4 KB
constexpr int kF32Slot = 4 * kF32Box + kF32BiasBytes;  // x_hi, x_lo, c_hi, c_lo, bias
constexpr int kF32Slots = 3;
constexpr int kF32EpiWarps = 4;
constexpr int kF32ProdWarp = 4, kF32MmaWarp = 5;
constexpr int kF32Threads = 32 * 6;
constexpr uint32_t kF32TmemCols = 256;        // two 128-column accumulators
constexpr int kF32Bars = 2 * kF32Slots + 4 + 1;
constexpr int kF32Used = kF32Slots * kF32Slot + 256 + kF32Bars * 8 + 16;
static_assert(kF32Slot % 1024 == 0, "slots keep the 1 KB alignment of the 128-byte swizzle");
static_assert(kF32Used + 1024 <= 232448, "shared memory (227 KB per CTA) exceeded");

struct F32Params {
  int N, K, nkb, ntiles, nunits;
  const float *xnorm;
  int32_t *labels;
  float *mindist;
  NearTies ties;
  uint32_t idesc;
  uint32_t dyn_bytes;
  DevCtl ctl;
};

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, tf32 inputs (fp32 storage, the
// low 13 mantissa bits unused), fp32 accumulate.
__device__ __forceinline__ void tc_mma_tf32(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                            uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

__device__ __forceinline__ uint64_t f32_desc_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
__device__ __forceinline__ uint64_t f32_desc_sw32(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(256 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}
__device__ __forceinline__ uint64_t f32_desc_ones(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)1 << 46);
}

__global__ void __launch_bounds__(kF32Threads, 1)
    assign_tf32_kernel(const __grid_constant__ CUtensorMap xhmap, const __grid_constant__ CUtensorMap xlmap,
                       const __grid_constant__ CUtensorMap chmap, const __grid_constant__ CUtensorMap clmap,
                       const __grid_constant__ CUtensorMap bmap, const F32Params p) {
  extern __shared__ __align__(1024) uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  if (pad + (uint32_t)kF32Used > p.dyn_bytes) {
    if (threadIdx.x == 0) record_status(p.ctl.status, -3);
    return;
  }
  uint8_t *sm = smem_raw + pad;
  const uint32_t s0 = raw + pad;
  float *ones = reinterpret_cast<float *>(sm + kF32Slots * kF32Slot);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + kF32Slots * kF32Slot + 256);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + kF32Bars);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);
  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (kF32Slots + s); };
  auto accfull = [&](int a) { return bar0 + 8u * (2 * kF32Slots + a); };
  auto accempty = [&](int a) { return bar0 + 8u * (2 * kF32Slots + 2 + a); };
  const uint32_t drain = bar0 + 8u * (2 * kF32Slots + 4);
  auto slot = [&](int s) { return s0 + (uint32_t)(s * kF32Slot); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kF32Slots; ++s) {
      mbar_init(full(s), 1);   // the producer's expect_tx
      mbar_init(empty(s), 1);  // the MMA commit once the slot's MMAs are done
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(accfull(a), 1);              // the MMA commit
      mbar_init(accempty(a), kF32EpiWarps);  // every epilogue warp
    }
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kF32ProdWarp && lane == 0) {
    tma_prefetch_desc(&xhmap);
    tma_prefetch_desc(&xlmap);
    tma_prefetch_desc(&chmap);
    tma_prefetch_desc(&clmap);
    tma_prefetch_desc(&bmap);
  }
  // the A operand of the bias step: 8 rows of (1, 1, 1, 0 | 0, 0, 0, 0) as
  // two no-swizzle core matrices
  if (threadIdx.x < 64) ones[threadIdx.x] = (threadIdx.x < 32 && (threadIdx.x & 3) < 3) ? 1.f : 0.f;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
  if (warp == kF32MmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kF32TmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kF32ProdWarp) {
    if (lane == 0) {
      // the split kernels that wrote the operands may still be draining
      asm volatile("griddepcontrol.wait;" ::: "memory");
      int st = 0;
      uint32_t sph = 0;
      bool ok = true, issued = false;
      for (int u = blockIdx.x; ok && u < p.nunits; u += gridDim.x) {
        for (int j = 0; ok && j < p.ntiles; ++j) {
          for (int kb = 0; kb < p.nkb; ++kb) {
            if (!(ok = mbar_wait(empty(st), sph ^ 1u, abort_flag, p.ctl))) break;
            const uint32_t sl = slot(st);
            mbar_arrive_expect_tx(full(st), 4 * kF32Box + (kb == 0 ? kF32BiasBytes : 0));
            tma_load_3d(sl, &xhmap, full(st), kb * kF32Blk, u * kF32Rows, 0);
            tma_load_3d(sl + kF32Box, &xlmap, full(st), kb * kF32Blk, u * kF32Rows, 0);
            tma_load_3d(sl + 2 * kF32Box, &chmap, full(st), kb * kF32Blk, j * kF32TileN, 0);
            tma_load_3d(sl + 3 * kF32Box, &clmap, full(st), kb * kF32Blk, j * kF32TileN, 0);
            if (kb == 0) tma_load_3d(sl + 4 * kF32Box, &bmap, full(st), 0, j * kF32TileN, 0);
            issued = true;
            if (++st == kF32Slots) {
              st = 0;
              sph ^= 1u;
            }
          }
        }
      }
      if (!ok && issued) {  // let copies already issued land before the CTA can exit
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 50000ull) {
        }
      }
    }
  } else if (warp == kF32MmaWarp) {
    if (lane == 0) {
      const uint64_t ones_desc = f32_desc_ones(smem_u32(ones));
      int st = 0, t = 0;
      uint32_t sph = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.nunits; u += gridDim.x) {
        for (int j = 0; ok && j < p.ntiles; ++j, ++t) {
          const int a = t & 1;
          if (!(ok = mbar_wait(accempty(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
          tc_fence_after();
          const uint32_t acc = tbase + (uint32_t)(a * kF32TileN);
          for (int kb = 0; kb < p.nkb; ++kb) {
            if (!(ok = mbar_wait(full(st), sph, abort_flag, p.ctl))) break;
            tc_fence_after();
            const uint32_t sl = slot(st);
            // accumulator = -|c|^2/2 (overwrites), then the three products
            if (kb == 0) tc_mma_tf32(acc, ones_desc, f32_desc_sw32(sl + 4 * kF32Box), p.idesc, 0u);
            const uint64_t xh = f32_desc_sw128(sl), xl = f32_desc_sw128(sl + kF32Box);
            const uint64_t ch = f32_desc_sw128(sl + 2 * kF32Box), cl = f32_desc_sw128(sl + 3 * kF32Box);
#pragma unroll
            for (int k = 0; k < 4; ++k) {  // 32-byte steps: start address + 2 (16-byte units)
              tc_mma_tf32(acc, xh + 2 * k, ch + 2 * k, p.idesc, 1u);
              tc_mma_tf32(acc, xh + 2 * k, cl + 2 * k, p.idesc, 1u);
              tc_mma_tf32(acc, xl + 2 * k, ch + 2 * k, p.idesc, 1u);
            }
            tc_commit(empty(st));  // the slot is free once these MMAs complete
            if (++st == kF32Slots) {
              st = 0;
              sph ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit(accfull(a));
        }
      }
      // every MMA issued completes before TMEM is released
      tc_commit(drain);
      mbar_wait_for(drain, 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------ epilogue ----
    const int r = warp * 32 + lane;  // row within the unit == TMEM lane
    const uint32_t t_row = tbase + ((uint32_t)(warp * 32) << 16);
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {  // both accumulators start out free
      mbar_arrive(accempty(0));
      mbar_arrive(accempty(1));
    }
    int t = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.nunits; u += gridDim.x) {
      const int row = u * kF32Rows + r;
      const bool valid = row < p.N;
      const float xn = valid ? __ldg(p.xnorm + row) : 0.f;
      const int ex = (p.ties.excl != nullptr && valid) ? p.ties.excl[row] : -1;  // left out (top-2), or -1
      Best bs;
      best_init(bs);
      auto fold = [&](uint32_t (&v)[32], int col) {
        mask_col(v, ex - col);
        fold_chunk(bs, v, col);
      };
      for (int j = 0; j < p.ntiles; ++j, ++t) {
        const int a = t & 1;
        if (!(ok = mbar_wait(accfull(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
        tc_fence_after();
        const uint32_t ta = t_row + (uint32_t)(a * kF32TileN);
        uint32_t va[32], vb[32];
        FK_TMEM_LD32(ta, va);
        FK_TMEM_LD32(ta + 32, vb);
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_WAIT_LD(vb);
        fold(va, j * kF32TileN);
        fold(vb, j * kF32TileN + 32);
        FK_TMEM_LD32(ta + 64, va);
        FK_TMEM_LD32(ta + 96, vb);
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_WAIT_LD(vb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(accempty(a));
        fold(va, j * kF32TileN + 64);
        fold(vb, j * kF32TileN + 96);
      }
      if (!ok) break;
      const int jm = best_pos(bs);
      const int bi = jm < 32 ? bs.base + jm : 0;
      const float s2 = fmaxf(bs.s2, second_in_chunk(bs, jm));
      if (valid) {
        p.labels[row] = bi;
        if (p.mindist) p.mindist[row] = fmaxf(0.f, fmaf(-2.f, bs.score, xn));
      }
      list_near_tie(p.ties, valid, bs.score, s2, bs.s3, xn, (size_t)row, bs.base2);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kF32MmaWarp) {
    tc_fence_after();
    tmem_dealloc(tbase, kF32TmemCols);
  }
}

// hi = v rounded to tf32 (nearest, ties away), lo = v - hi; norm[r] = |row|^2
// (fp32) when norm is not null.  One warp per row.
__global__ void __launch_bounds__(256) tf32_split_kernel(const float *__restrict__ V, long long rows, int D,
                                                         float *__restrict__ hi, float *__restrict__ lo,
                                                         float *__restrict__ norm) {
  const long long w = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  for (long long r = w; r < rows; r += ((long long)gridDim.x * blockDim.x) >> 5) {
    const float *v = V + r * D;
    float s = 0.f;
    for (int j = lane; j < D; j += 32) {
      const float x = v[j];
      uint32_t h;
      asm("cvt.rna.tf32.f32 %0, %1;" : "=r"(h) : "f"(x));
      const float hf = __uint_as_float(h);
      hi[r * D + j] = hf;
      lo[r * D + j] = x - hf;
      s = fmaf(x, x, s);
    }
    if (norm) {
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
      if (lane == 0) norm[r] = s;
    }
  }
}

static PFN_cuTensorMapEncodeTiled_v12000 f32_encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    cudaDriverEntryPointQueryResult q;
    void *f = nullptr;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

// rows x D fp32, loaded as 32-element (128-byte) x 128-row boxes, 128-byte swizzle
static bool f32_encode(CUtensorMap *m, const float *ptr, int D, int rows) {
  auto fn = f32_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, 1};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 4, (cuuint64_t)D * 4 * (cuuint64_t)rows};
  const cuuint32_t box[3] = {(cuuint32_t)kF32Blk, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(ptr), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// the prepared bias (Kpad rows of kBiasTerms fp32), 128 rows at a time, 32-byte swizzle
static bool f32_encode_bias(CUtensorMap *m, const float *bias, int Kpad) {
  auto fn = f32_encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kBiasTerms, (cuuint64_t)Kpad, 1};
  const cuuint64_t strides[2] = {(cuuint64_t)kBiasTerms * 4, (cuuint64_t)kBiasTerms * 4 * (cuuint64_t)Kpad};
  const cuuint32_t box[3] = {(cuuint32_t)kBiasTerms, 128, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(bias), dims, strides, box, estr,
            CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool tf32_shape_ok(int D) { return D % 4 == 0 && D >= 4 && D <= kMaxD; }

size_t tf32_workspace_bytes(int64_t N, int D, int K) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  return 2 * al((size_t)N * D * 4) + al((size_t)N * 4) + 2 * al((size_t)K * D * 4);
}

cudaError_t launch_tf32_split_points(const float *X, int N, int D, void *ws, cudaStream_t s) {
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  char *w = (char *)ws;
  float *xh = (float *)w; w += al((size_t)N * D * 4);
  float *xl = (float *)w; w += al((size_t)N * D * 4);
  float *xn = (float *)w;
  long long g = ((long long)N * 32 + 255) / 256;
  g = g < 4096 ? (g > 0 ? g : 1) : 4096;
  tf32_split_kernel<<<(int)g, 256, 0, s>>>(X, N, D, xh, xl, xn);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_assign_tf32(const float *X, const float *C, const float *bias, int N, int D, int K, int Kpad,
                               int32_t *labels, float *mindist, NearTies ties, void *ws, DevCtl ctl, int num_sms,
                               cudaStream_t s, bool x_split) {
  if (!tf32_shape_ok(D) || (uintptr_t)bias % 16 != 0) return cudaErrorNotSupported;
  if (Kpad < (K + kF32TileN - 1) / kF32TileN * kF32TileN) return cudaErrorInvalidValue;
  auto al = [](size_t v) { return (v + 255) / 256 * 256; };
  char *w = (char *)ws;
  float *xh = (float *)w; w += al((size_t)N * D * 4);
  float *xl = (float *)w; w += al((size_t)N * D * 4);
  float *xn = (float *)w; w += al((size_t)N * 4);
  float *ch = (float *)w; w += al((size_t)K * D * 4);
  float *cl = (float *)w;
  auto grid_for = [&](long long rows) {
    long long g = (rows * 32 + 255) / 256;
    return (int)(g < 4096 ? (g > 0 ? g : 1) : 4096);
  };
  if (!x_split) {  // (a Lloyd run splits X once: the points do not change)
    tf32_split_kernel<<<grid_for(N), 256, 0, s>>>(X, N, D, xh, xl, xn);
    count_launches(1);
  }
  tf32_split_kernel<<<grid_for(K), 256, 0, s>>>(C, K, D, ch, cl, nullptr);
  count_launches(1);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  CUtensorMap xhm, xlm, chm, clm, bm;
  if (!f32_encode(&xhm, xh, D, N) || !f32_encode(&xlm, xl, D, N) || !f32_encode(&chm, ch, D, K) ||
      !f32_encode(&clm, cl, D, K) || !f32_encode_bias(&bm, bias, Kpad))
    return cudaErrorNotSupported;
  F32Params p{};
  p.N = N;
  p.K = K;
  p.nkb = (D + kF32Blk - 1) / kF32Blk;
  p.ntiles = (K + kF32TileN - 1) / kF32TileN;
  p.nunits = (N + kF32Rows - 1) / kF32Rows;
  p.xnorm = xn;
  p.labels = labels;
  p.mindist = mindist;
  p.ties = ties;
  p.idesc = (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(kF32TileN >> 3) << 17) | ((uint32_t)(kF32Rows >> 4) << 24);
  p.ctl = ctl;
  static int configured[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int want = kF32Used + 1024;
  const int dyn = want < optin ? want : optin;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && !configured[dev]) {
      e = cudaFuncSetAttribute(assign_tf32_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
      if (e != cudaSuccess) return e;
      configured[dev] = 1;
    }
  }
  p.dyn_bytes = (uint32_t)dyn;
  const int grid = p.nunits < num_sms ? p.nunits : num_sms;
  assign_tf32_kernel<<<grid, kF32Threads, dyn, s>>>(xhm, xlm, chm, clm, bm, p);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk
