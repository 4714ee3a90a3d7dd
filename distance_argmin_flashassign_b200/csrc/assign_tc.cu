// assign_tc.cu -- FlashAssign on Blackwell tensor cores (tcgen05 + TMA + TMEM).
//
// Flash-KMeans (arXiv 2603.09229, abstract) fuses the distance computation
// with an online argmin so that the N x K distance matrix is never
// materialised in HBM.  On sm_100a that becomes:
//
//   * one persistent CTA per SM loops over "units" of 256 points (two 128-row
//     sub-tiles, the M of one tcgen05.mma);
//   * a TMA warp loads the unit's X rows once (kept resident while every
//     centroid tile streams past) and streams 256-centroid tiles of C through
//     a ring of shared-memory stages (128-byte swizzle, one 64-element k-block
//     per stage);
//   * one thread issues tcgen05.mma (M=128, N=256, K=16, fp32 accumulate)
//     into two TMEM accumulators of 128 x 256 fp32, one per sub-tile.  Each
//     accumulator already holds the bias -|c|^2/2 of its columns when the MMA
//     starts, so it ends holding the score s = <x,c> - |c|^2/2, whose arg-max
//     is the arg-min of |x - c|^2: no per-distance arithmetic is left for the
//     epilogue but the arg-max itself;
//   * four epilogue warpgroups drain the accumulators with tcgen05.ld:
//     warpgroups 0-1 own sub-tile 0, 2-3 own sub-tile 1, and within a pair
//     one scans columns [0,128) of every tile and the other [128,256).  Each
//     thread owns one point (TMEM lane == row).  Per 32-column chunk a
//     3-input-max tree (half an ALU op per score; the ALU pipe runs at half
//     rate and bounds this epilogue) gives the chunk maximum; when it beats
//     the point's running maximum (strict ">", so an earlier column keeps a
//     tie) the lane copies the chunk into a register-resident candidate.  The
//     lowest column of the candidate holding the maximum is found once per
//     unit.  After reading a chunk the thread writes the next tile's bias
//     into the same TMEM columns (tcgen05.st), re-arming the accumulator.
//     The two column halves of a point are merged at the end of the unit
//     (score, then lower index).
//
// Only labels (and optionally |x|^2 - 2 max s) leave the chip.  X, C and the
// bias are read; nothing else is written.
//
// Every wait is an mbarrier wait bounded in time; on expiry the CTA records
// FK_ERR_TIMEOUT, drains its in-flight copies and MMAs, frees TMEM and exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "fk_internal.h"

namespace fk {

constexpr int kRowsSub = 128;              // rows per sub-tile (MMA M)
constexpr int kSubs = 2;                   // sub-tiles per unit
constexpr int kRowsUnit = kRowsSub * kSubs;
constexpr int kTileN = 256;                // centroids per tile (MMA N)
constexpr int kBlkK = 64;                  // elements per k-block (128 bytes)
constexpr int kSubBytes = kRowsSub * 128;  // one sub-tile k-block, 16 KB
constexpr int kStageBytes = kTileN * 128;  // one centroid k-block, 32 KB
constexpr int kEpiWarps = 16;                 // four epilogue warpgroups
constexpr int kAccWarps = 8;                  // warps draining one accumulator
constexpr int kProducerWarp = 16, kMmaWarp = 17;
constexpr int kThreads = 32 * 18;
constexpr uint32_t kTmemCols = 512;        // two 256-column fp32 accumulators

template <int KB> struct TcCfg {
  static constexpr int XBUF = 2;                  // X double buffer (next unit prefetch)
  static constexpr int NST = KB == 1 ? 4 : 3;     // centroid stages
  static constexpr int X_BYTES = XBUF * kSubs * KB * kSubBytes;
  static constexpr int C_BYTES = NST * kStageBytes;
  static constexpr int XCHG_BYTES = kSubs * kRowsSub * 8;
  // full/empty per stage, xfull/xempty per X buffer, accfull/accempty per
  // accumulator, xchg full/empty, drain
  static constexpr int NBAR = 2 * NST + 2 * XBUF + 4 + 2 + 1;
  static constexpr int USED = X_BYTES + C_BYTES + XCHG_BYTES + NBAR * 8 + 16;
  static_assert(NST >= KB, "a whole centroid tile must fit in the stage ring");
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// 32 consecutive bias values (uniform address across the warp, L1 cached).
__device__ __forceinline__ void load_bias32(const float *p, uint32_t (&w)[32]) {
  const float4 *p4 = reinterpret_cast<const float4 *>(p);
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const float4 t = __ldg(p4 + e);
    w[4 * e] = __float_as_uint(t.x);
    w[4 * e + 1] = __float_as_uint(t.y);
    w[4 * e + 2] = __float_as_uint(t.z);
    w[4 * e + 3] = __float_as_uint(t.w);
  }
}

struct TcParams {
  int N, K, Kpad, ntiles, upb, total_units;
  uint32_t idesc;
  int is_bf16;
  uint32_t dyn_bytes;
  const float *bias;  // -|c|^2/2 per centroid, -inf in the padding
  int32_t *labels;
  float *mindist;
  DevCtl ctl;
};

template <int KB>
__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                     const TcParams p) {
  using Cfg = TcCfg<KB>;
  constexpr int NST = Cfg::NST, XBUF = Cfg::XBUF;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  if (pad + (uint32_t)Cfg::USED > p.dyn_bytes) {  // cannot happen with a 1 KB aligned window
    if (threadIdx.x == 0) record_status(p.ctl.status, -3);
    return;
  }
  uint8_t *sm = smem_raw + pad;
  const uint32_t sX = raw + pad;
  const uint32_t sC = sX + Cfg::X_BYTES;
  float2 *xchg = reinterpret_cast<float2 *>(sm + Cfg::X_BYTES + Cfg::C_BYTES);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Cfg::X_BYTES + Cfg::C_BYTES + Cfg::XCHG_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Cfg::NBAR);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };
  auto empty = [&](int s) { return bar0 + 8u * (NST + s); };
  auto xfull = [&](int x) { return bar0 + 8u * (2 * NST + x); };
  auto xempty = [&](int x) { return bar0 + 8u * (2 * NST + XBUF + x); };
  auto accfull = [&](int g) { return bar0 + 8u * (2 * NST + 2 * XBUF + g); };
  auto accempty = [&](int g) { return bar0 + 8u * (2 * NST + 2 * XBUF + 2 + g); };
  const uint32_t xchg_full = bar0 + 8u * (2 * NST + 2 * XBUF + 4);
  const uint32_t xchg_empty = xchg_full + 8u;
  const uint32_t drain = xchg_full + 16u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    for (int x = 0; x < XBUF; ++x) {
      mbar_init(xfull(x), 1);
      mbar_init(xempty(x), 1 + kEpiWarps);  // MMA commit + every epilogue warp
    }
    for (int g = 0; g < 2; ++g) {
      mbar_init(accfull(g), 1);
      mbar_init(accempty(g), kAccWarps);
    }
    mbar_init(xchg_full, kEpiWarps);
    mbar_init(xchg_empty, kEpiWarps);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&cmap);
  }
  if (warp == kMmaWarp) {
    tmem_alloc(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer ----
      uint32_t xb = 0, xph = 0, st = 0, sph = 0;
      uint32_t st_armed = 0, st_par = 0, x_armed = 0, x_par = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        const int b = u / p.upb, r0 = (u % p.upb) * kRowsUnit;
        if (!(ok = mbar_wait(xempty(xb), xph ^ 1u, abort_flag, p.ctl))) break;
        mbar_arrive_expect_tx(xfull(xb), kSubs * KB * kSubBytes);
        for (int g = 0; g < kSubs; ++g)
          for (int kb = 0; kb < KB; ++kb)
            tma_load_3d(sX + ((xb * kSubs + g) * KB + kb) * kSubBytes, &xmap, xfull(xb), kb * kBlkK,
                        r0 + g * kRowsSub, b);
        x_armed |= 1u << xb;
        x_par = (x_par & ~(1u << xb)) | (xph << xb);
        if (++xb == XBUF) { xb = 0; xph ^= 1u; }
        for (int j = 0; ok && j < p.ntiles; ++j) {
          for (int kb = 0; kb < KB; ++kb) {
            if (!(ok = mbar_wait(empty(st), sph ^ 1u, abort_flag, p.ctl))) break;
            mbar_arrive_expect_tx(full(st), kStageBytes);
            tma_load_3d(sC + st * kStageBytes, &cmap, full(st), kb * kBlkK, j * kTileN, b);
            st_armed |= 1u << st;
            st_par = (st_par & ~(1u << st)) | (sph << st);
            if (++st == NST) { st = 0; sph ^= 1u; }
          }
        }
      }
      // No bulk copy may still be writing this CTA's shared memory at exit.
      for (int s = 0; s < NST; ++s)
        if (st_armed >> s & 1u) mbar_wait_for(full(s), st_par >> s & 1u, 200000000ull);
      for (int x = 0; x < XBUF; ++x)
        if (x_armed >> x & 1u) mbar_wait_for(xfull(x), x_par >> x & 1u, 200000000ull);
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0) {
      // ------------------------------------------------- MMA issuer -----
      uint32_t xb = 0, xph = 0, st = 0, sph = 0, ae0 = 0, ae1 = 0;
      bool ok = true;
      for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x) {
        if (!(ok = mbar_wait(xfull(xb), xph, abort_flag, p.ctl))) break;
        const uint32_t xa0 = sX + (xb * kSubs + 0) * KB * kSubBytes;
        const uint32_t xa1 = sX + (xb * kSubs + 1) * KB * kSubBytes;
        for (int j = 0; ok && j < p.ntiles; ++j) {
          uint32_t stg[KB];
          for (int kb = 0; kb < KB; ++kb) {
            stg[kb] = st;
            if (!(ok = mbar_wait(full(st), sph, abort_flag, p.ctl))) break;
            if (++st == NST) { st = 0; sph ^= 1u; }
          }
          if (!ok) break;
          tc_fence_after();
          if (!(ok = mbar_wait(accempty(0), ae0, abort_flag, p.ctl))) break;
          ae0 ^= 1u;
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = desc_kmajor_sw128(xa0 + kb * kSubBytes);
            const uint64_t bd = desc_kmajor_sw128(sC + stg[kb] * kStageBytes);
#pragma unroll
            for (int k = 0; k < kBlkK / 16; ++k)
              tc_mma_f16(tbase, ad + 2 * k, bd + 2 * k, p.idesc, 1u);
          }
          tc_commit(accfull(0));
          if (!(ok = mbar_wait(accempty(1), ae1, abort_flag, p.ctl))) break;
          ae1 ^= 1u;
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = desc_kmajor_sw128(xa1 + kb * kSubBytes);
            const uint64_t bd = desc_kmajor_sw128(sC + stg[kb] * kStageBytes);
#pragma unroll
            for (int k = 0; k < kBlkK / 16; ++k)
              tc_mma_f16(tbase + kTileN, ad + 2 * k, bd + 2 * k, p.idesc, 1u);
          }
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) tc_commit(empty(stg[kb]));
          tc_commit(accfull(1));
        }
        if (!ok) break;
        tc_commit(xempty(xb));
        if (++xb == XBUF) { xb = 0; xph ^= 1u; }
      }
      // Every MMA this thread issued completes before TMEM is released.
      tc_commit(drain);
      mbar_wait_for(drain, 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------ epilogue ----
    const int wg = warp >> 2, q = warp & 3;
    const int g = wg >> 1;     // sub-tile (accumulator) of this warpgroup
    const int h = wg & 1;      // column half of every tile
    const int r = q * 32 + lane;  // row within the sub-tile == TMEM lane
    const uint32_t t_row = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(g * kTileN + h * 128);
    const uint32_t my_full = accfull(g), my_empty = accempty(g);
    // bias of tile j of the unit u, for this warpgroup's 128 columns
    auto bias_of = [&](int u, int j) {
      return p.bias + (size_t)(u / p.upb) * p.Kpad + j * kTileN + h * 128;
    };
    // Every accumulator starts each tile holding the bias: the first tile's
    // now, every later tile's while the previous tile is drained.
    if ((int)blockIdx.x < p.total_units) {
      const float *bp = bias_of(blockIdx.x, 0);
#pragma unroll 1
      for (int c = 0; c < 4; ++c) {
        uint32_t w[32];
        load_bias32(bp + c * 32, w);
        FK_TMEM_ST32(t_row + c * 32, w);
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) mbar_arrive(my_empty);

    uint32_t xb = 0, xph = 0, af = 0, xc = 0;
    bool ok = true;
    for (int u = blockIdx.x; ok && u < p.total_units; u += gridDim.x, xc ^= 1u) {
      const int b = u / p.upb, r0 = (u % p.upb) * kRowsUnit;
      if (!(ok = mbar_wait(xfull(xb), xph, abort_flag, p.ctl))) break;
      float xn = 0.f;
      if (p.mindist && h == 0) {  // |x|^2 of row r of sub-tile g, from the swizzled tile
        for (int kb = 0; kb < KB; ++kb) {
          const uint8_t *rowp = sm + ((xb * kSubs + g) * KB + kb) * kSubBytes + r * 128;
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint4 w = *reinterpret_cast<const uint4 *>(rowp + ((c ^ (r & 7)) << 4));
            const uint32_t ws[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              float lo, hi;
              if (p.is_bf16) {
                lo = __uint_as_float(ws[e] << 16);
                hi = __uint_as_float(ws[e] & 0xffff0000u);
              } else {
                const __half2 h2 = *reinterpret_cast<const __half2 *>(&ws[e]);
                lo = __low2float(h2);
                hi = __high2float(h2);
              }
              xn = fmaf(lo, lo, xn);
              xn = fmaf(hi, hi, xn);
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xempty(xb));
      if (++xb == XBUF) { xb = 0; xph ^= 1u; }

      // score s = <x,c> - |c|^2/2 (argmax s == argmin |x-c|^2); running max and
      // the 32-column chunk that first reached it
      float cbest = __int_as_float(0xff800000);
      int cbase = 0;
      uint32_t cand[32];
#pragma unroll
      for (int t = 0; t < 32; ++t) cand[t] = 0u;
      for (int j = 0; ok && j < p.ntiles; ++j) {
        const int col0 = j * kTileN + h * 128;
        int nu = u, nj = j + 1;  // the tile this accumulator holds next
        if (nj == p.ntiles) { nu = u + gridDim.x; nj = 0; }
        const float *nbp = nu < p.total_units ? bias_of(nu, nj) : nullptr;
        if (!(ok = mbar_wait(my_full, af, abort_flag, p.ctl))) break;
        af ^= 1u;
        tc_fence_after();
#pragma unroll 1
        for (int c = 0; c < 4; ++c) {
          uint32_t v[32];
          FK_TMEM_LD32(t_row + c * 32, v);
          FK_TMEM_WAIT_LD(v);
          // chunk maximum: 3-input-max tree, depth 4
          float l1[11];
#pragma unroll
          for (int i = 0; i < 10; ++i)
            l1[i] = fmax3(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
          l1[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
          const float l2a = fmax3(l1[0], l1[1], l1[2]), l2b = fmax3(l1[3], l1[4], l1[5]);
          const float l2c = fmax3(l1[6], l1[7], l1[8]), l2d = fmaxf(l1[9], l1[10]);
          const float m = fmaxf(fmax3(l2a, l2b, l2c), l2d);
          const bool imp = m > cbest;  // strict: an earlier column keeps a tie
          if (__any_sync(0xffffffffu, imp)) {
            if (imp) {
#pragma unroll
              for (int t = 0; t < 32; ++t) cand[t] = v[t];
              cbest = m;
              cbase = col0 + c * 32;
            }
          }
          if (nbp) {  // the next tile's bias goes where this chunk was read
            load_bias32(nbp + c * 32, v);
            FK_TMEM_ST32(t_row + c * 32, v);
          }
        }
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) mbar_arrive(my_empty);
      }
      if (!ok) break;
      // lowest column of the candidate chunk holding the maximum
      int j0 = 32, j1 = 32, j2 = 32, j3 = 32;
#pragma unroll
      for (int t = 28; t >= 0; t -= 4) {
        j0 = __uint_as_float(cand[t]) == cbest ? t : j0;
        j1 = __uint_as_float(cand[t + 1]) == cbest ? t + 1 : j1;
        j2 = __uint_as_float(cand[t + 2]) == cbest ? t + 2 : j2;
        j3 = __uint_as_float(cand[t + 3]) == cbest ? t + 3 : j3;
      }
      const int jm = min(min(j0, j1), min(j2, j3));
      int bi = jm < 32 ? cbase + jm : 0;
      float sb = cbest;
      // merge the two column halves of each point: warpgroup h == 0 writes
      if (u != (int)blockIdx.x && !(ok = mbar_wait(xchg_empty, xc ^ 1u, abort_flag, p.ctl))) break;
      if (h == 1) xchg[g * kRowsSub + r] = make_float2(sb, __int_as_float(bi));
      __syncwarp();
      if (lane == 0) mbar_arrive(xchg_full);
      if (!(ok = mbar_wait(xchg_full, xc, abort_flag, p.ctl))) break;
      if (h == 0) {
        const float2 o = xchg[g * kRowsSub + r];
        const int oi = __float_as_int(o.y);
        if (o.x > sb || (o.x == sb && oi < bi)) { sb = o.x; bi = oi; }
        const int row = r0 + g * kRowsSub + r;
        if (row < p.N) {
          const size_t o_ = (size_t)b * p.N + row;
          p.labels[o_] = bi;
          if (p.mindist) p.mindist[o_] = fmaxf(0.f, fmaf(-2.f, sb, xn));
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(xchg_empty);
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc(tbase, kTmemCols);
  }
}

// ------------------------------------------------------------------ host --
static PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
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

static bool encode_3d(CUtensorMap *m, DType dt, const void *ptr, int D, int rows, int B, int box_rows) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)D, (cuuint64_t)rows, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)D * 2, (cuuint64_t)D * 2 * (cuuint64_t)rows};
  const cuuint32_t box[3] = {(cuuint32_t)kBlkK, (cuuint32_t)box_rows, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, dt == kF16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3,
                  const_cast<void *>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                  CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_shape_ok(DType dt, int D) { return dt != kF32 && D % 8 == 0 && D >= 8 && D <= 128; }

bool tc_aligned(const void *X, const void *C) {
  return ((uintptr_t)X % 16 == 0) && ((uintptr_t)C % 16 == 0);
}

template <int KB>
static cudaError_t launch_kb(const CUtensorMap &xm, const CUtensorMap &cm, TcParams p, int num_sms,
                             cudaStream_t s) {
  static int configured_dev = -1;
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int want = TcCfg<KB>::USED + 1024;
  const int dyn = want < optin ? want : optin;
  {
    std::lock_guard<std::mutex> g(mu);
    if (configured_dev != dev) {
      cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel<KB>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
      if (e != cudaSuccess) return e;
      configured_dev = dev;
    }
  }
  p.dyn_bytes = (uint32_t)dyn;
  const int grid = p.total_units < num_sms ? p.total_units : num_sms;
  assign_tc_kernel<KB><<<grid, kThreads, dyn, s>>>(xm, cm, p);
  count_launches(1);
  return cudaGetLastError();
}

cudaError_t launch_assign_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N,
                             int D, int K, int Kpad, int32_t *labels, float *mindist, DevCtl ctl,
                             int num_sms, cudaStream_t s) {
  if (!tc_shape_ok(dt, D) || !tc_aligned(X, C)) return cudaErrorNotSupported;
  CUtensorMap xm, cm;
  if (!encode_3d(&xm, dt, X, D, N, B, kRowsSub) || !encode_3d(&cm, dt, C, D, K, B, kTileN))
    return cudaErrorNotSupported;
  TcParams p;
  p.N = N;
  p.K = K;
  p.Kpad = Kpad;
  p.ntiles = (K + kTileN - 1) / kTileN;
  p.upb = (N + kRowsUnit - 1) / kRowsUnit;
  p.total_units = p.upb * B;
  p.idesc = idesc_f16(dt == kBF16 ? 1 : 0, kRowsSub, kTileN);
  p.is_bf16 = dt == kBF16;
  p.bias = bias;
  p.labels = labels;
  p.mindist = mindist;
  p.ctl = ctl;
  p.dyn_bytes = 0;
  if (p.total_units == 0) return cudaSuccess;
  const int KB = (D + kBlkK - 1) / kBlkK;
  if (KB == 1) return launch_kb<1>(xm, cm, p, num_sms, s);
  return launch_kb<2>(xm, cm, p, num_sms, s);
}

}  // namespace fk
