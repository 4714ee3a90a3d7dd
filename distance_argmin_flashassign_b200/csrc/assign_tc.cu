// assign_tc.cu -- FlashAssign on Blackwell tensor cores (tcgen05 + TMA + TMEM),
// run by pairs of CTAs (cta_group::2).
//
// Flash-KMeans (arXiv 2603.09229, abstract) fuses the distance computation
// with an online argmin so that the N x K distance matrix is never
// materialised in HBM.  On sm_100a that becomes:
//
//   * clusters of two CTAs (one per SM) loop over "units" of 256 points; the
//     leader CTA owns rows [0,128) of a unit, the peer rows [128,256);
//   * in each CTA a TMA warp loads its 128 rows of X once per unit (kept
//     resident while every centroid tile streams past) and its half of every
//     256-centroid tile (128 centroids) through a ring of 16 KB stages
//     (128-byte swizzle, one 64-element k-block per stage);
//   * one thread of the leader issues tcgen05.mma with cta_group::2
//     (M = 256 across the pair, N = 256, K = 16, fp32 accumulate); each CTA's
//     TMEM receives its 128 rows x 256 columns.  Two such accumulators (all
//     512 TMEM columns) alternate over the tiles, and a tile ends with one
//     tcgen05.commit that reaches both CTAs.  There is no other commit: the
//     epilogue frees a tile's centroid stages once it has seen the tile
//     complete, and a unit's X buffer once it is done with the unit;
//   * every accumulator already holds the bias -|c|^2/2 of its columns when
//     the MMA starts, so it ends holding the score s = <x,c> - |c|^2/2, whose
//     arg-max is the arg-min of |x - c|^2;
//   * eight epilogue warps per CTA: warp (h, q) owns TMEM lanes [32q, 32q+32)
//     (one point per thread) and columns [128h, 128h+128) of every tile, read
//     as four 32-column chunks with the next chunk's tcgen05.ld in flight
//     while the current one is reduced.  A 3-input-max tree gives the chunk
//     maximum; when it beats the point's running maximum (strict ">", so an
//     earlier column keeps a tie) the lane copies the chunk into a
//     register-resident candidate.  Right after reading a chunk the thread
//     writes the bias of the tile that uses this accumulator next into the
//     same columns (tcgen05.st).  The lowest column of the candidate holding
//     the maximum is found once per unit, and the two column halves of a
//     point are merged at the end of the unit (score, then lower index),
//     together with |x|^2 for the returned squared distance;
//   * an accumulator goes back to the MMA thread when all 16 epilogue warps
//     of the pair have drained and re-armed it.  The peer's warps signal the
//     leader's barrier with a relaxed cluster-scope arrive, after
//     tcgen05.wait::ld / wait::st and tcgen05.fence::before_thread_sync: a
//     release at cluster scope would cost more than a third of a tile, and
//     those TMEM accesses are already complete when the arrive is issued.
//
// Only labels (and optionally |x|^2 - 2 max s) leave the chip.  X, C and the
// bias are read; nothing else is written.
//
// Every wait is an mbarrier wait bounded in time; on expiry the CTA records
// FK_ERR_TIMEOUT, lets its in-flight copies and MMAs finish (bounded), frees
// TMEM and exits.
#include <cudaTypedefs.h>

#include <mutex>

#include "fk_internal.h"

namespace fk {

constexpr int kRows = 128;                  // rows per CTA per unit
constexpr int kRowsUnit = 2 * kRows;        // rows per pair unit (MMA M)
constexpr int kTileN = 256;                 // centroids per tile (MMA N)
constexpr int kHalfN = kTileN / 2;          // centroids per CTA per tile
constexpr int kBlkK = 64;                   // elements per k-block (128 bytes)
constexpr int kXBytes = kRows * 128;        // one X k-block, 16 KB
constexpr int kStageBytes = kHalfN * 128;   // one centroid half k-block, 16 KB
constexpr int kAcc = 2;                     // accumulators
constexpr int kEpiWarps = 8;                // column half x lane quarter
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1;
constexpr int kThreads = 32 * (kEpiWarps + 2);
constexpr uint32_t kTmemCols = 512;         // two 256-column fp32 accumulators
constexpr uint16_t kBothCtas = 0x3;
static_assert(kAcc * kTileN <= (int)kTmemCols, "accumulators exceed TMEM");
static_assert(kTileN == kCentroidPad, "the bias is padded to whole tiles");

template <int KB> struct TcCfg {
  static constexpr int XBUF = 2;                 // X double buffer (next unit prefetch)
  static constexpr int NST = KB == 1 ? 11 : 9;   // centroid stages (16 KB)
  static constexpr int X_BYTES = XBUF * KB * kXBytes;
  static constexpr int C_BYTES = NST * kStageBytes;
  static constexpr int XCHG_BYTES = kRows * 16;  // one float4 per row
  // full/empty per stage, xfull/xempty per X buffer, accfull/accempty per
  // accumulator, xchg full/empty, drain
  static constexpr int NBAR = 2 * NST + 2 * XBUF + 2 * kAcc + 2 + 1;
  static constexpr int USED = X_BYTES + C_BYTES + XCHG_BYTES + NBAR * 8 + 16;
  static_assert(NST >= KB, "a whole centroid tile must fit in the stage ring");
  static_assert(USED + 1024 <= 232448, "shared memory (227 KB per CTA on sm_100) exceeded");
};

__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float r;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(r) : "f"(a), "f"(b), "f"(c));
  return r;
}

// Maximum of 32 scores: a 3-input-max tree of depth 4.
__device__ __forceinline__ float max32(const uint32_t (&v)[32]) {
  float l1[11];
#pragma unroll
  for (int i = 0; i < 10; ++i)
    l1[i] = fmax3(__uint_as_float(v[3 * i]), __uint_as_float(v[3 * i + 1]), __uint_as_float(v[3 * i + 2]));
  l1[10] = fmaxf(__uint_as_float(v[30]), __uint_as_float(v[31]));
  const float l2a = fmax3(l1[0], l1[1], l1[2]), l2b = fmax3(l1[3], l1[4], l1[5]);
  const float l2c = fmax3(l1[6], l1[7], l1[8]), l2d = fmaxf(l1[9], l1[10]);
  return fmaxf(fmax3(l2a, l2b, l2c), l2d);
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

// Running arg-max of one point over the chunks it has seen, in column order.
struct Best {
  float score;
  int base;           // first column of the candidate chunk
  uint32_t cand[32];  // the chunk that first reached `score`
};

// Fold one 32-column chunk (first column `col`) into the running arg-max.
// The candidate copy is written as x + 0 (add.rn.f32), which runs on the
// full-rate FMA pipe instead of the half-rate integer/logic pipe that the
// max tree already saturates; it keeps every value but turns -0 into +0,
// which compares equal, so the index search below finds the same column.
__device__ __forceinline__ void fold_chunk(Best &bs, const uint32_t (&v)[32], int col) {
  const float m = max32(v);
  const bool imp = m > bs.score;  // strict: an earlier column keeps a tie
  if (__any_sync(0xffffffffu, imp)) {
    if (imp) {
#pragma unroll
      for (int i = 0; i < 32; ++i) bs.cand[i] = __float_as_uint(__fadd_rn(__uint_as_float(v[i]), 0.f));
      bs.score = m;
      bs.base = col;
    }
  }
}

template <int KB>
__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                     const TcParams p) {
  using Cfg = TcCfg<KB>;
  constexpr int NST = Cfg::NST, XBUF = Cfg::XBUF;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t pad = (1024u - (raw & 1023u)) & 1023u;
  // Both CTAs of a pair see the same layout (same kernel, same dynamic size),
  // so either both fail this check or neither does.
  if (pad + (uint32_t)Cfg::USED > p.dyn_bytes) {
    if (threadIdx.x == 0) record_status(p.ctl.status, -3);
    return;
  }
  uint8_t *sm = smem_raw + pad;
  const uint32_t sX = raw + pad;
  const uint32_t sC = sX + Cfg::X_BYTES;
  float4 *xchg = reinterpret_cast<float4 *>(sm + Cfg::X_BYTES + Cfg::C_BYTES);
  uint64_t *bars = reinterpret_cast<uint64_t *>(sm + Cfg::X_BYTES + Cfg::C_BYTES + Cfg::XCHG_BYTES);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Cfg::NBAR);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };                                   // leader's
  auto empty = [&](int s) { return bar0 + 8u * (NST + s); };                          // each CTA
  auto xfull = [&](int x) { return bar0 + 8u * (2 * NST + x); };                      // leader's
  auto xempty = [&](int x) { return bar0 + 8u * (2 * NST + XBUF + x); };              // each CTA
  auto accfull = [&](int a) { return bar0 + 8u * (2 * NST + 2 * XBUF + a); };         // each CTA
  auto accempty = [&](int a) { return bar0 + 8u * (2 * NST + 2 * XBUF + kAcc + a); };  // leader's
  const uint32_t xchg_full = bar0 + 8u * (2 * NST + 2 * XBUF + 2 * kAcc);
  const uint32_t xchg_empty = xchg_full + 8u;
  const uint32_t drain = xchg_full + 16u;

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full(s), 1);   // the leader's expect_tx; bytes from both CTAs
      mbar_init(empty(s), 1);  // the epilogue, once the tile using the stage is complete
    }
    for (int x = 0; x < XBUF; ++x) {
      mbar_init(xfull(x), 1);
      mbar_init(xempty(x), kEpiWarps);  // this CTA's epilogue warps, after the unit
    }
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(accfull(a), 1);               // the MMA commit
      mbar_init(accempty(a), 2 * kEpiWarps);  // every epilogue warp of both CTAs
    }
    mbar_init(xchg_full, kEpiWarps / 2);   // the column-half-1 warps
    mbar_init(xchg_empty, kEpiWarps / 2);  // the column-half-0 warps
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == kProducerWarp && lane == 0) {
    tma_prefetch_desc(&xmap);
    tma_prefetch_desc(&cmap);
  }
  if (warp == kMmaWarp) {
    tmem_alloc_pair(smem_u32(tmem_slot), kTmemCols);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // every barrier of both CTAs exists before either signals the other
  tc_fence_after();
  const uint32_t tbase = *tmem_slot;

  if (warp == kProducerWarp) {
    if (lane == 0) {
      // ------------------------------------------------ TMA producer ----
      uint32_t xb = 0, xph = 0, st = 0, sph = 0;
      bool ok = true, issued = false;
      for (int u = pair; ok && u < p.total_units; u += npairs) {
        const int b = u / p.upb, r0 = (u % p.upb) * kRowsUnit + (int)rank * kRows;
        if (!(ok = mbar_wait(xempty(xb), xph ^ 1u, abort_flag, p.ctl))) break;
        if (leader) mbar_arrive_expect_tx(xfull(xb), 2 * KB * kXBytes);
        const uint32_t xbar = map_to_cta(xfull(xb), 0);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_3d_pair(sX + (xb * KB + kb) * kXBytes, &xmap, xbar, kb * kBlkK, r0, b);
        issued = true;
        if (++xb == XBUF) { xb = 0; xph ^= 1u; }
        for (int j = 0; ok && j < p.ntiles; ++j) {
          for (int kb = 0; kb < KB; ++kb) {
            if (!(ok = mbar_wait(empty(st), sph ^ 1u, abort_flag, p.ctl))) break;
            if (leader) mbar_arrive_expect_tx(full(st), 2 * kStageBytes);
            tma_load_3d_pair(sC + st * kStageBytes, &cmap, map_to_cta(full(st), 0), kb * kBlkK,
                             j * kTileN + (int)rank * kHalfN, b);
            if (++st == NST) { st = 0; sph ^= 1u; }
          }
        }
      }
      // After an abort, give copies already issued time to land in this CTA's
      // shared memory before it can exit (their barrier may be in the peer).
      if (!ok && issued) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 50000ull) {
        }
      }
    }
  } else if (warp == kMmaWarp) {
    if (lane == 0 && leader) {
      // ------------------------------------------------- MMA issuer -----
      uint32_t xb = 0, xph = 0, st = 0, sph = 0;
      int t = 0;  // tile counter: accumulator t % 2, its (t / 2)-th use
      bool ok = true;
      for (int u = pair; ok && u < p.total_units; u += npairs) {
        if (!(ok = mbar_wait(xfull(xb), xph, abort_flag, p.ctl))) break;
        const uint32_t xa = sX + xb * KB * kXBytes;
        for (int j = 0; ok && j < p.ntiles; ++j, ++t) {
          uint32_t stg[KB];
          for (int kb = 0; kb < KB; ++kb) {
            stg[kb] = st;
            if (!(ok = mbar_wait(full(st), sph, abort_flag, p.ctl))) break;
            if (++st == NST) { st = 0; sph ^= 1u; }
          }
          if (!ok) break;
          const int a = t & 1;
          // the accumulator was drained and re-armed with this tile's bias
          if (!(ok = mbar_wait(accempty(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
          tc_fence_after();
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = desc_kmajor_sw128(xa + kb * kXBytes);
            const uint64_t bd = desc_kmajor_sw128(sC + stg[kb] * kStageBytes);
#pragma unroll
            for (int k = 0; k < kBlkK / 16; ++k)
              tc_mma_f16_pair(tbase + a * kTileN, ad + 2 * k, bd + 2 * k, p.idesc, 1u);
          }
          tc_commit_pair(accfull(a), kBothCtas);
        }
        if (!ok) break;
        if (++xb == XBUF) { xb = 0; xph ^= 1u; }
      }
      // Every MMA this thread issued completes before TMEM is released (all
      // tcgen05 operations of this kernel use the pair form, this one too).
      tc_commit_pair(drain, 0x1);
      mbar_wait_for(drain, 0, 200000000ull);
    }
  } else {
    // ------------------------------------------------------ epilogue ----
    const int h = warp >> 2, q = warp & 3;  // column half, lane quarter
    const int r = q * 32 + lane;            // row within this CTA's 128 == TMEM lane
    const uint32_t t_row = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(h * kHalfN);
    // hand an accumulator back to the leader's MMA thread
    auto release_acc = [&](int a) {
      if (leader) mbar_arrive(accempty(a));
      else mbar_arrive_cluster_relaxed(map_to_cta(accempty(a), 0));
    };
    // Walks the pair's tiles in order and yields the bias of this warp's 128
    // columns of each (null past the last unit).
    struct BiasIter {
      const float *row;  // bias of the current unit's problem, this warp's half
      int u, j;
    } bi_ = {nullptr, pair, 0};
    auto bias_row = [&](int u) { return p.bias + (size_t)(u / p.upb) * p.Kpad + h * kHalfN; };
    bi_.row = bias_row(pair);
    auto next_bias = [&]() -> const float * {
      const float *r = bi_.u < p.total_units ? bi_.row + bi_.j * kTileN : nullptr;
      if (++bi_.j == p.ntiles) {
        bi_.j = 0;
        bi_.u += npairs;
        if (bi_.u < p.total_units) bi_.row = bias_row(bi_.u);
      }
      return r;
    };
    // Arm both accumulators with the bias of tiles 0 and 1.
#pragma unroll 1
    for (int a = 0; a < kAcc; ++a) {
      if (const float *bp = next_bias()) {
#pragma unroll 1
        for (int c = 0; c < kHalfN / 32; ++c) {
          uint32_t w[32];
          load_bias32(bp + c * 32, w);
          FK_TMEM_ST32(t_row + a * kTileN + c * 32, w);
        }
      }
    }
    tmem_wait_st();
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      release_acc(0);
      release_acc(1);
    }

    uint32_t xb = 0, xc = 0;
    int t = 0;  // the pair's tile counter
    bool ok = true;
    for (int u = pair; ok && u < p.total_units; u += npairs, xc ^= 1u) {
      const int b = u / p.upb;
      const int row = (u % p.upb) * kRowsUnit + (int)rank * kRows + r;
      Best bs;
      bs.score = __int_as_float(0xff800000);
      bs.base = 0;
#pragma unroll
      for (int i = 0; i < 32; ++i) bs.cand[i] = 0u;
      for (int j = 0; ok && j < p.ntiles; ++j, ++t) {
        const int a = t & 1;
        const float *nbp = next_bias();  // tile t + 2: the next one for this accumulator
        if (!(ok = mbar_wait(accfull(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
        tc_fence_after();
        if (h == 0 && q == 0 && lane == 0) {  // the MMA has consumed this tile's centroid stages
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) mbar_arrive(empty((t * KB + kb) % NST));
        }
        const uint32_t ta = t_row + a * kTileN;
        const int col = j * kTileN + h * kHalfN;
        uint32_t va[32], vb[32], w[32];
        if (nbp) load_bias32(nbp, w);
        FK_TMEM_LD32(ta, va);
        FK_TMEM_WAIT_LD(va);
        // chunk c is reduced while chunk c + 1 is on its way from TMEM; the
        // next tile's bias goes where chunk c was read
        FK_TMEM_LD32(ta + 32, vb);
        fold_chunk(bs, va, col);
        if (nbp) {
          FK_TMEM_ST32(ta, w);
          load_bias32(nbp + 32, w);
        }
        FK_TMEM_WAIT_LD(vb);
        FK_TMEM_LD32(ta + 64, va);
        fold_chunk(bs, vb, col + 32);
        if (nbp) {
          FK_TMEM_ST32(ta + 32, w);
          load_bias32(nbp + 64, w);
        }
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_LD32(ta + 96, vb);
        fold_chunk(bs, va, col + 64);
        if (nbp) {
          FK_TMEM_ST32(ta + 64, w);
          load_bias32(nbp + 96, w);
        }
        FK_TMEM_WAIT_LD(vb);
        fold_chunk(bs, vb, col + 96);
        if (nbp) FK_TMEM_ST32(ta + 96, w);
        tmem_wait_st();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(a);
      }
      if (!ok) break;
      // lowest column of the candidate chunk holding the maximum
      int j0 = 32, j1 = 32, j2 = 32, j3 = 32;
#pragma unroll
      for (int i = 28; i >= 0; i -= 4) {
        j0 = __uint_as_float(bs.cand[i]) == bs.score ? i : j0;
        j1 = __uint_as_float(bs.cand[i + 1]) == bs.score ? i + 1 : j1;
        j2 = __uint_as_float(bs.cand[i + 2]) == bs.score ? i + 2 : j2;
        j3 = __uint_as_float(bs.cand[i + 3]) == bs.score ? i + 3 : j3;
      }
      const int jm = min(min(j0, j1), min(j2, j3));
      const int bi = jm < 32 ? bs.base + jm : 0;
      // merge the two column halves of each point: half 1 hands over its
      // candidate and |x|^2, half 0 merges and writes
      if (h == 1) {
        if (u != pair && !(ok = mbar_wait(xchg_empty, xc ^ 1u, abort_flag, p.ctl))) break;
        float xn = 0.f;
        if (p.mindist) {
          // |x|^2 from the swizzled X tile: every MMA of this unit is done
          // (its last accumulator was full), so X is resident until this
          // CTA's epilogue warps have all arrived on xempty below
          for (int kb = 0; kb < KB; ++kb) {
            const uint8_t *rowp = sm + (xb * KB + kb) * kXBytes + r * 128;
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              const uint4 wv = *reinterpret_cast<const uint4 *>(rowp + ((c ^ (r & 7)) << 4));
              const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
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
        xchg[r] = make_float4(bs.score, __int_as_float(bi), xn, 0.f);
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(xchg_full);
          mbar_arrive(xempty(xb));
        }
      } else {
        if (!(ok = mbar_wait(xchg_full, xc, abort_flag, p.ctl))) break;
        const float4 o = xchg[r];
        float sb = bs.score;
        int bb = bi;
        const int oi = __float_as_int(o.y);
        if (o.x > sb || (o.x == sb && oi < bb)) { sb = o.x; bb = oi; }
        if (row < p.N) {
          const size_t o_ = (size_t)b * p.N + row;
          p.labels[o_] = bb;
          if (p.mindist) p.mindist[o_] = fmaxf(0.f, fmaf(-2.f, sb, o.z));
        }
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(xchg_empty);
          mbar_arrive(xempty(xb));
        }
      }
      if (++xb == XBUF) xb = 0;
    }
  }

  tc_fence_before();
  cluster_sync();  // neither CTA leaves while the other may still signal it
  if (warp == kMmaWarp) {
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tbase, kTmemCols);
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
  static int configured[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int want = TcCfg<KB>::USED + 1024;
  const int dyn = want < optin ? want : optin;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel<KB>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
      if (e != cudaSuccess) return e;
      configured[dev] = 1;
    }
  }
  p.dyn_bytes = (uint32_t)dyn;
  const int max_pairs = num_sms / 2 > 0 ? num_sms / 2 : 1;
  const int pairs = p.total_units < max_pairs ? p.total_units : max_pairs;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * pairs);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = dyn;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  cudaError_t e = cudaLaunchKernelEx(&cfg, assign_tc_kernel<KB>, xm, cm, p);
  count_launches(1);
  return e;
}

cudaError_t launch_assign_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N,
                             int D, int K, int Kpad, int32_t *labels, float *mindist, DevCtl ctl,
                             int num_sms, cudaStream_t s) {
  if (!tc_shape_ok(dt, D) || !tc_aligned(X, C)) return cudaErrorNotSupported;
  CUtensorMap xm, cm;
  if (!encode_3d(&xm, dt, X, D, N, B, kRows) || !encode_3d(&cm, dt, C, D, K, B, kHalfN))
    return cudaErrorNotSupported;
  TcParams p;
  p.N = N;
  p.K = K;
  p.Kpad = Kpad;
  p.ntiles = (K + kTileN - 1) / kTileN;
  p.upb = (N + kRowsUnit - 1) / kRowsUnit;
  p.total_units = p.upb * B;
  p.idesc = idesc_f16(dt == kBF16 ? 1 : 0, kRowsUnit, kTileN);
  p.is_bf16 = dt == kBF16;
  p.bias = bias;
  p.labels = labels;
  p.mindist = mindist;
  p.ctl = ctl;
  p.dyn_bytes = 0;
  if (p.total_units == 0) return cudaSuccess;
  if (Kpad < p.ntiles * kTileN) return cudaErrorInvalidValue;  // the bias must cover every tile
  const int KB = (D + kBlkK - 1) / kBlkK;
  if (KB == 1) return launch_kb<1>(xm, cm, p, num_sms, s);
  return launch_kb<2>(xm, cm, p, num_sms, s);
}

}  // namespace fk
