// assign_tc.cu -- FlashAssign on Blackwell tensor cores (tcgen05 + TMA + TMEM),
// run by pairs of CTAs (cta_group::2).
//
// Flash-KMeans (arXiv 2603.09229, abstract) fuses the distance computation
// with an online argmin so that the N x K distance matrix is never
// materialised in HBM.  On sm_100a that becomes:
//
//   * clusters of two CTAs (one per SM) loop over "units" of 256 points; the
//     leader CTA owns rows [0,128) of a unit, the peer rows [128,256);
//   * in each CTA one TMA warp streams its 128 rows of X per unit into a ring
//     of X buffers (kept resident while every centroid tile streams past;
//     deeper when a unit has at most two tiles), and another loads, per
//     256-centroid tile, its half (128 centroids) into a ring of tile slots:
//     the k-blocks of the centroids (128-byte swizzle, 64 elements each) and
//     their bias terms (32-byte rows: three tf32-exact terms of -|c|^2/2,
//     then zeros); a slot that already holds the wanted tile is reused;
//   * one thread of the leader issues the tile's MMAs with cta_group::2
//     (M = 256 across the pair, N = 256, fp32 accumulate; each CTA's TMEM
//     receives its 128 rows x 256 columns).  The first, of kind tf32 and
//     K = 8, multiplies a constant block of ones by the bias terms and so
//     overwrites the accumulator with -|c|^2/2 (exactly: the terms and their
//     partial sums are fp32-exact); the kind::f16 MMAs (K = 16) then add
//     <x,c>.  The accumulator ends holding the score s = <x,c> - |c|^2/2,
//     whose arg-max is the arg-min of |x - c|^2, and the epilogue has no
//     per-column arithmetic left but the arg-max.  (Giving every thread the
//     bias instead would move 128 bytes per thread per 32 columns through
//     L1, as much as L1 returns to the registers in a whole tile.)  Two
//     accumulators (all 512 TMEM columns) alternate over the tiles, and a
//     tile ends with one tcgen05.commit that reaches both CTAs.  There is no
//     other commit: the epilogue frees a tile slot once it has seen the tile
//     complete, and a unit's X buffer once it is done with the unit;
//   * eight epilogue warps per CTA: warp (h, q) owns TMEM lanes [32q, 32q+32)
//     (one point per thread) and columns [128h, 128h+128) of every tile, read
//     as two pairs of 32-column chunks (with one tile per unit, warp (h, q)
//     instead takes every other unit whole, on accumulator h, and no merge
//     is needed).  A 3-input-max tree gives the chunk
//     maximum; when it beats the point's running maximum (strict
//     ">", so an earlier column keeps a tie) the lane copies the chunk into a
//     register-resident candidate.  The lowest column of the candidate
//     holding the maximum is found once per unit, and the two column halves
//     of a point are merged at the end of the unit (score, then lower index),
//     together with |x|^2 for the returned squared distance;
//   * nothing is written back to TMEM, so an accumulator goes back to the MMA
//     thread as soon as all epilogue warps of the pair that read it have
//     LOADED their last chunk pair (issued while the pair before it is
//     folded): the reduction of that pair overlaps the next tile's MMAs.  The peer's warps signal the leader's barrier with a relaxed
//     cluster-scope arrive, after tcgen05.wait::ld and
//     tcgen05.fence::before_thread_sync: a release at cluster scope would cost
//     more than a third of a tile, and those TMEM reads are already complete
//     when the arrive is issued.
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
#include "tc_argmin.cuh"
#include "tc_gauss.cuh"

namespace fk {

constexpr int kRows = 128;                  // rows per CTA per unit
constexpr int kRowsUnit = 2 * kRows;        // rows per pair unit (MMA M)
constexpr int kTileN = 256;                 // centroids per tile (MMA N)
constexpr int kHalfN = kTileN / 2;          // centroids per CTA per tile
constexpr int kBlkK = 64;                   // elements per k-block (128 bytes)
constexpr int kXBytes = kRows * 128;        // one X k-block, 16 KB
constexpr int kStageBytes = kHalfN * 128;   // one centroid half k-block, 16 KB
constexpr int kBiasRow = kBiasTerms * 4;    // bias terms of one centroid, 32 bytes
constexpr int kBiasBytes = kHalfN * kBiasRow;  // bias terms of a half tile, 4 KB
constexpr int kOnesBytes = 256;             // the tf32 A operand of the bias step
constexpr int kAcc = 2;                     // accumulators
constexpr int kEpiWarps = 8;                // column half x lane quarter
// warp 8 loads X, warp 9 issues the MMAs, warp 10 loads the centroid tiles
constexpr int kProducerWarp = kEpiWarps, kMmaWarp = kEpiWarps + 1, kTileWarp = kEpiWarps + 2;
constexpr int kThreads = 32 * (kEpiWarps + 3);
constexpr uint32_t kTmemCols = 512;         // two 256-column fp32 accumulators
constexpr uint16_t kBothCtas = 0x3;
static_assert(kAcc * kTileN <= (int)kTmemCols, "accumulators exceed TMEM");
static_assert(kTileN == kCentroidPad, "the bias is padded to whole tiles");

// Shared-memory plan.  With many tiles per unit the X tile of the next unit
// has several tiles' time to load, and the ring holds as many tile slots as
// fit.  With at most two tiles per unit (small K, e.g. a batch of small
// problems) a unit's MMAs last less than one X load takes, so the deep-X
// plan (DX) keeps several units of X in flight and only two tile slots.
// Rows of up to 128 dimensions keep several X tiles and tile slots in
// flight; 129 to 256 dimensions (3 or 4 k-blocks) fit two tile slots and two
// X buffers (one at 4 k-blocks) in the 227 KB of shared memory.
template <int KB, bool DX> struct TcCfg {
  static constexpr int XBUF = KB >= 4 ? 1 : KB == 3 ? 2 : DX ? (KB == 1 ? 8 : 4) : 2;  // X buffers (units in flight)
  static constexpr int SLOT = KB * kStageBytes + kBiasBytes;  // one tile's centroids and bias terms
  static constexpr int NSLOT = KB >= 3 ? 2 : DX ? (KB == 1 ? 4 : 2) : (KB == 1 ? 9 : 4);  // tile slots in the ring
  static constexpr int X_BYTES = XBUF * KB * kXBytes;
  static constexpr int C_BYTES = NSLOT * SLOT;
  static constexpr int XCHG_BYTES = kRows * 32;    // two float4 per row
  // full/empty per slot, xfull/xempty per X buffer, accfull/accempty per
  // accumulator, xchg full/empty, drain, xready per X buffer
  static constexpr int NBAR = 2 * NSLOT + 2 * XBUF + 2 * kAcc + 2 + 1 + XBUF;
  static constexpr int USED = X_BYTES + C_BYTES + XCHG_BYTES + kOnesBytes + NBAR * 8 + 16;
  static_assert(SLOT % 1024 == 0, "slots keep the 1 KB alignment of the 128-byte swizzle");
  static_assert(USED + 1024 <= 232448, "shared memory (227 KB per CTA on sm_100) exceeded");
};

// Pair MMA of kind tf32 (K = 8 per instruction), same operand split as the
// kind::f16 form.
__device__ __forceinline__ void tc_mma_tf32_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                 uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::tf32 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Instruction descriptor of kind::tf32: fp32 accumulator, A and B tf32, both
// K-major, shape M x N.
constexpr uint32_t idesc_tf32(int M, int N) {
  return (1u << 4) | (2u << 7) | (2u << 10) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Shared-memory descriptor of the bias terms as TMA writes them: K-major rows
// of 32 bytes with the 32-byte swizzle (layout type 6), 8-row groups 256 B
// apart.  The base must be 256-byte aligned.
__device__ __forceinline__ uint64_t desc_kmajor_sw32(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(256 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)6 << 61);
}

// Shared-memory descriptor of the block of ones, without swizzle: the two
// 16-byte column groups of a row are core matrices 128 B apart (leading byte
// offset) and every 8-row group reads the same 8 rows (stride byte offset 0),
// so a 256-byte block serves all 128 rows.
__device__ __forceinline__ uint64_t desc_ones(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)(128 >> 4) << 16) | ((uint64_t)1 << 46);
}

struct TcParams {
  int N, K, Kpad, ntiles, upb, total_units;
  uint32_t idesc, idesc_bias;
  int is_bf16;
  uint32_t dyn_bytes;
  int32_t *labels;
  float *mindist;
  const float *xnorm;  // |x|^2 per row (B*N), or null: computed from the X tile
  NearTies ties;
  // Gaussian-sum epilogue: a = 2 beta log2(e); outputs (either may be null)
  float gs_a;
  float *gs_log;  // ln of the weighted Gauss sum per row
  float *gs_val;  // the weighted Gauss sum per row  // where points whose two best scores are too close to order are listed
  DevCtl ctl;
};

// The Gaussian-sum epilogue (GaussAcc, gauss_fold, gauss_merge) is in tc_gauss.cuh.

// ln and value of exp(-beta |x|^2) 2^(a M) S for a row.
__device__ __forceinline__ void gauss_store(const TcParams &p, const GaussAcc &g, float xn, size_t o) {
  const float l2 = lg2_approx(g.S) + p.gs_a * (g.M - 0.5f * xn);  // log2 of the sum
  if (p.gs_log) p.gs_log[o] = l2 * 0.6931471805599453f;
  if (p.gs_val) p.gs_val[o] = ex2_approx(l2);
}

template <int KB, bool DX, bool GS, bool EX>
__global__ void __launch_bounds__(kThreads, 1)
    assign_tc_kernel(const __grid_constant__ CUtensorMap xmap, const __grid_constant__ CUtensorMap cmap,
                     const __grid_constant__ CUtensorMap bmap, const TcParams p) {
  using Cfg = TcCfg<KB, DX>;
  constexpr int NST = Cfg::NSLOT, XBUF = Cfg::XBUF;
  extern __shared__ __align__(1024) uint8_t smem_raw[];

  const uint32_t rank = cluster_rank();
  const bool leader = rank == 0;
  const int pair = blockIdx.x >> 1, npairs = gridDim.x >> 1;
  // The pair's units: a contiguous range, so that consecutive units mostly
  // belong to the same problem (a batch of problems reuses its centroid
  // tiles from one unit to the next, see the producer).
  const int upp = (p.total_units + npairs - 1) / npairs;
  const int u_begin = pair * upp;
  const int u_end = u_begin + upp < p.total_units ? u_begin + upp : p.total_units;
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
  float *ones = reinterpret_cast<float *>(sm + Cfg::X_BYTES + Cfg::C_BYTES + Cfg::XCHG_BYTES);
  uint64_t *bars =
      reinterpret_cast<uint64_t *>(sm + Cfg::X_BYTES + Cfg::C_BYTES + Cfg::XCHG_BYTES + kOnesBytes);
  uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(bars + Cfg::NBAR);
  volatile int *abort_flag = reinterpret_cast<volatile int *>(tmem_slot + 1);

  const uint32_t bar0 = smem_u32(bars);
  auto full = [&](int s) { return bar0 + 8u * s; };                                   // leader's
  auto empty = [&](int s) { return bar0 + 8u * (NST + s); };                          // each CTA
  auto slot_c = [&](int s, int kb) { return sC + s * Cfg::SLOT + kb * kStageBytes; };
  auto slot_bias = [&](int s) { return sC + s * Cfg::SLOT + KB * kStageBytes; };
  auto xfull = [&](int x) { return bar0 + 8u * (2 * NST + x); };                      // leader's
  auto xempty = [&](int x) { return bar0 + 8u * (2 * NST + XBUF + x); };              // each CTA
  auto accfull = [&](int a) { return bar0 + 8u * (2 * NST + 2 * XBUF + a); };         // each CTA
  auto accempty = [&](int a) { return bar0 + 8u * (2 * NST + 2 * XBUF + kAcc + a); };  // leader's
  const uint32_t xchg_full = bar0 + 8u * (2 * NST + 2 * XBUF + 2 * kAcc);
  const uint32_t xchg_empty = xchg_full + 8u;
  const uint32_t drain = xchg_full + 16u;
  // (one tile per unit) the peer's X tile has landed: the leader's epilogue
  // sees the pair's xfull and tells the peer
  auto xready = [&](int x) { return drain + 8u + 8u * x; };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < NST; ++s) {
      mbar_init(full(s), 1);   // the leader's expect_tx; bytes from both CTAs
      mbar_init(empty(s), 1);  // the epilogue, once the tile using the slot is complete
    }
    // With one tile per unit and |x|^2 prepared, nothing but the MMAs reads an
    // X buffer: the MMA thread's commit frees it as soon as they complete.
    // Otherwise this CTA's epilogue warps of the unit free it after the unit.
    const bool x_by_mma = p.ntiles == 1 && p.xnorm != nullptr;
    for (int x = 0; x < XBUF; ++x) {
      mbar_init(xfull(x), 1);
      mbar_init(xempty(x), x_by_mma ? 1 : p.ntiles == 1 ? kEpiWarps / 2 : kEpiWarps);
      mbar_init(xready(x), 1);  // one leader warp of the unit (read in the peer, one tile per unit)
    }
    // With one tile per unit each unit is read by one warp of each lane
    // quarter (see the epilogue), else by all epilogue warps.
    const int readers = p.ntiles == 1 ? kEpiWarps / 2 : kEpiWarps;
    for (int a = 0; a < kAcc; ++a) {
      mbar_init(accfull(a), 1);             // the MMA commit
      mbar_init(accempty(a), 2 * readers);  // those epilogue warps of both CTAs
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
    tma_prefetch_desc(&bmap);
  }
  // The A operand of the bias step: 8 rows of (1, 1, 1, 0 | 0, 0, 0, 0) as
  // two no-swizzle core matrices (columns 0-3, then 4-7 at +128 B).
  if (threadIdx.x < kOnesBytes / 4) ones[threadIdx.x] = (threadIdx.x < 32 && (threadIdx.x & 3) < 3) ? 1.f : 0.f;
  asm volatile("fence.proxy.async.shared::cta;" ::: "memory");  // visible to the tensor cores
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
      // ------------------------------------------------- X producer -----
      // X streams up to XBUF units ahead of the MMAs, independently of the
      // centroid tiles (a unit of one or two tiles is over before one X
      // tile has loaded)
      uint32_t xb = 0, xph = 0;
      bool ok = true, issued = false;
      for (int u = u_begin; ok && u < u_end; ++u) {
        const int b = u / p.upb, r0 = (u % p.upb) * kRowsUnit + (int)rank * kRows;
        if (!(ok = mbar_wait(xempty(xb), xph ^ 1u, abort_flag, p.ctl))) break;
        if (leader) mbar_arrive_expect_tx(xfull(xb), 2 * KB * kXBytes);
        const uint32_t xbar = map_to_cta(xfull(xb), 0);
        for (int kb = 0; kb < KB; ++kb)
          tma_load_3d_pair(sX + (xb * KB + kb) * kXBytes, &xmap, xbar, kb * kBlkK, r0, b);
        issued = true;
        if (++xb == XBUF) { xb = 0; xph ^= 1u; }
      }
      // After an abort, give copies already issued time to land in this CTA's
      // shared memory before it can exit (their barrier may be in the peer).
      if (!ok && issued) {
        const uint64_t t0 = globaltimer();
        while (globaltimer() - t0 < 50000ull) {
        }
      }
    }
  } else if (warp == kTileWarp) {
    if (lane == 0) {
      // ---------------------------------------------- tile producer -----
      // The kernel may be launched before the one that prepared the
      // centroids and the bias has finished (programmatic stream
      // serialization): the centroid tiles wait until that kernel's writes
      // are visible.
      asm volatile("griddepcontrol.wait;" ::: "memory");
      uint32_t st = 0, sph = 0;
      bool ok = true, issued = false;
      // (problem, tile) + 1 held by each slot, 0 when not known: both CTAs of
      // the pair track it alike, so both skip or both load
      int held[NST];
      for (int i = 0; i < NST; ++i) held[i] = 0;
      for (int u = u_begin; ok && u < u_end; ++u) {
        const int b = u / p.upb;
        for (int j = 0; ok && j < p.ntiles; ++j) {
          if (!(ok = mbar_wait(empty(st), sph ^ 1u, abort_flag, p.ctl))) break;
          const int tag = b * p.ntiles + j + 1;
          if (held[st] == tag) {
            // the slot already holds this tile (same problem, one or two
            // tiles per unit): hand it over again without copying
            if (leader) mbar_arrive(full(st));
          } else {
            if (leader) mbar_arrive_expect_tx(full(st), 2 * (KB * kStageBytes + kBiasBytes));
            const uint32_t fbar = map_to_cta(full(st), 0);
            const int c0 = j * kTileN + (int)rank * kHalfN;
            for (int kb = 0; kb < KB; ++kb) tma_load_3d_pair(slot_c(st, kb), &cmap, fbar, kb * kBlkK, c0, b);
            tma_load_3d_pair(slot_bias(st), &bmap, fbar, 0, c0, b);
            held[st] = tag;
            issued = true;
          }
          if (++st == NST) { st = 0; sph ^= 1u; }
        }
      }
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
      const uint64_t ones_desc = desc_ones(smem_u32(ones));
      int t = 0;  // tile counter: accumulator t % 2, its (t / 2)-th use
      bool ok = true;
      for (int u = u_begin; ok && u < u_end; ++u) {
        if (!(ok = mbar_wait(xfull(xb), xph, abort_flag, p.ctl))) break;
        const uint32_t xa = sX + xb * KB * kXBytes;
        for (int j = 0; ok && j < p.ntiles; ++j, ++t) {
          const int sl = st;
          if (!(ok = mbar_wait(full(st), sph, abort_flag, p.ctl))) break;
          if (++st == NST) { st = 0; sph ^= 1u; }
          const int a = t & 1;
          // every epilogue warp of the pair has read the accumulator's last tile
          if (!(ok = mbar_wait(accempty(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
          tc_fence_after();
          const uint32_t acc = tbase + a * kTileN;
          // accumulator = 1*hi + 1*mid + 1*lo = -|c|^2/2 (overwrites)
          tc_mma_tf32_pair(acc, ones_desc, desc_kmajor_sw32(slot_bias(sl)), p.idesc_bias, 0u);
#pragma unroll
          for (int kb = 0; kb < KB; ++kb) {
            const uint64_t ad = desc_kmajor_sw128(xa + kb * kXBytes);
            const uint64_t bd = desc_kmajor_sw128(slot_c(sl, kb));
#pragma unroll
            for (int k = 0; k < kBlkK / 16; ++k) tc_mma_f16_pair(acc, ad + 2 * k, bd + 2 * k, p.idesc, 1u);
          }
          tc_commit_pair(accfull(a), kBothCtas);
        }
        if (!ok) break;
        if (p.ntiles == 1 && p.xnorm) tc_commit_pair(xempty(xb), kBothCtas);  // the unit's MMAs have read X
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
    // One tile per unit (small K): the two warps of a lane quarter take
    // alternate units whole, each on its own accumulator (unit u on u % 2),
    // so a warp has two tiles of MMA time to read it and no merge is needed.
    // Otherwise warp h takes columns [128h, 128h + 128) of every tile.
    const bool whole = p.ntiles == 1;
    const uint32_t t_row = tbase + ((uint32_t)(q * 32) << 16) + (uint32_t)(whole ? 0 : h * kHalfN);
    // hand an accumulator back to the leader's MMA thread
    auto release_acc = [&](int a) {
      if (leader) mbar_arrive(accempty(a));
      else mbar_arrive_cluster_relaxed(map_to_cta(accempty(a), 0));
    };
    // Partial |x|^2 of this thread's row over its 16-byte groups [g0, g1) (8
    // per k-block) from the swizzled X tile in buffer xb, which must have
    // landed (it stays resident until this CTA's warps of the unit have
    // arrived on xempty).  Squares of fp16/bf16 values are exact in fp32; the
    // sums run two at a time (packed fma).
    auto x_norm = [&](uint32_t xb, int g0, int g1) {
      uint32_t a0 = 0u, a1 = 0u;
      for (int gi = g0; gi < g1; ++gi) {
        const int kb = gi >> 3, c = gi & 7;
        const uint8_t *rowp = sm + (xb * KB + kb) * kXBytes + r * 128;
        const uint4 wv = *reinterpret_cast<const uint4 *>(rowp + ((c ^ (r & 7)) << 4));
        const uint32_t ws[4] = {wv.x, wv.y, wv.z, wv.w};
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          uint32_t lo, hi;
          if (p.is_bf16) {
            lo = ws[e] << 16;
            hi = ws[e] & 0xffff0000u;
          } else {
            const __half2 h2 = *reinterpret_cast<const __half2 *>(&ws[e]);
            lo = __float_as_uint(__low2float(h2));
            hi = __float_as_uint(__high2float(h2));
          }
          fma2(a0, a1, lo, hi);
        }
      }
      return __uint_as_float(a0) + __uint_as_float(a1);
    };
    // The accumulators start out free.
    tc_fence_before();
    __syncwarp();
    if (lane == 0) {
      if (whole) {
        release_acc(h);
      } else {
        release_acc(0);
        release_acc(1);
      }
    }

    if (whole) {
      bool ok = true;
      for (int u = u_begin + h; ok && u < u_end; u += 2) {
        const int t = u - u_begin, a = t & 1;  // a == h
        const int b = u / p.upb;
        const int row = (u % p.upb) * kRowsUnit + (int)rank * kRows + r;
        const uint32_t xb = (uint32_t)(t % XBUF);
        Best bs;
        GaussAcc ga{__int_as_float(0xff800000), 0.f};
        if constexpr (!GS) best_init(bs);
        int ex = -1;  // the centroid this point leaves out
        if constexpr (EX) ex = row < p.N ? __ldg(p.ties.excl + (size_t)b * p.N + row) : -1;
        auto fold = [&](uint32_t (&v)[32], int col) {
          if constexpr (EX) mask_col(v, ex - col);
          if constexpr (GS) gauss_fold(ga, v, p.gs_a);
          else fold_chunk(bs, v, col);
        };
        // |x|^2 of this thread's row while the unit is multiplied: the X tile
        // has landed once the pair's xfull completes (the leader sees it and
        // tells the peer)
        // (or read the prepared |x|^2, a load issued before the unit's wait)
        float xn;
        if (p.xnorm) {
          xn = row < p.N ? __ldg(p.xnorm + (size_t)b * p.N + row) : 0.f;
        } else {
          const uint32_t xph = (uint32_t)(t / XBUF) & 1u;
          if (leader) {
            if (!(ok = mbar_wait(xfull(xb), xph, abort_flag, p.ctl))) break;
            if (q == 0 && lane == 0) mbar_arrive_cluster(map_to_cta(xready(xb), 1));
          } else {
            if (!(ok = mbar_wait_acq_cluster(xready(xb), xph, abort_flag, p.ctl))) break;
          }
          xn = x_norm(xb, 0, KB * 8);
        }
        if (!(ok = mbar_wait(accfull(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
        tc_fence_after();
        if (q == 0 && lane == 0) mbar_arrive(empty(t % NST));  // the MMA is done with the slot
        const uint32_t ta = t_row + a * kTileN;
        uint32_t va[32], vb[32], vc[32];
        // eight chunks; each load is issued while the chunk before is folded
        FK_TMEM_LD32(ta, va);
        FK_TMEM_LD32(ta + 32, vb);
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_WAIT_LD(vb);
        FK_TMEM_LD32(ta + 64, vc);
        fold(va, 0);
        FK_TMEM_LD32(ta + 96, va);
        fold(vb, 32);
        FK_TMEM_WAIT_LD(vc);
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_LD32(ta + 128, vb);
        fold(vc, 64);
        FK_TMEM_LD32(ta + 160, vc);
        fold(va, 96);
        FK_TMEM_WAIT_LD(vb);
        FK_TMEM_WAIT_LD(vc);
        FK_TMEM_LD32(ta + 192, va);
        fold(vb, 128);
        FK_TMEM_LD32(ta + 224, vb);
        fold(vc, 160);
        FK_TMEM_WAIT_LD(va);
        FK_TMEM_WAIT_LD(vb);
        tc_fence_before();
        __syncwarp();
        if (lane == 0) release_acc(a);
        fold(va, 192);
        fold(vb, 224);
        const size_t o_ = (size_t)b * p.N + row;
        if constexpr (GS) {
          if (row < p.N) gauss_store(p, ga, xn, o_);
        } else {
          const int jm = best_pos(bs);
          const int bi = jm < 32 ? bs.base + jm : 0;
          const float s2 = fmaxf(bs.s2, second_in_chunk(bs, jm));
          if (row < p.N) {
            p.labels[o_] = bi;
            if (p.mindist) p.mindist[o_] = fmaxf(0.f, fmaf(-2.f, bs.score, xn));
          }
          list_near_tie(p.ties, row < p.N, bs.score, s2, bs.s3, xn, o_, bs.base2);
        }
        __syncwarp();
        if (lane == 0 && !p.xnorm) mbar_arrive(xempty(xb));  // (with |x|^2 prepared the MMA commit frees it)
      }
    } else {
      uint32_t xb = 0, xc = 0;
      int t = 0;  // the pair's tile counter
      bool ok = true;
      for (int u = u_begin; ok && u < u_end; ++u, xc ^= 1u) {
        const int b = u / p.upb;
        const int row = (u % p.upb) * kRowsUnit + (int)rank * kRows + r;
        Best bs;
        GaussAcc ga{__int_as_float(0xff800000), 0.f};
        if constexpr (!GS) best_init(bs);
        int ex = -1;  // the centroid this point leaves out
        if constexpr (EX) ex = row < p.N ? __ldg(p.ties.excl + (size_t)b * p.N + row) : -1;
        auto fold = [&](uint32_t (&v)[32], int c) {
          if constexpr (EX) mask_col(v, ex - c);
          if constexpr (GS) gauss_fold(ga, v, p.gs_a);
          else fold_chunk(bs, v, c);
        };
        // this column half's share of |x|^2, or (column half 0) the prepared
        // |x|^2, loaded now and used at the end of the unit
        float xn = 0.f;
        if (p.xnorm && h == 0 && row < p.N) xn = __ldg(p.xnorm + (size_t)b * p.N + row);
        for (int j = 0; ok && j < p.ntiles; ++j, ++t) {
          const int a = t & 1;
          if (!(ok = mbar_wait(accfull(a), (uint32_t)(t >> 1) & 1u, abort_flag, p.ctl))) break;
          tc_fence_after();
          if (h == 0 && q == 0 && lane == 0) mbar_arrive(empty(t % NST));  // the MMA is done with the slot
          const uint32_t ta = t_row + a * kTileN;
          const int col = j * kTileN + h * kHalfN;
          uint32_t va[32], vb[32], vc[32];
          // chunks 0 and 1; the loads of chunks 2 and 3 are issued while they
          // are folded (chunk 3 into chunk 0's registers once it is folded)
          FK_TMEM_LD32(ta, va);
          FK_TMEM_LD32(ta + 32, vb);
          FK_TMEM_WAIT_LD(va);
          FK_TMEM_WAIT_LD(vb);
          FK_TMEM_LD32(ta + 64, vc);
          fold(va, col);
          FK_TMEM_LD32(ta + 96, va);
          fold(vb, col + 32);
          // chunks 2 and 3: once they are in registers the accumulator is free
          FK_TMEM_WAIT_LD(vc);
          FK_TMEM_WAIT_LD(va);
          tc_fence_before();
          __syncwarp();
          if (lane == 0) release_acc(a);
          fold(vc, col + 64);
          fold(va, col + 96);
          // half of the row's |x|^2 per column half, while the unit's second
          // tile is multiplied (the first tile's MMAs have read X)
          if (j == 0 && !p.xnorm) xn = x_norm(xb, h * KB * 4, (h + 1) * KB * 4);
        }
        if (!ok) break;
        if constexpr (GS) {
          // merge the two column halves: half 1 hands over (M, S) and its
          // share of |x|^2, half 0 merges and writes
          if (h == 1) {
            if (u != u_begin && !(ok = mbar_wait(xchg_empty, xc ^ 1u, abort_flag, p.ctl))) break;
            xchg[2 * r] = make_float4(ga.M, ga.S, xn, 0.f);
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(xchg_full);
              mbar_arrive(xempty(xb));
            }
          } else {
            if (!(ok = mbar_wait(xchg_full, xc, abort_flag, p.ctl))) break;
            const float4 o = xchg[2 * r];
            const GaussAcc g = gauss_merge(ga, GaussAcc{o.x, o.y}, p.gs_a);
            if (row < p.N) gauss_store(p, g, xn + o.z, (size_t)b * p.N + row);
            __syncwarp();
            if (lane == 0) {
              mbar_arrive(xchg_empty);
              mbar_arrive(xempty(xb));
            }
          }
          if (++xb == XBUF) xb = 0;
          continue;
        }
        const int jm = best_pos(bs);
        const int bi = jm < 32 ? bs.base + jm : 0;
        const float s2in = second_in_chunk(bs, jm);
        // merge the two column halves of each point: half 1 hands over its
        // candidate and |x|^2, half 0 merges and writes
        if (h == 1) {
          if (u != u_begin && !(ok = mbar_wait(xchg_empty, xc ^ 1u, abort_flag, p.ctl))) break;
          xchg[2 * r] = make_float4(bs.score, __int_as_float(bi), xn, bs.s2);
          xchg[2 * r + 1] = make_float4(s2in, __int_as_float(bs.base2), bs.s3, 0.f);
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(xchg_full);
            mbar_arrive(xempty(xb));
          }
        } else {
          if (!(ok = mbar_wait(xchg_full, xc, abort_flag, p.ctl))) break;
          const float4 o = xchg[2 * r], o2 = xchg[2 * r + 1];
          const float xt = xn + o.z;
          const int oi = __float_as_int(o.y), ob2 = __float_as_int(o2.y);
          // winner: larger score, then lower column; runner-up chunk: the
          // better of the loser's best chunk and the winner's own runner-up
          const bool other_wins = o.x > bs.score || (o.x == bs.score && oi < bi);
          const float s1 = other_wins ? o.x : bs.score;
          const int b1 = other_wins ? oi : bi;
          const float w_s2 = other_wins ? o.w : bs.s2, w_in = other_wins ? o2.x : s2in;
          const int w_b2 = other_wins ? ob2 : bs.base2;
          const float l_s1 = other_wins ? bs.score : o.x;
          const int l_b1 = other_wins ? bi : oi;
          const float s2 = fmaxf(fmaxf(w_s2, w_in), l_s1);
          const int other = l_s1 > w_s2 ? (l_b1 & ~31) : w_b2;
          // third best among the other chunks: the winner's runner-up and third,
          // the loser's best chunk and runner-up
          const float w_s3 = other_wins ? o2.z : bs.s3, l_s2 = other_wins ? bs.s2 : o.w;
          const float s3 = l_s1 >= w_s2 ? fmaxf(w_s2, l_s2) : fmaxf(l_s1, w_s3);
          const size_t o_ = (size_t)b * p.N + row;
          if (row < p.N) {
            p.labels[o_] = b1;
            if (p.mindist) p.mindist[o_] = fmaxf(0.f, fmaf(-2.f, s1, xt));
          }
          list_near_tie(p.ties, row < p.N, s1, s2, s3, xt, o_, other);
          __syncwarp();
          if (lane == 0) {
            mbar_arrive(xchg_empty);
            mbar_arrive(xempty(xb));
          }
        }
        if (++xb == XBUF) xb = 0;
      }
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

// The prepared bias as B x Kpad rows of kBiasTerms fp32 terms, loaded half a
// tile (128 rows of 32 bytes) at a time with the 32-byte swizzle.
static bool encode_bias_3d(CUtensorMap *m, const float *bias, int Kpad, int B) {
  auto fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[3] = {(cuuint64_t)kBiasTerms, (cuuint64_t)Kpad, (cuuint64_t)B};
  const cuuint64_t strides[2] = {(cuuint64_t)kBiasRow, (cuuint64_t)kBiasRow * (cuuint64_t)Kpad};
  const cuuint32_t box[3] = {(cuuint32_t)kBiasTerms, (cuuint32_t)kHalfN, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = fn(m, CU_TENSOR_MAP_DATA_TYPE_FLOAT32, 3, const_cast<float *>(bias), dims, strides, box, estr,
                  CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_32B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                  CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

bool tc_shape_ok(DType dt, int D) { return dt != kF32 && D % 8 == 0 && D >= 8 && D <= 256; }

bool tc_aligned(const void *X, const void *C) {
  return ((uintptr_t)X % 16 == 0) && ((uintptr_t)C % 16 == 0);
}

template <int KB, bool DX, bool GS, bool EX>
static cudaError_t launch_kb(const CUtensorMap &xm, const CUtensorMap &cm, const CUtensorMap &bm, TcParams p,
                             int num_sms, cudaStream_t s) {
  static int configured[64] = {};
  static std::mutex mu;
  int dev = 0;
  cudaGetDevice(&dev);
  int optin = 0;
  cudaDeviceGetAttribute(&optin, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev);
  const int want = TcCfg<KB, DX>::USED + 1024;
  const int dyn = want < optin ? want : optin;
  {
    std::lock_guard<std::mutex> g(mu);
    if (dev < 64 && !configured[dev]) {
      cudaError_t e = cudaFuncSetAttribute(assign_tc_kernel<KB, DX, GS, EX>, cudaFuncAttributeMaxDynamicSharedMemorySize, dyn);
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
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  // may start while the previous kernel in the stream drains; the producer
  // waits for it before the first centroid load (see the kernel)
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  cudaError_t e = cudaLaunchKernelEx(&cfg, assign_tc_kernel<KB, DX, GS, EX>, xm, cm, bm, p);
  count_launches(1);
  return e;
}

// Tensor maps and parameters shared by the arg-min and Gaussian-sum launches.
static cudaError_t tc_setup(DType dt, const void *X, const void *C, const float *bias, int B, int N, int D, int K,
                            int Kpad, const float *xnorm, DevCtl ctl, CUtensorMap *xm, CUtensorMap *cm,
                            CUtensorMap *bm, TcParams *p) {
  if (!tc_shape_ok(dt, D) || !tc_aligned(X, C) || (uintptr_t)bias % 16 != 0) return cudaErrorNotSupported;
  if (!encode_3d(xm, dt, X, D, N, B, kRows) || !encode_3d(cm, dt, C, D, K, B, kHalfN) ||
      !encode_bias_3d(bm, bias, Kpad, B))
    return cudaErrorNotSupported;
  *p = TcParams{};
  p->N = N;
  p->K = K;
  p->Kpad = Kpad;
  p->ntiles = (K + kTileN - 1) / kTileN;
  p->upb = (N + kRowsUnit - 1) / kRowsUnit;
  p->total_units = p->upb * B;
  p->idesc = idesc_f16(dt == kBF16 ? 1 : 0, kRowsUnit, kTileN);
  p->idesc_bias = idesc_tf32(kRowsUnit, kTileN);
  p->is_bf16 = dt == kBF16;
  p->xnorm = xnorm;
  p->ctl = ctl;
  if (Kpad < p->ntiles * kTileN) return cudaErrorInvalidValue;  // the bias must cover every tile
  return cudaSuccess;
}

template <bool GS, bool EX>
static cudaError_t launch_any(const CUtensorMap &xm, const CUtensorMap &cm, const CUtensorMap &bm, const TcParams &p,
                              int D, int num_sms, cudaStream_t s) {
  if (p.total_units == 0) return cudaSuccess;
  const int KB = (D + kBlkK - 1) / kBlkK;
  const bool deep_x = p.ntiles <= 2;
  if (KB == 1)
    return deep_x ? launch_kb<1, true, GS, EX>(xm, cm, bm, p, num_sms, s) : launch_kb<1, false, GS, EX>(xm, cm, bm, p, num_sms, s);
  if (KB == 2)
    return deep_x ? launch_kb<2, true, GS, EX>(xm, cm, bm, p, num_sms, s) : launch_kb<2, false, GS, EX>(xm, cm, bm, p, num_sms, s);
  if (KB == 3)
    return deep_x ? launch_kb<3, true, GS, EX>(xm, cm, bm, p, num_sms, s) : launch_kb<3, false, GS, EX>(xm, cm, bm, p, num_sms, s);
  return deep_x ? launch_kb<4, true, GS, EX>(xm, cm, bm, p, num_sms, s) : launch_kb<4, false, GS, EX>(xm, cm, bm, p, num_sms, s);
}

cudaError_t launch_assign_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N,
                             int D, int K, int Kpad, const float *xnorm, int32_t *labels, float *mindist,
                             NearTies ties, DevCtl ctl, int num_sms, cudaStream_t s) {
  CUtensorMap xm, cm, bm;
  TcParams p;
  cudaError_t e = tc_setup(dt, X, C, bias, B, N, D, K, Kpad, xnorm, ctl, &xm, &cm, &bm, &p);
  if (e != cudaSuccess) return e;
  p.labels = labels;
  p.mindist = mindist;
  p.ties = ties;
  return ties.excl ? launch_any<false, true>(xm, cm, bm, p, D, num_sms, s)
                    : launch_any<false, false>(xm, cm, bm, p, D, num_sms, s);
}

cudaError_t launch_gauss_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N, int D, int K,
                            int Kpad, const float *xnorm, float beta, float *log_out, float *val_out, DevCtl ctl,
                            int num_sms, cudaStream_t s) {
  CUtensorMap xm, cm, bm;
  TcParams p;
  cudaError_t e = tc_setup(dt, X, C, bias, B, N, D, K, Kpad, xnorm, ctl, &xm, &cm, &bm, &p);
  if (e != cudaSuccess) return e;
  p.gs_a = 2.f * beta * 1.4426950408889634f;
  p.gs_log = log_out;
  p.gs_val = val_out;
  return launch_any<true, false>(xm, cm, bm, p, D, num_sms, s);
}

}  // namespace fk
