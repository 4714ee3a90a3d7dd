// fk_common.cuh -- device helpers shared by the libfk kernels (sm_100a).
//
// Thin inline-PTX wrappers for the Blackwell features the assignment kernel
// uses (mbarrier, TMA tensor loads, tcgen05 MMA / TMEM), the bounded wait
// used by every spin loop, and the device status word.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace fk {

// Device-side status codes (same values as the public fk_status codes).
enum : int { kStOk = 0, kStTimeout = -5, kStBadLabel = -7 };

enum DType : int { kF32 = 0, kF16 = 1, kBF16 = 2 };

// What every kernel that can fail needs: where to record the failure and how
// long a wait may spin before it gives up.
struct DevCtl {
  int *status;
  unsigned long long timeout_ns;
};

// Points the assignment kernels could not order with certainty: a point
// whose best and second-best fp32 scores (or distances) lie within `tau`
// times the magnitude they were accumulated from is listed as (global row
// b*N + i, first column of the second 32-centroid chunk to re-examine, or
// -1).  When a third chunk is that close too, the point is listed as
// (row, -2), from the other end of the list, for a comparison with every
// centroid.  The re-decision kernel (refine.cu) reads both parts, decides
// them exactly and resets the counts to 0.
struct NearTies {
  int2 *list;     // room for `cap` entries (B*N: a point is listed at most once)
  int *count;     // entries [0, *count), zero before the assignment kernel runs
  int *done;      // blocks of the re-decision kernel that have finished
  int *count_hi;  // entries [cap - *count_hi, cap), the full comparisons
  int cap;
  float tau;
  // null, or per point a centroid the assignment must leave out (the second
  // pass of the top-2 assignment excludes each point's nearest centroid)
  const int32_t *excl;
};

// Append the listed points of a warp (every lane calls this, `near` and
// `full` per lane): two-chunk points with one atomic add per warp from the
// front, full-comparison points one by one from the back.
__device__ __forceinline__ void list_append(const NearTies &t, bool near, bool full, int g, int other) {
  const bool two = near && !full;
  const unsigned fm = __ballot_sync(0xffffffffu, two);
  const int lane = threadIdx.x & 31;
  if (fm != 0u) {
    const int lead = __ffs(fm) - 1;
    int at = 0;
    if (lane == lead) at = atomicAdd(t.count, __popc(fm));
    at = __shfl_sync(0xffffffffu, at, lead);
    const int slot = at + __popc(fm & ((1u << lane) - 1u));
    if (two && slot < t.cap) t.list[slot] = make_int2(g, other);
  }
  if (near && full) {
    const int slot = t.cap - 1 - atomicAdd(t.count_hi, 1);
    if (slot >= 0) t.list[slot] = make_int2(g, -2);
  }
}

__device__ __forceinline__ void record_status(int *status, int code) {
  atomicCAS(status, 0, code);  // first error wins
}

__device__ __forceinline__ uint64_t globaltimer() {
  uint64_t t;
  asm volatile("mov.u64 %0, %%globaltimer;" : "=l"(t));
  return t;
}

__device__ __forceinline__ uint32_t smem_u32(const void *p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

template <typename T> __device__ __forceinline__ float to_f32(T v);
template <> __device__ __forceinline__ float to_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ float to_f32<__half>(__half v) { return __half2float(v); }
template <> __device__ __forceinline__ float to_f32<__nv_bfloat16>(__nv_bfloat16 v) {
  return __bfloat162float(v);
}
template <typename T> __device__ __forceinline__ T from_f32(float v);
template <> __device__ __forceinline__ float from_f32<float>(float v) { return v; }
template <> __device__ __forceinline__ __half from_f32<__half>(float v) { return __float2half_rn(v); }
template <> __device__ __forceinline__ __nv_bfloat16 from_f32<__nv_bfloat16>(float v) {
  return __float2bfloat16_rn(v);
}

// ------------------------------------------------------------- mbarrier ---
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}
__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}
__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
  asm volatile("{\n\t.reg .b64 st;\n\tmbarrier.arrive.shared::cta.b64 st, [%0];\n\t}" ::"r"(bar)
               : "memory");
}
__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
  asm volatile(
      "{\n\t.reg .b64 st;\n\tmbarrier.arrive.expect_tx.shared::cta.b64 st, [%0], %1;\n\t}" ::"r"(bar),
      "r"(bytes)
      : "memory");
}
__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity)
      : "memory");
  return ok != 0;
}

// The same test, but a thread whose phase is not complete is suspended until
// it completes or `sleep_ns` nanoseconds pass (the suspend-time hint).  A
// waiting thread that polls without it keeps issuing instructions and takes
// issue slots from the warps doing the work on its SM sub-partition.
__device__ __forceinline__ bool mbar_try_wait_sleep(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(sleep_ns)
      : "memory");
  return ok != 0;
}
// Longest single suspension of a waiting thread: the abort flag and the
// timeout are checked at least this often.
constexpr uint32_t kWaitSleepNs = 1000000u;

// Wait until the phase of parity `parity` of barrier `bar` has completed.
// Gives up (returns false) when *abort becomes non-zero or when the wait has
// lasted longer than ctl.timeout_ns; in the latter case it raises *abort and
// records kStTimeout.  No wait in this library is unbounded.
__device__ __forceinline__ bool mbar_wait(uint32_t bar, uint32_t parity, volatile int *abort,
                                          const DevCtl &ctl) {
  if (mbar_try_wait(bar, parity)) return true;
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > ctl.timeout_ns) {
      *abort = 1;
      record_status(ctl.status, kStTimeout);
      return false;
    }
  }
}

// mbar_wait for a barrier whose phase is completed by a thread of the other
// CTA of the pair with a cluster-scope release: the test acquires at cluster
// scope, so what that thread could see is visible here afterwards.
__device__ __forceinline__ bool mbar_try_wait_acq_cluster(uint32_t bar, uint32_t parity, uint32_t sleep_ns) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\tmbarrier.try_wait.parity.acquire.cluster.shared::cta.b64 p, [%1], %2, %3;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(bar), "r"(parity), "r"(sleep_ns)
      : "memory");
  return ok != 0;
}
__device__ __forceinline__ bool mbar_wait_acq_cluster(uint32_t bar, uint32_t parity, volatile int *abort,
                                                      const DevCtl &ctl) {
  const uint64_t t0 = globaltimer();
  for (;;) {
    if (mbar_try_wait_acq_cluster(bar, parity, kWaitSleepNs)) return true;
    if (*abort) return false;
    if (globaltimer() - t0 > ctl.timeout_ns) {
      *abort = 1;
      record_status(ctl.status, kStTimeout);
      return false;
    }
  }
}

// Same, bounded by `ns` only (used while draining after an abort).
__device__ __forceinline__ bool mbar_wait_for(uint32_t bar, uint32_t parity, uint64_t ns) {
  const uint64_t t0 = globaltimer();
  while (!mbar_try_wait_sleep(bar, parity, kWaitSleepNs)) {
    if (globaltimer() - t0 > ns) return false;
  }
  return true;
}

// ------------------------------------------------------------------ TMA ---
__device__ __forceinline__ void tma_prefetch_desc(const void *map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(map) : "memory");
}
// 3-D tiled bulk tensor load into this CTA's shared memory; completes
// `bytes` of transaction count on `bar`.  c0 is the innermost coordinate.
__device__ __forceinline__ void tma_load_3d(uint32_t dst, const void *map, uint32_t bar, int c0,
                                            int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// ---------------------------------------------------- CTA pair (cluster) ---
__device__ __forceinline__ uint32_t cluster_rank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}
// Address, in the cluster's shared window, of the same shared-memory offset in
// CTA `rank` of this cluster.
__device__ __forceinline__ uint32_t map_to_cta(uint32_t smem_addr, uint32_t rank) {
  uint32_t r;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(r) : "r"(smem_addr), "r"(rank));
  return r;
}
// Cluster-wide barrier (every thread of both CTAs); the warp is reconverged
// first and the per-thread form is used, so diverged warps are fine.
__device__ __forceinline__ void cluster_sync() {
  __syncwarp();
  asm volatile("barrier.cluster.arrive.release;\n\tbarrier.cluster.wait.acquire;" ::: "memory");
}
// Arrive once on a barrier given by its shared::cluster address (possibly in
// the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// The same arrival without release semantics: it publishes no generic-proxy
// writes, only that the arriving thread got this far.  A cluster-scope
// release costs a few hundred cycles on sm_100; where the only work to order
// is the arriving thread's own tcgen05.ld/st, already completed by
// tcgen05.wait::ld / wait::st, the relaxed form carries the hand-off.
__device__ __forceinline__ void mbar_arrive_cluster_relaxed(uint32_t cluster_bar) {
  asm volatile("mbarrier.arrive.relaxed.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_bar) : "memory");
}
// 3-D tiled TMA load issued by one CTA of a pair into its own shared memory,
// completing `bytes` of transaction count on a barrier that may live in the
// other CTA of the pair (given by its shared::cluster address).
__device__ __forceinline__ void tma_load_3d_pair(uint32_t dst, const void *map, uint32_t cluster_bar, int c0,
                                                 int c1, int c2) {
  asm volatile(
      "cp.async.bulk.tensor.3d.cta_group::2.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      " [%0], [%1, {%3, %4, %5}], [%2];" ::"r"(dst),
      "l"(map), "r"(cluster_bar), "r"(c0), "r"(c1), "r"(c2)
      : "memory");
}

// -------------------------------------------------------------- tcgen05 ---
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_alloc_pair(uint32_t dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// has completed.
__device__ __forceinline__ void tc_commit(uint32_t bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                   bar)
               : "memory");
}
// Pair form: arrive once on the barrier at offset `bar` in every CTA of
// `cta_mask` when the tcgen05 operations issued so far have completed.
__device__ __forceinline__ void tc_commit_pair(uint32_t bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64 [%0], %1;" ::"r"(
          bar),
      "h"(cta_mask)
      : "memory");
}
// Pair MMA issued by the leader CTA: A rows and B rows are split across the
// two CTAs at the same shared-memory offsets, each CTA's TMEM receives its own
// rows of D.
__device__ __forceinline__ void tc_mma_f16_pair(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                                uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}
// D[tmem] (+)= A[smem desc] * B[smem desc]^T, fp16/bf16 inputs, fp32 accumulate.
__device__ __forceinline__ void tc_mma_f16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc,
                                           uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\tsetp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Shared-memory matrix descriptor for a K-major operand stored with the
// 128-byte swizzle: rows of 128 B, 8-row groups 1024 B apart (stride byte
// offset), leading byte offset unused (1), descriptor version 1 (sm_100),
// layout type 2 = SWIZZLE_128B.  The tile base must be 1024-byte aligned; a
// K step of 16 two-byte elements advances the start address by 32 B.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t saddr) {
  return (uint64_t)((saddr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, A and B
// of the same 16-bit type (0 = fp16, 1 = bf16), both K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_f16(int ab_fmt, int M, int N) {
  return (1u << 4) | ((uint32_t)ab_fmt << 7) | ((uint32_t)ab_fmt << 10) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// tcgen05.ld, shape 32x32b, 32 repetitions: thread i of the warp receives
// 32 consecutive 32-bit columns of TMEM lane (warp quarter base + i).
#define FK_TMEM_LD32(taddr, v)                                                                  \
  asm volatile(                                                                                 \
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"  \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"        \
      : "=r"(v[0]), "=r"(v[1]), "=r"(v[2]), "=r"(v[3]), "=r"(v[4]), "=r"(v[5]), "=r"(v[6]),     \
        "=r"(v[7]), "=r"(v[8]), "=r"(v[9]), "=r"(v[10]), "=r"(v[11]), "=r"(v[12]), "=r"(v[13]), \
        "=r"(v[14]), "=r"(v[15]), "=r"(v[16]), "=r"(v[17]), "=r"(v[18]), "=r"(v[19]),           \
        "=r"(v[20]), "=r"(v[21]), "=r"(v[22]), "=r"(v[23]), "=r"(v[24]), "=r"(v[25]),           \
        "=r"(v[26]), "=r"(v[27]), "=r"(v[28]), "=r"(v[29]), "=r"(v[30]), "=r"(v[31])            \
      : "r"(taddr))

// tcgen05.st, shape 32x32b, 32 repetitions: thread i writes 32 consecutive
// columns of TMEM lane (warp quarter base + i).
#define FK_TMEM_ST32(taddr, v)                                                                  \
  asm volatile(                                                                                 \
      "tcgen05.st.sync.aligned.32x32b.x32.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,"  \
      "%14,%15,%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31,%32};"            \
      ::"r"(taddr), "r"(v[0]), "r"(v[1]), "r"(v[2]), "r"(v[3]), "r"(v[4]), "r"(v[5]), "r"(v[6]), \
      "r"(v[7]), "r"(v[8]), "r"(v[9]), "r"(v[10]), "r"(v[11]), "r"(v[12]), "r"(v[13]),          \
      "r"(v[14]), "r"(v[15]), "r"(v[16]), "r"(v[17]), "r"(v[18]), "r"(v[19]), "r"(v[20]),        \
      "r"(v[21]), "r"(v[22]), "r"(v[23]), "r"(v[24]), "r"(v[25]), "r"(v[26]), "r"(v[27]),        \
      "r"(v[28]), "r"(v[29]), "r"(v[30]), "r"(v[31])                                            \
      : "memory")

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Wait for every tcgen05.ld of this thread.  The registers are listed as
// read-write operands so the compiler cannot move their uses above the wait.
#define FK_TMEM_WAIT_LD(v)                                                                       \
  asm volatile("tcgen05.wait::ld.sync.aligned;"                                                  \
               : "+r"(v[0]), "+r"(v[1]), "+r"(v[2]), "+r"(v[3]), "+r"(v[4]), "+r"(v[5]),         \
                 "+r"(v[6]), "+r"(v[7]), "+r"(v[8]), "+r"(v[9]), "+r"(v[10]), "+r"(v[11]),       \
                 "+r"(v[12]), "+r"(v[13]), "+r"(v[14]), "+r"(v[15]), "+r"(v[16]), "+r"(v[17]),   \
                 "+r"(v[18]), "+r"(v[19]), "+r"(v[20]), "+r"(v[21]), "+r"(v[22]), "+r"(v[23]),   \
                 "+r"(v[24]), "+r"(v[25]), "+r"(v[26]), "+r"(v[27]), "+r"(v[28]), "+r"(v[29]),   \
                 "+r"(v[30]), "+r"(v[31])                                                        \
               :                                                                                 \
               : "memory")

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}

}  // namespace fk
