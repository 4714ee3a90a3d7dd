/*
 * fk.h -- C ABI of libfk, exact Lloyd k-means on NVIDIA B200 (sm_100a).
 *
 * The operation is the one "Flash-KMeans: Fast and Memory-Efficient Exact
 * K-Means" (arXiv 2603.09229) states in its abstract: one Lloyd iteration is an
 * assignment stage (the nearest of K centroids for each of N points in D
 * dimensions) followed by a centroid-update stage (each centroid becomes the
 * mean of the points assigned to it), computed exactly -- the k-means math is
 * unchanged, only the execution is reorganised (same abstract; the Japanese
 * Hacker News summary, section "what Flash-KMeans changes"):
 *   - FlashAssign fuses the distance computation with an online argmin, so the
 *     N x K distance matrix is never written to HBM;
 *   - the sort-inverse update groups points by cluster id (an inverse map with
 *     segment offsets) and sums each segment locally instead of scattering
 *     atomics into the centroid sums;
 *   - chunked-stream overlap streams inputs larger than device memory from the
 *     host, overlapping the copy of one chunk with the compute of another.
 *
 * Conventions shared by every entry point
 *   Layout     X is row-major N x D (batched: B x N x D, problem-major);
 *              centroids K x D (batched B x K x D); labels N (B x N) int32;
 *              everything contiguous, no strides.
 *   dtype      FK_F32, FK_F16 or FK_BF16 tags the element type of X (and of C
 *              where C is given in the input type).  Arithmetic accumulates in
 *              fp32.  fp16/bf16 assignment runs on tcgen05 tensor cores when
 *              D is a multiple of 8 and 8 <= D <= 256; fp32 assignment of one
 *              problem with D a multiple of 4 (16-byte aligned X and C) runs on
 *              them as three tf32 passes on split hi/lo operands; every other
 *              case runs on a CUDA-core kernel.
 *   Distances  label[i] = argmin_k |x_i - c_k|^2 with ties to the LOWEST k
 *              (the pages are silent on ties).  mindist[i] = that squared
 *              distance, clamped at 0.  The tensor path ranks by
 *              <x,c> - |c|^2/2 in fp32 (mindist = |x|^2 - 2 * best score).
 *   Exactness  Every assignment ends with an exact re-decision of the
 *              points whose best and second-best fp32 values lie within the
 *              fp32 rounding width of each other: their distances to the
 *              centroids of the two 32-centroid chunks holding those values
 *              (or to every centroid, when a third chunk is as close) are
 *              recomputed as sum_j (x_j - c_j)^2 in fp64, j ascending, and
 *              the first minimum is taken; such a point's mindist is that
 *              fp64 distance rounded to fp32.  The labels are then those of
 *              the fp64 definition on the same (rounded) inputs.
 *   Update     C_k = mean of the points with label k, in fp32; a cluster
 *              that receives no point keeps its previous centroid and gets
 *              count 0 (the pages are silent on empty clusters).
 *   Memory     Pointers documented as "device" must be device memory of the
 *              current CUDA device; "host" means host memory (pinned memory
 *              gives asynchronous copies, pageable memory still works).  All
 *              device arrays are owned by the caller.  The library keeps a
 *              per-(device, stream) scratch cache that it grows on demand with
 *              stream-ordered allocation; fk_release_workspace() returns it.
 *              Device pointers to X and C must be 16-byte aligned for the
 *              tensor-core path (else the CUDA-core kernel is used).
 *   Streams    stream is a cudaStream_t (NULL = legacy default stream).
 *              fk_assign / fk_update and their batched forms only enqueue work
 *              and return; fk_lloyd* and fk_lloyd_ooc synchronise the stream
 *              before returning.  Calls that share a device and a stream are
 *              ordered; concurrent calls on different streams use separate
 *              scratch.
 *   Errors     Every entry point returns an fk_status.  Argument errors are
 *              detected on the host before any work is enqueued (nothing is
 *              written).  Errors found on the device (a label outside [0, K)
 *              given to fk_update, a wait that ran out of time) are recorded in
 *              a per-device status word that fk_sync() returns and clears;
 *              the synchronous entry points return it themselves.
 *              fk_last_error_message() describes the last non-OK status of
 *              the calling thread.
 *   Limits     1 <= D <= 1024; 1 <= K <= 2^22 (B*K <= 2^22); 1 <= B <= 65535;
 *              0 <= N, B*N < 2^31; K <= N is NOT required.
 */
#ifndef FK_H_
#define FK_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define FK_API __attribute__((visibility("default")))
#else
#define FK_API
#endif

typedef struct CUstream_st *fk_stream_t; /* identical to cudaStream_t */

typedef enum { FK_F32 = 0, FK_F16 = 1, FK_BF16 = 2 } fk_dtype;

typedef int fk_status;
enum {
  FK_OK = 0,
  FK_ERR_INVALID_ARG = -1, /* bad pointer, size or dtype                       */
  FK_ERR_UNSUPPORTED = -2, /* valid request the library cannot serve          */
  FK_ERR_CUDA = -3,        /* a CUDA runtime call failed (no device, launch)   */
  FK_ERR_OOM = -4,         /* device or pinned allocation failed               */
  FK_ERR_TIMEOUT = -5,     /* a device-side wait exceeded its time limit       */
  FK_ERR_HOST_IO = -6,     /* a host<->device copy failed (out-of-core path)   */
  FK_ERR_BAD_LABEL = -7    /* fk_update saw a label outside [0, K)             */
};

/* ------------------------------------------------------------------------
 * fk_assign -- assignment stage (FlashAssign).
 *   Flash-KMeans abstract: FlashAssign computes each distance and folds it
 *   into a running argmin on chip, so the N x K distances are never stored.
 *   X        device, N x D, dtype dt
 *   C        device, K x D, dtype dt (centroids already in the input type)
 *   labels   device, N int32 (out)
 *   mindist  device, N fp32 (out) or NULL
 *   N may be 0 (nothing is launched).
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_assign(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K,
                    int32_t *labels, float *mindist, fk_stream_t stream);

/* fk_assign_batched -- B independent assignment problems in one launch.
 *   Flash-KMeans abstract (FlashAssign) applied per problem; the batch of
 *   independent problems in one launch is this library's reading of the
 *   batched online-clustering use the Flash-KMeans pages motivate.
 *   X B x N x D, C B x K x D, labels B x N, mindist B x N or NULL (device).
 *   Problem b compares rows of X[b] only with centroids of C[b]; labels are
 *   in [0, K) within each problem. */
FK_API fk_status fk_assign_batched(const void *X, int B, int64_t N, int D, fk_dtype dt, const void *C,
                            int K, int32_t *labels, float *mindist, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * Two-phase assignment for callers that iterate (Lloyd loops, benchmarks).
 *
 * fk_bias_len -- number of floats of the prepared bias for B problems of K
 *   centroids: 8 per centroid, K rounded up to the 256-centroid tile, per
 *   problem.
 * fk_prepare_centroids -- the preparation step of the assignment stage:
 *   C_dt = C32 rounded to dt (round-to-nearest-even; a plain copy for
 *   FK_F32, skipped when C_dt == C32) and the bias b_k = -|C_dt[k]|^2 / 2,
 *   computed in fp32.  The tensor-core kernel ranks centroids by
 *   <x, c> + b, which orders them exactly as the squared distance does; its
 *   tensor cores add b themselves, so each centroid's bias is stored as a
 *   32-byte row of 8 floats: three terms that tf32 holds exactly and whose
 *   sum is b exactly, then five zeros.  Padded centroids get (-inf, 0, ...)
 *   so they never win.  One kernel.
 *   C32 device B x K x D fp32; C_dt device B x K x D of dt; bias device
 *   fk_bias_len(B, K) floats, 16-byte aligned for the tensor-core path (a
 *   less aligned bias sends fk_assign_prepared to the CUDA-core kernel).
 * fk_prepare_points -- the row norms of the assignment stage:
 *   xnorm[i] = |x_i|^2 in fp32 for the B*N rows of X (device, B x N x D of
 *   dt; xnorm device, B*N floats).  X does not change between Lloyd
 *   iterations, so an iterating caller computes this once.  One kernel.
 * fk_assign_prepared -- fk_assign_batched against prepared centroids and
 *   bias, and optionally the prepared row norms (xnorm, or NULL: the
 *   tensor-core kernel then sums them from its X tiles).  Launches two
 *   kernels: the assignment kernel (the CUDA-core kernel, which computes
 *   direct differences, reads neither the bias nor xnorm) and the exact
 *   re-decision of near-ties (see "Exactness" below).
 * ------------------------------------------------------------------------ */
FK_API int64_t fk_bias_len(int B, int K);
FK_API fk_status fk_prepare_centroids(const float *C32, int B, int K, int D, fk_dtype dt, void *C_dt,
                                      float *bias, fk_stream_t stream);
FK_API fk_status fk_prepare_points(const void *X, int B, int64_t N, int D, fk_dtype dt, float *xnorm,
                                   fk_stream_t stream);
FK_API fk_status fk_assign_prepared(const void *X, int B, int64_t N, int D, fk_dtype dt, const void *C_dt,
                                    int K, const float *bias, const float *xnorm, int32_t *labels,
                                    float *mindist, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_update -- centroid-update stage (sort-inverse update).
 *   Flash-KMeans abstract: the update builds an explicit inverse map from
 *   clusters to their points and sums each cluster's segment locally instead
 *   of scattering contended atomics.  Here: a stable radix sort of the labels gives the inverse
 *   map (point ids grouped by cluster) and segment offsets; each segment is
 *   summed in fp32 by contention-free reductions, partial sums of segments
 *   that cross work-chunk borders are combined in a fixed order (the result is
 *   deterministic), and divided by the count.
 *   X        device, N x D, dtype dt
 *   labels   device, N int32, each in [0, K)
 *   C        device, K x D fp32, in: previous centroids, out: new centroids
 *            (rows of empty clusters are left untouched)
 *   counts   device, K int32 (out) or NULL
 *   A label outside [0, K) is counted in cluster 0 and reported as
 *   FK_ERR_BAD_LABEL by fk_sync().
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_update(const void *X, const int32_t *labels, int64_t N, int D, fk_dtype dt, int K,
                    float *C, int32_t *counts, fk_stream_t stream);

/* fk_update_batched -- B independent update problems (labels B x N, C B x K
 * x D fp32 in/out, counts B x K or NULL), one sort over B*K segments.
 * Flash-KMeans abstract (sort-inverse update) applied per problem, in one
 * launch per kernel for the whole batch. */
FK_API fk_status fk_update_batched(const void *X, const int32_t *labels, int B, int64_t N, int D,
                            fk_dtype dt, int K, float *C, int32_t *counts, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_update_noalloc -- fk_update for callers that must not allocate.
 *   The paper has no counterpart: this entry point exists for users whose
 *   code cannot tolerate a library allocating device memory (work recorded
 *   under CUDA stream capture, frameworks that own all device memory through
 *   their own pool, loops that cannot afford an allocation or the implicit
 *   synchronisation of freeing).  It computes exactly what fk_update computes
 *   for one problem, with the same kernels and the same arguments, but takes
 *   its scratch from a 32 MiB array compiled into the library instead of the
 *   allocation cache; it calls no cudaMalloc, cudaFree or other allocating
 *   routine.
 *   Limits: the scratch needed, 16 N + 4 2^b ceil(N / 4096) + 4 (K + 1) +
 *   8 D ceil(N / R) bytes (b: bits per sort pass, at most 11; R >= 128 rows
 *   per gather worker), must fit the 32 MiB array less 256 bytes -- about
 *   1.55 million points at D = 128 and K = 1,024, about 0.41 million at
 *   D = 1,024; larger requests return FK_ERR_UNSUPPORTED with the needed size
 *   in fk_last_error_message().
 *   Set-up: the first call on each device looks up the array's device address
 *   (no allocation); make that first call before any stream capture.  A
 *   failed lookup is retried by the next call.  The
 *   array exists on every device where the library's code was loaded and is
 *   held until the process exits.
 *   Sharing: all calls in the process share the one array and it keeps the
 *   last call's contents; calls that can overlap on the GPU (different
 *   streams, or different host threads on one device) race and corrupt each
 *   other -- order them on one stream.
 *   Errors: argument errors as fk_update.  Labels outside [0, K) are counted
 *   in cluster 0 like fk_update, but this variant does not report them
 *   through fk_sync().  Asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_update_noalloc(const void *X, const int32_t *labels, int64_t N, int D, fk_dtype dt, int K,
                                   float *C, int32_t *counts, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_assign_top2 -- the two nearest centroids of every point (soft /
 * multi-assignment of border points).
 *   Flash-GMM abstract (the "similar papers" sidebar of the FlashDiffusion
 *   page): border vectors are placed in several clusters, without a
 *   materialised point x cluster matrix.  Here the assignment stage runs
 *   twice on the fused kernels: label1[i] = argmin_k |x_i - c_k|^2 and
 *   label2[i] = argmin over k != label1[i], both with ties to the LOWEST k
 *   and both exact in the sense of fk_assign (near-ties re-decided in fp64).
 *   dist1 / dist2 (either may be NULL): those squared distances as fk_assign
 *   reports mindist.  K == 1: label2 = -1 and dist2 = +inf.
 *   X, C, label1, label2, dist1, dist2 on the device; shapes, dtypes and
 *   paths as fk_assign; label1 and label2 must not alias.  Asynchronous on
 *   `stream`.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_assign_top2(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K,
                                int32_t *label1, int32_t *label2, float *dist1, float *dist2,
                                fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_lloyd -- `iters` Lloyd iterations, device resident.
 *   Flash-KMeans abstract: one iteration is the assignment stage followed by
 *   the centroid-update stage; the Japanese Hacker News summary, key points:
 *   the k-means mathematics itself is unchanged.
 *   Iteration t assigns X against C_t rounded (round-to-nearest-even) to the
 *   input type (fp16/bf16; fp32 uses C_t as is), then sets C_{t+1} = the
 *   cluster means in fp32.  On return C holds C_iters, labels the last
 *   assignment (made against C_{iters-1}), mindist (or NULL) its squared
 *   distances and counts (or NULL) its cluster sizes.  iters >= 1.
 *   X device N x D; C device K x D fp32 in/out; labels device N int32.
 *   Synchronises `stream`; returns the first device-side error, if any.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_lloyd(const void *X, int64_t N, int D, fk_dtype dt, float *C, int K,
                   int32_t *labels, float *mindist, int32_t *counts, int iters,
                   fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_lloyd_fused -- fk_lloyd in a single pass over X per iteration, for
 * problems whose centroids fit in shared memory (K x D about 25,000 values
 * at most; FK_ERR_UNSUPPORTED otherwise).
 *   Flash-KMeans abstract: the assignment stage followed by the update
 *   stage, with chunked-stream overlap; here both stages share one read of
 *   X: each CTA adds the rows it has just assigned into its own per-cluster
 *   partial sums, and after a grid-wide barrier the partial sums are combined
 *   in CTA order and divided.  All iterations run in one cooperative launch.
 *   Labels are exact as in fk_lloyd (near-ties re-decided in fp64); the
 *   centroid sums are added in a different (fixed) order than fk_lloyd's, so
 *   C agrees with it to fp32 rounding, not bit for bit.  Arguments, results
 *   and errors as fk_lloyd.  Synchronises `stream`.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_lloyd_fused(const void *X, int64_t N, int D, fk_dtype dt, float *C, int K,
                         int32_t *labels, float *mindist, int32_t *counts, int iters,
                         fk_stream_t stream);

/* fk_lloyd_batched -- fk_lloyd over B independent problems in one launch per
 * stage (shapes as in fk_assign_batched / fk_update_batched); the iteration
 * follows the Flash-KMeans abstract for each problem. */
FK_API fk_status fk_lloyd_batched(const void *X, int B, int64_t N, int D, fk_dtype dt, float *C, int K,
                           int32_t *labels, float *mindist, int32_t *counts, int iters,
                           fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_lloyd_ooc -- out-of-core Lloyd with chunked-stream overlap.
 *   Flash-KMeans abstract ("chunked-stream overlap"); the Japanese summary
 *   adds that PCIe transfers overlap compute when the input exceeds VRAM.
 *   X_host stays in host memory: every iteration streams it in chunks of
 *   chunk_rows rows through a ring of device buffers; the copy of chunk c+1
 *   runs on a side stream while chunk c is assigned and its per-cluster sums
 *   are accumulated (fp64 accumulators, no atomics).  The iteration ends by
 *   dividing.  The result equals fk_lloyd on the same data up to the
 *   summation order of the means.
 *   X_host       host, N x D dtype dt (pinned for overlap)
 *   C_host       host, K x D fp32, in/out
 *   labels_host  host, N int32 (out, last iteration) or NULL
 *   counts_host  host, K int32 (out) or NULL
 *   chunk_rows   rows per chunk, >= 1 (clamped to N); the 2 chunk buffers and
 *                the per-chunk scratch come from the library's scratch cache
 *                for (device, stream), kept for later calls (fk_release_workspace
 *                frees it), together with a side copy stream and its events.
 *   Synchronous: returns when C_host (and labels/counts) are written.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_lloyd_ooc(const void *X_host, int64_t N, int D, fk_dtype dt, float *C_host, int K,
                       int32_t *labels_host, int32_t *counts_host, int iters, int64_t chunk_rows,
                       fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_gauss_sum -- weighted Gauss sums on the assignment engine.
 *   "Fast Gauss Sums via Flash Attention", abstract: Gauss kernel sums with
 *   arbitrary signed weights, evaluated in fused tiles without writing the
 *   N x K kernel matrix; FlashDiffusion, Figure 4 caption: the same
 *   matrix-free Gaussian kernel applied to a vector (Kv: pass C = X, w = v).
 *     G[i] = sum_k w[k] exp(-beta |x_i - c_k|^2)
 *   computed like the assignment (same tensor-core tiles, inputs in dt,
 *   fp32 accumulation), with a running log-sum-exp per point instead of the
 *   arg-min.
 *   X        device, N x D, dtype dt
 *   C        device, K x D, dtype dt
 *   w        device, K fp32, or NULL (every weight 1)
 *   w_signed 0: the weights are taken as >= 0 (negative entries count as 0),
 *            one pass over X; 1: any sign, G is the positive part less the
 *            negative part (two passes)
 *   beta     > 0
 *   G        device, N fp32 (out) or NULL; may underflow or overflow in fp32
 *   logG     device, N fp32 (out) or NULL: ln G (NaN where G <= 0)
 *   fp16/bf16 with D % 8 == 0, D <= 256 run on tcgen05; other inputs (fp32
 *   included) on a CUDA-core kernel.  Asynchronous on `stream`.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_gauss_sum(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K, const float *w,
                              int w_signed, float beta, float *G, float *logG, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * fk_seed_kmeanspp -- k-means++ seeding on the GPU.
 *   The Japanese Hacker News summary of Flash-KMeans (discussion section):
 *   seeding (k-means++) is the step before Lloyd's iterations, outside the
 *   paper's target.  Centre 0 is point floor(u[0] N); centre t is drawn with
 *   probability proportional to D2(x) = min over the centres so far of
 *   |x - c|^2, with these reproducible rules: D2 is sum_j (x_j - c_j)^2 in
 *   fp64, j ascending, each operation rounded; the weights are the integers
 *   floor(D2 2^s) with s = 61 - e - L, where the largest D2 after the first
 *   centre is m 2^e (m in [1/2, 1)) and 2^L >= N, so that the total stays
 *   below 2^61; r = floor(u[t] T) for the weights' total T
 *   (T - 1 if that rounds up to T), and the centre is the first point whose
 *   running weight exceeds r; with T = 0 it is point floor(u[t] N).
 *   X        device, N x D, dtype dt, N >= 1
 *   u        host, K doubles in [0, 1): the draws (the caller's generator)
 *   centers  device, K int32 (out): row indices of the chosen centres
 *   Scratch 8 N bytes and a little more.  One kernel per centre when a row
 *   is a whole number of 16 bytes (16-byte aligned X), two otherwise.
 *   Synchronises `stream`.
 * ------------------------------------------------------------------------ */
FK_API fk_status fk_seed_kmeanspp(const void *X, int64_t N, int D, fk_dtype dt, int K, const double *u,
                                  int32_t *centers, fk_stream_t stream);

/* ------------------------------------------------------------------------
 * Status, diagnostics and control.
 * ------------------------------------------------------------------------ */

/* Synchronise `stream`, then return and clear the current device's status
 * word (FK_ERR_BAD_LABEL, FK_ERR_TIMEOUT) or a CUDA error; FK_OK otherwise. */
FK_API fk_status fk_sync(fk_stream_t stream);

/* Static description of a status code (never NULL). */
FK_API const char *fk_status_string(fk_status s);

/* Last non-OK status returned to the calling thread (FK_OK if none), and a
 * human-readable message for it.  Reading does not clear it. */
FK_API fk_status fk_get_last_error(void);
FK_API const char *fk_last_error_message(void);

/* Number of kernels this library has launched in this process (all devices). */
FK_API uint64_t fk_launch_count(void);

/* Which assignment kernel fk_assign would run for this request:
 * 1 = tcgen05 tensor-core kernel (fp32: three tf32 passes), 2 = CUDA-core
 * kernel, or a negative status for an invalid request (or, under a forced
 * tensor path, one it cannot serve).  Host-only: queries no device; a tensor
 * answer still needs 16-byte aligned X and C at the call. */
FK_API int fk_assign_path(int64_t N, int D, fk_dtype dt, int K, int B);

/* Force the assignment kernel: 0 = automatic (default), 1 = tensor-core
 * (requests it cannot serve fail with FK_ERR_UNSUPPORTED), 2 = CUDA-core.
 * Process-wide; used by tests to compare the two kernels on one input. */
FK_API fk_status fk_set_assign_path(int path);

/* Time limit of every device-side wait loop, in nanoseconds (default 2e9).
 * A wait that exceeds it makes the kernel stop, release what it holds and
 * record FK_ERR_TIMEOUT.  0 restores the default. */
FK_API fk_status fk_set_wait_timeout_ns(uint64_t ns);

/* Self-test of the wait-timeout mechanism: runs one small kernel that waits
 * on a shared-memory barrier nothing will complete, bounded by `ns`; returns
 * the status the kernel recorded (FK_ERR_TIMEOUT when the mechanism works).
 * Synchronises `stream`. */
FK_API fk_status fk_debug_wait_timeout(uint64_t ns, fk_stream_t stream);

/* Free the scratch cached for the current device (all streams).  The caller
 * must ensure no fk_* work is still running on that device. */
FK_API fk_status fk_release_workspace(void);

/* Test hook: arm one host-side fault, which fires once and disarms itself.
 *   what = 1: in the next fk_lloyd_ooc call, chunk copy number `at` (0 = the
 *             first chunk of the first iteration, counting on across
 *             iterations) is not issued and the call fails with
 *             FK_ERR_HOST_IO, as when a copy fails: the call waits for the
 *             work it already queued on both of its streams and returns;
 *   what = 2: the next growth of the scratch cache fails as when the device
 *             is out of memory (FK_ERR_OOM; nothing is queued);
 *   what = 0: disarm.
 * Nothing is injected on the device.  Process-wide. */
FK_API fk_status fk_debug_inject(int what, int64_t at);

/* Library version, major * 10000 + minor * 100 + patch (101: 0.1.1). */
FK_API int fk_version(void);

#ifdef __cplusplus
}
#endif
#endif /* FK_H_ */
