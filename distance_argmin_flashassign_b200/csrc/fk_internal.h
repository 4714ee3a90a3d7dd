// fk_internal.h -- host-side interface between the C ABI (fk_api.cu) and the
// kernel files.  Every launcher enqueues on `s`, counts its launches and
// returns the CUDA error of the launch.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "fk_common.cuh"

namespace fk {

void count_launches(int n);
// Set the calling thread's last error (fk_get_last_error / fk_last_error_message).
int record_error(int status, const char *msg);

constexpr int kMaxD = 1024;        // largest D the library accepts
constexpr int kCentroidPad = 256;  // centroid tile of the tensor-core kernel
inline int pad_k(int K) { return (K + kCentroidPad - 1) / kCentroidPad * kCentroidPad; }
// Floats of prepared bias per (padded) centroid: three tf32-exact terms of
// -|c|^2/2, then zeros, one 32-byte row per centroid (the K = 8 operand of a
// tf32 MMA step).
constexpr int kBiasTerms = 8;
inline size_t bias_bytes(int B, int K) { return (size_t)B * pad_k(K) * kBiasTerms * sizeof(float); }
inline size_t dtype_size(DType dt) { return dt == kF32 ? 4 : 2; }

// ---- assign_tf32.cu: fp32 assignment on tensor cores (three tf32 passes) ---
bool tf32_shape_ok(int D);
size_t tf32_workspace_bytes(int64_t N, int D, int K);
// One problem; ws of tf32_workspace_bytes(N, D, K).  cudaErrorNotSupported when
// the shape or the tensor maps do not fit.
// x_split: the workspace already holds X's split and |x|^2 (from
// launch_tf32_split_points on the same X), so only C is split.
cudaError_t launch_assign_tf32(const float *X, const float *C, const float *bias, int N, int D, int K, int Kpad,
                               int32_t *labels, float *mindist, NearTies ties, void *ws, DevCtl ctl, int num_sms,
                               cudaStream_t s, bool x_split = false);
// The split of X (hi, lo) and |x|^2 into the workspace of launch_assign_tf32.
cudaError_t launch_tf32_split_points(const float *X, int N, int D, void *ws, cudaStream_t s);

// ---- fused.cu: single-pass Lloyd iterations (centroids in shared memory) ---
// True when K x D fits the single-pass kernel's shared memory.
bool lloyd_fused_fits(int K, int D);
size_t lloyd_fused_workspace_bytes(int K, int D, int num_sms);
// `iters` Lloyd iterations of one problem in one cooperative launch (semantics
// of fk_lloyd).  cudaErrorNotSupported when the shape does not fit.
cudaError_t launch_lloyd_fused(DType dt, const void *X, int N, int D, int K, float *C, int32_t *labels,
                               float *mindist, int32_t *counts, int iters, void *ws, DevCtl ctl, int num_sms,
                               cudaStream_t s);

// ---- prep.cu: centroid bias (row norms of the assignment stage) -----------
// bias[b*Kpad + j] = -|C[b][j]|^2 / 2 in fp32 for j < K, -inf for K <= j < Kpad.
cudaError_t launch_bias(DType dt, const void *C, int B, int K, int Kpad, int D, float *bias,
                        cudaStream_t s);
// xnorm[r] = |X[r]|^2 (fp32) for the `rows` rows of D elements of X.
cudaError_t launch_point_norms(DType dt, const void *X, long long rows, int D, float *xnorm, cudaStream_t s);
// p[0 .. n) = v.
cudaError_t launch_fill_f32(float *p, long long n, float v, cudaStream_t s);
// Cdt = C32 rounded to dt (round-to-nearest-even) and bias of Cdt.
cudaError_t launch_round_bias(DType dt, const float *C32, int B, int K, int Kpad, int D, void *Cdt,
                              float *bias, cudaStream_t s);

// Relative width of the near-tie test of the CUDA-core kernel for rows of D
// dimensions: (D + 8) units of fp32 rounding, the classical bound on the
// error of an fp32 sum of D + 8 terms (the squared differences), times the
// magnitude summed (the two distances).
inline float near_tie_tau_simt(int D) { return (float)(D + 8) * 5.9604644775390625e-8f; }
// The same for the tensor-core kernel: 16 units of fp32 rounding (2^-20)
// times a bound on |x|^2 + |c|^2 for rows of up to 128 dimensions, scaled by
// D / 128 above that (the accumulation error grows with the number of
// products summed).  Its accumulation order is the hardware's; on the five
// workloads no point whose score gap exceeded 1.3e-7 (|x|^2 + |c|^2) was
// misordered, eight times below this width.
constexpr float kNearTieTauTc = 9.5367431640625e-7f;
inline float near_tie_tau_tc(int D) { return D > 128 ? kNearTieTauTc * (float)D / 128.f : kNearTieTauTc; }
// The fp32 tensor-core path (three tf32 passes) adds the split's error, below
// 2.5 2^-21 of sum |x_j c_j| (the dropped lo x lo product and the lo parts'
// own tf32 rounding): four times the 16-bit path's width.
inline float near_tie_tau_tf32(int D) { return 4.f * near_tie_tau_tc(D); }

// ---- assign_simt.cu: CUDA-core assignment (any dtype, any D) --------------
cudaError_t launch_assign_simt(DType dt, const void *X, const void *C, int B, int N, int D, int K,
                               int32_t *labels, float *mindist, NearTies ties, cudaStream_t s);

// ---- Gauss sums: sum_k w_k exp(-beta |x_i - c_k|^2) ------------------------
// Bias of the tensor-core Gauss-sum epilogue for the weights of one sign
// (prep.cu); one problem.
cudaError_t launch_gauss_bias(DType dt, const void *C, int K, int Kpad, int D, const float *w, int sign, float beta,
                              float *bias, cudaStream_t s);
// Tensor-core pass (assign_tc.cu): ln and/or value of the sum of one sign part.
cudaError_t launch_gauss_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N, int D, int K,
                            int Kpad, const float *xnorm, float beta, float *log_out, float *val_out, DevCtl ctl,
                            int num_sms, cudaStream_t s);
// CUDA-core pass (gauss.cu) for the other inputs.
cudaError_t launch_gauss_simt(DType dt, const void *X, const void *C, int N, int D, int K, const float *w, int sign,
                              float beta, float *log_out, float *val_out, cudaStream_t s);
// G = e^lp - e^ln and ln G (gauss.cu).
cudaError_t launch_gauss_combine(const float *lp, const float *ln, int N, float *log_out, float *val_out,
                                 cudaStream_t s);

// ---- seed.cu: k-means++ seeding ---------------------------------------------
size_t seed_workspace_bytes(int64_t N, int D, int K);
// centers[0..K) from the caller's uniforms u_host[0..K) (host memory).
cudaError_t launch_seed(DType dt, const void *X, int N, int D, int K, const double *u_host, int32_t *centers, void *ws,
                        cudaStream_t s);

// ---- refine.cu: exact re-decision of listed near-ties ---------------------
cudaError_t launch_refine(DType dt, const void *X, const void *C, int N, int D, int K, NearTies t,
                          int32_t *labels, float *mindist, int num_sms, cudaStream_t s);

// ---- assign_tc.cu: tcgen05 assignment (fp16/bf16, D % 8 == 0, D <= 128) --
bool tc_shape_ok(DType dt, int D);
bool tc_aligned(const void *X, const void *C);
// Returns cudaErrorNotSupported if the tensor maps could not be encoded.
// xnorm: |x|^2 per row (B*N floats), or null (computed in the kernel).
cudaError_t launch_assign_tc(DType dt, const void *X, const void *C, const float *bias, int B, int N,
                             int D, int K, int Kpad, const float *xnorm, int32_t *labels, float *mindist,
                             NearTies ties, DevCtl ctl, int num_sms, cudaStream_t s);

// ---- update.cu: sort-inverse update ---------------------------------------
enum UpdateMode : int { kMean = 0, kAccumulate = 1 };
struct UpdateArgs {
  DType dt;
  const void *X;          // B*N rows of D elements
  const int32_t *labels;  // B*N
  int B, N, D, K;
  float *C;               // kMean: B*K x D fp32 in/out
  int32_t *counts;        // kMean: B*K or null
  double *acc;            // kAccumulate: B*K x D fp64 running sums
  long long *cnt;         // kAccumulate: B*K running counts
  UpdateMode mode;
};
// Device workspace of launch_update for B problems of Ntot / B points and
// Ktot / B clusters each.
size_t update_workspace_bytes(int64_t Ntot, int64_t Ktot, int D, int B);
cudaError_t launch_update(const UpdateArgs &a, void *ws, size_t ws_bytes, DevCtl ctl,
                          int num_sms, cudaStream_t s);
// C[k] = acc[k] / cnt[k] (fp32) where cnt[k] > 0, counts[k] = cnt[k]; acc and
// cnt are reset to zero.
cudaError_t launch_divide_accumulated(double *acc, long long *cnt, int Ktot, int D, float *C,
                                      int32_t *counts, cudaStream_t s);

// ---- fk_api.cu: timeout self-test kernel -----------------------------------
cudaError_t launch_wait_probe(DevCtl ctl, cudaStream_t s);

}  // namespace fk
