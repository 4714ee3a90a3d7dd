// fk_api.cu -- the C ABI of libfk (see include/fk.h): argument checks, the
// per-device state (SM count, status word, scratch cache), dispatch of the
// assignment kernel, the Lloyd drivers and the out-of-core driver.
#include <atomic>
#include <cstdio>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "../../include/fk.h"
#include "fk_internal.h"

namespace fk {

static std::atomic<unsigned long long> g_launches{0};
void count_launches(int n) { g_launches.fetch_add((unsigned long long)n, std::memory_order_relaxed); }

static std::atomic<unsigned long long> g_timeout_ns{2000000000ull};
static std::atomic<int> g_assign_path{0};

// Host-side fault injection for tests (fk_debug_inject): one armed fault,
// disarmed when it fires.  Nothing is done on the device.
static std::atomic<int> g_inject{0};            // 0 none, 1 chunk copy, 2 scratch allocation
static std::atomic<long long> g_inject_at{-1};  // chunk copy number within the next out-of-core call
static bool inject_fires(int what, long long at = -1) {
  int w = what;
  if (g_inject.load() != what || (at >= 0 && g_inject_at.load() != at)) return false;
  return g_inject.compare_exchange_strong(w, 0);
}

static thread_local fk_status t_last = FK_OK;
static thread_local std::string t_msg;

static fk_status fail(fk_status s, const std::string &msg) {
  t_last = s;
  t_msg = msg;
  return s;
}

// Record a non-OK status as the calling thread's last error (used by entry
// points defined in other files).
int record_error(int status, const char *msg) { return fail(status, msg); }

static fk_status cuda_fail(cudaError_t e, const char *where) {
  const fk_status s = e == cudaErrorMemoryAllocation ? FK_ERR_OOM : FK_ERR_CUDA;
  return fail(s, std::string(where) + ": " + cudaGetErrorString(e));
}

struct Scratch {
  void *ptr = nullptr;
  size_t bytes = 0;
  // the fp32 tensor-core path's split operands (x and c as tf32 hi and lo
  // parts, |x|^2), apart from the caller's scratch
  void *aux = nullptr;
  size_t aux_bytes = 0;
  // near-tie list counters of the assignment kernels (count, done), zeroed
  // once on allocation; the re-decision kernel leaves them zero
  int *ties_ctl = nullptr;
  // out-of-core driver: side copy stream and ring events, created on first use
  cudaStream_t copy = nullptr;
  cudaEvent_t ready[2] = {nullptr, nullptr}, freed[2] = {nullptr, nullptr};
};

struct DevState {
  std::mutex mu;
  bool ready = false;
  int sms = 0;
  int *status = nullptr;
  std::map<cudaStream_t, Scratch> scratch;
};
constexpr int kMaxDevices = 64;
static DevState g_dev[kMaxDevices];

static fk_status device_state(DevState **out) {
  int dev = -1;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return cuda_fail(e, "cudaGetDevice");
  if (dev < 0 || dev >= kMaxDevices) return fail(FK_ERR_UNSUPPORTED, "device index out of range");
  DevState &d = g_dev[dev];
  std::lock_guard<std::mutex> g(d.mu);
  if (!d.ready) {
    e = cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceGetAttribute");
    e = cudaMalloc(&d.status, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMalloc(status)");
    e = cudaMemset(d.status, 0, sizeof(int));
    if (e != cudaSuccess) return cuda_fail(e, "cudaMemset(status)");
    d.ready = true;
  }
  *out = &d;
  return FK_OK;
}

static DevCtl ctl_of(const DevState &d) { return DevCtl{d.status, g_timeout_ns.load()}; }

// Scratch for (device, stream), grown with stream-ordered allocation.
static fk_status scratch(DevState &d, cudaStream_t s, size_t need, void **out) {
  std::lock_guard<std::mutex> g(d.mu);
  Scratch &w = d.scratch[s];
  if (w.bytes < need) {
    if (inject_fires(2)) return fail(FK_ERR_OOM, "scratch allocation failed (injected by fk_debug_inject)");
    if (w.ptr) cudaFreeAsync(w.ptr, s);
    w.ptr = nullptr;
    w.bytes = 0;
    const size_t want = need + need / 4 + 4096;
    cudaError_t e = cudaMallocAsync(&w.ptr, want, s);
    if (e != cudaSuccess) {
      w.ptr = nullptr;
      cudaGetLastError();
      return cuda_fail(e, "cudaMallocAsync(scratch)");
    }
    w.bytes = want;
  }
  *out = w.ptr;
  return FK_OK;
}

static fk_status aux_scratch(DevState &d, cudaStream_t s, size_t need, void **out) {
  std::lock_guard<std::mutex> g(d.mu);
  Scratch &w = d.scratch[s];
  if (w.aux_bytes < need) {
    if (inject_fires(2)) return fail(FK_ERR_OOM, "scratch allocation failed (injected by fk_debug_inject)");
    if (w.aux) cudaFreeAsync(w.aux, s);
    w.aux = nullptr;
    w.aux_bytes = 0;
    const size_t want = need + need / 4 + 4096;
    cudaError_t e = cudaMallocAsync(&w.aux, want, s);
    if (e != cudaSuccess) {
      w.aux = nullptr;
      cudaGetLastError();
      return cuda_fail(e, "cudaMallocAsync(split operands)");
    }
    w.aux_bytes = want;
  }
  *out = w.aux;
  return FK_OK;
}

// Copy stream and events of the out-of-core driver for (device, stream).
static fk_status ooc_streams(DevState &d, cudaStream_t s, Scratch **out) {
  std::lock_guard<std::mutex> g(d.mu);
  Scratch &w = d.scratch[s];
  if (!w.copy) {
    cudaError_t e = cudaStreamCreateWithFlags(&w.copy, cudaStreamNonBlocking);
    for (int i = 0; e == cudaSuccess && i < 2; ++i) {
      e = cudaEventCreateWithFlags(&w.ready[i], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&w.freed[i], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(e, "out-of-core stream/event creation");
  }
  *out = &w;
  return FK_OK;
}

static size_t al256(size_t v) { return (v + 255) / 256 * 256; }

// Bytes of scratch the near-tie list of an assignment of `rows` points takes.
static size_t ties_bytes(int64_t rows) { return al256((size_t)rows * sizeof(int2)); }

// The near-tie list of an assignment on (device, stream): `list` is scratch
// of ties_bytes(rows); the counters are allocated (and zeroed) on first use.
static fk_status near_ties(DevState &d, cudaStream_t s, void *list, int64_t rows, int D, NearTies *out) {
  int *ctl = nullptr;
  {
    std::lock_guard<std::mutex> g(d.mu);
    Scratch &w = d.scratch[s];
    if (!w.ties_ctl) {
      cudaError_t e = cudaMallocAsync((void **)&w.ties_ctl, 256, s);
      if (e == cudaSuccess) e = cudaMemsetAsync(w.ties_ctl, 0, 256, s);
      if (e != cudaSuccess) {
        if (w.ties_ctl) cudaFreeAsync(w.ties_ctl, s);
        w.ties_ctl = nullptr;
        cudaGetLastError();
        return cuda_fail(e, "cudaMallocAsync(near-tie counters)");
      }
    }
    ctl = w.ties_ctl;
  }
  out->list = (int2 *)list;
  out->cap = (int)rows;
  out->count = ctl;
  out->done = ctl + 1;
  out->count_hi = ctl + 2;
  out->tau = near_tie_tau_simt(D);
  out->excl = nullptr;
  return FK_OK;
}

static bool valid_dtype(fk_dtype dt) { return dt == FK_F32 || dt == FK_F16 || dt == FK_BF16; }

static fk_status check_sizes(int B, int64_t N, int D, int K, fk_dtype dt) {
  if (!valid_dtype(dt)) return fail(FK_ERR_INVALID_ARG, "unknown dtype");
  if (B < 1 || B > 65535) return fail(FK_ERR_INVALID_ARG, "B must be in [1, 65535]");
  if (N < 0) return fail(FK_ERR_INVALID_ARG, "N must be >= 0");
  if (D < 1 || D > 1024) return fail(FK_ERR_INVALID_ARG, "D must be in [1, 1024]");
  if (K < 1) return fail(FK_ERR_INVALID_ARG, "K must be >= 1");
  if ((long long)B * N >= (1ll << 31)) return fail(FK_ERR_INVALID_ARG, "B*N must be < 2^31");
  if ((long long)B * K > (1ll << 22)) return fail(FK_ERR_INVALID_ARG, "B*K must be <= 2^22");
  return FK_OK;
}

// 1 = tensor-core kernel (fp16/bf16: kind::f16; fp32: three tf32 passes),
// 2 = CUDA-core kernel.
static bool tensor_shape_ok(DType dt, int D) { return dt == kF32 ? tf32_shape_ok(D) : tc_shape_ok(dt, D); }
static int choose_path(DType dt, int D) {
  const int forced = g_assign_path.load();
  if (forced == 2) return 2;
  if (forced == 1) return tensor_shape_ok(dt, D) ? 1 : -1;
  return tensor_shape_ok(dt, D) ? 1 : 2;
}

// Assignment of B problems.  cn (the prepared bias of C: kBiasTerms floats per
// padded centroid) may be null, in which case the tensor path computes it into
// scratch at `cn_ws`.  `ties_ws` is scratch of ties_bytes(B * N) for the
// near-tie list; the points listed there are re-decided exactly (refine.cu)
// by a second kernel.  xnorm (|x|^2 per point) may be null: the tensor-core
// kernel then computes it from its X tiles.
static fk_status run_assign(DevState &d, DType dt, const void *X, int B, int N, int D, const void *C, int K,
                            const float *cn, float *cn_ws, void *ties_ws, const float *xnorm, int32_t *labels,
                            float *mindist, cudaStream_t s, const int32_t *excl = nullptr, bool x_split = false) {
  NearTies ties;
  fk_status st = near_ties(d, s, ties_ws, (int64_t)B * N, D, &ties);
  if (st != FK_OK) return st;
  ties.excl = excl;
  const int path = choose_path(dt, D);
  if (path < 0) return fail(FK_ERR_UNSUPPORTED, "tensor-core path forced for an unsupported shape");
  bool done = false;
  if (path == 1 && dt == kF32) {
    // fp32: three tf32 passes (one problem at a time; a batch runs on CUDA cores)
    if (B == 1 && tc_aligned(X, C) && (!cn || (uintptr_t)cn % 16 == 0)) {
      const int Kpad = pad_k(K);
      if (!cn) {
        cudaError_t e = launch_bias(dt, C, B, K, Kpad, D, cn_ws, s);
        if (e != cudaSuccess) return cuda_fail(e, "bias kernel");
        cn = cn_ws;
      }
      void *aux = nullptr;
      if ((st = aux_scratch(d, s, tf32_workspace_bytes(N, D, K), &aux)) != FK_OK) return st;
      NearTies tt = ties;
      tt.tau = near_tie_tau_tf32(D);
      cudaError_t e = launch_assign_tf32((const float *)X, (const float *)C, cn, N, D, K, Kpad, labels, mindist, tt,
                                         aux, ctl_of(d), d.sms, s, x_split);
      if (e == cudaSuccess) {
        done = true;
      } else {
        if (e != cudaErrorNotSupported) return cuda_fail(e, "tf32 tensor-core assign kernel");
        cudaGetLastError();
        if (g_assign_path.load() == 1) return fail(FK_ERR_UNSUPPORTED, "tensor maps could not be encoded");
      }
    } else if (g_assign_path.load() == 1) {
      return fail(FK_ERR_UNSUPPORTED, "the fp32 tensor-core path takes one problem with 16-byte aligned X and C");
    }
  } else if (path == 1 && tc_aligned(X, C) && (!cn || (uintptr_t)cn % 16 == 0)) {
    const int Kpad = pad_k(K);
    if (!cn) {
      cudaError_t e = launch_bias(dt, C, B, K, Kpad, D, cn_ws, s);
      if (e != cudaSuccess) return cuda_fail(e, "bias kernel");
      cn = cn_ws;
    }
    NearTies tt = ties;
    tt.tau = near_tie_tau_tc(D);
    cudaError_t e =
        launch_assign_tc(dt, X, C, cn, B, N, D, K, Kpad, xnorm, labels, mindist, tt, ctl_of(d), d.sms, s);
    if (e == cudaSuccess) {
      done = true;
    } else {
      if (e != cudaErrorNotSupported) return cuda_fail(e, "tensor-core assign kernel");
      cudaGetLastError();
      if (g_assign_path.load() == 1) return fail(FK_ERR_UNSUPPORTED, "tensor maps could not be encoded");
    }
  } else if (path == 1 && g_assign_path.load() == 1) {
    return fail(FK_ERR_UNSUPPORTED, "tensor-core path needs 16-byte aligned X, C and bias");
  }
  if (!done) {
    cudaError_t e = launch_assign_simt(dt, X, C, B, N, D, K, labels, mindist, ties, s);
    if (e != cudaSuccess) return cuda_fail(e, "CUDA-core assign kernel");
  }
  cudaError_t e = launch_refine(dt, X, C, N, D, K, ties, labels, mindist, d.sms, s);
  if (e != cudaSuccess) return cuda_fail(e, "near-tie re-decision kernel");
  return FK_OK;
}

static fk_status read_status(DevState &d, cudaStream_t s) {
  cudaError_t e = cudaStreamSynchronize(s);
  if (e != cudaSuccess) return cuda_fail(e, "cudaStreamSynchronize");
  int h = 0;
  e = cudaMemcpy(&h, d.status, sizeof(int), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "status read");
  if (h != 0) {
    cudaMemset(d.status, 0, sizeof(int));
    return fail((fk_status)h, h == FK_ERR_TIMEOUT ? "a device-side wait exceeded its time limit"
                              : h == FK_ERR_BAD_LABEL ? "a label outside [0, K) was given to the update"
                                                      : "device-side error");
  }
  return FK_OK;
}

// ------------------------------------------------------------ wait probe --
__global__ void wait_probe_kernel(DevCtl ctl) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  if (threadIdx.x == 0) {
    mbar_init(smem_u32(&bar), 1);
    abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();
  if (threadIdx.x == 0) mbar_wait(smem_u32(&bar), 0, &abort_flag, ctl);  // nothing ever arrives
}

cudaError_t launch_wait_probe(DevCtl ctl, cudaStream_t s) {
  wait_probe_kernel<<<1, 32, 0, s>>>(ctl);
  count_launches(1);
  return cudaGetLastError();
}

}  // namespace fk

using namespace fk;

// =================================================================== ABI ===
extern "C" {

fk_status fk_assign_batched(const void *X, int B, int64_t N, int D, fk_dtype dt, const void *C, int K,
                            int32_t *labels, float *mindist, fk_stream_t stream) {
  fk_status st = check_sizes(B, N, D, K, dt);
  if (st != FK_OK) return st;
  if (N == 0) return FK_OK;
  if (!X || !C || !labels) return fail(FK_ERR_INVALID_ARG, "X, C and labels must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void *ws = nullptr;
  const size_t cnb = al256(bias_bytes(B, K));
  if ((st = scratch(*d, s, cnb + ties_bytes((int64_t)B * N), &ws)) != FK_OK) return st;
  return run_assign(*d, (DType)dt, X, B, (int)N, D, C, K, nullptr, (float *)ws, (char *)ws + cnb, nullptr, labels,
                    mindist, s);
}

fk_status fk_assign(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K, int32_t *labels,
                    float *mindist, fk_stream_t stream) {
  return fk_assign_batched(X, 1, N, D, dt, C, K, labels, mindist, stream);
}

fk_status fk_assign_top2(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K, int32_t *label1,
                         int32_t *label2, float *dist1, float *dist2, fk_stream_t stream) {
  fk_status st = check_sizes(1, N, D, K, dt);
  if (st != FK_OK) return st;
  if (N == 0) return FK_OK;
  if (!X || !C || !label1 || !label2) return fail(FK_ERR_INVALID_ARG, "X, C, label1 and label2 must not be NULL");
  if (label1 == label2) return fail(FK_ERR_INVALID_ARG, "label1 and label2 must not alias");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void *ws = nullptr;
  const size_t cnb = al256(bias_bytes(1, K));
  if ((st = scratch(*d, s, cnb + ties_bytes(N), &ws)) != FK_OK) return st;
  const DType t = (DType)dt;
  // pass 1: the nearest centroid
  st = run_assign(*d, t, X, 1, (int)N, D, C, K, nullptr, (float *)ws, (char *)ws + cnb, nullptr, label1, dist1, s);
  if (st != FK_OK) return st;
  if (K == 1) {  // no second centroid
    cudaError_t e = cudaMemsetAsync(label2, 0xff, (size_t)N * 4, s);
    if (e == cudaSuccess && dist2) e = launch_fill_f32(dist2, N, __builtin_huge_valf(), s);
    return e == cudaSuccess ? FK_OK : cuda_fail(e, "second-label fill");
  }
  // pass 2: the nearest of the others (each point leaves its label1 out)
  return run_assign(*d, t, X, 1, (int)N, D, C, K, nullptr, (float *)ws, (char *)ws + cnb, nullptr, label2, dist2, s,
                    label1);
}

int64_t fk_bias_len(int B, int K) {
  if (B < 1 || K < 1) return 0;
  return (int64_t)B * pad_k(K) * kBiasTerms;
}

fk_status fk_prepare_centroids(const float *C32, int B, int K, int D, fk_dtype dt, void *C_dt, float *bias,
                               fk_stream_t stream) {
  fk_status st = check_sizes(B, 0, D, K, dt);
  if (st != FK_OK) return st;
  if (!C32 || !C_dt || !bias) return fail(FK_ERR_INVALID_ARG, "C32, C_dt and bias must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const DType t = (DType)dt;
  cudaError_t e;
  if (t == kF32 && C_dt == (const void *)C32)
    e = launch_bias(t, C32, B, K, pad_k(K), D, bias, s);
  else
    e = launch_round_bias(t, C32, B, K, pad_k(K), D, C_dt, bias, s);
  if (e != cudaSuccess) return cuda_fail(e, "centroid prep kernel");
  return FK_OK;
}

fk_status fk_prepare_points(const void *X, int B, int64_t N, int D, fk_dtype dt, float *xnorm,
                            fk_stream_t stream) {
  fk_status st = check_sizes(B, N, D, 1, dt);
  if (st != FK_OK) return st;
  if (N == 0) return FK_OK;
  if (!X || !xnorm) return fail(FK_ERR_INVALID_ARG, "X and xnorm must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaError_t e = launch_point_norms((DType)dt, X, (long long)B * N, D, xnorm, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "point norm kernel");
  return FK_OK;
}

fk_status fk_assign_prepared(const void *X, int B, int64_t N, int D, fk_dtype dt, const void *C_dt, int K,
                             const float *bias, const float *xnorm, int32_t *labels, float *mindist,
                             fk_stream_t stream) {
  fk_status st = check_sizes(B, N, D, K, dt);
  if (st != FK_OK) return st;
  if (N == 0) return FK_OK;
  if (!X || !C_dt || !labels || !bias) return fail(FK_ERR_INVALID_ARG, "X, C_dt, bias and labels must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void *ws = nullptr;
  if ((st = scratch(*d, s, ties_bytes((int64_t)B * N), &ws)) != FK_OK) return st;
  return run_assign(*d, (DType)dt, X, B, (int)N, D, C_dt, K, bias, nullptr, ws, xnorm, labels, mindist, s);
}

fk_status fk_update_batched(const void *X, const int32_t *labels, int B, int64_t N, int D, fk_dtype dt,
                            int K, float *C, int32_t *counts, fk_stream_t stream) {
  fk_status st = check_sizes(B, N, D, K, dt);
  if (st != FK_OK) return st;
  if (!C) return fail(FK_ERR_INVALID_ARG, "C must not be NULL");
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    if (counts) {
      cudaError_t e = cudaMemsetAsync(counts, 0, (size_t)B * K * 4, s);
      if (e != cudaSuccess) return cuda_fail(e, "cudaMemsetAsync(counts)");
    }
    return FK_OK;
  }
  if (!X || !labels) return fail(FK_ERR_INVALID_ARG, "X and labels must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  const size_t need = update_workspace_bytes((int64_t)B * N, (int64_t)B * K, D, B);
  void *ws = nullptr;
  if ((st = scratch(*d, s, need, &ws)) != FK_OK) return st;
  UpdateArgs a{};
  a.dt = (DType)dt;
  a.X = X;
  a.labels = labels;
  a.B = B;
  a.N = (int)N;
  a.D = D;
  a.K = K;
  a.C = C;
  a.counts = counts;
  a.mode = kMean;
  cudaError_t e = launch_update(a, ws, need, ctl_of(*d), d->sms, s);
  if (e != cudaSuccess) return cuda_fail(e, "update kernels");
  return FK_OK;
}

fk_status fk_update(const void *X, const int32_t *labels, int64_t N, int D, fk_dtype dt, int K, float *C,
                    int32_t *counts, fk_stream_t stream) {
  return fk_update_batched(X, labels, 1, N, D, dt, K, C, counts, stream);
}

fk_status fk_lloyd_batched(const void *X, int B, int64_t N, int D, fk_dtype dt, float *C, int K,
                           int32_t *labels, float *mindist, int32_t *counts, int iters, fk_stream_t stream) {
  fk_status st = check_sizes(B, N, D, K, dt);
  if (st != FK_OK) return st;
  if (iters < 1) return fail(FK_ERR_INVALID_ARG, "iters must be >= 1");
  if (!C) return fail(FK_ERR_INVALID_ARG, "C must not be NULL");
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) return fk_update_batched(X, labels, B, 0, D, dt, K, C, counts, stream);
  if (!X || !labels) return fail(FK_ERR_INVALID_ARG, "X and labels must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  const DType t = (DType)dt;
  const int Kpad = pad_k(K);
  const size_t upd = al256(update_workspace_bytes((int64_t)B * N, (int64_t)B * K, D, B));
  const size_t cnb = al256(bias_bytes(B, K));
  const size_t cdb = t == kF32 ? 0 : al256((size_t)B * K * D * dtype_size(t));
  const size_t tb = ties_bytes((int64_t)B * N);
  const size_t xb = t == kF32 ? 0 : al256((size_t)B * N * 4);
  void *ws = nullptr;
  if ((st = scratch(*d, s, upd + cnb + cdb + tb + xb, &ws)) != FK_OK) return st;
  float *cn = (float *)((char *)ws + upd);
  void *Cdt = t == kF32 ? (void *)C : (void *)((char *)ws + upd + cnb);
  void *tl = (char *)ws + upd + cnb + cdb;
  float *xn = t == kF32 ? nullptr : (float *)((char *)ws + upd + cnb + cdb + tb);
  if (xn) {  // |x|^2 once for all iterations (X does not change)
    cudaError_t e = launch_point_norms(t, X, (long long)B * N, D, xn, s);
    if (e != cudaSuccess) return cuda_fail(e, "point norm kernel");
  }

  UpdateArgs a{};
  a.dt = t;
  a.X = X;
  a.labels = labels;
  a.B = B;
  a.N = (int)N;
  a.D = D;
  a.K = K;
  a.C = C;
  a.counts = counts;
  a.mode = kMean;
  // fp32 on the tensor path: X's tf32 split is made once for all iterations
  bool x_split = false;
  if (t == kF32 && B == 1 && choose_path(t, D) == 1 && tc_aligned(X, C) && (uintptr_t)cn % 16 == 0) {
    void *aux = nullptr;
    if ((st = aux_scratch(*d, s, tf32_workspace_bytes(N, D, K), &aux)) != FK_OK) return st;
    cudaError_t e = launch_tf32_split_points((const float *)X, (int)N, D, aux, s);
    if (e != cudaSuccess) return cuda_fail(e, "tf32 split kernel");
    x_split = true;
  }
  for (int it = 0; it < iters; ++it) {
    {  // the centroids as the assignment reads them (fp16/bf16: rounded) and their bias
      cudaError_t e = t != kF32 ? launch_round_bias(t, C, B, K, Kpad, D, Cdt, cn, s)
                                : launch_bias(t, C, B, K, Kpad, D, cn, s);
      if (e != cudaSuccess) return cuda_fail(e, "centroid prep kernel");
    }
    st = run_assign(*d, t, X, B, (int)N, D, Cdt, K, cn, nullptr, tl, xn, labels, it == iters - 1 ? mindist : nullptr,
                    s, nullptr, x_split);
    if (st != FK_OK) return st;
    cudaError_t e = launch_update(a, ws, upd, ctl_of(*d), d->sms, s);
    if (e != cudaSuccess) return cuda_fail(e, "update kernels");
  }
  return read_status(*d, s);
}

fk_status fk_lloyd(const void *X, int64_t N, int D, fk_dtype dt, float *C, int K, int32_t *labels,
                   float *mindist, int32_t *counts, int iters, fk_stream_t stream) {
  return fk_lloyd_batched(X, 1, N, D, dt, C, K, labels, mindist, counts, iters, stream);
}

fk_status fk_lloyd_fused(const void *X, int64_t N, int D, fk_dtype dt, float *C, int K, int32_t *labels,
                         float *mindist, int32_t *counts, int iters, fk_stream_t stream) {
  fk_status st = check_sizes(1, N, D, K, dt);
  if (st != FK_OK) return st;
  if (iters < 1) return fail(FK_ERR_INVALID_ARG, "iters must be >= 1");
  if (!C) return fail(FK_ERR_INVALID_ARG, "C must not be NULL");
  if (!lloyd_fused_fits(K, D)) return fail(FK_ERR_UNSUPPORTED, "K x D is too large for the single-pass kernel");
  if (N == 0) return fk_update_batched(X, labels, 1, 0, D, dt, K, C, counts, stream);
  if (!X || !labels) return fail(FK_ERR_INVALID_ARG, "X and labels must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void *ws = nullptr;
  if ((st = scratch(*d, s, lloyd_fused_workspace_bytes(K, D, d->sms), &ws)) != FK_OK) return st;
  const cudaError_t e = launch_lloyd_fused((DType)dt, X, (int)N, D, K, C, labels, mindist, counts, iters, ws,
                                           ctl_of(*d), d->sms, s);
  if (e == cudaErrorNotSupported) {
    cudaGetLastError();
    return fail(FK_ERR_UNSUPPORTED, "the single-pass kernel cannot be made resident on this device");
  }
  if (e != cudaSuccess) return cuda_fail(e, "single-pass Lloyd kernel");
  return read_status(*d, s);
}

fk_status fk_lloyd_ooc(const void *X_host, int64_t N, int D, fk_dtype dt, float *C_host, int K,
                       int32_t *labels_host, int32_t *counts_host, int iters, int64_t chunk_rows,
                       fk_stream_t stream) {
  fk_status st = check_sizes(1, N, D, K, dt);
  if (st != FK_OK) return st;
  if (iters < 1) return fail(FK_ERR_INVALID_ARG, "iters must be >= 1");
  if (chunk_rows < 1) return fail(FK_ERR_INVALID_ARG, "chunk_rows must be >= 1");
  if (!C_host) return fail(FK_ERR_INVALID_ARG, "C_host must not be NULL");
  if (N == 0) {
    if (counts_host) memset(counts_host, 0, (size_t)K * 4);
    return FK_OK;
  }
  if (!X_host) return fail(FK_ERR_INVALID_ARG, "X_host must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  const DType t = (DType)dt;
  cudaStream_t s = (cudaStream_t)stream;
  const int64_t rows = chunk_rows < N ? chunk_rows : N;
  const int64_t nchunks = (N + rows - 1) / rows;
  const size_t es = dtype_size(t);
  const int Kpad = pad_k(K);

  // device buffers, carved from the scratch cache of (device, stream)
  const size_t b_ring = al256((size_t)rows * D * es), b_lab = al256((size_t)rows * 4);
  const size_t b_c32 = al256((size_t)K * D * 4), b_cdt = t == kF32 ? 0 : al256((size_t)K * D * es);
  const size_t b_cn = al256(bias_bytes(1, K)), b_acc = al256((size_t)K * D * 8);
  const size_t b_cnt = al256((size_t)K * 8), b_counts = al256((size_t)K * 4);
  const size_t b_upd = al256(update_workspace_bytes(rows, K, D, 1));
  const size_t b_ties = ties_bytes(rows);
  const size_t total = 2 * b_ring + 2 * b_lab + b_c32 + b_cdt + b_cn + b_acc + b_cnt + b_counts + b_upd + b_ties;

  Scratch *sc = nullptr;
  char *mem = nullptr;
  fk_status rc = FK_OK;
  cudaError_t e;
  if ((rc = ooc_streams(*d, s, &sc)) != FK_OK) return rc;
  if ((rc = scratch(*d, s, total, (void **)&mem)) != FK_OK) return rc;
  {
    cudaStream_t cs = sc->copy;
    cudaEvent_t *ready = sc->ready, *freed = sc->freed;
#define FK_TRY(call, what, code)        \
  do {                                  \
    e = (call);                         \
    if (e != cudaSuccess) {             \
      rc = code == FK_ERR_CUDA ? cuda_fail(e, what) : fail(code, std::string(what) + ": " + cudaGetErrorString(e)); \
      goto done;                        \
    }                                   \
  } while (0)
    char *p = mem;
    char *ring[2] = {p, p + b_ring};
    p += 2 * b_ring;
    int32_t *lab[2] = {(int32_t *)p, (int32_t *)(p + b_lab)};
    p += 2 * b_lab;
    float *c32 = (float *)p; p += b_c32;
    void *cdt = t == kF32 ? (void *)c32 : (void *)p; p += b_cdt;
    float *cn = (float *)p; p += b_cn;
    double *acc = (double *)p; p += b_acc;
    long long *cnt = (long long *)p; p += b_cnt;
    int32_t *cnts = (int32_t *)p; p += b_counts;
    void *tl = (void *)p; p += b_ties;
    void *upd = (void *)p;

    // Order the copy stream after everything already queued on `s` (the
    // scratch may just have been allocated there, or read by an earlier call).
    FK_TRY(cudaEventRecord(freed[0], s), "cudaEventRecord", FK_ERR_CUDA);
    FK_TRY(cudaEventRecord(freed[1], s), "cudaEventRecord", FK_ERR_CUDA);
    FK_TRY(cudaMemcpyAsync(c32, C_host, (size_t)K * D * 4, cudaMemcpyHostToDevice, s), "copy of C to the device",
           FK_ERR_HOST_IO);
    UpdateArgs a{};
    a.dt = t;
    a.B = 1;
    a.D = D;
    a.K = K;
    a.acc = acc;
    a.cnt = cnt;
    a.mode = kAccumulate;
    long long copy_no = 0;  // chunk copies issued by this call
    for (int it = 0; it < iters; ++it) {
      FK_TRY(cudaMemsetAsync(acc, 0, (size_t)K * D * 8, s), "cudaMemsetAsync", FK_ERR_CUDA);
      FK_TRY(cudaMemsetAsync(cnt, 0, (size_t)K * 8, s), "cudaMemsetAsync", FK_ERR_CUDA);
      if (t != kF32)
        FK_TRY(launch_round_bias(t, c32, 1, K, Kpad, D, cdt, cn, s), "centroid prep kernel", FK_ERR_CUDA);
      else
        FK_TRY(launch_bias(t, c32, 1, K, Kpad, D, cn, s), "centroid prep kernel", FK_ERR_CUDA);
      for (int64_t c = 0; c < nchunks; ++c) {
        const int slot = (int)(c & 1);
        const int64_t r0 = c * rows;
        const int nr = (int)((N - r0) < rows ? (N - r0) : rows);
        // copy stream: chunk c into its slot once the compute that last read the slot is done
        if (inject_fires(1, copy_no)) {
          rc = fail(FK_ERR_HOST_IO, "host-to-device copy of chunk " + std::to_string(c) + " of iteration " +
                                        std::to_string(it) + " not issued (injected by fk_debug_inject)");
          goto done;
        }
        ++copy_no;
        FK_TRY(cudaStreamWaitEvent(cs, freed[slot], 0), "cudaStreamWaitEvent", FK_ERR_CUDA);
        FK_TRY(cudaMemcpyAsync(ring[slot], (const char *)X_host + (size_t)r0 * D * es, (size_t)nr * D * es,
                               cudaMemcpyHostToDevice, cs),
               "host-to-device copy of a chunk", FK_ERR_HOST_IO);
        FK_TRY(cudaEventRecord(ready[slot], cs), "cudaEventRecord", FK_ERR_CUDA);
        // compute stream: assign the chunk and accumulate its per-cluster sums
        FK_TRY(cudaStreamWaitEvent(s, ready[slot], 0), "cudaStreamWaitEvent", FK_ERR_CUDA);
        rc = run_assign(*d, t, ring[slot], 1, nr, D, cdt, K, cn, nullptr, tl, nullptr, lab[slot], nullptr, s);
        if (rc != FK_OK) goto done;
        if (it == iters - 1 && labels_host)
          FK_TRY(cudaMemcpyAsync(labels_host + r0, lab[slot], (size_t)nr * 4, cudaMemcpyDeviceToHost, s),
                 "device-to-host copy of labels", FK_ERR_HOST_IO);
        a.X = ring[slot];
        a.labels = lab[slot];
        a.N = nr;
        FK_TRY(launch_update(a, upd, b_upd, ctl_of(*d), d->sms, s), "update kernels", FK_ERR_CUDA);
        FK_TRY(cudaEventRecord(freed[slot], s), "cudaEventRecord", FK_ERR_CUDA);
      }
      FK_TRY(launch_divide_accumulated(acc, cnt, K, D, c32, cnts, s), "divide kernel", FK_ERR_CUDA);
    }
    FK_TRY(cudaMemcpyAsync(C_host, c32, (size_t)K * D * 4, cudaMemcpyDeviceToHost, s), "copy of C to the host",
           FK_ERR_HOST_IO);
    if (counts_host)
      FK_TRY(cudaMemcpyAsync(counts_host, cnts, (size_t)K * 4, cudaMemcpyDeviceToHost, s),
             "copy of counts to the host", FK_ERR_HOST_IO);
    rc = read_status(*d, s);
  }
done:
#undef FK_TRY
  if (rc != FK_OK) {  // leave nothing of this call running on the side stream
    cudaStreamSynchronize(sc->copy);
    cudaStreamSynchronize(s);
  }
  return rc;
}

fk_status fk_gauss_sum(const void *X, int64_t N, int D, fk_dtype dt, const void *C, int K, const float *w,
                       int w_signed, float beta, float *G, float *logG, fk_stream_t stream) {
  fk_status st = check_sizes(1, N, D, K, dt);
  if (st != FK_OK) return st;
  if (!(beta > 0.f) || !(beta < 3.0e38f)) return fail(FK_ERR_INVALID_ARG, "beta must be a positive finite number");
  if (w_signed != 0 && w_signed != 1) return fail(FK_ERR_INVALID_ARG, "w_signed must be 0 or 1");
  if (w_signed && !w) return fail(FK_ERR_INVALID_ARG, "w_signed needs w");
  if (!G && !logG) return fail(FK_ERR_INVALID_ARG, "G and logG must not both be NULL");
  if (N == 0) return FK_OK;
  if (!X || !C) return fail(FK_ERR_INVALID_ARG, "X and C must not be NULL");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  const DType t = (DType)dt;
  const int Kpad = pad_k(K);
  const size_t cnb = al256(bias_bytes(1, K)), lb = w_signed ? al256((size_t)N * 4) : 0;
  void *ws = nullptr;
  if ((st = scratch(*d, s, cnb + 2 * lb, &ws)) != FK_OK) return st;
  float *bias = (float *)ws;
  float *lp = w_signed ? (float *)((char *)ws + cnb) : logG;
  float *lneg = w_signed ? (float *)((char *)ws + cnb + lb) : nullptr;
  const bool tc = choose_path(t, D) == 1 && tc_aligned(X, C);
  for (int part = 0; part < (w_signed ? 2 : 1); ++part) {
    const int sign = part == 0 ? 1 : -1;
    float *lo = part == 0 ? lp : lneg;
    float *vo = w_signed ? nullptr : G;
    cudaError_t e = cudaErrorNotSupported;
    if (tc) {
      e = launch_gauss_bias(t, C, K, Kpad, D, w, sign, beta, bias, s);
      if (e != cudaSuccess) return cuda_fail(e, "Gauss-sum bias kernel");
      e = launch_gauss_tc(t, X, C, bias, 1, (int)N, D, K, Kpad, nullptr, beta, lo, vo, ctl_of(*d), d->sms, s);
      if (e != cudaSuccess && e != cudaErrorNotSupported) return cuda_fail(e, "tensor-core Gauss-sum kernel");
      if (e != cudaSuccess) cudaGetLastError();
    }
    if (e != cudaSuccess) {
      e = launch_gauss_simt(t, X, C, (int)N, D, K, w, sign, beta, lo, vo, s);
      if (e != cudaSuccess) return cuda_fail(e, "CUDA-core Gauss-sum kernel");
    }
  }
  if (w_signed) {
    cudaError_t e = launch_gauss_combine(lp, lneg, (int)N, logG, G, s);
    if (e != cudaSuccess) return cuda_fail(e, "Gauss-sum combine kernel");
  }
  return FK_OK;
}

fk_status fk_seed_kmeanspp(const void *X, int64_t N, int D, fk_dtype dt, int K, const double *u, int32_t *centers,
                           fk_stream_t stream) {
  fk_status st = check_sizes(1, N, D, K, dt);
  if (st != FK_OK) return st;
  if (N < 1) return fail(FK_ERR_INVALID_ARG, "N must be >= 1");
  if (!X || !u || !centers) return fail(FK_ERR_INVALID_ARG, "X, u and centers must not be NULL");
  for (int t = 0; t < K; ++t)
    if (!(u[t] >= 0.0 && u[t] < 1.0)) return fail(FK_ERR_INVALID_ARG, "every u[t] must lie in [0, 1)");
  DevState *d;
  if ((st = device_state(&d)) != FK_OK) return st;
  cudaStream_t s = (cudaStream_t)stream;
  void *ws = nullptr;
  if ((st = scratch(*d, s, seed_workspace_bytes(N, D, K), &ws)) != FK_OK) return st;
  cudaError_t e = launch_seed((DType)dt, X, (int)N, D, K, u, centers, ws, s);
  if (e != cudaSuccess) return cuda_fail(e, "seeding kernels");
  return read_status(*d, s);
}

fk_status fk_sync(fk_stream_t stream) {
  DevState *d;
  fk_status st = device_state(&d);
  if (st != FK_OK) return st;
  return read_status(*d, (cudaStream_t)stream);
}

const char *fk_status_string(fk_status s) {
  switch (s) {
    case FK_OK: return "ok";
    case FK_ERR_INVALID_ARG: return "invalid argument";
    case FK_ERR_UNSUPPORTED: return "unsupported request";
    case FK_ERR_CUDA: return "CUDA error";
    case FK_ERR_OOM: return "out of memory";
    case FK_ERR_TIMEOUT: return "device-side wait timed out";
    case FK_ERR_HOST_IO: return "host/device copy failed";
    case FK_ERR_BAD_LABEL: return "label outside [0, K)";
    default: return "unknown status";
  }
}

fk_status fk_get_last_error(void) { return t_last; }
const char *fk_last_error_message(void) { return t_msg.c_str(); }
uint64_t fk_launch_count(void) { return g_launches.load(); }

int fk_assign_path(int64_t N, int D, fk_dtype dt, int K, int B) {
  if (!valid_dtype(dt) || B < 1 || N < 0 || D < 1 || D > 1024 || K < 1) return FK_ERR_INVALID_ARG;
  const int path = choose_path((DType)dt, D);
  // the fp32 tensor path takes one problem at a time; a batch runs on CUDA cores
  if (path == 1 && (DType)dt == kF32 && B > 1) return g_assign_path.load() == 1 ? FK_ERR_UNSUPPORTED : 2;
  return path;
}

fk_status fk_set_assign_path(int path) {
  if (path < 0 || path > 2) return fail(FK_ERR_INVALID_ARG, "path must be 0, 1 or 2");
  g_assign_path.store(path);
  return FK_OK;
}

fk_status fk_set_wait_timeout_ns(uint64_t ns) {
  g_timeout_ns.store(ns == 0 ? 2000000000ull : (unsigned long long)ns);
  return FK_OK;
}

fk_status fk_debug_wait_timeout(uint64_t ns, fk_stream_t stream) {
  DevState *d;
  fk_status st = device_state(&d);
  if (st != FK_OK) return st;
  DevCtl c = ctl_of(*d);
  c.timeout_ns = ns;
  cudaError_t e = launch_wait_probe(c, (cudaStream_t)stream);
  if (e != cudaSuccess) return cuda_fail(e, "wait probe kernel");
  return read_status(*d, (cudaStream_t)stream);
}

fk_status fk_release_workspace(void) {
  DevState *d;
  fk_status st = device_state(&d);
  if (st != FK_OK) return st;
  std::lock_guard<std::mutex> g(d->mu);
  for (auto &kv : d->scratch) {
    if (kv.second.ptr) cudaFreeAsync(kv.second.ptr, kv.first);
    if (kv.second.aux) cudaFreeAsync(kv.second.aux, kv.first);
    if (kv.second.ties_ctl) cudaFreeAsync(kv.second.ties_ctl, kv.first);
  }
  cudaError_t e = cudaDeviceSynchronize();
  for (auto &kv : d->scratch) {  // the out-of-core side streams are idle now
    Scratch &w = kv.second;
    if (w.copy) cudaStreamDestroy(w.copy);
    for (int i = 0; i < 2; ++i) {
      if (w.ready[i]) cudaEventDestroy(w.ready[i]);
      if (w.freed[i]) cudaEventDestroy(w.freed[i]);
    }
  }
  d->scratch.clear();
  if (e != cudaSuccess) return cuda_fail(e, "cudaDeviceSynchronize");
  return FK_OK;
}

fk_status fk_debug_inject(int what, int64_t at) {
  if (what < 0 || what > 2 || (what == 1 && at < 0)) return fail(FK_ERR_INVALID_ARG, "what must be 0, 1 or 2");
  g_inject_at.store(what == 1 ? at : -1);
  g_inject.store(what);
  return FK_OK;
}

int fk_version(void) { return 101; }

}  // extern "C"
