// noalloc.cu -- fk_update_noalloc: the centroid update without any device
// memory allocation.
//
// fk_update takes its scratch (sorted keys and point ids, digit histograms,
// segment offsets, boundary partial sums) from a cache it grows with
// cudaMallocAsync.  Some callers cannot let a library allocate: code running
// while a stream is being captured into a CUDA graph, frameworks that reserve
// all device memory up front for their own pool, and latency-critical loops
// that must not pay for an allocation or the synchronisation that freeing
// memory can imply.  This file gives them the same update with its scratch in
// one statically sized device array that is part of the library image.
#include <mutex>
#include <string>

#include "../../include/fk.h"
#include "fk_internal.h"

namespace fk {

// 32 MiB.  A call needs 16 N + 4 2^b ceil(N / 4096) + 4 (K + 1) +
// 8 D ceil(N / R) bytes (each term rounded up to 256; b = bits per sort pass,
// at most 11; R >= 128 sorted positions per gather worker): about 1.55
// million points at D = 128 and K = 1,024, about 0.41 million at D = 1,024.
// The need is computed per call and larger problems are refused.  The array
// is created on each device when this file's code is first loaded there and
// stays until the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr size_t kNoAllocStatusBytes = 256;  // device status word, then the scratch
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
  std::mutex mu;
  bool ready = false;             // set only once the lookup has succeeded
  unsigned char *base = nullptr;  // device address of g_noalloc_scratch
  int sms = 0;
};
constexpr int kNoAllocMaxDevices = 64;
static NoAllocDevice g_noalloc_dev[kNoAllocMaxDevices];

}  // namespace fk

using namespace fk;

extern "C" fk_status fk_update_noalloc(const void *X, const int32_t *labels, int64_t N, int D, fk_dtype dt,
                                       int K, float *C, int32_t *counts, fk_stream_t stream) {
  if (dt != FK_F32 && dt != FK_F16 && dt != FK_BF16) return record_error(FK_ERR_INVALID_ARG, "unknown dtype");
  if (N < 0 || N >= (1ll << 31)) return record_error(FK_ERR_INVALID_ARG, "N must be in [0, 2^31)");
  if (D < 1 || D > 1024) return record_error(FK_ERR_INVALID_ARG, "D must be in [1, 1024]");
  if (K < 1 || K > (1 << 22)) return record_error(FK_ERR_INVALID_ARG, "K must be in [1, 2^22]");
  if (!C) return record_error(FK_ERR_INVALID_ARG, "C must not be NULL");
  cudaStream_t s = (cudaStream_t)stream;
  if (N == 0) {
    if (counts && cudaMemsetAsync(counts, 0, (size_t)K * 4, s) != cudaSuccess)
      return record_error(FK_ERR_CUDA, "cudaMemsetAsync(counts) failed");
    return FK_OK;
  }
  if (!X || !labels) return record_error(FK_ERR_INVALID_ARG, "X and labels must not be NULL");
  const size_t need = update_workspace_bytes(N, K, D, 1);
  if (need > kNoAllocScratchBytes - kNoAllocStatusBytes) {
    const std::string msg = "fk_update_noalloc needs " + std::to_string(need) +
                            " bytes of scratch; its static scratch holds " +
                            std::to_string(kNoAllocScratchBytes - kNoAllocStatusBytes) + " bytes";
    return record_error(FK_ERR_UNSUPPORTED, msg.c_str());
  }
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= kNoAllocMaxDevices)
    return record_error(FK_ERR_CUDA, "no usable current CUDA device");
  NoAllocDevice &nd = g_noalloc_dev[dev];
  // Once per device, with that device current: the host-side name of the
  // array is not a device address, so ask the runtime for the real one.  A
  // failed lookup is not remembered; the next call tries again.
  unsigned char *base = nullptr;
  int sms = 0;
  {
    std::lock_guard<std::mutex> g(nd.mu);
    if (!nd.ready) {
      void *p = nullptr;
      cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      int n = 0;
      if (e == cudaSuccess) e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
      if (e != cudaSuccess || !p) {
        cudaGetLastError();
        return record_error(FK_ERR_CUDA, (std::string("cudaGetSymbolAddress(static scratch): ") +
                                          cudaGetErrorString(e)).c_str());
      }
      nd.base = static_cast<unsigned char *>(p);
      nd.sms = n;
      nd.ready = true;
    }
    base = nd.base;
    sms = nd.sms;
  }
  int *status = reinterpret_cast<int *>(base);
  // The status word must start each call at zero; the rest is fully written
  // before it is read.
  if (cudaMemsetAsync(status, 0, sizeof(int), s) != cudaSuccess)
    return record_error(FK_ERR_CUDA, "cudaMemsetAsync(status) failed");
  UpdateArgs a{};
  a.dt = (DType)dt;
  a.X = X;
  a.labels = labels;
  a.B = 1;
  a.N = (int)N;
  a.D = D;
  a.K = K;
  a.C = C;
  a.counts = counts;
  a.mode = kMean;
  const cudaError_t e = launch_update(a, base + kNoAllocStatusBytes, kNoAllocScratchBytes - kNoAllocStatusBytes,
                                      DevCtl{status, 2000000000ull}, sms, s);
  if (e != cudaSuccess) return record_error(FK_ERR_CUDA, (std::string("update kernels: ") + cudaGetErrorString(e)).c_str());
  return FK_OK;
}
