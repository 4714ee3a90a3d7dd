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

// 32 MiB: enough for about 1.5 million points at D = 128 (the exact need is
// computed per call and larger problems are refused).  The array is created
// on each device when this file's code is first loaded there and stays until
// the process exits.
constexpr size_t kNoAllocScratchBytes = size_t(32) << 20;
constexpr size_t kNoAllocStatusBytes = 256;  // device status word, then the scratch
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

struct NoAllocDevice {
  std::once_flag once;
  cudaError_t err = cudaSuccess;
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
  // array is not a device address, so ask the runtime for the real one.
  std::call_once(nd.once, [&nd, dev] {
    void *p = nullptr;
    nd.err = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (nd.err == cudaSuccess) nd.err = cudaDeviceGetAttribute(&nd.sms, cudaDevAttrMultiProcessorCount, dev);
    nd.base = static_cast<unsigned char *>(p);
  });
  if (nd.err != cudaSuccess || !nd.base)
    return record_error(FK_ERR_CUDA, (std::string("cudaGetSymbolAddress(static scratch): ") +
                                      cudaGetErrorString(nd.err)).c_str());
  int *status = reinterpret_cast<int *>(nd.base);
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
  const cudaError_t e = launch_update(a, nd.base + kNoAllocStatusBytes, kNoAllocScratchBytes - kNoAllocStatusBytes,
                                      DevCtl{status, 2000000000ull}, nd.sms, s);
  if (e != cudaSuccess) return record_error(FK_ERR_CUDA, (std::string("update kernels: ") + cudaGetErrorString(e)).c_str());
  return FK_OK;
}
