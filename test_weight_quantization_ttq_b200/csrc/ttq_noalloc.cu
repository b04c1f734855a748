// ttq_act_norm_noalloc: the per-channel activation statistic for callers
// that cannot allocate device memory and have no workspace to hand over.
// Its scratch (the fp64 partial sums of the token splits, the merge tickets
// and a status word) lives in one fixed array compiled into the library.
#include <mutex>

#include "ttq.h"
#include "ttq_device.cuh"
#include "ttq_kernels.h"

namespace ttq {
namespace {

constexpr int64_t kNoAllocMaxChannels = 16384;  // largest d accepted
constexpr int64_t kNoAllocMaxSplits = 16;       // token splits of the statistic pass
constexpr size_t kNoAllocHeaderBytes = 4096;    // status word + merge tickets
constexpr size_t kNoAllocScratchBytes =
    kNoAllocHeaderBytes + kNoAllocMaxSplits * kNoAllocMaxChannels * sizeof(double);
constexpr int kPlanSMs = 148;  // the same split plan as ttq_act_norm

// Every GPU that loads the library holds this array (2 MiB + 4 KiB) until
// the process exits.  Host code must not pass its name to a kernel: on the
// host it is only a stand-in, so its device address is looked up below.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

// Device address of the scratch array on the current device, looked up with
// that device current and cached per device; null on failure.  A device
// reset (cudaDeviceReset, or the primary context released and created
// again) loads the library's module anew, possibly elsewhere, so a cached
// address that no longer names device memory of this device is looked up
// again.
bool still_valid(const void* p, int dev) {
  cudaPointerAttributes a;
  if (cudaPointerGetAttributes(&a, p) != cudaSuccess) {
    (void)cudaGetLastError();  // clear the non-sticky error of the query
    return false;
  }
  return a.type == cudaMemoryTypeDevice && a.device == dev;
}

void* noalloc_scratch() {
  static void* addr[64] = {};
  static std::mutex mu;
  int dev = -1;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return nullptr;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr || !still_valid(addr[dev], dev)) {
    void* p = nullptr;
    if (cudaGetSymbolAddress(&p, g_noalloc_scratch) != cudaSuccess) {
      addr[dev] = nullptr;
      return nullptr;
    }
    addr[dev] = p;
  }
  return addr[dev];
}

}  // namespace
}  // namespace ttq

extern "C" ttq_status ttq_act_norm_noalloc(const void* X, ttq_dtype dtype, int64_t d, int64_t T,
                                           float p, float lambda, float alpha, float* D,
                                           float* D_rsqrt, void* stream) {
  using namespace ttq;
  if (dtype != TTQ_F32 && dtype != TTQ_BF16) return TTQ_ERR_INVALID_ARG;
  if (d < 8 || d % 8 != 0 || T < 0) return TTQ_ERR_INVALID_ARG;
  if ((T > 0 && X == nullptr) || D == nullptr || D_rsqrt == nullptr) return TTQ_ERR_INVALID_ARG;
  if (!(p >= 1.0f) || !(lambda >= 0.0f) || !(alpha >= 0.0f) || !(p <= 3.402823466e38f) ||
      !(lambda <= 3.402823466e38f) || !(alpha <= 3.402823466e38f))
    return TTQ_ERR_INVALID_ARG;
  const auto misaligned = [](const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) != 0; };
  if ((X && misaligned(X)) || misaligned(D) || misaligned(D_rsqrt)) return TTQ_ERR_INVALID_ARG;
  if (d > kNoAllocMaxChannels) return TTQ_ERR_UNSUPPORTED;  // beyond the fixed scratch
  int64_t splits = 1, rps = 1;
  act_norm_plan(d, T, kPlanSMs, &splits, &rps);
  if (splits > kNoAllocMaxSplits) return TTQ_ERR_UNSUPPORTED;
  uint8_t* scratch = static_cast<uint8_t*>(noalloc_scratch());
  if (scratch == nullptr) return TTQ_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  // the status word and the merge tickets must start at zero
  if (cudaMemsetAsync(scratch, 0, kNoAllocHeaderBytes, s) != cudaSuccess) return TTQ_ERR_CUDA;
  uint32_t* status = reinterpret_cast<uint32_t*>(scratch);
  double* partial = reinterpret_cast<double*>(scratch + kNoAllocHeaderBytes);
  const cudaError_t e = launch_act_norm(X, dtype == TTQ_F32, d, T, p, lambda, alpha, splits, rps,
                                        partial, status + 64, D, D_rsqrt, nullptr, nullptr,
                                        status, s, false);
  return e == cudaSuccess ? TTQ_OK : TTQ_ERR_CUDA;
}
