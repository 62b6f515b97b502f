// Library-owned scratch for moe_permute_static: one fixed device array per
// device, so that entry point allocates nothing.  Its address is looked up
// with that device current and cached per device once the lookup succeeds; a
// failed lookup is not cached, so the next call tries again.
#include "internal.cuh"

#include <mutex>

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

}  // namespace

cudaError_t static_scratch_address(void** out) {
  constexpr int kMaxDev = 64;
  static std::mutex mu;
  static void* addr[kMaxDev];
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);   // the current device: the one the lookup resolves for
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::lock_guard<std::mutex> lock(mu);
  if (addr[dev] == nullptr) {
    void* p = nullptr;
    e = cudaGetSymbolAddress(&p, g_static_scratch);
    if (e == cudaSuccess && (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 255u) != 0))
      e = cudaErrorInvalidDevicePointer;
    if (e != cudaSuccess) {
      (void)cudaGetLastError();   // leave no error behind for the caller's next launch check
      return e;
    }
    addr[dev] = p;
  }
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace moe
