// Library-owned scratch for moe_permute_static: one fixed device array per
// device, so that entry point allocates nothing.  Its address is looked up
// once per device, with that device current, and cached.
#include "internal.cuh"

#include <mutex>

namespace moe {
namespace {

static __device__ __align__(256) unsigned char g_static_scratch[MOE_STATIC_SCRATCH_BYTES];

}  // namespace

cudaError_t static_scratch_address(void** out) {
  constexpr int kMaxDev = 64;
  static void* addr[kMaxDev];
  static cudaError_t err[kMaxDev];
  static std::once_flag once[kMaxDev];
  *out = nullptr;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);   // the current device: the one the lookup resolves for
  if (e != cudaSuccess) return e;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  std::call_once(once[dev], [&] {
    void* p = nullptr;
    err[dev] = cudaGetSymbolAddress(&p, g_static_scratch);
    if (err[dev] == cudaSuccess && (p == nullptr || (reinterpret_cast<uintptr_t>(p) & 255u) != 0))
      err[dev] = cudaErrorInvalidDevicePointer;
    addr[dev] = (err[dev] == cudaSuccess) ? p : nullptr;
  });
  if (err[dev] != cudaSuccess) return err[dev];
  *out = addr[dev];
  return cudaSuccess;
}

}  // namespace moe
