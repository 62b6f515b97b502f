// Weight preparation: bf16 -> fp16 (round to nearest even, saturating), used
// once at load time to give W2 to the layer when the hidden activation is fp16
// (both tcgen05 kind::f16 operands of the second layer must share a type).
#include "internal.cuh"

namespace {

__device__ __forceinline__ __half bf16_to_f16(__nv_bfloat16 v) {
  float f = __bfloat162float(v);                       // exact
  if (fabsf(f) > 65504.f) f = copysignf(65504.f, f);   // NaN passes through
  return __float2half_rn(f);
}

__global__ void convert_kernel(const __nv_bfloat16* __restrict__ src, __half* __restrict__ dst, size_t n) {
  const size_t nvec = n / 8;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < nvec; i += stride) {
    const uint4 v = __ldg(reinterpret_cast<const uint4*>(src) + i);
    const __nv_bfloat16* b = reinterpret_cast<const __nv_bfloat16*>(&v);
    uint4 o;
    __half* h = reinterpret_cast<__half*>(&o);
#pragma unroll
    for (int j = 0; j < 8; ++j) h[j] = bf16_to_f16(b[j]);
    reinterpret_cast<uint4*>(dst)[i] = o;
  }
  // tail of fewer than 8 elements
  const size_t t = nvec * 8 + (size_t)blockIdx.x * blockDim.x + threadIdx.x;
  if (t < n) dst[t] = bf16_to_f16(src[t]);
}

}  // namespace

namespace moe {
cudaError_t launch_convert_bf16_f16(const void* src, void* dst, size_t n, cudaStream_t s) {
  if (n == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const size_t want = (n / 8 + 255) / 256;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)di.sms * 8));
  convert_kernel<<<grid, 256, 0, s>>>(static_cast<const __nv_bfloat16*>(src), static_cast<__half*>(dst), n);
  return cudaGetLastError();
}
}  // namespace moe

extern "C" moe_status moe_convert_bf16_to_f16(const void* src, void* dst, size_t n, moe_stream_t stream) {
  if (n == 0) return MOE_OK;
  if (src == nullptr || dst == nullptr) return MOE_ERR_ARG;
  if ((reinterpret_cast<uintptr_t>(src) & 15u) || (reinterpret_cast<uintptr_t>(dst) & 15u)) return MOE_ERR_ARG;
  const uintptr_t s0 = reinterpret_cast<uintptr_t>(src), d0 = reinterpret_cast<uintptr_t>(dst);
  if (s0 < d0 + 2 * n && d0 < s0 + 2 * n) return MOE_ERR_ARG;   // overlap
  (void)cudaGetLastError();   // do not report an earlier caller's stale error as ours
  moe::DeviceInfo di;
  if (moe::device_info(&di) != cudaSuccess) return MOE_ERR_CUDA;
  const size_t nvec = n / 8;
  const int threads = 256;
  const size_t want = (nvec + threads - 1) / threads;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>(want, (size_t)di.sms * 8));
  convert_kernel<<<grid, threads, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
      static_cast<const __nv_bfloat16*>(src), static_cast<__half*>(dst), n);
  return cudaGetLastError() == cudaSuccess ? MOE_OK : MOE_ERR_CUDA;
}
