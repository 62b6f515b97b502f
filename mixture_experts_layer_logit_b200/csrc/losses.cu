// Small element-wise kernels around the layer: the layer-wise adaptive
// aux-loss coefficient, and the shared expert's segment and sum.
//
// The layer-wise adaptive aux-loss coefficient on the device (Skywork-MoE
// release, "2.自适应的Aux Loss"; slides, slide 7: raise a layer's coefficient
// when its token drop rate rises, lower it when it falls).  One thread reads
// the drop rate the layer's forward left in moe_stats and updates the
// coefficient in place, so a training step needs no host synchronisation.
#include "internal.cuh"

#include <algorithm>

namespace moe {
namespace {

__global__ void aux_coef_kernel(const moe_stats* __restrict__ stats, float* __restrict__ coef, float beta,
                                float xi) {
  pdl_wait();   // the forward that wrote the statistics
  if (threadIdx.x == 0) *coef = aux_coef_step(*coef, stats->drop_rate, beta, xi);
}

__global__ void fill_segment_kernel(int32_t* seg, int rows) {
  pdl_wait();
  pdl_launch_dependents();
  if (threadIdx.x == 0) {
    seg[0] = 0;
    seg[1] = rows;
  }
}

// out += add, element by element, 16-byte vectors (n a multiple of 4)
__global__ void __launch_bounds__(256) add_rows_kernel(float* __restrict__ out, const float* __restrict__ add,
                                                        size_t n) {
  pdl_wait();
  pdl_launch_dependents();
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += (size_t)gridDim.x * blockDim.x) {
    float4 a = reinterpret_cast<float4*>(out)[i];
    const float4 b = __ldg(reinterpret_cast<const float4*>(add) + i);
    a.x += b.x;
    a.y += b.y;
    a.z += b.z;
    a.w += b.w;
    reinterpret_cast<float4*>(out)[i] = a;
  }
}

}  // namespace

cudaError_t launch_fill_segment(int32_t* seg, int rows, cudaStream_t s) {
  return launch_pdl(fill_segment_kernel, dim3(1), dim3(32), 0, s, seg, rows);
}

cudaError_t launch_add_rows(float* out, const float* add, size_t n, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t e = device_info(&di);
  if (e != cudaSuccess) return e;
  const int grid = (int)std::max<size_t>(1, std::min<size_t>((n / 4 + 255) / 256, (size_t)di.sms * 8));
  return launch_pdl(add_rows_kernel, dim3(grid), dim3(256), 0, s, out, add, n);
}

cudaError_t launch_aux_coef_update(const moe_stats* stats, float* coef, float beta, float xi, cudaStream_t s) {
  return launch_pdl(aux_coef_kernel, dim3(1), dim3(32), 0, s, stats, coef, beta, xi);
}

}  // namespace moe
