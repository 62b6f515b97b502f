// The layer-wise adaptive aux-loss coefficient on the device (Skywork-MoE
// release, "2.自适应的Aux Loss"; slides, slide 7: raise a layer's coefficient
// when its token drop rate rises, lower it when it falls).  One thread reads
// the drop rate the layer's forward left in moe_stats and updates the
// coefficient in place, so a training step needs no host synchronisation.
#include "internal.cuh"

namespace moe {
namespace {

__global__ void aux_coef_kernel(const moe_stats* __restrict__ stats, float* __restrict__ coef, float beta,
                                float xi) {
  pdl_wait();   // the forward that wrote the statistics
  if (threadIdx.x == 0) *coef = aux_coef_step(*coef, stats->drop_rate, beta, xi);
}

}  // namespace

cudaError_t launch_aux_coef_update(const moe_stats* stats, float* coef, float beta, float xi, cudaStream_t s) {
  return launch_pdl(aux_coef_kernel, dim3(1), dim3(32), 0, s, stats, coef, beta, xi);
}

}  // namespace moe
