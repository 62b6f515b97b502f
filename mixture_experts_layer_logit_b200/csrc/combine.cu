// Step 5 of the layer: un-permute and combine.
//
// out[t] = sum over kept slots j (slot order, fp32 accumulation) of
// w[t, j] * yp[row_of[t, j]]; a token whose slots were all dropped gets 0, the
// residual path outside the layer carrying it (Megatron-Core best-practice
// page, "MoE负载均衡的挑战与应对").  The sum itself is the definition of the
// layer output (FastMoE announcement, "1. MoE 设计").
//
// One warp per (token, column slice).  A token's row of 16-byte vectors is
// dealt to `nslice` warps: slice s takes vectors s*32 + lane, then every
// 32*nslice after that.  Each lane issues the k row reads of a vector back to
// back.  A large batch keeps nslice = 1 (one warp walks the whole row).  A
// small one (decode) splits its rows so that enough warps keep reads in
// flight: otherwise each warp would wait on d/128 serial read latencies.
#include "internal.cuh"

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kTokPerBlock = kThreads / 32;

template <typename TX> struct Pack;
template <> struct Pack<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void acc(const uint4& v, float w, float* a) {
    a[0] = fmaf(w, __uint_as_float(v.x), a[0]);
    a[1] = fmaf(w, __uint_as_float(v.y), a[1]);
    a[2] = fmaf(w, __uint_as_float(v.z), a[2]);
    a[3] = fmaf(w, __uint_as_float(v.w), a[3]);
  }
  __device__ __forceinline__ static uint4 store(const float* a) {
    return make_uint4(__float_as_uint(a[0]), __float_as_uint(a[1]), __float_as_uint(a[2]),
                      __float_as_uint(a[3]));
  }
};
template <typename TX, int KB>
__global__ void __launch_bounds__(kThreads)
combine_kernel(const TX* __restrict__ yp, const int32_t* __restrict__ row_of,
               const float* __restrict__ topk_w, TX* __restrict__ out, int T, int d, int k, int nslice) {
  constexpr int N = Pack<TX>::N;
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x * kTokPerBlock + warp;
  const int t = g / nslice, sl = g - t * nslice;
  if (t >= T) return;
  int rows[KB];
  float ws[KB];
  const int A = T * k;
#pragma unroll
  for (int j = 0; j < KB; ++j) {
    rows[j] = (j < k) ? __ldg(row_of + (size_t)t * k + j) : -1;
    if (rows[j] >= A) rows[j] = -1;   // outside the permuted buffer: treated as dropped
    ws[j] = (j < k) ? __ldg(topk_w + (size_t)t * k + j) : 0.f;
  }
  const int nvec = d / N;
  uint4* o = reinterpret_cast<uint4*>(out + (size_t)t * d);
  for (int v = sl * 32 + lane; v < nvec; v += 32 * nslice) {
    uint4 in[KB];
#pragma unroll
    for (int j = 0; j < KB; ++j)
      if (rows[j] >= 0) in[j] = __ldg(reinterpret_cast<const uint4*>(yp + (size_t)rows[j] * d) + v);
    float a[N];
#pragma unroll
    for (int i = 0; i < N; ++i) a[i] = 0.f;
#pragma unroll
    for (int j = 0; j < KB; ++j)
      if (rows[j] >= 0) Pack<TX>::acc(in[j], ws[j], a);
    o[v] = Pack<TX>::store(a);
  }
}

// any k: rows read slot by slot
template <typename TX>
__global__ void __launch_bounds__(kThreads)
combine_generic_kernel(const TX* __restrict__ yp, const int32_t* __restrict__ row_of,
                       const float* __restrict__ topk_w, TX* __restrict__ out, int T, int d, int k,
                       int nslice) {
  constexpr int N = Pack<TX>::N;
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int g = blockIdx.x * kTokPerBlock + warp;
  const int t = g / nslice, sl = g - t * nslice;
  if (t >= T) return;
  const int nvec = d / N;
  uint4* o = reinterpret_cast<uint4*>(out + (size_t)t * d);
  for (int v = sl * 32 + lane; v < nvec; v += 32 * nslice) {
    float a[N];
#pragma unroll
    for (int i = 0; i < N; ++i) a[i] = 0.f;
    for (int j = 0; j < k; ++j) {
      const int r = row_of[(size_t)t * k + j];
      if (r < 0 || r >= T * k) continue;
      Pack<TX>::acc(__ldg(reinterpret_cast<const uint4*>(yp + (size_t)r * d) + v), topk_w[(size_t)t * k + j], a);
    }
    o[v] = Pack<TX>::store(a);
  }
}

// Column slices per token: doubled while the batch gives fewer than 32 warps
// per SM, and never more than one 32-vector group per slice.
int num_slices(const moe_config& c, int N, int sms) {
  const int groups = (c.d / N + 31) / 32;
  const long long want = 32LL * sms;
  int ns = 1;
  while (ns < groups && (long long)c.T * ns < want) ns *= 2;
  return ns < groups ? ns : (groups > 0 ? groups : 1);
}

template <typename TX>
cudaError_t launch_t(const moe_config& c, const void* yp, const int32_t* row_of, const float* w,
                     void* out, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int ns = num_slices(c, Pack<TX>::N, di.sms);
  const long long grid = ((long long)c.T * ns + kTokPerBlock - 1) / kTokPerBlock;
  if (grid > 0x7fffffffLL) return cudaErrorInvalidConfiguration;
  const TX* y = static_cast<const TX*>(yp);
  TX* o = static_cast<TX*>(out);
  const dim3 g((unsigned)grid), b(kThreads);
  if (c.k <= 1) return launch_pdl(combine_kernel<TX, 1>, g, b, 0, s, y, row_of, w, o, c.T, c.d, c.k, ns);
  if (c.k <= 2) return launch_pdl(combine_kernel<TX, 2>, g, b, 0, s, y, row_of, w, o, c.T, c.d, c.k, ns);
  if (c.k <= 4) return launch_pdl(combine_kernel<TX, 4>, g, b, 0, s, y, row_of, w, o, c.T, c.d, c.k, ns);
  if (c.k <= 8) return launch_pdl(combine_kernel<TX, 8>, g, b, 0, s, y, row_of, w, o, c.T, c.d, c.k, ns);
  return launch_pdl(combine_generic_kernel<TX>, g, b, 0, s, y, row_of, w, o, c.T, c.d, c.k, ns);
}

}  // namespace

// Expert outputs (yp) and the layer output are fp32 for both element types:
// with bf16 yp and out, the two last roundings alone can reach 2^-8 |out|,
// close to the whole output tolerance on the largest elements.
cudaError_t launch_combine(const moe_config& c, const void* yp, const int32_t* row_of,
                           const float* topk_w, void* out, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  return launch_t<float>(c, yp, row_of, topk_w, out, s);
}

}  // namespace moe
