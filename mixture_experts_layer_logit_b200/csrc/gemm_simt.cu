// Step 4 on CUDA cores for the fp32 layer: grouped GEMM over the expert
// segments with FFMA only (TF32 tensor cores would round the inputs to 10
// mantissa bits, too coarse for a 1e-4 relative tolerance).
//
// Experts: two-layer ReLU MLP (FastMoE announcement, Transformer-XL experiment)
// or SwiGLU with the gate projection stored before the up projection
// (Megatron-Core best-practice page, "从HuggingFace到Megatron的权重转换要点").
// One 64x64 output tile per iteration of a grid-stride loop over the tile
// table built from offsets[] on the device.
#include "internal.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;
enum { kPlain = 0, kRelu = 1, kSwiglu = 2 };

template <int MODE>
__global__ void __launch_bounds__(kThreads)
simt_grouped_gemm(const float* __restrict__ A, const float* __restrict__ B, float* __restrict__ C,
                  const int32_t* __restrict__ offsets, int E, int K, int Nout, int NB, int F, int rows_alloc,
                  int EW, uint32_t* __restrict__ status) {
  __shared__ int tstart[kMaxExperts + 1];
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  __shared__ float Bu[MODE == kSwiglu ? kBK : 1][kBN + 4];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int nt = (Nout + kBN - 1) / kBN;
  if (warp == 0) {
    if (!tile_table_warp(offsets, E, kBM, nt, rows_alloc, tstart, lane) && lane == 0 && blockIdx.x == 0)
      atomicOr(status, MOE_DEV_BOUNDS);   // offsets[] unusable: no tile is scheduled
  }
  __syncthreads();
  const int total = tstart[E];
  const int ty = tid >> 4, tx = tid & 15;

  for (int L = blockIdx.x; L < total; L += gridDim.x) {
    const int e = tile_expert(tstart, E, L);
    const int we = e % EW;   // weight block of segment e
    const int seg0 = offsets[e], M = offsets[e + 1] - seg0;
    const int mt = (M + kBM - 1) / kBM;
    const int local = L - tstart[e];
    const int nti = local / mt, mti = local - nti * mt;
    const int row0 = seg0 + mti * kBM, n0 = nti * kBN;
    // rows past the T*k-row buffers (only reachable with corrupt offsets) are skipped
    const int rows = max(0, min(min(kBM, M - mti * kBM), rows_alloc - row0));
    float acc[4][4], accu[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = accu[i][j] = 0.f;

    for (int k0 = 0; k0 < K; k0 += kBK) {
      for (int i = tid; i < kBM * kBK; i += kThreads) {
        const int r = i / kBK, kk = i % kBK;
        As[kk][r] = (r < rows && k0 + kk < K) ? A[(size_t)(row0 + r) * K + k0 + kk] : 0.f;
      }
      for (int i = tid; i < kBN * kBK; i += kThreads) {
        const int n = i / kBK, kk = i % kBK;
        const bool ok = (n0 + n < Nout) && (k0 + kk < K);
        Bs[kk][n] = ok ? B[((size_t)we * NB + n0 + n) * K + k0 + kk] : 0.f;
        if (MODE == kSwiglu) Bu[kk][n] = ok ? B[((size_t)we * NB + F + n0 + n) * K + k0 + kk] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kBK; ++kk) {
        float a[4], b[4], u[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          b[j] = Bs[kk][tx + 16 * j];
          if (MODE == kSwiglu) u[j] = Bu[kk][tx + 16 * j];
        }
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
            if (MODE == kSwiglu) accu[i][j] = fmaf(a[i], u[j], accu[i][j]);
          }
      }
      __syncthreads();
    }
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int r = ty * 4 + i, n = n0 + tx + 16 * j;
        if (r >= rows || n >= Nout) continue;
        float v = acc[i][j];
        if (MODE == kRelu) v = fmaxf(v, 0.f);
        if (MODE == kSwiglu) v = v / (1.f + expf(-v)) * accu[i][j];
        C[(size_t)(row0 + r) * Nout + n] = v;
      }
  }
}

}  // namespace

cudaError_t launch_grouped_plain_simt(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
                                      const void* B, int K, int Nout, float* out, uint32_t* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const long long tiles = ((long long)rows_alloc / kBM + c.E) * ((Nout + kBN - 1) / kBN);
  simt_grouped_gemm<kPlain><<<(int)std::min<long long>(tiles, 8LL * di.sms), kThreads, 0, s>>>(
      static_cast<const float*>(A), static_cast<const float*>(B), out, offsets, c.E, K, Nout, Nout, 0, rows_alloc,
      c.E, status);
  return cudaGetLastError();
}

cudaError_t launch_expert_ffn_simt(const moe_config& c, const void* xp, const int32_t* offsets,
                                   const void* w1, const void* w2, void* h, void* yp, uint32_t* status,
                                   cudaStream_t s, int e_mod) {
  const int EW = e_mod > 0 ? e_mod : c.E;
  if (c.T == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const long long A = (long long)c.T * c.k;
  const long long mt_max = A / kBM + c.E;
  auto grid_for = [&](int N) {
    const long long tiles = mt_max * ((N + kBN - 1) / kBN);
    return (int)std::min<long long>(tiles, 8LL * di.sms);
  };
  const float* X = static_cast<const float*>(xp);
  float* H = static_cast<float*>(h);
  if (c.act == MOE_ACT_SWIGLU)
    simt_grouped_gemm<kSwiglu><<<grid_for(c.F), kThreads, 0, s>>>(X, static_cast<const float*>(w1), H,
                                                                   offsets, c.E, c.d, c.F, 2 * c.F, c.F, (int)A,
                                                                   EW, status);
  else
    simt_grouped_gemm<kRelu><<<grid_for(c.F), kThreads, 0, s>>>(X, static_cast<const float*>(w1), H,
                                                                 offsets, c.E, c.d, c.F, c.F, 0, (int)A, EW, status);
  err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  simt_grouped_gemm<kPlain><<<grid_for(c.d), kThreads, 0, s>>>(H, static_cast<const float*>(w2),
                                                                static_cast<float*>(yp), offsets, c.E,
                                                                c.F, c.d, c.d, 0, (int)A, EW, status);
  return cudaGetLastError();
}

}  // namespace moe
