// The backward of step 4 on CUDA cores for the fp32 layer (the grouped GEMMs
// of the tensor-core backward, gemm_bwd.cu, in FFMA): dh = dy W2[e] with the
// activation backward in the epilogue, dxp = du W1[e], and the weight
// gradients over each expert's padded rows.  64 x 64 output tiles.
#include "internal.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int kBM = 64, kBN = 64, kBK = 16, kThreads = 256;
enum { kDgradAct = 0, kDgradPlain = 1, kWgrad = 2 };
enum { kRelu = 0, kSwiglu = 1 };

struct SimtBwdParams {
  const int32_t* offsets;   // padded segment offsets [E+1]
  int E, rows_alloc;
  const float* A;           // kDgrad*: [rows][K] (row-major, K contiguous); kWgrad: [rows][M]
  const float* B;           // kDgrad*: [E*K][Nout] (rows along K); kWgrad: [rows][N]
  int K, Nout, M, N;
  float* out;
  uint32_t* status;
  const float* u;           // kDgradAct
  const float* wrow;
  float* du;
  float* hw;
  float* dwpart;            // [ceil(F / 64)][rows]
  int F, F1;
};

template <int MODE, int ACT>
__global__ void __launch_bounds__(kThreads)
simt_bwd_gemm(const SimtBwdParams p) {
  __shared__ int tstart[kMaxExperts + 1];
  __shared__ float As[kBK][kBM + 4];
  __shared__ float Bs[kBK][kBN + 4];
  __shared__ float red[kBM][17];
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int ncols = MODE == kWgrad ? p.N : p.Nout;
  const int nt = (ncols + kBN - 1) / kBN;
  pdl_wait();
  pdl_launch_dependents();
  int total;
  if (MODE == kWgrad) {
    total = p.E * ((p.M + kBM - 1) / kBM) * nt;
  } else {
    if (warp == 0) {
      if (!tile_table_warp(p.offsets, p.E, kBM, nt, p.rows_alloc, tstart, lane) && lane == 0 && blockIdx.x == 0)
        atomicOr(p.status, MOE_DEV_BOUNDS);
    }
    __syncthreads();
    total = tstart[p.E];
  }
  const int ty = tid >> 4, tx = tid & 15;
  for (int L = blockIdx.x; L < total; L += gridDim.x) {
    int e, row0 = 0, rows = 0, m0 = 0, n0, k0, klen;
    if (MODE == kWgrad) {
      const int mt = (p.M + kBM - 1) / kBM;
      e = L / (mt * nt);
      const int r = L - e * mt * nt;
      const int ni = r / mt, mi = r - ni * mt;
      m0 = mi * kBM;
      n0 = ni * kBN;
      rows = min(kBM, p.M - m0);
      k0 = p.offsets[e];
      klen = p.offsets[e + 1] - k0;
    } else {
      e = tile_expert(tstart, p.E, L);
      const int seg0 = p.offsets[e], Mseg = p.offsets[e + 1] - seg0;
      const int mt = (Mseg + kBM - 1) / kBM;
      const int local = L - tstart[e];
      const int nti = local / mt, mti = local - nti * mt;
      row0 = seg0 + mti * kBM;
      rows = max(0, min(min(kBM, Mseg - mti * kBM), p.rows_alloc - row0));
      n0 = nti * kBN;
      k0 = 0;
      klen = p.K;
    }
    float acc[4][4];
#pragma unroll
    for (int i = 0; i < 4; ++i)
#pragma unroll
      for (int j = 0; j < 4; ++j) acc[i][j] = 0.f;
    for (int kk0 = 0; kk0 < klen; kk0 += kBK) {
      for (int i = tid; i < kBM * kBK; i += kThreads) {
        if (MODE == kWgrad) {   // A rows along K: coalesced along m
          const int kk = i / kBM, r = i % kBM;
          As[kk][r] = (r < rows && kk0 + kk < klen) ? p.A[(size_t)(k0 + kk0 + kk) * p.M + m0 + r] : 0.f;
        } else {
          const int r = i / kBK, kk = i % kBK;
          As[kk][r] = (r < rows && kk0 + kk < klen) ? p.A[(size_t)(row0 + r) * p.K + kk0 + kk] : 0.f;
        }
      }
      for (int i = tid; i < kBN * kBK; i += kThreads) {
        const int kk = i / kBN, n = i % kBN;
        const bool ok = (n0 + n < ncols) && (kk0 + kk < klen);
        const size_t brow = MODE == kWgrad ? (size_t)(k0 + kk0 + kk) : (size_t)e * p.K + kk0 + kk;
        Bs[kk][n] = ok ? p.B[brow * ncols + n0 + n] : 0.f;
      }
      __syncthreads();
#pragma unroll
      for (int kk = 0; kk < kBK; ++kk) {
        float a[4], b[4];
#pragma unroll
        for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
        for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
      }
      __syncthreads();
    }
    if (MODE == kDgradAct) {
      float part[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const int r = ty * 4 + i;
        if (r >= rows) continue;
        const int row = row0 + r;
        const float w = p.wrow[row];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int f = n0 + tx + 16 * j;
          if (f >= p.F) continue;
          const float g = acc[i][j], a = p.u[(size_t)row * p.F1 + f];
          float h;
          if (ACT == kSwiglu) {
            const float v = p.u[(size_t)row * p.F1 + p.F + f];
            const float s = 1.f / (1.f + expf(-a));
            const float silu = a * s;
            h = silu * v;
            p.du[(size_t)row * p.F1 + f] = w * g * v * s * (1.f + a * (1.f - s));
            p.du[(size_t)row * p.F1 + p.F + f] = w * g * silu;
          } else {
            h = fmaxf(a, 0.f);
            p.du[(size_t)row * p.F1 + f] = a > 0.f ? w * g : 0.f;
          }
          p.hw[(size_t)row * p.F + f] = w * h;
          part[i] += g * h;
        }
      }
      // the row sums over this tile's columns, in a fixed order
#pragma unroll
      for (int i = 0; i < 4; ++i) red[ty * 4 + i][tx] = part[i];
      __syncthreads();
      if (tid < kBM && tid < rows) {
        float s = 0.f;
        for (int x = 0; x < 16; ++x) s += red[tid][x];
        p.dwpart[(size_t)(n0 / kBN) * p.rows_alloc + row0 + tid] = s;
      }
      __syncthreads();
    } else {
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int r = ty * 4 + i, n = n0 + tx + 16 * j;
          if (r >= rows || n >= ncols) continue;
          if (MODE == kWgrad) p.out[(size_t)e * p.M * p.N + (size_t)(m0 + r) * p.N + n] = acc[i][j];
          else p.out[(size_t)(row0 + r) * p.Nout + n] = acc[i][j];
        }
    }
  }
}

template <int MODE, int ACT>
cudaError_t launch_s(const SimtBwdParams& p, int grid, cudaStream_t s) {
  return launch_pdl(simt_bwd_gemm<MODE, ACT>, dim3(grid), dim3(kThreads), 0, s, p);
}

}  // namespace

int bwd_simt_col_tile() { return kBN; }

cudaError_t launch_expert_backward_simt(const moe_config& c, const BwdState& st, const void* w1, const void* w2,
                                        float* dw1, float* dw2, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const long long mt_max = (long long)st.rows_alloc / kBM + c.E;
  auto grid_for = [&](long long tiles) { return (int)std::max<long long>(1, std::min<long long>(tiles, 8LL * di.sms)); };
  SimtBwdParams p{};
  p.offsets = st.pad_offsets;
  p.E = c.E;
  p.rows_alloc = st.rows_alloc;
  p.status = st.status;
  p.F = c.F;
  p.F1 = F1;
  // dh = dout_perm W2[e] (B rows along K = d), the activation backward in the epilogue
  p.A = static_cast<const float*>(st.dout_perm);
  p.B = static_cast<const float*>(w2);
  p.K = c.d;
  p.Nout = c.F;
  p.u = st.u;
  p.wrow = st.wrow;
  p.du = static_cast<float*>(st.du);
  p.hw = static_cast<float*>(st.hw);
  p.dwpart = st.dwpart;
  const long long nF = (c.F + kBN - 1) / kBN, nd = (c.d + kBN - 1) / kBN;
  err = (c.act == MOE_ACT_SWIGLU) ? launch_s<kDgradAct, kSwiglu>(p, grid_for(mt_max * nF), s)
                                  : launch_s<kDgradAct, kRelu>(p, grid_for(mt_max * nF), s);
  if (err != cudaSuccess) return err;
  // dxp = du W1[e] (B rows along K = F1)
  p.A = static_cast<const float*>(st.du);
  p.B = static_cast<const float*>(w1);
  p.K = F1;
  p.Nout = c.d;
  p.out = st.dxp;
  if ((err = launch_s<kDgradPlain, kRelu>(p, grid_for(mt_max * nd), s)) != cudaSuccess) return err;
  // dW2[e] = dout_perm_e^T (w h)_e, dW1[e] = du_e^T xp_e
  p.A = static_cast<const float*>(st.dout_perm);
  p.B = static_cast<const float*>(st.hw);
  p.M = c.d;
  p.N = c.F;
  p.out = dw2;
  if ((err = launch_s<kWgrad, kRelu>(p, grid_for((long long)c.E * nd * nF), s)) != cudaSuccess) return err;
  p.A = static_cast<const float*>(st.du);
  p.B = static_cast<const float*>(st.xp);
  p.M = F1;
  p.N = c.d;
  p.out = dw1;
  return launch_s<kWgrad, kRelu>(p, grid_for((long long)c.E * ((F1 + kBM - 1) / kBM) * nd), s);
}

}  // namespace moe
