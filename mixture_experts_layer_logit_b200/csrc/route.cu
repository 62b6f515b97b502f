// Steps 1-2 of the layer: gate GEMM, optional gating-logit normalisation,
// softmax and top-k, one CTA per chunk of kChunk tokens.
//
// Gate: one fully-connected layer z = x W_gate^T (+ b) (FastMoE announcement,
// "特色二").  Normalisation (Skywork-MoE release, "Gating Logits归一化操作";
// slides, slide 6): z_hat = lambda (z - mean) / std over the experts of a token,
// population std, zero spread -> 0.  Top-k on z_hat (or z), ties to the lower
// expert index (FastMoE announcement, "图4": the top-2 gate activates the two
// highest-scoring experts).  Weights: the selected experts' softmax
// probabilities renormalised to sum to 1.
//
// The CTA also leaves, for the permutation step, its per-expert histogram, its
// per-expert sum of softmax probabilities (for the Switch aux loss), its
// near-tie count and its sum of squared log-partitions (the router z-loss;
// Megatron-Core best-practice page, "Megatron-Core MoE的关键特性") in the
// scratch workspace.
#include "internal.cuh"

#include <math.h>

namespace moe {
namespace {

constexpr int kThreads = 256;
constexpr int kKC = 32;          // model-width slice staged per iteration

template <typename TX> struct VecLoad;
template <> struct VecLoad<float> {
  static constexpr int N = 4;
  __device__ __forceinline__ static void load(const float* p, float* o) {
    float4 v = __ldg(reinterpret_cast<const float4*>(p));
    o[0] = v.x; o[1] = v.y; o[2] = v.z; o[3] = v.w;
  }
};
template <> struct VecLoad<__nv_bfloat16> {
  static constexpr int N = 8;
  __device__ __forceinline__ static void load(const __nv_bfloat16* p, float* o) {
    uint4 v = __ldg(reinterpret_cast<const uint4*>(p));
    const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&v);
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      float2 f = __bfloat1622float2(h[i]);
      o[2 * i] = f.x; o[2 * i + 1] = f.y;
    }
  }
};

// Dynamic shared memory of one CTA for NJ (experts padded to EP = 16 NJ).
template <int NJ>
struct RouteSmem {
  static constexpr int EP = 16 * NJ;
  static constexpr size_t xs = 0;                                          // float [64][kKC+1]
  static constexpr size_t ws = xs + sizeof(float) * 64 * (kKC + 1);        // float [EP][kKC+1]
  static constexpr size_t zs = ws + sizeof(float) * EP * (kKC + 1);        // float [kChunk][EP+1]
  static constexpr size_t selp = zs + sizeof(float) * kChunk * (EP + 1);   // float [8][EP]
  static constexpr size_t seli = selp + sizeof(float) * 8 * EP;            // int   [8][EP]
  static constexpr size_t pbuf = seli + sizeof(int) * 8 * EP;              // float [8][EP]
  static constexpr size_t hist = pbuf + sizeof(float) * 8 * EP;            // int   [EP]
  static constexpr size_t misc = hist + sizeof(int) * EP;                  // int   [4]
  static constexpr size_t zpart = misc + 16;                               // float [8] per-warp z-loss sums
  static constexpr size_t total = zpart + sizeof(float) * (kThreads / 32);
};

template <int NJ, typename TX>
__global__ void __launch_bounds__(kThreads)
route_kernel(const TX* __restrict__ x, const TX* __restrict__ wg, const float* __restrict__ bg,
             int T, int d, int E, int k, float lam,
             int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ gap_out,
             int32_t* __restrict__ hist_out, float* __restrict__ psum_out, int32_t* __restrict__ ntie_out,
             float* __restrict__ zsum_out, int nch, uint32_t* __restrict__ status) {
  using L = RouteSmem<NJ>;
  constexpr int EP = L::EP;
  constexpr int V = VecLoad<TX>::N;
  constexpr int EPL = (EP + 31) / 32;   // expert values per lane in the epilogue
  extern __shared__ __align__(16) unsigned char smem[];
  float (*xs)[kKC + 1] = reinterpret_cast<float (*)[kKC + 1]>(smem + L::xs);
  float (*wsm)[kKC + 1] = reinterpret_cast<float (*)[kKC + 1]>(smem + L::ws);
  float (*zs)[EP + 1] = reinterpret_cast<float (*)[EP + 1]>(smem + L::zs);
  float (*selp)[EP] = reinterpret_cast<float (*)[EP]>(smem + L::selp);
  int (*seli)[EP] = reinterpret_cast<int (*)[EP]>(smem + L::seli);
  float (*pbuf)[EP] = reinterpret_cast<float (*)[EP]>(smem + L::pbuf);
  int* shist = reinterpret_cast<int*>(smem + L::hist);
  int* misc = reinterpret_cast<int*>(smem + L::misc);
  float* zpart = reinterpret_cast<float*>(smem + L::zpart);

  const int tid = threadIdx.x;
  const int chunk = blockIdx.x;
  const int t0 = chunk * kChunk;
  const int rows = min(kChunk, T - t0);

  for (int e = tid; e < EP; e += kThreads) shist[e] = 0;
  if (tid == 0) misc[0] = 0;

  // ---- gate GEMM: z[kChunk][EP] = x . wg^T in fp32, 64 token rows at a time
  const int ty = tid >> 4, tx = tid & 15;
  for (int half = 0; half < kChunk / 64; ++half) {
  float acc[4][NJ];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) acc[i][j] = 0.f;

  for (int k0 = 0; k0 < d; k0 += kKC) {
    // stage x: 64 rows x kKC columns
    for (int v = tid; v < 64 * (kKC / V); v += kThreads) {
      const int r = v / (kKC / V), c = (v % (kKC / V)) * V;
      float f[V];
      if (half * 64 + r < rows && k0 + c < d) {
        VecLoad<TX>::load(x + (size_t)(t0 + half * 64 + r) * d + k0 + c, f);
      } else {
#pragma unroll
        for (int q = 0; q < V; ++q) f[q] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < V; ++q) xs[r][c + q] = f[q];
    }
    for (int v = tid; v < EP * (kKC / V); v += kThreads) {
      const int r = v / (kKC / V), c = (v % (kKC / V)) * V;
      float f[V];
      if (r < E && k0 + c < d) {
        VecLoad<TX>::load(wg + (size_t)r * d + k0 + c, f);
      } else {
#pragma unroll
        for (int q = 0; q < V; ++q) f[q] = 0.f;
      }
#pragma unroll
      for (int q = 0; q < V; ++q) wsm[r][c + q] = f[q];
    }
    __syncthreads();
#pragma unroll 8
    for (int kk = 0; kk < kKC; ++kk) {
      float a[4], b[NJ];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = xs[ty * 4 + i][kk];
#pragma unroll
      for (int j = 0; j < NJ; ++j) b[j] = wsm[tx + 16 * j][kk];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < NJ; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < NJ; ++j) {
      const int e = tx + 16 * j;
      zs[half * 64 + ty * 4 + i][e] = acc[i][j] + ((bg != nullptr && e < E) ? bg[e] : 0.f);
    }
  }
  __syncthreads();

  // ---- routing epilogue: one warp per token, lane holds experts lane + 32 i
  const int warp = tid >> 5, lane = tid & 31;
  float pacc[EPL];
#pragma unroll
  for (int i = 0; i < EPL; ++i) pacc[i] = 0.f;
  float zacc = 0.f;   // this warp's rows: sum of squared log-partitions (router z-loss)

  for (int r = warp; r < rows; r += kThreads / 32) {
    const int t = t0 + r;
    float v[EPL];
    bool ok[EPL];
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      const int e = lane + 32 * i;
      ok[i] = e < E;
      v[i] = ok[i] ? zs[r][e] : 0.f;
    }
    if (lam > 0.f) {
      float s = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) s += ok[i] ? v[i] : 0.f;
      const float mu = warp_sum(s) / (float)E;
      float q = 0.f;
#pragma unroll
      for (int i = 0; i < EPL; ++i) {
        const float dv = v[i] - mu;
        q += ok[i] ? dv * dv : 0.f;
      }
      const float sd = sqrtf(warp_sum(q) / (float)E);
#pragma unroll
      for (int i = 0; i < EPL; ++i) v[i] = (sd == 0.f) ? 0.f : lam * (v[i] - mu) / sd;   // NaN spread stays NaN
    }
    float m = -INFINITY;
#pragma unroll
    for (int i = 0; i < EPL; ++i) if (ok[i]) m = fmaxf(m, v[i]);
    m = warp_max(m);
    float p[EPL], ps = 0.f;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      p[i] = ok[i] ? expf(v[i] - m) : 0.f;
      ps += p[i];
    }
    const float psum_row = warp_sum(ps);
    const float inv = 1.f / psum_row;
    const float lse = m + logf(psum_row);
    zacc += lse * lse;
#pragma unroll
    for (int i = 0; i < EPL; ++i) {
      p[i] *= inv;
      pacc[i] += p[i];
    }

    // top-k by repeated warp argmax; equal scores -> lower expert index; a NaN
    // or -inf score is never taken, so a row with fewer than k scores above
    // -inf keeps empty slots (out of range: dropped by the permutation, and
    // flagged)
    unsigned taken = 0u;
    float kth = 0.f, gap = INFINITY;
    const int rounds = (k < E) ? k + 1 : k;
    for (int j = 0; j < rounds; ++j) {
      float bv = -INFINITY;
      int bi = 0x7fffffff;
#pragma unroll
      for (int i = 0; i < EPL; ++i)
        if (ok[i] && !((taken >> i) & 1u) && v[i] > bv) {
          bv = v[i];
          bi = lane + 32 * i;
        }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, o);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, o);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (j < k) {
        float pv = 0.f;
        if ((bi & 31) == lane) {
#pragma unroll
          for (int i = 0; i < EPL; ++i)
            if (bi == lane + 32 * i) { pv = p[i]; taken |= 1u << i; }
        }
        pv = __shfl_sync(0xffffffffu, pv, bi & 31);
        if (lane == 0) { seli[warp][j] = bi; selp[warp][j] = pv; }
        kth = bv;
      } else {
        gap = kth - bv;
      }
    }
    __syncwarp();
    float sel = 0.f;
    for (int j = 0; j < k; ++j) sel += selp[warp][j];   // fixed slot order
    const float rs = 1.f / sel;
    for (int j = lane; j < k; j += 32) {
      const int e = seli[warp][j];
      topk_idx[(size_t)t * k + j] = e;
      topk_w[(size_t)t * k + j] = selp[warp][j] * rs;
      if ((unsigned)e < (unsigned)E) atomicAdd(&shist[e], 1);
      else atomicOr(status, MOE_DEV_BOUNDS);
    }
    if (lane == 0) {
      gap_out[t] = gap;
      if (gap < MOE_NEAR_TIE_GAP) atomicAdd(&misc[0], 1);
    }
    __syncwarp();
  }

  // ---- per-chunk outputs for the permutation step
#pragma unroll
  for (int i = 0; i < EPL; ++i) {
    const int e = lane + 32 * i;
    if (e < EP) pbuf[warp][e] = pacc[i];
  }
  if (lane == 0) zpart[warp] = zacc;
  __syncthreads();
  for (int e = tid; e < E; e += kThreads) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) s += pbuf[w][e];
    psum_out[(size_t)chunk * E + e] = s;
    hist_out[(size_t)e * nch + chunk] = shist[e];
  }
  if (tid == 0) {
    ntie_out[chunk] = misc[0];
    float z = 0.f;
#pragma unroll
    for (int w = 0; w < kThreads / 32; ++w) z += zpart[w];   // fixed warp order
    zsum_out[chunk] = z;
  }
}

// The totals of a standalone route, in one launch: P_e = sum over chunks of
// psum / T, one warp per expert (lanes stride over the chunks, then a
// fixed-order butterfly sum: deterministic); with z_loss, the last block's
// first warp adds the chunks' squared log-partitions (double) and divides by
// T.  Launched with programmatic dependent launch: it waits here for the
// route kernel's results.
__global__ void route_totals_kernel(const float* __restrict__ psum, const float* __restrict__ zsum, int nch,
                                    int E, int T, float* __restrict__ prob_mean, float* __restrict__ z_loss) {
  pdl_wait();
  pdl_launch_dependents();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (z_loss != nullptr && blockIdx.x == gridDim.x - 1) {
    if (warp != 0) return;
    double s = 0.0;
    for (int c = lane; c < nch; c += 32) s += (double)zsum[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(0xffffffffu, s, o);
    if (lane == 0) *z_loss = (float)(s / (double)T);
    return;
  }
  const int e = blockIdx.x * (blockDim.x / 32) + warp;
  if (prob_mean == nullptr || e >= E) return;
  float s = 0.f;
  for (int c = lane; c < nch; c += 32) s += psum[(size_t)c * E + e];
  s = warp_sum(s);
  if (lane == 0) prob_mean[e] = s / (float)T;
}

template <int NJ, typename TX>
cudaError_t launch_route_nj(const moe_config& c, const void* x, const void* wg, const float* bg,
                            int32_t* idx, float* w, float* gap, int32_t* hist, float* psum,
                            int32_t* ntie, float* zsum, uint32_t* status, cudaStream_t s) {
  const size_t smem = RouteSmem<NJ>::total;
  auto kern = route_kernel<NJ, TX>;
  cudaError_t err = set_smem_once<route_kernel<NJ, TX>>(smem);
  if (err != cudaSuccess) return err;
  const int nch = num_chunks(c.T);
  kern<<<nch, kThreads, smem, s>>>(static_cast<const TX*>(x), static_cast<const TX*>(wg), bg,
                                   c.T, c.d, c.E, c.k, c.lambda, idx, w, gap, hist, psum, ntie, zsum, nch,
                                   status);
  return cudaGetLastError();
}

template <typename TX>
cudaError_t launch_route_t(const moe_config& c, const void* x, const void* wg, const float* bg,
                           int32_t* idx, float* w, float* gap, int32_t* hist, float* psum,
                           int32_t* ntie, float* zsum, uint32_t* status, cudaStream_t s) {
  if (c.E <= 16) return launch_route_nj<1, TX>(c, x, wg, bg, idx, w, gap, hist, psum, ntie, zsum, status, s);
  if (c.E <= 32) return launch_route_nj<2, TX>(c, x, wg, bg, idx, w, gap, hist, psum, ntie, zsum, status, s);
  if (c.E <= 64) return launch_route_nj<4, TX>(c, x, wg, bg, idx, w, gap, hist, psum, ntie, zsum, status, s);
  if (c.E <= 128) return launch_route_nj<8, TX>(c, x, wg, bg, idx, w, gap, hist, psum, ntie, zsum, status, s);
  return launch_route_nj<16, TX>(c, x, wg, bg, idx, w, gap, hist, psum, ntie, zsum, status, s);
}

}  // namespace

cudaError_t launch_route(const moe_config& c, const void* x, const void* wg, const float* bg,
                         int32_t* topk_idx, float* topk_w, float* gap,
                         int32_t* hist, float* psum, int32_t* ntie, float* zsum, uint32_t* status,
                         cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  if (route_tc_supported(c))
    return launch_route_tc(c, x, wg, bg, topk_idx, topk_w, gap, hist, psum, ntie, zsum, status, s);
  if (c.dtype == MOE_DTYPE_BF16)
    return launch_route_t<__nv_bfloat16>(c, x, wg, bg, topk_idx, topk_w, gap, hist, psum, ntie, zsum, status, s);
  return launch_route_t<float>(c, x, wg, bg, topk_idx, topk_w, gap, hist, psum, ntie, zsum, status, s);
}

cudaError_t launch_route_totals(const moe_config& c, const float* psum, const float* zsum, float* prob_mean,
                                float* z_loss, cudaStream_t s) {
  if (prob_mean == nullptr && z_loss == nullptr) return cudaSuccess;
  const int blocks = (prob_mean != nullptr ? (c.E + 7) / 8 : 0) + (z_loss != nullptr ? 1 : 0);
  return launch_pdl(route_totals_kernel, dim3(blocks), dim3(256), 0, s, psum, zsum, num_chunks(c.T), c.E, c.T,
                    prob_mean, z_loss);
}

}  // namespace moe
