// The backward of the layer around the expert GEMMs: the padded permutation
// the backward GEMMs run on, the gradient of the gate (through the renormalised
// top-k weights, the softmax, the aux loss, the z-loss and the gating-logit
// normalisation), and the gradients of x and of the gate weights.
//
// The forward's discrete choices (the top-k selection, the capacity drops and
// the counts of the aux loss) carry no gradient: the backward reads them from
// the forward's workspace.  The pages' figures for the layer are training
// figures (FastMoE announcement, "特色三"); the normalisation is the Skywork
// release's ("Gating Logits归一化操作"), the aux loss the Switch form the
// Skywork slides build on (slide 4) and the z-loss the one the Megatron-Core
// best-practice page names ("Megatron-Core MoE的关键特性").
#include "internal.cuh"

#include <math.h>

#include <algorithm>

#include <type_traits>

namespace moe {
namespace {

constexpr int kPad = 64;   // rows of a backward segment: a multiple of the GEMMs' k-block

// max |dout| over the batch, as the bits of a non-negative float (their
// integer order is the float order), for the fp16 operands' scale.
__global__ void __launch_bounds__(256)
dout_amax_kernel(const float* __restrict__ dout, size_t n, unsigned* __restrict__ amax) {
  pdl_wait();
  pdl_launch_dependents();
  float m = 0.f;
  const size_t stride = (size_t)gridDim.x * blockDim.x;
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n / 4; i += stride) {
    const float4 v = __ldg(reinterpret_cast<const float4*>(dout) + i);
    m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
  }
  m = warp_max(m);
  if ((threadIdx.x & 31) == 0) atomicMax(amax, __float_as_uint(m));
}

// One warp: padded offsets, pad_offsets[e] = sum over e' < e of kept rounded
// up to 64; and the scale of the fp16 operands: s = 2^(10 - ceil(log2 max|dout|)),
// a power of two that brings max|s dout| into [512, 1024) (an all-zero or
// non-finite dout keeps s = 1).
__global__ void bwd_prep_kernel(const int32_t* __restrict__ offsets, int E, int32_t* __restrict__ pad_offsets,
                                const unsigned* __restrict__ amax, float* __restrict__ scale) {
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x;
  if (lane == 0) {
    float s = 1.f;
    if (amax != nullptr) {
      const float a = __uint_as_float(*amax);
      if (a > 0.f && isfinite(a)) {
        int ex;
        (void)frexpf(a, &ex);   // a = m 2^ex, m in [0.5, 1)
        s = ldexpf(1.f, 10 - ex);
      }
    }
    scale[0] = s;
    scale[1] = 1.f / s;   // exact: s is a power of two
  }
  constexpr int PER = kMaxExperts / 32;
  int loc[PER], sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    int v = 0;
    if (e < E) {
      const int kept = offsets[e + 1] - offsets[e];
      v = (kept + kPad - 1) / kPad * kPad;
    }
    loc[i] = v;
    sum += v;
  }
  int incl = sum;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(0xffffffffu, incl, o);
    if (lane >= o) incl += u;
  }
  int run = incl - sum;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    if (e < E) pad_offsets[e] = run;
    run += loc[i];
  }
  if (lane == 31) pad_offsets[E] = incl;
}

__device__ __forceinline__ int find_segment(const int32_t* off, int E, int r) {
  int lo = 0, hi = E - 1;   // the largest e with off[e] <= r
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (off[mid] <= r) lo = mid; else hi = mid - 1;
  }
  return lo;
}

__device__ __forceinline__ uint32_t pack_bf16x2(float a, float b) {
  __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  return *reinterpret_cast<uint32_t*>(&h);
}

// One warp per padded row: the token of the row (kept rows of the forward's
// permutation, each expert's segment moved to its padded start), its gate
// weight, and the row's x and s * dout in the GEMMs' operand type TG (bf16 or
// fp16 on the bf16 path: fp16 saturates at +-65504 and sets MOE_DEV_RANGE;
// fp32 on the fp32 path).  Padding rows and rows past the last segment are zero.
template <typename TG> struct OpType;
template <> struct OpType<__nv_bfloat16> {
  __device__ __forceinline__ static uint32_t pack(float a, float b, bool&) { return pack_bf16x2(a, b); }
};
template <> struct OpType<__half> {
  __device__ __forceinline__ static uint32_t pack(float a, float b, bool& over) {
    const bool oa = fabsf(a) > 65504.f, ob = fabsf(b) > 65504.f;
    over |= oa | ob;
    __half2 h = __floats2half2_rn(oa ? copysignf(65504.f, a) : a, ob ? copysignf(65504.f, b) : b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
};

template <typename TX, typename TG>
__global__ void __launch_bounds__(256)
bwd_gather_kernel(const TX* __restrict__ x, const float* __restrict__ dout, const int32_t* __restrict__ offsets,
                  const int32_t* __restrict__ pad_offsets, const int32_t* __restrict__ src_tok,
                  const int32_t* __restrict__ row_of, const float* __restrict__ topk_w, int E, int T, int k, int d,
                  int rows_alloc, const float* __restrict__ scale, TG* __restrict__ xp, TG* __restrict__ dout_perm,
                  float* __restrict__ wrow, uint32_t* __restrict__ status) {
  __shared__ int32_t s_off[kMaxExperts + 1], s_pad[kMaxExperts + 1];
  pdl_wait();
  pdl_launch_dependents();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) {
    s_off[e] = offsets[e];
    s_pad[e] = pad_offsets[e];
  }
  __syncthreads();
  const int lane = threadIdx.x & 31;
  const int pr = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (pr >= rows_alloc) return;
  const float sc = scale[0];
  int t = -1;
  float w = 0.f;
  if (pr < s_pad[E]) {
    const int e = find_segment(s_pad, E, pr);
    const int i = pr - s_pad[e];
    if (i < s_off[e + 1] - s_off[e]) {
      const int row = s_off[e] + i;
      t = src_tok[row];
      if ((unsigned)t >= (unsigned)T) {
        if (lane == 0) atomicOr(status, MOE_DEV_BOUNDS);
        t = -1;
      } else {
        for (int j = 0; j < k; ++j)
          if (row_of[(size_t)t * k + j] == row) w = topk_w[(size_t)t * k + j];
      }
    }
  }
  if (lane == 0) wrow[pr] = w;
  if constexpr (sizeof(TG) == 2) {
    const int nvec = d / 8;   // 8 elements = 16 bytes
    uint4* xo = reinterpret_cast<uint4*>(xp + (size_t)pr * d);
    uint4* go = reinterpret_cast<uint4*>(dout_perm + (size_t)pr * d);
    bool over = false;
    for (int v = lane; v < nvec; v += 32) {
      uint4 xv = make_uint4(0u, 0u, 0u, 0u), gv = xv;
      if (t >= 0) {
        xv = __ldg(reinterpret_cast<const uint4*>(x + (size_t)t * d) + v);
        if constexpr (std::is_same<TG, __half>::value) {   // bf16 x -> fp16 (exact inside the fp16 range)
          const __nv_bfloat162* b = reinterpret_cast<const __nv_bfloat162*>(&xv);
          uint32_t o[4];
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const float2 f = __bfloat1622float2(b[q]);
            o[q] = OpType<__half>::pack(f.x, f.y, over);
          }
          xv = make_uint4(o[0], o[1], o[2], o[3]);
        }
        const float4 a = __ldg(reinterpret_cast<const float4*>(dout + (size_t)t * d) + 2 * v);
        const float4 b = __ldg(reinterpret_cast<const float4*>(dout + (size_t)t * d) + 2 * v + 1);
        gv = make_uint4(OpType<TG>::pack(sc * a.x, sc * a.y, over), OpType<TG>::pack(sc * a.z, sc * a.w, over),
                        OpType<TG>::pack(sc * b.x, sc * b.y, over), OpType<TG>::pack(sc * b.z, sc * b.w, over));
      }
      xo[v] = xv;
      go[v] = gv;
    }
    if (__any_sync(0xffffffffu, over) && lane == 0) atomicOr(status, MOE_DEV_RANGE);
  } else {
    const int nvec = d / 4;
    float4* xo = reinterpret_cast<float4*>(xp + (size_t)pr * d);
    float4* go = reinterpret_cast<float4*>(dout_perm + (size_t)pr * d);
    for (int v = lane; v < nvec; v += 32) {
      float4 xv = make_float4(0.f, 0.f, 0.f, 0.f), gv = xv;
      if (t >= 0) {
        xv = __ldg(reinterpret_cast<const float4*>(x + (size_t)t * d) + v);
        gv = __ldg(reinterpret_cast<const float4*>(dout + (size_t)t * d) + v);
        gv = make_float4(sc * gv.x, sc * gv.y, sc * gv.z, sc * gv.w);
      }
      xo[v] = xv;
      go[v] = gv;
    }
  }
}

// Gate logits in fp32 (the forward keeps them on chip only), as partial sums
// over slices of the model width: zpart[s][t][e] = sum over slice s of
// x[t, c] W_gate[e, c].  The reader adds the bias and the slices in slice
// order.  A block computes 32 tokens x 16 experts (two per thread), the
// slice staged 32 columns at a time; the slices (blockIdx.z) put enough
// blocks in flight when T is small.
constexpr int kLT = 32, kLK = 32, kLE = 16;
template <typename TX>
__global__ void __launch_bounds__(256)
logits_kernel(const TX* __restrict__ x, const TX* __restrict__ wg, int T, int d, int E, int kslice,
              float* __restrict__ zpart) {
  __shared__ float xs[kLT][kLK + 1];
  __shared__ float ws[kLE][kLK + 1];
  pdl_wait();
  pdl_launch_dependents();
  const int t0 = blockIdx.x * kLT, e0 = blockIdx.y * kLE;
  const int ks = blockIdx.z;
  const int kbeg = ks * kslice, kend = min(d, kbeg + kslice);
  const int tid = threadIdx.x;
  // thread (tt, eg): token t0 + tt, experts e0 + eg and e0 + eg + 8
  const int tt = tid & 31, eg = tid >> 5;
  float acc0 = 0.f, acc1 = 0.f;
  for (int k0 = kbeg; k0 < kend; k0 += kLK) {
#pragma unroll
    for (int i = tid; i < kLT * kLK; i += 256) {
      const int r = i / kLK, c = i % kLK;
      xs[r][c] = (t0 + r < T && k0 + c < kend) ? to_float(x[(size_t)(t0 + r) * d + k0 + c]) : 0.f;
    }
#pragma unroll
    for (int i = tid; i < kLE * kLK; i += 256) {
      const int r = i / kLK, c = i % kLK;
      ws[r][c] = (e0 + r < E && k0 + c < kend) ? to_float(wg[(size_t)(e0 + r) * d + k0 + c]) : 0.f;
    }
    __syncthreads();
#pragma unroll 8
    for (int c = 0; c < kLK; ++c) {
      const float xv = xs[tt][c];
      acc0 = fmaf(xv, ws[eg][c], acc0);
      acc1 = fmaf(xv, ws[eg + 8][c], acc1);
    }
    __syncthreads();
  }
  if (t0 + tt < T) {
    float* zs = zpart + ((size_t)ks * T + t0 + tt) * E;
    if (e0 + eg < E) zs[e0 + eg] = acc0;
    if (e0 + eg + 8 < E) zs[e0 + eg + 8] = acc1;
  }
}

// One warp per token: the gradient of the scores and the logits.
//   dw[j]  = sum over the layer-2 column tiles of the kept row's G h partial
//            (0 for a dropped slot);
//   dp     = (dw_i - sum_j w_j dw_j) / sum(p_sel) on the selected experts,
//            plus aux_coef * E * f_e / T everywhere (f_e = counts_e / (T k));
//   ds     = p (dp - <dp, p>) + z_coef * (2 / T) * lse * p;
//   dz     = ds, or through z_hat = lambda (z - mean) / std:
//            (lambda / std) (ds - mean(ds) - n mean(ds n)), 0 at zero spread.
// The softmax is recomputed from the fp32 logits the way the route kernel
// computes it.  Lanes hold experts lane + 32 i.
__global__ void __launch_bounds__(256)
gate_bwd_kernel(const float* __restrict__ zpart, int nks, const float* __restrict__ bg,
                const int32_t* __restrict__ topk_idx, const float* __restrict__ topk_w,
                const int32_t* __restrict__ row_of, const int32_t* __restrict__ offsets,
                const int32_t* __restrict__ pad_offsets, const int32_t* __restrict__ counts,
                const float* __restrict__ dwpart, int nt2, int rows_alloc, int T, int E, int k, float lam,
                float aux_coef, float z_coef, float* __restrict__ dz, float* __restrict__ dw_out) {
  constexpr int PER = kMaxExperts / 32;
  pdl_wait();
  pdl_launch_dependents();
  const int lane = threadIdx.x & 31;
  const int t = blockIdx.x * (blockDim.x / 32) + (threadIdx.x >> 5);
  if (t >= T) return;
  float zv[PER], s[PER], p[PER];
  bool ok[PER];
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane + 32 * i;
    ok[i] = e < E;
    float zz = 0.f;
    if (ok[i]) {
      zz = (bg != nullptr) ? bg[e] : 0.f;
      for (int sl = 0; sl < nks; ++sl) zz += zpart[((size_t)sl * T + t) * E + e];
    }
    zv[i] = zz;
  }
  float mu = 0.f, sd = 0.f;
  if (lam > 0.f) {
    float a = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) a += zv[i];
    mu = warp_sum(a) / (float)E;
    float q = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const float dv = ok[i] ? zv[i] - mu : 0.f;
      q += dv * dv;
    }
    sd = sqrtf(warp_sum(q) / (float)E);
#pragma unroll
    for (int i = 0; i < PER; ++i) s[i] = (sd == 0.f) ? 0.f : lam * (zv[i] - mu) / sd;   // as the forward
  } else {
#pragma unroll
    for (int i = 0; i < PER; ++i) s[i] = zv[i];
  }
  float m = -INFINITY;
#pragma unroll
  for (int i = 0; i < PER; ++i) if (ok[i]) m = fmaxf(m, s[i]);
  m = warp_max(m);
  float S = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    p[i] = ok[i] ? expf(s[i] - m) : 0.f;
    S += p[i];
  }
  S = warp_sum(S);
  const float invS = 1.f / S;
#pragma unroll
  for (int i = 0; i < PER; ++i) p[i] *= invS;
  const float lse = m + logf(S);

  // the gate weights' gradient, slot by slot (dw of the warp's token in shared memory)
  __shared__ float dwsm[8][kMaxExperts];
  float* dws = dwsm[threadIdx.x >> 5];
  float dp[PER];
  const float aux_scale = aux_coef * (float)E / ((float)T * (float)T * (float)k);
#pragma unroll
  for (int i = 0; i < PER; ++i) dp[i] = ok[i] ? aux_scale * (float)counts[lane + 32 * i] : 0.f;
  float wdw = 0.f, psel = 0.f;
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[(size_t)t * k + j];
    const int row = row_of[(size_t)t * k + j];
    float dwj = 0.f;
    if (lane == 0 && row >= 0 && (unsigned)e < (unsigned)E) {
      const int pr = pad_offsets[e] + (row - offsets[e]);
      if ((unsigned)pr < (unsigned)rows_alloc)
        for (int n = 0; n < nt2; ++n) dwj += dwpart[(size_t)n * rows_alloc + pr];   // fixed order
    }
    dwj = __shfl_sync(0xffffffffu, dwj, 0);
    if (lane == 0) {
      dws[j] = dwj;
      if (dw_out != nullptr) dw_out[(size_t)t * k + j] = dwj;
    }
    wdw += topk_w[(size_t)t * k + j] * dwj;
    // the selected probability, from the lane that holds expert e
    float pe = 0.f;
#pragma unroll
    for (int i = 0; i < PER; ++i) if (lane + 32 * i == e) pe = p[i];
    psel += __shfl_sync(0xffffffffu, pe, e & 31);
  }
  __syncwarp();
  for (int j = 0; j < k; ++j) {
    const int e = topk_idx[(size_t)t * k + j];
    const float g = (dws[j] - wdw) / psel;
#pragma unroll
    for (int i = 0; i < PER; ++i) if (lane + 32 * i == e) dp[i] += g;
  }
  float dpp = 0.f;
#pragma unroll
  for (int i = 0; i < PER; ++i) dpp += dp[i] * p[i];
  dpp = warp_sum(dpp);
  float ds[PER];
  const float zs = z_coef * 2.f / (float)T * lse;
#pragma unroll
  for (int i = 0; i < PER; ++i) ds[i] = ok[i] ? p[i] * (dp[i] - dpp) + zs * p[i] : 0.f;
  if (lam > 0.f) {
    if (sd != 0.f) {
      float a = 0.f, b = 0.f;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const float n = ok[i] ? (zv[i] - mu) / sd : 0.f;
        a += ds[i];
        b += ds[i] * n;
      }
      a = warp_sum(a) / (float)E;
      b = warp_sum(b) / (float)E;
#pragma unroll
      for (int i = 0; i < PER; ++i) {
        const float n = (zv[i] - mu) / sd;
        ds[i] = (lam / sd) * (ds[i] - a - n * b);
      }
    } else {
#pragma unroll
      for (int i = 0; i < PER; ++i) ds[i] = 0.f;
    }
  }
#pragma unroll
  for (int i = 0; i < PER; ++i)
    if (ok[i]) dz[(size_t)t * E + lane + 32 * i] = ds[i];
}

// dx[t, c] = sum over kept slots (slot order) of dxp[padded row, c]
//          + sum_e dz[t, e] W_gate[e, c];  16 tokens x 512 columns per block
// (4 consecutive columns per thread when d is a multiple of 4).  The padded
// rows of the block's slots are found once, into shared memory, so that the
// row loads of different tokens are independent.
template <typename TX>
__global__ void __launch_bounds__(128)
dx_kernel(const float* __restrict__ dxp, const float* __restrict__ dz, const TX* __restrict__ wg,
          const int32_t* __restrict__ topk_idx, const int32_t* __restrict__ row_of,
          const int32_t* __restrict__ offsets, const int32_t* __restrict__ pad_offsets, int T, int E, int k, int d,
          int rows_alloc, float* __restrict__ dx) {
  constexpr int TT = 16, V = 4;
  __shared__ float dzs[TT][kMaxExperts + 1];
  __shared__ int prow[TT * kMaxExperts];
  pdl_wait();
  pdl_launch_dependents();
  const int t0 = blockIdx.x * TT;
  for (int i = threadIdx.x; i < TT * E; i += blockDim.x) {
    const int r = i / E, e = i % E;
    dzs[r][e] = (t0 + r < T) ? dz[(size_t)(t0 + r) * E + e] : 0.f;
  }
  for (int i = threadIdx.x; i < TT * k; i += blockDim.x) {
    const int r = i / k, j = i % k, t = t0 + r;
    int pr = -1;
    if (t < T) {
      const int row = row_of[(size_t)t * k + j];
      const int e = topk_idx[(size_t)t * k + j];
      if (row >= 0 && (unsigned)e < (unsigned)E) {
        pr = pad_offsets[e] + (row - offsets[e]);
        if ((unsigned)pr >= (unsigned)rows_alloc) pr = -1;
      }
    }
    prow[i] = pr;
  }
  __syncthreads();
  const int nt = min(TT, T - t0);
  if ((d & (V - 1)) == 0) {
    const int c = (blockIdx.y * blockDim.x + threadIdx.x) * V;
    if (c >= d) return;
    float4 acc[TT];
#pragma unroll
    for (int r = 0; r < TT; ++r) acc[r] = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int e = 0; e < E; ++e) {
      const float w0 = to_float(wg[(size_t)e * d + c]), w1 = to_float(wg[(size_t)e * d + c + 1]);
      const float w2 = to_float(wg[(size_t)e * d + c + 2]), w3 = to_float(wg[(size_t)e * d + c + 3]);
#pragma unroll
      for (int r = 0; r < TT; ++r) {
        const float zv = dzs[r][e];
        acc[r].x = fmaf(zv, w0, acc[r].x);
        acc[r].y = fmaf(zv, w1, acc[r].y);
        acc[r].z = fmaf(zv, w2, acc[r].z);
        acc[r].w = fmaf(zv, w3, acc[r].w);
      }
    }
#pragma unroll
    for (int r = 0; r < TT; ++r) {
      if (r >= nt) continue;
      float4 v = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int j = 0; j < k; ++j) {
        const int pr = prow[r * k + j];
        if (pr < 0) continue;
        const float4 a = __ldcs(reinterpret_cast<const float4*>(dxp + (size_t)pr * d + c));
        v.x += a.x;
        v.y += a.y;
        v.z += a.z;
        v.w += a.w;
      }
      __stcs(reinterpret_cast<float4*>(dx + (size_t)(t0 + r) * d + c),
             make_float4(v.x + acc[r].x, v.y + acc[r].y, v.z + acc[r].z, v.w + acc[r].w));
    }
  } else {
    for (int c = (blockIdx.y * blockDim.x + threadIdx.x) * V, cend = min(d, c + V); c < cend; ++c) {
      for (int r = 0; r < nt; ++r) {
        float a = 0.f;
        for (int e = 0; e < E; ++e) a = fmaf(dzs[r][e], to_float(wg[(size_t)e * d + c]), a);
        float v = 0.f;
        for (int j = 0; j < k; ++j) {
          const int pr = prow[r * k + j];
          if (pr >= 0) v += dxp[(size_t)pr * d + c];
        }
        dx[(size_t)(t0 + r) * d + c] = v + a;
      }
    }
  }
}

// dW_gate partials: part[s][e][c] = sum over tokens of split s of dz[t, e] x[t, c]
// (and the bias gradient in column d of a [E][d + 1] partial), then a fixed-order
// sum over the splits.
template <typename TX>
__global__ void __launch_bounds__(128)
dwg_partial_kernel(const float* __restrict__ dz, const TX* __restrict__ x, int T, int E, int d, int tok_per_split,
                   float* __restrict__ part) {
  constexpr int EB = 16;   // experts per block
  __shared__ float dzs[64][EB];
  pdl_wait();
  pdl_launch_dependents();
  const int split = blockIdx.z;
  const int e0 = blockIdx.y * EB;
  const int c = blockIdx.x * 128 + threadIdx.x;   // c == d: the bias column
  const int ta = split * tok_per_split, tb = min(T, ta + tok_per_split);
  float acc[EB];
#pragma unroll
  for (int i = 0; i < EB; ++i) acc[i] = 0.f;
  for (int t0 = ta; t0 < tb; t0 += 64) {
    for (int i = threadIdx.x; i < 64 * EB; i += 128) {
      const int r = i / EB, e = e0 + i % EB;
      dzs[r][i % EB] = (t0 + r < tb && e < E) ? dz[(size_t)(t0 + r) * E + e] : 0.f;
    }
    __syncthreads();
    if (c <= d) {
      const int n = min(64, tb - t0);
      for (int r = 0; r < n; ++r) {
        const float xv = (c < d) ? to_float(x[(size_t)(t0 + r) * d + c]) : 1.f;
#pragma unroll
        for (int i = 0; i < EB; ++i) acc[i] = fmaf(dzs[r][i], xv, acc[i]);
      }
    }
    __syncthreads();
  }
  if (c <= d) {
#pragma unroll
    for (int i = 0; i < EB; ++i)
      if (e0 + i < E) part[((size_t)split * E + e0 + i) * (d + 1) + c] = acc[i];
  }
}

__global__ void dwg_reduce_kernel(const float* __restrict__ part, int nsplit, int E, int d, float* __restrict__ dwg,
                                  float* __restrict__ dbg) {
  pdl_wait();
  pdl_launch_dependents();
  const size_t n = (size_t)E * (d + 1);
  for (size_t i = (size_t)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (size_t)gridDim.x * blockDim.x) {
    float s = 0.f;
    for (int sp = 0; sp < nsplit; ++sp) s += part[(size_t)sp * n + i];
    const int e = (int)(i / (d + 1)), c = (int)(i % (d + 1));
    if (c < d) dwg[(size_t)e * d + c] = s;
    else if (dbg != nullptr) dbg[e] = s;
  }
}

template <typename TX, typename TG>
cudaError_t launch_bwd_front_t(const moe_config& c, const void* x, const float* dout, const BwdState& st,
                               cudaStream_t s) {
  cudaError_t e;
  if (st.f16) {   // max |dout| for the scale of the fp16 operands
    if ((e = cudaMemsetAsync(st.amax, 0, sizeof(unsigned), s)) != cudaSuccess) return e;
    DeviceInfo di;
    if ((e = device_info(&di)) != cudaSuccess) return e;
    const size_t n = (size_t)c.T * c.d;   // d is a multiple of 16: whole float4 vectors
    const int grid = (int)std::max<size_t>(1, std::min<size_t>((n / 4 + 255) / 256, (size_t)di.sms * 4));
    if ((e = launch_pdl(dout_amax_kernel, dim3(grid), dim3(256), 0, s, dout, n, st.amax)) != cudaSuccess) return e;
  }
  e = launch_pdl(bwd_prep_kernel, dim3(1), dim3(32), 0, s, st.offsets, c.E, st.pad_offsets,
                 (const unsigned*)(st.f16 ? st.amax : nullptr), st.scale);
  if (e != cudaSuccess) return e;
  const int rows = st.rows_alloc;
  return launch_pdl(bwd_gather_kernel<TX, TG>, dim3((rows + 7) / 8), dim3(256), 0, s, static_cast<const TX*>(x),
                    dout, st.offsets, (const int32_t*)st.pad_offsets, st.src_tok, st.row_of, st.topk_w, c.E, c.T,
                    c.k, c.d, rows, (const float*)st.scale, static_cast<TG*>(st.xp), static_cast<TG*>(st.dout_perm),
                    st.wrow, st.status);
}

template <typename TX>
cudaError_t launch_bwd_gate_t(const moe_config& c, const void* x, const void* wg, const float* bg,
                              const BwdState& st, float aux_coef, float z_coef, float* dx, float* dwg, float* dbg,
                              float* dw_out, cudaStream_t s) {
  const TX* X = static_cast<const TX*>(x);
  const TX* WG = static_cast<const TX*>(wg);
  const int nks = bwd_logit_slices(c);
  const int kslice = (c.d + nks - 1) / nks;
  cudaError_t e = launch_pdl(logits_kernel<TX>, dim3((c.T + kLT - 1) / kLT, (c.E + kLE - 1) / kLE, nks), dim3(256),
                             0, s, X, WG, c.T, c.d, c.E, kslice, st.z);
  if (e != cudaSuccess) return e;
  // column tiles of the dh GEMM, each of which left one partial of dw per row
  const int col = c.dtype == MOE_DTYPE_BF16 ? bwd_tc_col_tile() : bwd_simt_col_tile();
  const int nt2 = (c.F + col - 1) / col;
  e = launch_pdl(gate_bwd_kernel, dim3((c.T + 7) / 8), dim3(256), 0, s, (const float*)st.z, nks, bg, st.topk_idx,
                 st.topk_w, st.row_of, st.offsets, (const int32_t*)st.pad_offsets, st.counts,
                 (const float*)st.dwpart, nt2, st.rows_alloc, c.T, c.E, c.k, c.lambda, aux_coef, z_coef, st.dz,
                 dw_out);
  if (e != cudaSuccess) return e;
  e = launch_pdl(dx_kernel<TX>, dim3((c.T + 15) / 16, (c.d + 511) / 512), dim3(128), 0, s, (const float*)st.dxp,
                 (const float*)st.dz, WG, st.topk_idx, st.row_of, st.offsets, (const int32_t*)st.pad_offsets, c.T,
                 c.E, c.k, c.d, st.rows_alloc, dx);
  if (e != cudaSuccess) return e;
  e = launch_pdl(dwg_partial_kernel<TX>, dim3((c.d + 1 + 127) / 128, (c.E + 15) / 16, st.nsplit), dim3(128), 0, s,
                 (const float*)st.dz, X, c.T, c.E, c.d, st.tok_per_split, st.dwg_part);
  if (e != cudaSuccess) return e;
  return launch_pdl(dwg_reduce_kernel, dim3(148), dim3(256), 0, s, (const float*)st.dwg_part, st.nsplit, c.E,
                    c.d, dwg, dbg);
}

}  // namespace

int bwd_pad_rows() { return kPad; }

// Model-width slices of the logits recompute: enough 32 x 16 blocks for
// about four waves of 148 SMs, at most 8, each slice at least 32 columns.
int bwd_logit_slices(const moe_config& c) {
  const int blocks = ((c.T + kLT - 1) / kLT) * ((c.E + kLE - 1) / kLE);
  const int want = blocks > 0 ? (4 * 148 + blocks - 1) / blocks : 1;
  return std::max(1, std::min({want, 8, (c.d + kLK - 1) / kLK}));
}

cudaError_t launch_bwd_front(const moe_config& c, const void* x, const float* dout, const BwdState& st,
                             cudaStream_t s) {
  if (c.dtype == MOE_DTYPE_BF16) {
    if (st.f16) return launch_bwd_front_t<__nv_bfloat16, __half>(c, x, dout, st, s);
    return launch_bwd_front_t<__nv_bfloat16, __nv_bfloat16>(c, x, dout, st, s);
  }
  return launch_bwd_front_t<float, float>(c, x, dout, st, s);
}

cudaError_t launch_bwd_gate(const moe_config& c, const void* x, const void* wg, const float* bg, const BwdState& st,
                            float aux_coef, float z_coef, float* dx, float* dwg, float* dbg, float* dw_out,
                            cudaStream_t s) {
  if (c.dtype == MOE_DTYPE_BF16)
    return launch_bwd_gate_t<__nv_bfloat16>(c, x, wg, bg, st, aux_coef, z_coef, dx, dwg, dbg, dw_out, s);
  return launch_bwd_gate_t<float>(c, x, wg, bg, st, aux_coef, z_coef, dx, dwg, dbg, dw_out, s);
}

}  // namespace moe
