// The expert MLP with FP8 weights in the MX form: E4M3 elements and one
// power-of-two (UE8M0) scale per 32 consecutive elements along the reduction,
// run by tcgen05.mma kind::mxf8f6f4 with the scales in TMEM.
//
// Skywork-MoE serves its model with FP8 weights (Skywork-MoE release,
// inference section: 146 GB of FP8 weights on 8 x 4090); the pages fix no
// FP8 format.  This is the block-scaled form the B200 tensor cores take
// natively.  A block's scale is 2^X with X the least integer that brings
// every |v| / 2^X within 448 (no element saturates); elements round to the
// nearest E4M3 value, ties to even.  Both expert layers run on it: the
// weights are quantised once (moe_prepare_mxfp8_weights), the layer-1 input
// rows and the hidden activation per call.  For the decode-sized layers the
// expert step streams the touched experts' weights from HBM, so halving
// their bytes halves the step.
//
// Layouts (all row-major):
//   elements : [rows][K] bytes;
//   scales   : atoms of 512 bytes, atom (r / 128) * (K / 128) + k / 128 for
//              row r, element k; inside it, byte 16 (r % 32) + 4 ((r % 128) / 32)
//              + (k / 32) % 4.  One atom is exactly what one
//              tcgen05.cp.32x128b.warpx4 moves to TMEM: the scales of 128
//              rows for a 128-element K stage, row r in lane r % 32 (and its
//              three copies), column (r % 128) / 32, byte = the 32-element block.
//   W1 of a SwiGLU expert is stored with its rows interleaved by 64: rows
//   [128 b, 128 b + 64) are gate rows [64 b, 64 b + 64) and the next 64 the
//   matching up rows, so one 128-row weight tile feeds both halves.
//   Activation rows are padded per expert to multiples of 128, so that a
//   128-row tile never spans two experts and its scales are whole atoms.
#include "gemm_common.cuh"

#include <cuda_fp8.h>

#include <algorithm>

namespace moe {
namespace {

using namespace tc;

constexpr int MB = 128, MN = 128, MK = 128;   // tile rows, columns, K elements (bytes) per stage
constexpr int STAGES = 6;
constexpr int A_BYTES = MB * MK, B_BYTES = MN * MK;   // 16 KB each
constexpr int SF_BYTES = 512;                         // one scale atom per operand
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;                     // scale columns after the two 128-column accumulators
constexpr int kMxPad = 128;

enum { kMxRelu = 0, kMxSwiglu = 1, kMxOut = 2 };

// Least X with amax <= 448 * 2^X (-127 for 0); the UE8M0 byte is X + 127.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  int e;
  const float m = frexpf(amax, &e);   // amax = m 2^e, m in [0.5, 1)
  const int X = (2.f * m <= 1.75f) ? e - 9 : e - 8;
  return max(-127, min(127, X));
}

__device__ __forceinline__ size_t sf_offset(int r, int k, int K) {
  return ((size_t)(r / 128) * (K / 128) + k / 128) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + (k / 32) % 4;
}

// 32 fp32 values -> 32 E4M3 bytes (scaled by 2^-X), round to nearest even.
__device__ __forceinline__ void quantize32(const float (&v)[32], int X, uint4& lo, uint4& hi) {
  const float s = ldexpf(1.f, -X);
  uint32_t w[8];
#pragma unroll
  for (int i = 0; i < 8; ++i) {
    const __nv_fp8x2_storage_t a = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i] * s, v[4 * i + 1] * s),
                                                             __NV_SATFINITE, __NV_E4M3);
    const __nv_fp8x2_storage_t b = __nv_cvt_float2_to_fp8x2(make_float2(v[4 * i + 2] * s, v[4 * i + 3] * s),
                                                             __NV_SATFINITE, __NV_E4M3);
    w[i] = (uint32_t)a | ((uint32_t)b << 16);
  }
  lo = make_uint4(w[0], w[1], w[2], w[3]);
  hi = make_uint4(w[4], w[5], w[6], w[7]);
}

// One thread per 32-element block of a bf16 matrix [rows][K]: E4M3 bytes and
// the block's scale.  src_row(r) maps a destination row to its source row
// (-1: a zero row).  Used for the weights (with the SwiGLU interleave) and
// for the padded layer-1 input rows.
struct RowMapIdentity {
  __device__ int operator()(int r) const { return r; }
};
struct RowMapSwiglu {   // destination row of an expert's interleaved W1 -> source row
  int F;
  __device__ int operator()(int r) const {
    const int F1 = 2 * F, e = r / F1, i = r - e * F1, b = i / 128, j = i % 128;
    return e * F1 + (j < 64 ? 64 * b + j : F + 64 * b + (j - 64));
  }
};
struct RowMapPadded {   // padded activation row -> kept permuted row (-1: padding; -2: past the last segment)
  const int32_t* offsets;
  const int32_t* pad;
  int E;
  __device__ int operator()(int r) const {
    if (r >= pad[E]) return -2;
    int lo = 0, hi = E - 1;
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (pad[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int i = r - pad[lo];
    return i < offsets[lo + 1] - offsets[lo] ? offsets[lo] + i : -1;
  }
};

template <typename Map>
__global__ void __launch_bounds__(256)
mx_quantize_kernel(const __nv_bfloat16* __restrict__ src, int rows, int K, Map map, uint8_t* __restrict__ q,
                   uint8_t* __restrict__ sf) {
  pdl_wait();
  pdl_launch_dependents();
  const int nb = K / 32;
  const size_t nblk = (size_t)rows * nb;
  for (size_t b = (size_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += (size_t)gridDim.x * blockDim.x) {
    const int r = (int)(b / nb), kb = (int)(b - (size_t)r * nb);
    const int sr = map(r);
    if (sr == -2) continue;   // no tile reads rows past the last segment
    float v[32];
    if (sr >= 0) {
      const uint4* p = reinterpret_cast<const uint4*>(src + (size_t)sr * K + 32 * kb);
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const uint4 u = __ldg(p + i);
        const __nv_bfloat162* h = reinterpret_cast<const __nv_bfloat162*>(&u);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float2 f = __bfloat1622float2(h[j]);
          v[8 * i + 2 * j] = f.x;
          v[8 * i + 2 * j + 1] = f.y;
        }
      }
    } else {
#pragma unroll
      for (int i = 0; i < 32; ++i) v[i] = 0.f;
    }
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 32; ++i) amax = fmaxf(amax, fabsf(v[i]));
    const int X = mx_exponent(amax);
    uint4 lo, hi;
    quantize32(v, X, lo, hi);
    uint4* qo = reinterpret_cast<uint4*>(q + (size_t)r * K + 32 * kb);
    qo[0] = lo;
    qo[1] = hi;
    sf[sf_offset(r, 32 * kb, K)] = (uint8_t)(X + 127);
  }
}

// Padded offsets: every expert's kept rows rounded up to a multiple of 128
// (one warp; 8 experts per lane, then a shuffle scan).
__global__ void mx_pad_kernel(const int32_t* __restrict__ offsets, int E, int32_t* __restrict__ pad) {
  pdl_wait();
  pdl_launch_dependents();
  constexpr int PER = kMaxExperts / 32;
  const int lane = threadIdx.x;
  int loc[PER], sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    loc[i] = (e < E) ? (offsets[e + 1] - offsets[e] + kMxPad - 1) / kMxPad * kMxPad : 0;
    sum += loc[i];
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
    if (e < E) pad[e] = run;
    run += loc[i];
  }
  if (lane == 31) pad[E] = incl;
}

struct MxParams {
  const int32_t* pad;        // [E+1] padded segment offsets (multiples of 128)
  const int32_t* offsets;    // [E+1] kept offsets (kMxOut: the unpadded row of each padded row)
  int E, K, Nout;            // Nout: output columns (layer 1: h columns F; layer 2: d)
  int b_rows;                // weight rows per expert (F1 or d)
  int rows_pad;              // padded rows allocated
  const uint8_t* sfa;        // A scales (activation rows, atoms over K)
  const uint8_t* sfb;        // B scales (weight rows, atoms over K)
  uint8_t* hq;               // layer 1: [rows_pad][F] E4M3 h
  uint8_t* hs;               // layer 1: h scales (atoms over F)
  float* out;                // kMxOut: yp [rows][d] fp32 at the kept (unpadded) rows
  uint32_t* status;
};

struct MxTail {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];
};
constexpr size_t kMxSmem = 1024 + (size_t)STAGES * STAGE_BYTES + (size_t)STAGES * 2 * SF_BYTES +
                           gemm::kStagingBytes + sizeof(MxTail);
static_assert(kMxSmem <= 227 * 1024, "shared memory of one CTA");

// MODE kMxRelu / kMxSwiglu: layer 1, h = act(xq W1q^T) quantised into hq/hs;
// kMxOut: layer 2, yp = hq W2q^T in fp32 at the kept rows.
template <int MODE>
__global__ void __launch_bounds__(kThreads, 1)
tc_mx_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const MxParams p) {
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);
  const uint32_t sf_base = base + (uint32_t)(STAGES * STAGE_BYTES);
  unsigned char* staging = sbase + (size_t)STAGES * STAGE_BYTES + (size_t)STAGES * 2 * SF_BYTES;
  MxTail* tail = reinterpret_cast<MxTail*>(staging + gemm::kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt = (p.b_rows == 0) ? 0 : ((MODE == kMxOut ? p.Nout : (MODE == kMxSwiglu ? 2 * p.Nout : p.Nout)) +
                                        MN - 1) / MN;
  const int nkb = p.K / MK;

  const uint32_t full0 = smem_u32(&tail->full[0]), empty0 = smem_u32(&tail->empty[0]);
  const uint32_t tfull0 = smem_u32(&tail->tfull[0]), tempty0 = smem_u32(&tail->tempty[0]);
  const uint32_t drain = smem_u32(&tail->drain);
  const volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 4);
    }
    mbar_init(drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tail->tmem_base)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  pdl_wait();
  pdl_launch_dependents();
  if (warp == 0) {
    if (!tile_table_warp(p.pad, p.E, MB, nt, p.rows_pad, tail->tstart, lane) && lane == 0 && blockIdx.x == 0)
      atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  for (int e = threadIdx.x; e <= p.E; e += kThreads) tail->seg[e] = p.pad[e];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  const int total = tail->tstart[p.E];

  auto decode = [&](int L, int& e, int& row0, int& n0) {
    e = tile_expert(tail->tstart, p.E, L);
    const int M = tail->seg[e + 1] - tail->seg[e];
    const int mt = (M + MB - 1) / MB;
    const int local = L - tail->tstart[e];
    const int nti = local / mt, mti = local - nti * mt;
    row0 = tail->seg[e] + mti * MB;
    n0 = nti * MN;   // weight-row offset inside the expert (SwiGLU: interleaved rows)
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        int e, row0, n0;
        decode(L, e, row0, n0);
        const int brow = e * p.b_rows + n0;
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint32_t sfs = sf_base + (uint32_t)(s * 2 * SF_BYTES);
          mbar_expect_tx(full0 + 8 * s, STAGE_BYTES + 2 * SF_BYTES);
          tma_load_2d(sa, &tmA, full0 + 8 * s, kb * MK, row0);
          tma_load_2d(sa + A_BYTES, &tmB, full0 + 8 * s, kb * MK, brow);
          bulk_load(sfs, p.sfa + ((size_t)(row0 / 128) * nkb + kb) * SF_BYTES, SF_BYTES, full0 + 8 * s);
          bulk_load(sfs + SF_BYTES, p.sfb + ((size_t)(brow / 128) * nkb + kb) * SF_BYTES, SF_BYTES, full0 + 8 * s);
          ++it;
        }
      }
      if (!ok) {
        atomicOr(p.status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
      }
      for (int i = max(0, it - STAGES); i < it; ++i)
        mbar_wait(full0 + 8 * (i % STAGES), (uint32_t)(i / STAGES) & 1u, nullptr, kDrainNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int it = 0, tl = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x, ++tl) {
        const int acc = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * MN);
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint32_t sfs = sf_base + (uint32_t)(s * 2 * SF_BYTES);
          // this stage's scales to TMEM (4 columns each), ahead of its MMAs in issue order
          const uint32_t tsfa = tmem + kSfCol0 + (uint32_t)(8 * s), tsfb = tsfa + 4;
          tc_cp_32x128b_x4(tsfa, sdesc_rows16(sfs));
          tc_cp_32x128b_x4(tsfb, sdesc_rows16(sfs + SF_BYTES));
          const uint64_t ad = sdesc(sa), bd = sdesc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < MK / 32; ++kk)
            tc_mma_mx(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc_mx_e4m3(MB, MN, kk),
                      tsfa | ((uint32_t)kk << 30), tsfb | ((uint32_t)kk << 30), (kb | kk) != 0);
          tc_commit(empty0 + 8 * s);
          ++it;
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);
      }
      if (!ok) {
        atomicOr(p.status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
      }
      tc_commit(drain);
      mbar_wait(drain, 0, nullptr, kDrainNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * gemm::kStageWarpBytes);
    int tl = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tl) {
      int e, row0, n0;
      decode(L, e, row0, n0);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * MN);
      const int prow = row0 + q * 32 + lane;   // this thread's padded row
      if (MODE != kMxOut) {
        // h columns of the tile: ReLU 128 from n0; SwiGLU 64 from n0 / 2 (gate then up in TMEM)
        const int hcols = (MODE == kMxSwiglu) ? MN / 2 : MN;
        const int h0 = (MODE == kMxSwiglu) ? n0 / 2 : n0;
#pragma unroll 1
        for (int blk = 0; blk < hcols / 32; ++blk) {
          uint32_t a[32], u[32];
          tmem_ld32(tb + blk * 32, a);
          if (MODE == kMxSwiglu) tmem_ld32(tb + MN / 2 + blk * 32, u);
          tmem_wait_ld();
          float h[32];
          float amax = 0.f;
#pragma unroll
          for (int i = 0; i < 32; ++i) {
            const float g = __uint_as_float(a[i]);
            h[i] = (MODE == kMxSwiglu) ? g / (1.f + __expf(-g)) * __uint_as_float(u[i]) : fmaxf(g, 0.f);
            amax = fmaxf(amax, fabsf(h[i]));
          }
          const int X = mx_exponent(amax);
          uint4 lo, hi;
          quantize32(h, X, lo, hi);
          const int c = h0 + blk * 32;
          if (c < p.Nout && prow < p.rows_pad) {
            uint4* dst = reinterpret_cast<uint4*>(p.hq + (size_t)prow * p.Nout + c);
            dst[0] = lo;
            dst[1] = hi;
            p.hs[sf_offset(prow, c, p.Nout)] = (uint8_t)(X + 127);
          }
        }
      } else {
        // fp32 rows to the kept row each padded row came from (padding rows are dropped)
        const int i = prow - tail->seg[e];
        const int kept = p.offsets[e + 1] - p.offsets[e];
        const int row = (i < kept) ? p.offsets[e] + i : -1;
#pragma unroll 1
        for (int blk = 0; blk < MN / 32; ++blk) {
          uint32_t a[32];
          tmem_ld32(tb + blk * 32, a);
          tmem_wait_ld();
          __syncwarp();
#pragma unroll
          for (int v = 0; v < 8; ++v)
            stg[lane * 8 + (v ^ (lane & 7))] = make_uint4(a[4 * v], a[4 * v + 1], a[4 * v + 2], a[4 * v + 3]);
          __syncwarp();
          const int col0 = n0 + blk * 32;
#pragma unroll
          for (int t = 0; t < 8; ++t) {
            const int rr = t * 4 + (lane >> 3), cc = lane & 7;
            const int trow = __shfl_sync(0xffffffffu, row, rr);
            const int col = col0 + cc * 4;
            if (trow >= 0 && col < p.Nout)
              *reinterpret_cast<uint4*>(p.out + (size_t)trow * p.Nout + col) = stg[rr * 8 + (cc ^ (rr & 7))];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
    }
    if (!ok && lane == 0) {
      atomicOr(p.status, MOE_DEV_TIMEOUT);
      tail->abort_flag = 1;
    }
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

template <int MODE>
cudaError_t launch_mx(const CUtensorMap& ma, const CUtensorMap& mb, const MxParams& p, int grid, cudaStream_t s) {
  cudaError_t err = set_smem_once<tc_mx_gemm<MODE>>(kMxSmem);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_mx_gemm<MODE>, dim3(grid), dim3(kThreads), kMxSmem, s, ma, mb, p);
}

template <typename Map>
cudaError_t launch_quantize(const __nv_bfloat16* src, int rows, int K, Map map, uint8_t* q, uint8_t* sf,
                            cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const size_t nblk = (size_t)rows * (K / 32);
  const int grid = (int)std::max<size_t>(1, std::min<size_t>((nblk + 255) / 256, (size_t)di.sms * 8));
  return launch_pdl(mx_quantize_kernel<Map>, dim3(grid), dim3(256), 0, s, src, rows, K, map, q, sf);
}

}  // namespace

int mx_pad_rows() { return kMxPad; }

size_t mx_scale_bytes(size_t rows, size_t K) { return (rows / 128) * (K / 128) * 512; }

cudaError_t launch_mx_prepare_weights(const moe_config& c, const void* w1, const void* w2, void* w1q, void* w1s,
                                      void* w2q, void* w2s, cudaStream_t s) {
  const int F1 = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  const auto* W1 = static_cast<const __nv_bfloat16*>(w1);
  const auto* W2 = static_cast<const __nv_bfloat16*>(w2);
  cudaError_t e = (c.act == MOE_ACT_SWIGLU)
                      ? launch_quantize(W1, c.E * F1, c.d, RowMapSwiglu{c.F}, static_cast<uint8_t*>(w1q),
                                        static_cast<uint8_t*>(w1s), s)
                      : launch_quantize(W1, c.E * F1, c.d, RowMapIdentity{}, static_cast<uint8_t*>(w1q),
                                        static_cast<uint8_t*>(w1s), s);
  if (e != cudaSuccess) return e;
  return launch_quantize(W2, c.E * c.d, c.F, RowMapIdentity{}, static_cast<uint8_t*>(w2q),
                         static_cast<uint8_t*>(w2s), s);
}

cudaError_t launch_mx_experts(const moe_config& c, const MxBuffers& b, const void* w1q, const void* w1s,
                              const void* w2q, const void* w2s, float* yp, uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int F1 = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  // padded rows and the layer-1 input rows in E4M3
  if ((err = launch_pdl(mx_pad_kernel, dim3(1), dim3(32), 0, s, b.offsets, c.E, b.pad)) != cudaSuccess) return err;
  if ((err = launch_quantize(static_cast<const __nv_bfloat16*>(b.xp), b.rows_pad, c.d,
                             RowMapPadded{b.offsets, b.pad, c.E}, static_cast<uint8_t*>(b.xq),
                             static_cast<uint8_t*>(b.xs), s)) != cudaSuccess)
    return err;
  const long long mt_max = b.rows_pad / MB;
  CUtensorMap ma, mb;
  MxParams p{};
  p.pad = b.pad;
  p.offsets = b.offsets;
  p.E = c.E;
  p.rows_pad = b.rows_pad;
  p.status = status;
  // layer 1: h = act(xq W1q^T), quantised in the epilogue
  if (!make_map_u8(&ma, b.xq, (uint64_t)b.rows_pad, (uint64_t)c.d) ||
      !make_map_u8(&mb, w1q, (uint64_t)c.E * F1, (uint64_t)c.d))
    return cudaErrorInvalidValue;
  p.K = c.d;
  p.Nout = c.F;
  p.b_rows = F1;
  p.sfa = static_cast<const uint8_t*>(b.xs);
  p.sfb = static_cast<const uint8_t*>(w1s);
  p.hq = static_cast<uint8_t*>(b.hq);
  p.hs = static_cast<uint8_t*>(b.hs);
  int grid = (int)std::min<long long>(mt_max * ((F1 + MN - 1) / MN), di.sms);
  err = (c.act == MOE_ACT_SWIGLU) ? launch_mx<kMxSwiglu>(ma, mb, p, std::max(grid, 1), s)
                                  : launch_mx<kMxRelu>(ma, mb, p, std::max(grid, 1), s);
  if (err != cudaSuccess) return err;
  // layer 2: yp = hq W2q^T (fp32), written at the kept rows
  if (!make_map_u8(&ma, b.hq, (uint64_t)b.rows_pad, (uint64_t)c.F) ||
      !make_map_u8(&mb, w2q, (uint64_t)c.E * c.d, (uint64_t)c.F))
    return cudaErrorInvalidValue;
  p.K = c.F;
  p.Nout = c.d;
  p.b_rows = c.d;
  p.sfa = static_cast<const uint8_t*>(b.hs);
  p.sfb = static_cast<const uint8_t*>(w2s);
  p.out = yp;
  grid = (int)std::min<long long>(mt_max * ((c.d + MN - 1) / MN), di.sms);
  return launch_mx<kMxOut>(ma, mb, p, std::max(grid, 1), s);
}

}  // namespace moe
