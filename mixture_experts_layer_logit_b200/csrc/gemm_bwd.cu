// The backward of step 4 on the tensor cores: the gradients of the expert
// layers as grouped GEMMs over the same expert segments as the forward.
//
// The layer's figures on the pages are training figures (FastMoE
// announcement, "特色三": the single-GPU multi-expert speed-up is a training
// speed-up), and Megatron-Core's GroupedGEMM (best-practice page,
// "Megatron-Core MoE的关键特性") merges the experts' small GEMMs in the
// backward as in the forward.  With dy = w * dout on a kept row (the combine
// reversed), u the first layer's pre-activation and h = act(u):
//
//   dh  = dy W2[e]             grouped over rows, K = d       (kDgradAct)
//   du  = dh * act'(u)         in that GEMM's epilogue, with dw = <dout, y>
//   dxp = du W1[e]             grouped over rows, K = F1      (kDgradPlain)
//   dW2[e] = dy_e^T h_e        grouped over K = the expert's rows (kWgrad)
//   dW1[e] = du_e^T xp_e       grouped over K = the expert's rows (kWgrad)
//
// The rows are those of the forward's permutation with every expert's
// segment padded with zero rows to a multiple of 64, so that a k-block of the
// weight gradients never crosses into the next expert.  No operand is
// transposed in memory: W2[e] ([d, F]) and W1[e] ([F1, d]) are read as
// MN-major B operands of the first two, and the row-major activations as
// MN-major A and B operands of the weight gradients (tcgen05 takes either
// major-ness through the smem descriptor and the instruction descriptor).
//
// Roles as in the forward's 1-SM grouped GEMM: warp 0 lane 0 issues the TMA
// loads, warp 1 lane 0 the MMAs (128 x 256 x 16, fp32 in TMEM, two
// accumulators), warps 2-5 the epilogue.  Every wait is bounded; a role that
// gives up sets MOE_DEV_TIMEOUT and stops the others.
#include "gemm_common.cuh"

#include <algorithm>

namespace moe {
namespace {

using namespace tc;
using namespace gemm;

constexpr int BM = 128;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 48 KB
constexpr int kMNBox = 64 * BK * 2;               // one MN-major box: 64 MN elements x 64 K rows, 8 KB
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

enum { kDgradAct = 0, kDgradPlain = 1, kWgrad = 2 };
constexpr int kDwCols = 128;   // columns of F per partial of dw (half a 256-column tile)

struct Tail {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];
};
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + kStagingBytes + sizeof(Tail);
static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");

struct BwdParams {
  const int32_t* offsets;   // [E+1] padded segment offsets (multiples of 64)
  int E;
  int K;                    // kDgrad*: reduction length (d or F1)
  int Nout;                 // kDgrad*: output columns (F or d)
  int b_krows;              // kDgrad*: B rows per expert (= K; B is MN-major [E*K, Nout])
  int M, N;                 // kWgrad: output rows and columns of each expert's gradient
  int rows_alloc;           // padded rows of the row buffers
  float* out;               // fp32: [rows][Nout] (kDgradPlain) or [E][M][N] (kWgrad)
  uint32_t* status;
  // kDgradAct epilogue
  const float* u;           // [rows][F1] pre-activation
  const float* wrow;        // [rows] gate weight of each padded row (0 on padding)
  void* du;                 // [rows][F1]  (operand type)
  void* hw;                 // [rows][F]   w * h (operand type)
  float* dwpart;            // [nt][rows] per column tile: sum over its columns of dh/w * h
  int F, F1;
  const float* scale;       // [2]: s, 1/s -- the operands hold s * dout; results linear in dout are scaled by 1/s
};

// Two fp32 values -> one 32-bit pair of the operand type (round to nearest
// even); fp16 saturates at +-65504 and notes it in `over`.
template <bool F16>
__device__ __forceinline__ uint32_t pack_op(float a, float b, bool& over) {
  return pack_hidden<F16>(a, b, over);
}

// An epilogue warp's 32 rows x BN fp32 columns from TMEM, times `scale`, into
// out[rows][Nout] (columns from n0; rows [wrow0, wrow0 + nrows)), turned
// around in shared memory so that the stores write whole 128-byte lines.
__device__ __forceinline__ void store_scaled(float* out, int Nout, uint32_t tb, int wrow0, int nrows, int n0,
                                             float scale, uint4* stg, int lane) {
#pragma unroll 1
  for (int blk = 0; blk < BN / 32; ++blk) {
    uint32_t a[32];
    tmem_ld32(tb + blk * 32, a);
    tmem_wait_ld();
    uint4 v[8];
#pragma unroll
    for (int i = 0; i < 8; ++i)
      v[i] = make_uint4(__float_as_uint(scale * __uint_as_float(a[4 * i])),
                        __float_as_uint(scale * __uint_as_float(a[4 * i + 1])),
                        __float_as_uint(scale * __uint_as_float(a[4 * i + 2])),
                        __float_as_uint(scale * __uint_as_float(a[4 * i + 3])));
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) stg[lane * 8 + (i ^ (lane & 7))] = v[i];
    __syncwarp();
    const int col0 = n0 + blk * 32;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int rr = it * 4 + (lane >> 3), cc = lane & 7;
      const int col = col0 + cc * 4;
      if (rr < nrows && col < Nout)
        *reinterpret_cast<uint4*>(out + (size_t)(wrow0 + rr) * Nout + col) = stg[rr * 8 + (cc ^ (rr & 7))];
    }
  }
}

struct BwdTile {
  int e, row0, rows, m0, n0, k0, nkb;
};

// Tile L.  kDgrad*: rows of expert e's segment (as the forward's tiles, from
// the tile table); kWgrad: output block (m0, n0) of expert e, its K range the
// expert's padded rows.
template <int MODE>
__device__ __forceinline__ BwdTile bwd_tile(const Tail* tail, const BwdParams& p, int L) {
  BwdTile t;
  if (MODE == kWgrad) {
    const int mt = (p.M + BM - 1) / BM, nt = (p.N + BN - 1) / BN;
    t.e = L / (mt * nt);
    const int r = L - t.e * mt * nt;
    const int ni = r / mt, mi = r - ni * mt;
    t.m0 = mi * BM;
    t.n0 = ni * BN;
    t.row0 = t.m0;
    t.rows = min(BM, p.M - t.m0);
    t.k0 = tail->seg[t.e];
    t.nkb = (tail->seg[t.e + 1] - t.k0) / BK;
  } else {
    const TileCoord c = decode_tile<kPlain, BM>(tail->tstart, tail->seg, p.E, L);
    t.e = c.e;
    t.row0 = c.row0;
    t.rows = c.rows;
    t.m0 = 0;
    t.n0 = c.n0;
    t.k0 = 0;
    t.nkb = (p.K + BK - 1) / BK;
  }
  return t;
}

// The activation backward of one epilogue warp on its 32 rows and the
// 32-column blocks [blk0, blk1) of a 256-column tile of G = dout_perm W2[e]
// (fp32 in TMEM): with u the pre-activation (staged through shared memory 32
// columns at a time), h = act(u), w the row's gate weight: dh = w G,
// du = dh act'(u), hw = w h (the B operand of dW2), and the row's sums of
// G h over each 128-column half of the tile (its parts of dw = <dout, y>,
// one partial per 128 columns of F).  [blk0, blk1) is a whole number of halves.
template <int ACT, bool F16>
__device__ __forceinline__ void act_backward_tile(const BwdParams& p, uint32_t tb, int wrow0, int nrows, int n0,
                                                  int blk0, int blk1, uint4* stg, int lane, float inv_s,
                                                  bool& over) {
  const int row = wrow0 + lane;
  const bool live = lane < nrows;
  const float w = live ? p.wrow[row] : 0.f;
  const int nhalf = (p.F + kDwCols - 1) / kDwCols;
  float dwp = 0.f;
#pragma unroll 1
  for (int blk = blk0; blk < blk1; ++blk) {
    const int f0 = n0 + blk * 32;
    if (f0 < p.F) {
    uint32_t g[32];
    tmem_ld32(tb + blk * 32, g);
    tmem_wait_ld();
    // the u blocks of the warp's rows (gate, and for SwiGLU then up) in
    // 16-byte vectors, coalesced, turned around in shared memory
    float ug[32], uv[32];
#pragma unroll
    for (int part = 0; part < (ACT == kSwiglu ? 2 : 1); ++part) {
      const int c0 = (part == 0 ? f0 : p.F + f0);
      __syncwarp();
#pragma unroll
      for (int it = 0; it < 8; ++it) {
        const int rr = it * 4 + (lane >> 3), cc = lane & 7;
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (rr < nrows && f0 + cc * 4 < p.F)
          v = *reinterpret_cast<const uint4*>(p.u + (size_t)(wrow0 + rr) * p.F1 + c0 + cc * 4);
        stg[rr * 8 + (cc ^ (rr & 7))] = v;
      }
      __syncwarp();
      float* dst = part == 0 ? ug : uv;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        const uint4 v = stg[lane * 8 + (i ^ (lane & 7))];
        dst[4 * i] = __uint_as_float(v.x);
        dst[4 * i + 1] = __uint_as_float(v.y);
        dst[4 * i + 2] = __uint_as_float(v.z);
        dst[4 * i + 3] = __uint_as_float(v.w);
      }
    }
    uint32_t du_g[16], du_v[16], hwp[16];
#pragma unroll
    for (int i = 0; i < 32; i += 2) {
      float dg[2], dv[2], hh[2];
#pragma unroll
      for (int j = 0; j < 2; ++j) {
        const float gv = (f0 + i + j < p.F) ? __uint_as_float(g[i + j]) : 0.f;
        const float a = ug[i + j];
        float h, du_first, du_second = 0.f;
        if (ACT == kSwiglu) {
          const float s = 1.f / (1.f + __expf(-a));
          const float silu = a * s;
          const float v = uv[i + j];
          h = silu * v;
          const float dh = w * gv;
          du_first = dh * v * s * (1.f + a * (1.f - s));
          du_second = dh * silu;
        } else {
          h = fmaxf(a, 0.f);
          du_first = a > 0.f ? w * gv : 0.f;
        }
        dwp += gv * h;
        dg[j] = du_first;
        dv[j] = du_second;
        hh[j] = w * h;
      }
      bool o = false;
      du_g[i / 2] = pack_op<F16>(dg[0], dg[1], o);
      du_v[i / 2] = pack_op<F16>(dv[0], dv[1], o);
      hwp[i / 2] = pack_op<F16>(hh[0], hh[1], o);
      over |= o && live && (f0 + i < p.F);
    }
    if (live) {
      // 32 bf16 = 64 bytes per row and block; F is a multiple of 16, so a
      // block ends at F on a 16-column boundary
      const int nv = min(4, (p.F - f0) / 8);
      uint4* dg_row = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.du) + (size_t)row * p.F1 + f0);
      uint4* hw_row = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.hw) + (size_t)row * p.F + f0);
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        if (q < nv) {
          dg_row[q] = make_uint4(du_g[4 * q], du_g[4 * q + 1], du_g[4 * q + 2], du_g[4 * q + 3]);
          hw_row[q] = make_uint4(hwp[4 * q], hwp[4 * q + 1], hwp[4 * q + 2], hwp[4 * q + 3]);
        }
      }
      if (ACT == kSwiglu) {
        uint4* dv_row = reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.du) + (size_t)row * p.F1 + p.F + f0);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          if (q < nv) dv_row[q] = make_uint4(du_v[4 * q], du_v[4 * q + 1], du_v[4 * q + 2], du_v[4 * q + 3]);
      }
    }
    }
    if ((blk & 3) == 3) {   // end of a 128-column half: its partial of dw
      const int hi = n0 / kDwCols + blk / 4;
      if (live && hi < nhalf) p.dwpart[(size_t)hi * p.rows_alloc + row] = dwp * inv_s;
      dwp = 0.f;
    }
  }
}

// A_MN / B_MN: the operand is MN-major in memory (rows along K).  F16: both
// operands fp16 (else bf16).
template <int MODE, int ACT, bool A_MN, bool B_MN, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
tc_bwd_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB, const BwdParams p) {
  constexpr uint32_t kIdesc = idesc_f16kind(BM, BN, F16) | (A_MN ? kIdescAMN : 0u) | (B_MN ? kIdescBMN : 0u);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* staging = smem_raw + (base - raw) + (size_t)STAGES * STAGE_BYTES;
  Tail* tail = reinterpret_cast<Tail*>(staging + kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int ncols = (MODE == kWgrad) ? p.N : p.Nout;
  const int nt = (ncols + BN - 1) / BN;

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
  bool table_ok = true;
  if (warp == 0) {
    if (MODE == kWgrad) {
      // every expert's segment must be a whole number of k-blocks inside the buffer
      bool ok = true;
      for (int e = lane; e < p.E; e += 32) {
        const int a = p.offsets[e], b = p.offsets[e + 1];
        ok &= a >= 0 && b >= a && b <= p.rows_alloc && (a % BK) == 0 && (b % BK) == 0;
      }
      table_ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) tail->tstart[p.E] = table_ok ? p.E * ((p.M + BM - 1) / BM) * nt : 0;
    } else {
      table_ok = tile_table_warp(p.offsets, p.E, BM, nt, p.rows_alloc, tail->tstart, lane);
    }
    if (!table_ok && lane == 0 && blockIdx.x == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  for (int e = threadIdx.x; e <= p.E; e += kThreads) tail->seg[e] = p.offsets[e];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  const int total = tail->tstart[p.E];

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int it = 0;
      bool ok = true;
      for (int L = blockIdx.x; L < total && ok; L += gridDim.x) {
        const BwdTile t = bwd_tile<MODE>(tail, p, L);
        for (int kb = 0; kb < t.nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          mbar_expect_tx(full0 + 8 * s, STAGE_BYTES);
          if (A_MN) {   // A rows along K: two 64-column boxes of the tile's 128 M columns
            const int krow = t.k0 + kb * BK;
            tma_load_2d(sa, &tmA, full0 + 8 * s, t.m0, krow);
            tma_load_2d(sa + kMNBox, &tmA, full0 + 8 * s, t.m0 + 64, krow);
          } else {
            tma_load_2d(sa, &tmA, full0 + 8 * s, kb * BK, t.row0);
          }
          // B is MN-major in every mode: four 64-column boxes of the 256 N columns
          const int brow = (MODE == kWgrad) ? t.k0 + kb * BK : t.e * p.b_krows + kb * BK;
#pragma unroll
          for (int i = 0; i < 4; ++i)
            tma_load_2d(sa + A_BYTES + i * kMNBox, &tmB, full0 + 8 * s, t.n0 + 64 * i, brow);
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
        const BwdTile t = bwd_tile<MODE>(tail, p, L);
        const int acc = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < t.nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint64_t ad = A_MN ? sdesc_mn(sa, kMNBox) : sdesc(sa);
          const uint64_t bd = sdesc_mn(sa + A_BYTES, kMNBox);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            // K-major: 16 elements = 32 bytes along the swizzled row; MN-major:
            // 16 rows = 2048 bytes (the descriptor counts 16-byte units)
            const uint64_t astep = A_MN ? (uint64_t)(128 * kk) : (uint64_t)(2 * kk);
            tc_mma(d_tmem, ad + astep, bd + (uint64_t)(128 * kk), kIdesc, (kb | kk) != 0);
          }
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
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * kStageWarpBytes);
    const float inv_s = p.scale[1];
    int tl = 0;
    bool ok = true;
    bool over = false;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tl) {
      const BwdTile t = bwd_tile<MODE>(tail, p, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if (MODE == kWgrad) {
        const int m0 = t.m0 + q * 32;
        const int nrows = max(0, min(32, p.M - m0));
        if (nrows > 0) {
          if (t.nkb > 0) {
            store_scaled(p.out + (size_t)t.e * p.M * p.N, p.N, tb, m0, nrows, t.n0, inv_s, stg, lane);
          } else if (lane < nrows) {   // an expert without rows: its gradient is zero
            float* dst = p.out + (size_t)t.e * p.M * p.N + (size_t)(m0 + lane) * p.N;
            for (int c = t.n0; c < min(t.n0 + BN, p.N); c += 4)
              *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      } else {
        const int wrow0 = t.row0 + q * 32;
        int nrows = min(32, t.rows - q * 32);
        if (nrows > 0 && wrow0 + nrows > p.rows_alloc) {
          if (lane == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
          nrows = p.rows_alloc - wrow0;
        }
        if (nrows > 0) {
          if (MODE == kDgradAct)
            act_backward_tile<ACT, F16>(p, tb, wrow0, nrows, t.n0, 0, BN / 32, stg, lane, inv_s, over);
          else
            store_scaled(p.out, p.Nout, tb, wrow0, nrows, t.n0, inv_s, stg, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);
    }
    if (F16 && __any_sync(0xffffffffu, over) && lane == 0) atomicOr(p.status, MOE_DEV_RANGE);
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

// ------------------------------------------------------------ 2-SM pair tiles
// The same GEMMs on tiles of 256 x 256 computed by a pair of CTAs on two SMs
// of one cluster (tcgen05.mma.cta_group::2), as the forward's pair kernel:
// CTA r of the pair loads its half of the A tile (kDgrad*: rows
// [128 r, 128 r + 128) of the tile's activation rows; kWgrad: output rows
// [m0 + 128 r, +128), MN-major) and its half of the B tile (N columns
// [n0 + 128 r, +128), MN-major), to the same shared-memory offsets; the even
// CTA issues the MMA (M = 256, N = 256, K = 16) and each CTA's TMEM receives
// its 128 rows x 256 columns.  Per SM and k-block this loads 32 KB for
// 128 x 256 x 64 multiply-adds where the 1-SM tile loads 48 KB: the 1-SM
// kernels are bound by how fast an SM takes in its loads, not by the tensor
// pipe.  Barriers, aborts and teardown as in the forward's pair kernel.
constexpr int PM = 256, HM = PM / 2, HN = BN / 2;
constexpr int PSTAGES = 6;
constexpr int PA_BYTES = HM * BK * 2;              // 16 KB
constexpr int PB_BYTES = HN * BK * 2;              // 16 KB
constexpr int PSTAGE_BYTES = PA_BYTES + PB_BYTES;

struct PTail {
  unsigned long long full[PSTAGES], empty[PSTAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];
};
// The dh GEMM's epilogue (the activation backward, reading u and writing du
// and w h) is the heaviest: it runs on eight warps, two per TMEM lane
// quadrant, each taking one 128-column half of the tile, with five stages so
// that their staging fits; the other modes keep four warps and six stages.
__host__ __device__ constexpr int pair_epi_warps(int mode) { return mode == kDgradAct ? 8 : 4; }
__host__ __device__ constexpr int pair_threads(int mode) { return 64 + 32 * pair_epi_warps(mode); }
__host__ __device__ constexpr int pair_stages(int mode) { return mode == kDgradAct ? 5 : PSTAGES; }
constexpr size_t pair_smem_bytes(int mode) {
  return 1024 + (size_t)pair_stages(mode) * PSTAGE_BYTES + (size_t)pair_epi_warps(mode) * kStageWarpBytes +
         sizeof(PTail);
}
static_assert(pair_smem_bytes(kDgradAct) <= 227 * 1024 && pair_smem_bytes(kWgrad) <= 227 * 1024,
              "shared memory of one CTA");

// Tile L of the pair kernels (256-row / 256-column tiles).
template <int MODE>
__device__ __forceinline__ BwdTile bwd_tile_pair(const PTail* tail, const BwdParams& p, int L) {
  BwdTile t;
  if (MODE == kWgrad) {
    const int mt = (p.M + PM - 1) / PM, nt = (p.N + BN - 1) / BN;
    t.e = L / (mt * nt);
    const int r = L - t.e * mt * nt;
    const int ni = r / mt, mi = r - ni * mt;
    t.m0 = mi * PM;
    t.n0 = ni * BN;
    t.row0 = t.m0;
    t.rows = min(PM, p.M - t.m0);
    t.k0 = tail->seg[t.e];
    t.nkb = (tail->seg[t.e + 1] - t.k0) / BK;
  } else {
    const TileCoord c = decode_tile<kPlain, PM>(tail->tstart, tail->seg, p.E, L);
    t.e = c.e;
    t.row0 = c.row0;
    t.rows = c.rows;
    t.m0 = 0;
    t.n0 = c.n0;
    t.k0 = 0;
    t.nkb = (p.K + BK - 1) / BK;
  }
  return t;
}

template <int MODE, int ACT, bool A_MN, bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(pair_threads(MODE), 1)
tc_bwd_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                 const BwdParams p) {
  constexpr uint32_t kIdesc = idesc_f16kind(PM, BN, F16) | (A_MN ? kIdescAMN : 0u) | kIdescBMN;
  constexpr int kEpi = pair_epi_warps(MODE), kPT = pair_threads(MODE), kST = pair_stages(MODE);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // the same offset in both CTAs
  unsigned char* staging = smem_raw + (base - raw) + (size_t)kST * PSTAGE_BYTES;
  PTail* tail = reinterpret_cast<PTail*>(staging + (size_t)kEpi * kStageWarpBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = (int)cluster_id(), npairs = (int)cluster_count();
  const int ncols = (MODE == kWgrad) ? p.N : p.Nout;
  const int nt = (ncols + BN - 1) / BN;

  const uint32_t full0 = smem_u32(&tail->full[0]), empty0 = smem_u32(&tail->empty[0]);
  const uint32_t tfull0 = smem_u32(&tail->tfull[0]), tempty0 = smem_u32(&tail->tempty[0]);
  const uint32_t drain = smem_u32(&tail->drain);
  const volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < kST; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, 2 * kEpi);
    }
    mbar_init(drain, 1);
    tail->abort_flag = 0;
    fence_mbar_init_cluster();
  }
  if (warp == 1) {   // the same warp in both CTAs allocates the pair's TMEM
    asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tail->tmem_base)), "r"(kTmemCols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB)) : "memory");
  }
  pdl_wait();
  pdl_launch_dependents();
  if (warp == 0) {
    bool table_ok = true;
    if (MODE == kWgrad) {
      // every expert's segment must be a whole number of k-blocks inside the buffer
      bool ok = true;
      for (int e = lane; e < p.E; e += 32) {
        const int a = p.offsets[e], b = p.offsets[e + 1];
        ok &= a >= 0 && b >= a && b <= p.rows_alloc && (a % BK) == 0 && (b % BK) == 0;
      }
      table_ok = __all_sync(0xffffffffu, ok);
      if (lane == 0) tail->tstart[p.E] = table_ok ? p.E * ((p.M + PM - 1) / PM) * nt : 0;
    } else {
      table_ok = tile_table_warp(p.offsets, p.E, PM, nt, p.rows_alloc, tail->tstart, lane);
    }
    if (!table_ok && lane == 0 && blockIdx.x == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  for (int e = threadIdx.x; e <= p.E; e += kPT) tail->seg[e] = p.offsets[e];
  tc_fence_before();
  cluster_sync();              // both CTAs: barriers initialised, TMEM allocated, tile tables built
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  const int total = tail->tstart[p.E];
  // the even CTA's barriers and the peer's abort flag, as cluster addresses
  const uint32_t full0_lead = cluster_addr(full0, 0), tempty0_lead = cluster_addr(tempty0, 0);
  const uint32_t abort_peer = cluster_addr(smem_u32(&tail->abort_flag), rank ^ 1u);
  auto give_up = [&]() {
    atomicOr(p.status, MOE_DEV_TIMEOUT);
    tail->abort_flag = 1;
    st_cluster_u32(abort_peer, 1u);
  };

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------ TMA producer
      int it = 0;
      bool ok = true;
      for (int L = pair; L < total && ok; L += npairs) {
        const BwdTile t = bwd_tile_pair<MODE>(tail, p, L);
        const int ncol = t.n0 + HN * (int)rank;
        for (int kb = 0; kb < t.nkb; ++kb) {
          const int s = it % kST;
          const uint32_t ph = (uint32_t)(it / kST) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * PSTAGE_BYTES);
          if (rank == 0) mbar_expect_tx(full0 + 8 * s, 2 * PSTAGE_BYTES);   // both halves
          if (A_MN) {   // this CTA's 128 M columns, rows along K: two 64-column boxes
            const int krow = t.k0 + kb * BK, mcol = t.m0 + HM * (int)rank;
            tma_load_2d_pair(sa, &tmA, full0_lead + 8 * s, mcol, krow);
            tma_load_2d_pair(sa + kMNBox, &tmA, full0_lead + 8 * s, mcol + 64, krow);
          } else {
            tma_load_2d_pair(sa, &tmA, full0_lead + 8 * s, kb * BK, t.row0 + HM * (int)rank);
          }
          // B, MN-major: this CTA's 128 of the 256 N columns
          const int brow = (MODE == kWgrad) ? t.k0 + kb * BK : t.e * p.b_krows + kb * BK;
          tma_load_2d_pair(sa + PA_BYTES, &tmB, full0_lead + 8 * s, ncol, brow);
          tma_load_2d_pair(sa + PA_BYTES + kMNBox, &tmB, full0_lead + 8 * s, ncol + 64, brow);
          ++it;
        }
      }
      if (!ok) give_up();
      if (rank == 0) {
        // the loads still in flight (of both CTAs) complete on these barriers
        for (int i = max(0, it - kST); i < it; ++i)
          mbar_wait(full0 + 8 * (i % kST), (uint32_t)(i / kST) & 1u, nullptr, kDrainNs);
      } else if (!ok) {
        // loads of this CTA whose phase the even CTA never armed: give them
        // time to land before the shared memory can be released
        const unsigned long long t0 = now_ns();
        while (now_ns() - t0 < 1000000ull) {
        }
      }
    }
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ------------------------------------------------------- MMA issuer
      int it = 0, tl = 0;
      bool ok = true;
      for (int L = pair; L < total && ok; L += npairs, ++tl) {
        const BwdTile t = bwd_tile_pair<MODE>(tail, p, L);
        const int acc = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < t.nkb; ++kb) {
          const int s = it % kST;
          const uint32_t ph = (uint32_t)(it / kST) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)(s * PSTAGE_BYTES);
          const uint64_t ad = A_MN ? sdesc_mn(sa, kMNBox) : sdesc(sa);
          const uint64_t bd = sdesc_mn(sa + PA_BYTES, kMNBox);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t astep = A_MN ? (uint64_t)(128 * kk) : (uint64_t)(2 * kk);
            tc_mma_pair(d_tmem, ad + astep, bd + (uint64_t)(128 * kk), kIdesc, (kb | kk) != 0);
          }
          tc_commit_pair(empty0 + 8 * s, 0x3);   // stage s free again in both CTAs
          ++it;
        }
        if (!ok) break;
        tc_commit_pair(tfull0 + 8 * acc, 0x3);   // accumulator ready in both CTAs
      }
      if (!ok) give_up();
      tc_commit_pair(drain, 0x1);                // every MMA issued above has completed
      mbar_wait(drain, 0, nullptr, kDrainNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3, half = (warp - 2) >> 2;   // half: 0, or 1 for the dh GEMM's second four warps
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * kStageWarpBytes);
    const float inv_s = p.scale[1];
    int tl = 0;
    bool ok = true;
    bool over = false;
    for (int L = pair; L < total; L += npairs, ++tl) {
      const BwdTile t = bwd_tile_pair<MODE>(tail, p, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      if (MODE == kWgrad) {
        const int m0 = t.m0 + HM * (int)rank + q * 32;
        const int nrows = max(0, min(32, p.M - m0));
        if (nrows > 0) {
          if (t.nkb > 0) {
            store_scaled(p.out + (size_t)t.e * p.M * p.N, p.N, tb, m0, nrows, t.n0, inv_s, stg, lane);
          } else if (lane < nrows) {   // an expert without rows: its gradient is zero
            float* dst = p.out + (size_t)t.e * p.M * p.N + (size_t)(m0 + lane) * p.N;
            for (int c = t.n0; c < min(t.n0 + BN, p.N); c += 4)
              *reinterpret_cast<float4*>(dst + c) = make_float4(0.f, 0.f, 0.f, 0.f);
          }
        }
      } else {
        const int wrow0 = t.row0 + HM * (int)rank + q * 32;
        int nrows = min(32, t.rows - HM * (int)rank - q * 32);
        if (nrows > 0 && wrow0 + nrows > p.rows_alloc) {
          if (lane == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
          nrows = p.rows_alloc - wrow0;
        }
        if (nrows > 0) {
          if (MODE == kDgradAct)
            act_backward_tile<ACT, F16>(p, tb, wrow0, nrows, t.n0, 4 * half, 4 * half + 4, stg, lane, inv_s,
                                        over);
          else
            store_scaled(p.out, p.Nout, tb, wrow0, nrows, t.n0, inv_s, stg, lane);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0_lead + 8 * acc);   // accumulator free again
    }
    if (F16 && __any_sync(0xffffffffu, over) && lane == 0) atomicOr(p.status, MOE_DEV_RANGE);
    if (!ok && lane == 0) give_up();
  }

  tc_fence_before();
  __syncthreads();
  cluster_sync();              // the pair's MMAs and loads are done with both CTAs' shared memory
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(kTmemCols) : "memory");
  }
}

template <int MODE, int ACT, bool A_MN, bool F16>
cudaError_t launch_bwd_pair(const CUtensorMap& ma, const CUtensorMap& mb, const BwdParams& p, int pairs,
                            cudaStream_t s) {
  constexpr size_t smem = pair_smem_bytes(MODE);
  cudaError_t err = set_smem_once<tc_bwd_gemm_pair<MODE, ACT, A_MN, F16>>(smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_bwd_gemm_pair<MODE, ACT, A_MN, F16>, dim3(2 * pairs), dim3(pair_threads(MODE)), smem, s, ma,
                    mb, p);
}

template <int MODE, int ACT, bool A_MN, bool B_MN, bool F16>
cudaError_t launch_bwd(const CUtensorMap& ma, const CUtensorMap& mb, const BwdParams& p, int grid, cudaStream_t s) {
  cudaError_t err = set_smem_once<tc_bwd_gemm<MODE, ACT, A_MN, B_MN, F16>>(kSmemBytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_bwd_gemm<MODE, ACT, A_MN, B_MN, F16>, dim3(grid), dim3(kThreads), kSmemBytes, s, ma, mb, p);
}

template <bool F16>
cudaError_t launch_backward_t(const moe_config& c, const BwdState& st, const void* w1, const void* w2, float* dw1,
                              float* dw2, int sms, bool pair, cudaStream_t s) {
  const int max_pairs = std::max(1, sms / 2);
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const uint64_t R = (uint64_t)st.rows_alloc;
  const long long mt_max = (long long)(R / BM) + c.E;
  CUtensorMap ma, mb;
  BwdParams p{};
  p.offsets = st.pad_offsets;
  p.E = c.E;
  p.rows_alloc = st.rows_alloc;
  p.status = st.status;
  p.scale = st.scale;
  cudaError_t err;

  // dh = dout_perm W2[e] (K = d), its activation backward in the epilogue
  if (!make_map(&ma, st.dout_perm, R, (uint64_t)c.d, F16) ||
      !make_map(&mb, w2, (uint64_t)c.E * c.d, (uint64_t)c.F, F16, 64))
    return cudaErrorInvalidValue;
  p.K = c.d;
  p.Nout = c.F;
  p.b_krows = c.d;
  p.u = st.u;
  p.wrow = st.wrow;
  p.du = st.du;
  p.hw = st.hw;
  p.dwpart = st.dwpart;
  p.F = c.F;
  p.F1 = F1;
  const long long pt_max = (long long)(R / PM) + c.E;   // pair m-tiles at most
  if (pair) {
    const int pairs = (int)std::min<long long>(pt_max * ((c.F + BN - 1) / BN), max_pairs);
    err = (c.act == MOE_ACT_SWIGLU) ? launch_bwd_pair<kDgradAct, kSwiglu, false, F16>(ma, mb, p, pairs, s)
                                    : launch_bwd_pair<kDgradAct, kRelu, false, F16>(ma, mb, p, pairs, s);
  } else {
    const int grid = (int)std::min<long long>(mt_max * ((c.F + BN - 1) / BN), sms);
    err = (c.act == MOE_ACT_SWIGLU) ? launch_bwd<kDgradAct, kSwiglu, false, true, F16>(ma, mb, p, grid, s)
                                    : launch_bwd<kDgradAct, kRelu, false, true, F16>(ma, mb, p, grid, s);
  }
  if (err != cudaSuccess) return err;

  // dxp = du W1[e] (K = F1)
  if (!make_map(&ma, st.du, R, (uint64_t)F1, F16) ||
      !make_map(&mb, w1, (uint64_t)c.E * F1, (uint64_t)c.d, F16, 64))
    return cudaErrorInvalidValue;
  p.K = F1;
  p.Nout = c.d;
  p.b_krows = F1;
  p.out = st.dxp;
  err = pair ? launch_bwd_pair<kDgradPlain, kRelu, false, F16>(
                   ma, mb, p, (int)std::min<long long>(pt_max * ((c.d + BN - 1) / BN), max_pairs), s)
             : launch_bwd<kDgradPlain, kRelu, false, true, F16>(
                   ma, mb, p, (int)std::min<long long>(mt_max * ((c.d + BN - 1) / BN), sms), s);
  if (err != cudaSuccess) return err;

  // dW2[e] = dout_perm_e^T (w h)_e: M = d, N = F, K = the expert's padded rows
  if (!make_map(&ma, st.dout_perm, R, (uint64_t)c.d, F16, 64) || !make_map(&mb, st.hw, R, (uint64_t)c.F, F16, 64))
    return cudaErrorInvalidValue;
  p.M = c.d;
  p.N = c.F;
  p.out = dw2;
  if (pair)
    err = launch_bwd_pair<kWgrad, kRelu, true, F16>(
        ma, mb, p,
        (int)std::min<long long>((long long)c.E * ((c.d + PM - 1) / PM) * ((c.F + BN - 1) / BN), max_pairs), s);
  else
    err = launch_bwd<kWgrad, kRelu, true, true, F16>(
        ma, mb, p, (int)std::min<long long>((long long)c.E * ((c.d + BM - 1) / BM) * ((c.F + BN - 1) / BN), sms),
        s);
  if (err != cudaSuccess) return err;

  // dW1[e] = du_e^T xp_e: M = F1, N = d
  if (!make_map(&ma, st.du, R, (uint64_t)F1, F16, 64) || !make_map(&mb, st.xp, R, (uint64_t)c.d, F16, 64))
    return cudaErrorInvalidValue;
  p.M = F1;
  p.N = c.d;
  p.out = dw1;
  if (pair)
    return launch_bwd_pair<kWgrad, kRelu, true, F16>(
        ma, mb, p, (int)std::min<long long>((long long)c.E * ((F1 + PM - 1) / PM) * ((c.d + BN - 1) / BN), max_pairs),
        s);
  return launch_bwd<kWgrad, kRelu, true, true, F16>(
      ma, mb, p, (int)std::min<long long>((long long)c.E * ((F1 + BM - 1) / BM) * ((c.d + BN - 1) / BN), sms), s);
}

}  // namespace

cudaError_t launch_expert_backward_tc(const moe_config& c, const BwdState& st, const void* w1, const void* w2,
                                      float* dw1, float* dw2, bool pair, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  return st.f16 ? launch_backward_t<true>(c, st, w1, w2, dw1, dw2, di.sms, pair, s)
                : launch_backward_t<false>(c, st, w1, w2, dw1, dw2, di.sms, pair, s);
}

int bwd_tc_col_tile() { return kDwCols; }

}  // namespace moe
