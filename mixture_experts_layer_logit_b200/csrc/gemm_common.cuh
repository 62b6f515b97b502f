// Pieces shared by the grouped expert GEMMs on the tensor cores (the 1-SM
// kernel in gemm_tc.cu and the 2-SM pair kernel in gemm_tc2.cu): parameters,
// tile decoding and the TMEM -> global epilogue with the fused activation.
//
// Experts: two-layer ReLU MLP (FastMoE announcement, Transformer-XL
// experiment) or SwiGLU whose W1 holds the gate rows before the up rows
// (Megatron-Core best-practice page, "从HuggingFace到Megatron的权重转换要点").
#pragma once

#include "tc_ptx.cuh"

namespace moe {
namespace gemm {

using namespace tc;

constexpr int BN = 256, BK = 64;
// kPlain: layer 2 into fp32 yp; kCombine: layer 2 added, gate-weighted, into
// the token rows of the layer output (the combine of step 5 fused in).
enum { kPlain = 0, kRelu = 1, kSwiglu = 2, kCombine = 3 };

// Epilogue staging: each epilogue warp turns its 32 rows x 128 bytes of output
// around in shared memory so that the global stores write whole 128-byte lines.
constexpr int kStageWarpBytes = 32 * 128;
constexpr size_t kStagingBytes = 4 * kStageWarpBytes;

struct Params {
  const int32_t* offsets;
  void* out;            // [rows][Nout]: 16-bit h (layer 1) or fp32 yp (layer 2)
  int E, K, Nout;
  int b_rows;           // B rows per expert
  int up_off;           // SwiGLU: first up row inside an expert's B block
  int rows_alloc;       // rows of the A and output buffers (T*k); stores stop there
  uint32_t* status;
  const int32_t* src_tok;   // kCombine: token of each permuted row
  const float* row_w;       // kCombine: gate weight of each permuted row
  int out_rows;             // kCombine: token rows of the output
  int e_mod;                // weight blocks: segment e uses block e % e_mod (0: e itself)
};

// Weight block of segment e: segments may outnumber the experts whose
// weights are given (the segments of several source ranks, each holding the
// same local experts in turn).
__device__ __forceinline__ int weight_block(const Params& p, int e) { return p.e_mod > 0 ? e % p.e_mod : e; }

// Two fp32 values -> one 32-bit pair of the hidden type (round to nearest
// even).  fp16 saturates at +-65504 (NaN passes through) and notes it in `over`.
template <bool F16>
__device__ __forceinline__ uint32_t pack_hidden(float a, float b, bool& over) {
  if constexpr (F16) {
    const bool oa = fabsf(a) > 65504.f, ob = fabsf(b) > 65504.f;
    over |= oa | ob;
    a = oa ? copysignf(65504.f, a) : a;
    b = ob ? copysignf(65504.f, b) : b;
    __half2 h = __floats2half2_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  } else {
    __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
    return *reinterpret_cast<uint32_t*>(&h);
  }
}

struct TileCoord {
  int e, row0, rows, n0;
};

// m-tiles per group of the second layer's tile order (see decode_tile).
constexpr int kL2Group = 8;

// Tile L of the table: expert, first permuted row, rows inside the expert's
// segment (up to TM) and first output column.  Within an expert the m-tiles
// of one n-tile are consecutive, so the CTAs running at the same time share
// a weight tile in L2.  For the second layer (K = F, long rows of h) the
// expert's m-tiles go in groups of kL2Group: all n-tiles of a group before
// the next group.  A wave of tiles then reads about as many h rows as weight
// rows (a 2-D block of the output) instead of every h row of the expert for
// a few weight tiles, and stays inside L2.
template <int MODE, int TM>
__device__ __forceinline__ TileCoord decode_tile(const int* tstart, const int32_t* offsets, int E, int L) {
  TileCoord c;
  c.e = tile_expert(tstart, E, L);
  const int seg0 = offsets[c.e];
  const int M = offsets[c.e + 1] - seg0;
  const int mt = (M + TM - 1) / TM;
  const int local = L - tstart[c.e];
  int nti, mti;
  if ((MODE == kPlain || MODE == kCombine) && mt > kL2Group) {
    const int nt = (tstart[c.e + 1] - tstart[c.e]) / mt;
    const int grp = local / (kL2Group * nt);
    const int gsize = min(kL2Group, mt - grp * kL2Group);
    const int rem = local - grp * kL2Group * nt;
    nti = rem / gsize;
    mti = grp * kL2Group + (rem - nti * gsize);
  } else {
    nti = local / mt;
    mti = local - nti * mt;
  }
  c.row0 = seg0 + mti * TM;
  c.rows = min(TM, M - mti * TM);
  c.n0 = nti * (MODE == kSwiglu ? BN / 2 : BN);
  return c;
}

// One epilogue warp: drains TMEM lanes 32q..32q+31 (base address `tb`, BN
// fp32 columns) and stores rows [wrow0, wrow0 + nrows) of the output from
// column n0.  One block = 128 bytes of output per row: 32 fp32 columns (layer
// 2) or 64 16-bit hidden columns (layer 1).  Thread `lane` owns TMEM row
// wrow0 + lane; the block is turned around in shared memory (16-byte chunk i
// of row r at slot i ^ (r & 7), conflict-free both ways) and written as
// 4 rows x 128 contiguous bytes per store instruction.  ReLU / silu(gate)*up
// and the rounding of h run here, in fp32.
//
// kCombine: out[src_tok[row]] += row_w[row] * y with 16-byte fp32 reductions
// (out zeroed beforehand).  A token receives at most two such additions (k <=
// 2), onto an exact zero, so the result does not depend on their order.
template <int MODE, bool F16>
__device__ __forceinline__ void store_tile(const Params& p, uint32_t tb, int wrow0, int nrows, int n0,
                                           uint4* stg, int lane, bool& over) {
  constexpr bool kF32Out = (MODE == kPlain || MODE == kCombine);
  constexpr int kBlocks = kF32Out ? BN / 32 : (MODE == kRelu ? BN / 64 : BN / 128);
  constexpr int kPer16 = kF32Out ? 4 : 8;
  // rows past the segment (the next expert's rows, or unwritten rows past
  // the kept ones) are computed but never stored: only stored rows may
  // report an fp16 overflow
  bool row_over = false;
  int tok = 0;
  float wgt = 0.f;
  if (MODE == kCombine && lane < nrows) {
    tok = p.src_tok[wrow0 + lane];
    wgt = p.row_w[wrow0 + lane];
    if ((unsigned)tok >= (unsigned)p.out_rows) atomicOr(p.status, MOE_DEV_BOUNDS);   // skipped below
  }
#pragma unroll 1
  for (int blk = 0; blk < kBlocks; ++blk) {
    uint4 v[8];
    if (kF32Out) {
      uint32_t a[32];
      tmem_ld32(tb + blk * 32, a);
      tmem_wait_ld();
#pragma unroll
      for (int i = 0; i < 8; ++i) v[i] = make_uint4(a[4 * i], a[4 * i + 1], a[4 * i + 2], a[4 * i + 3]);
    } else {
#pragma unroll
      for (int hf = 0; hf < 2; ++hf) {
        uint32_t a[32], u[32];
        if (MODE == kRelu) {
          tmem_ld32(tb + blk * 64 + hf * 32, a);
        } else {   // SwiGLU: gate columns, then the up columns BN/2 further
          tmem_ld32(tb + blk * 64 + hf * 32, a);
          tmem_ld32(tb + BN / 2 + blk * 64 + hf * 32, u);
        }
        tmem_wait_ld();
#pragma unroll
        for (int i = 0; i < 4; ++i) {
          uint32_t pk[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            float a0 = __uint_as_float(a[8 * i + 2 * j]), a1 = __uint_as_float(a[8 * i + 2 * j + 1]);
            if (MODE == kRelu) {
              a0 = fmaxf(a0, 0.f);
              a1 = fmaxf(a1, 0.f);
            } else {
              const float u0 = __uint_as_float(u[8 * i + 2 * j]), u1 = __uint_as_float(u[8 * i + 2 * j + 1]);
              // silu(a) = a / (1 + e^-a) with the fast division (a few ulp; the
              // denominator overflows to +inf only where silu is -0 anyway)
              a0 = __fdividef(a0, 1.f + __expf(-a0)) * u0;
              a1 = __fdividef(a1, 1.f + __expf(-a1)) * u1;
            }
            pk[j] = pack_hidden<F16>(a0, a1, row_over);
          }
          v[hf * 4 + i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
        }
      }
    }
    __syncwarp();
#pragma unroll
    for (int i = 0; i < 8; ++i) stg[lane * 8 + (i ^ (lane & 7))] = v[i];
    __syncwarp();
    const int col0 = n0 + blk * 8 * kPer16;
#pragma unroll
    for (int it = 0; it < 8; ++it) {
      const int rr = it * 4 + (lane >> 3), cc = lane & 7;
      const uint4 val = stg[rr * 8 + (cc ^ (rr & 7))];
      const int col = col0 + cc * kPer16;
      if (MODE == kCombine) {
        const int t = __shfl_sync(0xffffffffu, tok, rr);
        const float w = __shfl_sync(0xffffffffu, wgt, rr);
        if (rr < nrows && col < p.Nout && (unsigned)t < (unsigned)p.out_rows) {
          float* dst = static_cast<float*>(p.out) + (size_t)t * p.Nout + col;
          asm volatile("red.global.add.v4.f32 [%0], {%1, %2, %3, %4};"
                       ::"l"(dst), "f"(w * __uint_as_float(val.x)), "f"(w * __uint_as_float(val.y)),
                         "f"(w * __uint_as_float(val.z)), "f"(w * __uint_as_float(val.w))
                       : "memory");
        }
        continue;
      }
      if (rr < nrows && col < p.Nout) {
        const size_t off = (size_t)(wrow0 + rr) * p.Nout + col;
        if (MODE == kPlain) *reinterpret_cast<uint4*>(static_cast<float*>(p.out) + off) = val;
        else *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off) = val;
      }
    }
  }
  over |= row_over && lane < nrows;
}

// Layer-2 modes read fp16 operands when the hidden type is fp16.
constexpr bool layer2(int mode) { return mode == kPlain || mode == kCombine; }

// Rows of one epilogue warp that may be stored: inside the tile's segment
// part and inside the buffers (offsets[] beyond the buffers: skip and flag).
__device__ __forceinline__ int warp_rows(const Params& p, int wrow0, int rows_left, int lane) {
  int nrows = min(32, rows_left);
  if (nrows > 0 && wrow0 + nrows > p.rows_alloc) {
    if (lane == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
    nrows = p.rows_alloc - wrow0;
  }
  return nrows;
}

}  // namespace gemm
}  // namespace moe
