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
constexpr int B_BYTES = MN * MK;                      // 16 KB
constexpr int SF_BYTES = 512;                         // one scale atom per operand
constexpr int kMaxStages = 8;

// Stage layouts.  Wide: A and B tiles of 128 rows (16 KB each), 6 stages.
// Narrow, for batches of at most 64 tokens (a token takes an expert at most
// once, so no expert has more than 64 kept rows): A holds 64 rows (8 KB) and
// 8 stages keep 128 KB of weight tiles in flight per SM instead of 96 KB.  The
// MMA still reads 128 A rows, the last 64 from the stage's own B tile: those
// rows of the accumulator are computed and never stored (their epilogue warps
// are not live).
template <bool NARROW>
struct MxStages {
  static constexpr int kARows = NARROW ? 64 : MB;
  static constexpr int kABytes = kARows * MK;
  static constexpr int kStages = NARROW ? 8 : 6;
  static constexpr int kStageBytes = kABytes + B_BYTES;
  static_assert(kStages <= kMaxStages && kStageBytes % 1024 == 0, "stages of 1 KB-aligned tiles");
};
constexpr int kEpiWarps = 8;                         // two per TMEM lane quadrant
constexpr int kThreads = 64 + 32 * kEpiWarps;
constexpr uint32_t kTmemCols = 512;
constexpr uint32_t kSfCol0 = 256;                     // scale columns after the two 128-column accumulators
constexpr int kMxPad = 128;
constexpr int kQueue = 4;                             // claimed tiles in flight between the roles

enum { kMxRelu = 0, kMxSwiglu = 1 };

// Least X with amax <= 448 * 2^X (-127 for 0); the UE8M0 byte is X + 127.
// From the bit fields: amax = 1.m 2^(E-127), and 448 = 1.75 2^8, so X = E - 135
// when 1.m <= 1.75 (mantissa bits <= 0x600000), else E - 134.  A subnormal
// amax (< 2^-126) gives an X below -127, clamped; no finite float gives more
// than 120.
__device__ __forceinline__ int mx_exponent(float amax) {
  if (!(amax > 0.f)) return -127;
  const uint32_t b = __float_as_uint(amax);
  const int E = (int)(b >> 23);
  if (E == 0) return -127;
  return min(127, E - 135 + ((b & 0x7fffffu) > 0x600000u ? 1 : 0));
}

// 2^-X as a float, for X in [-127, 120] (exponent field 127 - X in [7, 254]).
__device__ __forceinline__ float mx_inv_scale(int X) { return __uint_as_float((uint32_t)(127 - X) << 23); }

__device__ __forceinline__ size_t sf_offset(int r, int k, int K) {
  return ((size_t)(r / 128) * (K / 128) + k / 128) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + (k / 32) % 4;
}

// 32 fp32 values -> 32 E4M3 bytes (scaled by 2^-X), round to nearest even.
__device__ __forceinline__ void quantize32(const float (&v)[32], int X, uint4& lo, uint4& hi) {
  const float s = mx_inv_scale(X);
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

// One 32-element block of a bf16 row -> 32 E4M3 bytes at q and the block's
// scale byte at sf (row r of the destination, block kb of K / 32).
__device__ __forceinline__ void quantize_block(const __nv_bfloat16* __restrict__ src, int r, int kb, int K,
                                               uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  float v[32];
  const uint4* p = reinterpret_cast<const uint4*>(src + 32 * kb);
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

// The weights, once: one thread per 32-element block.  The map takes a
// destination row to its source row (identity, or the SwiGLU interleave).
struct RowMapIdentity {
  __device__ int operator()(int r) const { return r; }
};
struct RowMapSwiglu {   // destination row of an expert's interleaved W1 <- source row
  int F;
  __device__ int operator()(int r) const {
    const int F1 = 2 * F, e = r / F1, i = r - e * F1, b = i / 128, j = i % 128;
    return e * F1 + (j < 64 ? 64 * b + j : F + 64 * b + (j - 64));
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
    quantize_block(src + (size_t)map(r) * K, r, kb, K, q, sf);
  }
}

// The layer-1 input rows, per call: every CTA first derives the padded
// segment offsets (each expert's kept rows rounded up to a multiple of 128;
// one warp, 8 experts per lane and a shuffle scan); CTA 0 publishes them and
// zeroes the expert kernel's tile and dependency counters.  Then one thread
// per 32-element block of a kept row, written at its row of the expert's
// padded segment.  Padding rows stay unwritten: every row of an MMA tile is
// computed from its own A row only, and no output of a padding row is
// stored as a kept row.
__global__ void __launch_bounds__(256)
mx_quantize_rows_kernel(const __nv_bfloat16* __restrict__ xp, int rows_max, int rows_pad, int K,
                        const int32_t* __restrict__ offsets, int E, int32_t* __restrict__ pad_out,
                        int* __restrict__ ctr, int nctr, uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  __shared__ int s_off[kMaxExperts + 1], s_pad[kMaxExperts + 1];
  pdl_wait();
  pdl_launch_dependents();
  for (int e = threadIdx.x; e <= E; e += blockDim.x) s_off[e] = offsets[e];
  __syncthreads();
  if (threadIdx.x < 32) {
    constexpr int PER = kMaxExperts / 32;
    const int lane = threadIdx.x;
    int loc[PER], sum = 0;
#pragma unroll
    for (int i = 0; i < PER; ++i) {
      const int e = lane * PER + i;
      loc[i] = (e < E) ? (s_off[e + 1] - s_off[e] + kMxPad - 1) / kMxPad * kMxPad : 0;
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
      if (e < E) s_pad[e] = run;
      run += loc[i];
    }
    if (lane == 31) s_pad[E] = incl;
  }
  __syncthreads();
  if (blockIdx.x == 0) {
    for (int e = threadIdx.x; e <= E; e += blockDim.x) pad_out[e] = s_pad[e];
    for (int i = threadIdx.x; i < nctr; i += blockDim.x) ctr[i] = 0;
  }
  const int nb = K / 32;
  const int kept = min(s_off[E], rows_max);
  const size_t nblk = (size_t)kept * nb;
  for (size_t b = (size_t)blockIdx.x * blockDim.x + threadIdx.x; b < nblk; b += (size_t)gridDim.x * blockDim.x) {
    const int i = (int)(b / nb), kb = (int)(b - (size_t)i * nb);
    int lo = 0, hi = E - 1;   // the largest e with offsets[e] <= i holds row i
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_off[mid] <= i) lo = mid; else hi = mid - 1;
    }
    const int r = s_pad[lo] + (i - s_off[lo]);
    if ((unsigned)r < (unsigned)rows_pad) quantize_block(xp + (size_t)i * K, r, kb, K, q, sf);
  }
}

struct MxParams {
  const int32_t* pad;        // [E+1] padded segment offsets (multiples of 128)
  const int32_t* offsets;    // [E+1] kept offsets
  int E, d, F, F1;           // model width, hidden width, layer-1 weight rows per expert (F or 2F)
  int rows_pad;              // padded rows allocated
  const uint8_t* xs;         // layer-1 A scales (the quantised input rows)
  const uint8_t* w1s;        // layer-1 B scales
  const uint8_t* w2s;        // layer-2 B scales
  uint8_t* hq;               // [rows_pad][F] E4M3 h: layer-1 output, layer-2 A
  uint8_t* hs;               // its scales
  float* out;                // yp [rows][d] fp32 at the kept (unpadded) rows
  uint32_t* status;
  int* sched;                // tile counter, zeroed beforehand
  int* dep;                  // per padded m-tile: layer-1 epilogue warps done; zeroed beforehand
};

struct MxTail {
  unsigned long long full[kMaxStages], empty[kMaxStages], tfull[2], tempty[2], drain;
  unsigned long long qfull[kQueue], qempty[kQueue];
  uint32_t tmem_base;
  int abort_flag;
  int queue[kQueue];
  int tstart1[kMaxExperts + 1];   // layer-1 tile table
  int tstart2[kMaxExperts + 1];   // layer-2 tile table
  int seg[kMaxExperts + 1];
  int cnt[kMaxExperts + 1];       // kept rows of each expert (the rest of its padded segment is padding)
};
template <bool NARROW>
constexpr size_t mx_smem() {
  using Lay = MxStages<NARROW>;
  return 1024 + (size_t)Lay::kStages * Lay::kStageBytes + (size_t)Lay::kStages * 2 * SF_BYTES +
         gemm::kStagingBytes + sizeof(MxTail);
}
static_assert(mx_smem<false>() <= 227 * 1024 && mx_smem<true>() <= 227 * 1024, "shared memory of one CTA");

struct MxTile {
  bool l2;
  int e, row0, n0, m;   // expert, first padded row, first output column (layer 1: weight row), m-tile
};

// Tile L of the two tables (layer 1 first).  Within an expert the m-tiles of
// one n-tile are consecutive, so CTAs running at the same time share a weight
// tile in L2.
__device__ __forceinline__ MxTile mx_tile(const MxTail* t, int E, int T1, int L) {
  MxTile r;
  r.l2 = L >= T1;
  const int* ts = r.l2 ? t->tstart2 : t->tstart1;
  const int Ll = r.l2 ? L - T1 : L;
  r.e = tile_expert(ts, E, Ll);
  const int mt = (t->seg[r.e + 1] - t->seg[r.e]) / MB;
  const int local = Ll - ts[r.e];
  const int nti = local / mt, mti = local - nti * mt;
  r.row0 = t->seg[r.e] + mti * MB;
  r.n0 = nti * MN;
  r.m = r.row0 / MB;
  return r;
}

// Both expert layers in one persistent launch, tiles drawn from one counter:
// every layer-1 tile (h = act(xq W1q^T), quantised in the epilogue), then
// every layer-2 tile (yp = hq W2q^T in fp32 at the kept rows).  A layer-2
// tile needs its m-tile's h from every layer-1 n-tile: each epilogue warp of
// a finished layer-1 tile adds 1 to the m-tile's counter (a release after
// its stores), and the producer of a layer-2 tile waits for kEpiWarps x nt1
// (acquire, then a proxy fence so that its TMA and bulk reads see them).
// Tiles are claimed in increasing order, so a claimed layer-2 tile only
// waits for layer-1 tiles already claimed by running CTAs, which never wait.
// Roles: warp 0 claims tiles and issues the TMA and scale loads, warp 1 the
// scale copies to TMEM and the MMAs, warps 2-9 the epilogue; the claimed
// tiles pass between them through a 4-slot queue in shared memory.
template <int ACT, bool NARROW>
__global__ void __launch_bounds__(kThreads, 1)
tc_mx_mlp(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
          const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2, const MxParams p) {
  constexpr int STAGES = MxStages<NARROW>::kStages;
  constexpr int STAGE_BYTES = MxStages<NARROW>::kStageBytes;
  constexpr int A_BYTES = MxStages<NARROW>::kABytes;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);
  const uint32_t sf_base = base + (uint32_t)(STAGES * STAGE_BYTES);
  unsigned char* staging = sbase + (size_t)STAGES * STAGE_BYTES + (size_t)STAGES * 2 * SF_BYTES;
  MxTail* tail = reinterpret_cast<MxTail*>(staging + gemm::kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt1 = p.F1 / MN, nt2 = p.d / MN;
  const int nkb1 = p.d / MK, nkb2 = p.F / MK;

  const uint32_t full0 = smem_u32(&tail->full[0]), empty0 = smem_u32(&tail->empty[0]);
  const uint32_t tfull0 = smem_u32(&tail->tfull[0]), tempty0 = smem_u32(&tail->tempty[0]);
  const uint32_t qfull0 = smem_u32(&tail->qfull[0]), qempty0 = smem_u32(&tail->qempty[0]);
  const uint32_t drain = smem_u32(&tail->drain);
  const volatile int* abort_flag = &tail->abort_flag;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(tfull0 + 8 * a, 1);
      mbar_init(tempty0 + 8 * a, kEpiWarps);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(qfull0 + 8 * q, 1);
      mbar_init(qempty0 + 8 * q, 1 + kEpiWarps);   // the MMA lane and the epilogue warps
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
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA1)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB1)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmA2)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmB2)) : "memory");
  }
  pdl_wait();   // pad[], the quantised rows and the zeroed counters come from earlier kernels
  pdl_launch_dependents();
  if (warp == 0) {
    const bool ok1 = tile_table_warp(p.pad, p.E, MB, nt1, p.rows_pad, tail->tstart1, lane);
    const bool ok2 = tile_table_warp(p.pad, p.E, MB, nt2, p.rows_pad, tail->tstart2, lane);
    if (!(ok1 && ok2) && lane == 0 && blockIdx.x == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  for (int e = threadIdx.x; e <= p.E; e += kThreads) {
    tail->seg[e] = p.pad[e];
    tail->cnt[e] = (e < p.E) ? p.offsets[e + 1] - p.offsets[e] : 0;
    // the narrow layout holds 64 A rows: more kept rows than that would be
    // computed from the B tile, so the launch is flagged (the host picks it
    // only when no expert can have more)
    if (NARROW && tail->cnt[e] > MxStages<true>::kARows && blockIdx.x == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  const int T1 = tail->tstart1[p.E];
  const int total = T1 + tail->tstart2[p.E];

  if (warp == 0) {
    if (lane == 0) {
      // ---------------------------------------------- tile claimer + TMA producer
      int it = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int q = n % kQueue;
        const uint32_t qph = (uint32_t)(n / kQueue) & 1u;
        if (!mbar_wait(qempty0 + 8 * q, qph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
        int L = atomicAdd(p.sched, 1);
        if (L >= total) L = -1;
        tail->queue[q] = L;
        mbar_arrive(qfull0 + 8 * q);
        if (L < 0) break;
        const MxTile t = mx_tile(tail, p.E, T1, L);
        const CUtensorMap* mA = t.l2 ? &tmA2 : &tmA1;
        const CUtensorMap* mB = t.l2 ? &tmB2 : &tmB1;
        const uint8_t* sfa = t.l2 ? p.hs : p.xs;
        const uint8_t* sfb = t.l2 ? p.w2s : p.w1s;
        const int brow = t.e * (t.l2 ? p.d : p.F1) + t.n0;
        const int nkb = t.l2 ? nkb2 : nkb1;
        if (t.l2) {   // the h rows of this m-tile: every layer-1 n-tile, every epilogue warp
          if (!wait_flag_geq(p.dep + t.m, kEpiWarps * nt1, abort_flag, kWaitNs)) { ok = false; break; }
          fence_proxy_async_global();
        }
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint32_t sfs = sf_base + (uint32_t)(s * 2 * SF_BYTES);
          mbar_expect_tx(full0 + 8 * s, STAGE_BYTES + 2 * SF_BYTES);
          tma_load_2d(sa, mA, full0 + 8 * s, kb * MK, t.row0);
          tma_load_2d(sa + A_BYTES, mB, full0 + 8 * s, kb * MK, brow);
          bulk_load(sfs, sfa + ((size_t)(t.row0 / 128) * nkb + kb) * SF_BYTES, SF_BYTES, full0 + 8 * s);
          bulk_load(sfs + SF_BYTES, sfb + ((size_t)(brow / 128) * nkb + kb) * SF_BYTES, SF_BYTES, full0 + 8 * s);
          ++it;
        }
      }
      if (!ok) {
        atomicOr(p.status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
      }
      for (int i = max(0, it - STAGES); i < it; ++i)   // loads still in flight
        mbar_wait(full0 + 8 * (i % STAGES), (uint32_t)(i / STAGES) & 1u, nullptr, kDrainNs);
    }
  } else if (warp == 1) {
    if (lane == 0) {
      // ------------------------------------------------------- MMA issuer
      int it = 0, tl = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int q = n % kQueue;
        const uint32_t qph = (uint32_t)(n / kQueue) & 1u;
        if (!mbar_wait(qfull0 + 8 * q, qph, abort_flag, kWaitNs)) { ok = false; break; }
        const int L = tail->queue[q];
        mbar_arrive(qempty0 + 8 * q);
        if (L < 0) break;
        const int nkb = (L >= T1) ? nkb2 : nkb1;
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
        ++tl;
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
    // Eight warps: warp w drains TMEM lane quadrant w % 4; the two warps of a
    // quadrant split the tile's 32-column blocks.  A warp whose 32 rows are
    // all padding only takes part in the barriers and the counters (padding
    // rows are computed from their own A rows and never stored as kept rows).
    const int qw = warp & 3, half = (warp - 2) >> 2;
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)qw * gemm::kStageWarpBytes);
    int tl = 0;
    bool ok = true;
    for (int n = 0;; ++n) {
      const int q = n % kQueue;
      const uint32_t qph = (uint32_t)(n / kQueue) & 1u;
      ok = mbar_wait(qfull0 + 8 * q, qph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int L = tail->queue[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty0 + 8 * q);
      if (L < 0) break;
      const MxTile t = mx_tile(tail, p.E, T1, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(qw * 32) << 16) + (uint32_t)(acc * MN);
      const int local0 = t.row0 - tail->seg[t.e] + qw * 32;   // first row of this warp inside the expert
      const bool live = local0 < tail->cnt[t.e];
      const int prow = t.row0 + qw * 32 + lane;                // this thread's padded row
      if (!t.l2) {
        // h columns of the tile: ReLU 128 from n0 (4 blocks); SwiGLU 64 from
        // n0 / 2 (2 blocks; gate columns, then the up columns MN / 2 further)
        constexpr int kBlk = (ACT == kMxSwiglu) ? MN / 64 : MN / 32;
        const int h0 = (ACT == kMxSwiglu) ? t.n0 / 2 : t.n0;
        if (live) {
#pragma unroll 1
          for (int blk = half; blk < kBlk; blk += 2) {
            uint32_t a[32], u[32];
            tmem_ld32(tb + blk * 32, a);
            if (ACT == kMxSwiglu) tmem_ld32(tb + MN / 2 + blk * 32, u);
            tmem_wait_ld();
            float h[32];
            float amax = 0.f;
#pragma unroll
            for (int i = 0; i < 32; ++i) {
              const float g = __uint_as_float(a[i]);
              h[i] = (ACT == kMxSwiglu) ? __fdividef(g, 1.f + __expf(-g)) * __uint_as_float(u[i]) : fmaxf(g, 0.f);
              amax = fmaxf(amax, fabsf(h[i]));
            }
            const int X = mx_exponent(amax);
            uint4 lo, hi;
            quantize32(h, X, lo, hi);
            const int c = h0 + blk * 32;
            uint4* dst = reinterpret_cast<uint4*>(p.hq + (size_t)prow * p.F + c);
            dst[0] = lo;
            dst[1] = hi;
            p.hs[sf_offset(prow, c, p.F)] = (uint8_t)(X + 127);
          }
        }
        // this warp's share of the tile is written: count it for the m-tile
        // (__syncwarp orders the lanes' stores before lane 0's release, which
        // carries them to GPU scope)
        __syncwarp();
        if (lane == 0) red_release_gpu_add(p.dep + t.m, 1);
      } else if (half == 0 && live) {
        // fp32 rows to the kept row each padded row came from (padding rows are dropped)
        const int i = prow - tail->seg[t.e];
        const int row = (i < tail->cnt[t.e]) ? p.offsets[t.e] + i : -1;
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
          const int col0 = t.n0 + blk * 32;
#pragma unroll
          for (int r8 = 0; r8 < 8; ++r8) {
            const int rr = r8 * 4 + (lane >> 3), cc = lane & 7;
            const int trow = __shfl_sync(0xffffffffu, row, rr);
            if (trow >= 0)
              *reinterpret_cast<uint4*>(p.out + (size_t)trow * p.d + col0 + cc * 4) = stg[rr * 8 + (cc ^ (rr & 7))];
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);   // accumulator free again
      ++tl;
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

template <int ACT, bool NARROW>
cudaError_t launch_mx(const CUtensorMap& a1, const CUtensorMap& b1, const CUtensorMap& a2, const CUtensorMap& b2,
                      const MxParams& p, int grid, cudaStream_t s) {
  constexpr size_t smem = mx_smem<NARROW>();
  cudaError_t err = set_smem_once<tc_mx_mlp<ACT, NARROW>>(smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_mx_mlp<ACT, NARROW>, dim3(grid), dim3(kThreads), smem, s, a1, b1, a2, b2, p);
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
  const int mt_max = b.rows_pad / MB;
  // the padded segments (and zeroed counters), the kept layer-1 input rows in E4M3
  {
    const int rows_max = c.T * c.k;
    const size_t nblk = (size_t)rows_max * (c.d / 32);
    const int grid = (int)std::max<size_t>(1, std::min<size_t>((nblk + 255) / 256, (size_t)di.sms * 8));
    err = launch_pdl(mx_quantize_rows_kernel, dim3(grid), dim3(256), 0, s,
                     static_cast<const __nv_bfloat16*>(b.xp), rows_max, b.rows_pad, c.d, b.offsets, c.E, b.pad,
                     b.ctr,
                     1 + mt_max, static_cast<uint8_t*>(b.xq), static_cast<uint8_t*>(b.xs));
    if (err != cudaSuccess) return err;
  }
  // both layers in one launch: h = act(xq W1q^T) quantised in the epilogue,
  // then yp = hq W2q^T (fp32) at the kept rows
  const bool narrow = c.T <= MxStages<true>::kARows;
  const uint32_t a_rows = narrow ? MxStages<true>::kARows : MxStages<false>::kARows;
  CUtensorMap a1, b1, a2, b2;
  if (!make_map_u8(&a1, b.xq, (uint64_t)b.rows_pad, (uint64_t)c.d, a_rows) ||
      !make_map_u8(&b1, w1q, (uint64_t)c.E * F1, (uint64_t)c.d) ||
      !make_map_u8(&a2, b.hq, (uint64_t)b.rows_pad, (uint64_t)c.F, a_rows) ||
      !make_map_u8(&b2, w2q, (uint64_t)c.E * c.d, (uint64_t)c.F))
    return cudaErrorInvalidValue;
  MxParams p{};
  p.pad = b.pad;
  p.offsets = b.offsets;
  p.E = c.E;
  p.d = c.d;
  p.F = c.F;
  p.F1 = F1;
  p.rows_pad = b.rows_pad;
  p.xs = static_cast<const uint8_t*>(b.xs);
  p.w1s = static_cast<const uint8_t*>(w1s);
  p.w2s = static_cast<const uint8_t*>(w2s);
  p.hq = static_cast<uint8_t*>(b.hq);
  p.hs = static_cast<uint8_t*>(b.hs);
  p.out = yp;
  p.status = status;
  p.sched = b.ctr;
  p.dep = b.ctr + 1;
  const int grid = (int)std::max<long long>(1, std::min<long long>((long long)mt_max * (F1 / MN + c.d / MN), di.sms));
  if (narrow)
    return (c.act == MOE_ACT_SWIGLU) ? launch_mx<kMxSwiglu, true>(a1, b1, a2, b2, p, grid, s)
                                     : launch_mx<kMxRelu, true>(a1, b1, a2, b2, p, grid, s);
  return (c.act == MOE_ACT_SWIGLU) ? launch_mx<kMxSwiglu, false>(a1, b1, a2, b2, p, grid, s)
                                   : launch_mx<kMxRelu, false>(a1, b1, a2, b2, p, grid, s);
}

}  // namespace moe
