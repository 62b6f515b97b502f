// Step 4, and with k <= 2 step 5, in one persistent launch: both expert
// layers (and the fused combine) with the tiles of the two layers drawn from
// one dynamic queue.
//
// The experts' two layers are grouped GEMMs over the expert segments
// (Megatron-Core best-practice page, "Megatron-Core MoE的关键特性":
// GroupedGEMM; FastMoE announcement, Transformer-XL experiment: ReLU MLP;
// SwiGLU with the gate rows first, Megatron-Core page,
// "从HuggingFace到Megatron的权重转换要点"), and the output of a token is the
// gate-weighted sum of its experts' outputs (FastMoE announcement,
// "1. MoE 设计").
//
// Two separate launches leave SMs idle at the end of each layer (the layers'
// 128 x 256 tiles fill 4.3 and 2.2 waves on the FastMoE layer, 2.8 and 2.05
// on the top-6 decode layer).  Here one grid of one CTA per SM takes tiles
// from a global counter: first every layer-1 tile (h = act(xp W1^T)), then
// every layer-2 tile.  With COMB (k <= 2) a layer-2 tile adds w * (h W2^T)
// into the token row of out (at most two additions per output); without it,
// it stores the fp32 rows of yp for the separate combine kernel.  A
// layer-2 tile needs the h rows of its m-tile from all layer-1 n-tiles: each
// epilogue warp of a finished layer-1 tile adds 1 to the m-tile's counter
// (a release after its h stores), and the TMA producer of a
// layer-2 tile waits for the counter to reach 4 x the layer-1 n-tile count
// (acquire, then a proxy fence so that its TMA reads see those stores).  Tiles are claimed in increasing
// order, so a claimed layer-2 tile only waits for layer-1 tiles already
// claimed by running CTAs, which never wait themselves.
//
// Batches of at most 64 tokens (decode) take m-tiles of 64 rows and one more
// stage of weight tiles in flight (MlpLayout).
//
// Roles as in the 1-SM grouped GEMM (warp 0 TMA producer and tile claimer,
// warp 1 MMA issuer, warps 2-5 epilogue); the producer passes each claimed
// tile to the other roles through a 4-slot queue in shared memory.  Every
// wait is bounded (~2 s) and a role that gives up sets MOE_DEV_TIMEOUT and
// stops the others.
#include "gemm_common.cuh"

#include <algorithm>
#include <atomic>

namespace moe {
namespace {

using namespace tc;
using namespace gemm;

constexpr int BM = 128;                           // MMA rows
constexpr int B_BYTES = BN * BK * 2;              // 32 KB
constexpr int kMaxStages = 5;
constexpr int kNarrowRows = 64;

// Stage layouts.  Wide: m-tiles of 128 rows, A 16 KB + B 32 KB, 4 stages.
// Narrow, for batches of at most 64 tokens: m-tiles of 64 rows (a decode
// expert has at most 64), A 8 KB, and 5 stages keep 160 KB of weight tiles
// in flight per SM instead of 128 KB.  The MMA still reads 128 A rows, the
// last 64 from the stage's own B tile; those accumulator rows are computed
// and never stored (a tile's rows end at 64).
template <bool NARROW>
struct MlpLayout {
  static constexpr int kTileRows = NARROW ? kNarrowRows : BM;
  static constexpr int kABytes = kTileRows * BK * 2;
  static constexpr int kStages = NARROW ? 5 : 4;
  static constexpr int kStageBytes = kABytes + B_BYTES;
  static_assert(kStages <= kMaxStages && kStageBytes % 1024 == 0, "stages of 1 KB-aligned tiles");
};
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
constexpr int kQueue = 4;                         // claimed tiles in flight between the roles

struct Tail {
  unsigned long long full[kMaxStages], empty[kMaxStages], tfull[2], tempty[2], drain;
  unsigned long long qfull[kQueue], qempty[kQueue];
  uint32_t tmem_base;
  int abort_flag;
  int queue[kQueue];
  int tstart1[kMaxExperts + 1];   // layer-1 tile table
  int tstart2[kMaxExperts + 1];   // layer-2 tile table
  int mstart[kMaxExperts + 1];    // first m-tile of each expert (dependency counters)
  int seg[kMaxExperts + 1];       // copy of offsets[]
};
template <bool NARROW>
constexpr size_t mlp_smem() {
  return 1024 + (size_t)MlpLayout<NARROW>::kStages * MlpLayout<NARROW>::kStageBytes + kStagingBytes + sizeof(Tail);
}
static_assert(mlp_smem<false>() <= 227 * 1024 && mlp_smem<true>() <= 227 * 1024, "shared memory of one CTA");

struct MlpParams {
  const int32_t* offsets;
  void* h;                  // [rows][F] hidden (16-bit)
  float* out;               // COMB: [T][d] layer output, zeroed beforehand; else [rows][d] yp
  const int32_t* src_tok;   // token of each permuted row
  const float* row_w;       // gate weight of each permuted row
  int E, d, F;
  int F1;                   // W1 rows per expert (F or 2F)
  int T;                    // token rows of out
  int rows_alloc;           // rows of xp and h
  int* sched;               // [0]: next tile to claim; zeroed beforehand
  int* dep;                 // per global m-tile: layer-1 n-tiles finished; zeroed beforehand
  uint32_t* status;
  unsigned long long wait_ns;   // limit of every bounded wait (kWaitNs unless a test shortens it)
  int dep_extra;                // added to the layer-2 dependency target (0 unless a test sets it)
  int e_mod;                    // weight blocks: segment e uses block e % e_mod
};

// the tile's layer, coordinates and global m-tile index
struct MlpTile {
  bool l2;
  TileCoord c;
  int m;
};

template <int ACT, int TM>
__device__ __forceinline__ MlpTile mlp_tile(const Tail* tail, int E, int T1, int L) {
  MlpTile t;
  t.l2 = L >= T1;
  t.c = t.l2 ? decode_tile<kCombine, TM>(tail->tstart2, tail->seg, E, L - T1)
             : decode_tile<ACT, TM>(tail->tstart1, tail->seg, E, L);
  t.m = tail->mstart[t.c.e] + (t.c.row0 - tail->seg[t.c.e]) / TM;
  return t;
}

template <int ACT, bool F16, bool COMB, bool NARROW>
__global__ void __launch_bounds__(kThreads, 1)
tc_expert_mlp(const __grid_constant__ CUtensorMap tmA1, const __grid_constant__ CUtensorMap tmB1,
              const __grid_constant__ CUtensorMap tmA2, const __grid_constant__ CUtensorMap tmB2,
              const MlpParams p) {
  constexpr int TM = MlpLayout<NARROW>::kTileRows;
  constexpr int STAGES = MlpLayout<NARROW>::kStages;
  constexpr int A_BYTES = MlpLayout<NARROW>::kABytes;
  constexpr int STAGE_BYTES = MlpLayout<NARROW>::kStageBytes;
  constexpr uint32_t kIdesc1 = idesc_f16kind(BM, BN, false);   // xp, W1: bf16
  constexpr uint32_t kIdesc2 = idesc_f16kind(BM, BN, F16);     // h, W2: the hidden type
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* staging = smem_raw + (base - raw) + (size_t)STAGES * STAGE_BYTES;
  Tail* tail = reinterpret_cast<Tail*>(staging + kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nt1 = (ACT == kSwiglu) ? (p.F + BN / 2 - 1) / (BN / 2) : (p.F + BN - 1) / BN;
  const int nt2 = (p.d + BN - 1) / BN;
  const int nkb1 = (p.d + BK - 1) / BK, nkb2 = (p.F + BK - 1) / BK;

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
      mbar_init(tempty0 + 8 * a, 4);
    }
    for (int q = 0; q < kQueue; ++q) {
      mbar_init(qfull0 + 8 * q, 1);
      mbar_init(qempty0 + 8 * q, 1 + 4);   // the MMA lane and the 4 epilogue warps
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
  pdl_wait();                  // offsets[], xp, out zeroed, counters zeroed: earlier kernels
  pdl_launch_dependents();
  bool table_ok = true;
  if (warp == 0) {
    table_ok = tile_table_warp(p.offsets, p.E, TM, nt1, p.rows_alloc, tail->tstart1, lane);
    table_ok &= tile_table_warp(p.offsets, p.E, TM, nt2, p.rows_alloc, tail->tstart2, lane);
    table_ok &= tile_table_warp(p.offsets, p.E, TM, 1, p.rows_alloc, tail->mstart, lane);
    if (!table_ok && lane == 0 && blockIdx.x == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
  }
  for (int e = threadIdx.x; e <= p.E; e += kThreads) tail->seg[e] = p.offsets[e];
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;
  const int T1 = tail->tstart1[p.E];
  const int total = T1 + tail->tstart2[p.E];

  Params p1{p.offsets, p.h, p.E, p.d, p.F, p.F1, p.F, p.rows_alloc, p.status, nullptr, nullptr, 0};
  Params p2{p.offsets, p.out, p.E, p.F, p.d, p.d, 0, p.rows_alloc, p.status, p.src_tok, p.row_w, p.T};

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------ tile claimer + TMA producer
      int it = 0;
      bool ok = true;
      for (int n = 0; ok; ++n) {
        const int q = n % kQueue;
        const uint32_t qph = (uint32_t)(n / kQueue) & 1u;
        if (!mbar_wait(qempty0 + 8 * q, qph ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        int L = atomicAdd(p.sched, 1);
        if (L >= total) L = -1;
        tail->queue[q] = L;
        mbar_arrive(qfull0 + 8 * q);
        if (L < 0) break;
        const MlpTile t = mlp_tile<ACT, TM>(tail, p.E, T1, L);
        const CUtensorMap* mA = t.l2 ? &tmA2 : &tmA1;
        const CUtensorMap* mB = t.l2 ? &tmB2 : &tmB1;
        int b0, b1;
        if (!t.l2) {
          b0 = (t.c.e % p.e_mod) * p.F1 + t.c.n0;
          b1 = (ACT == kSwiglu) ? b0 + p.F : b0 + BN / 2;
        } else {
          b0 = (t.c.e % p.e_mod) * p.d + t.c.n0;
          b1 = b0 + BN / 2;
        }
        if (t.l2) {   // the h rows of this m-tile: every layer-1 n-tile, 4 epilogue warps each
          if (!wait_flag_geq(p.dep + t.m, 4 * nt1 + p.dep_extra, abort_flag, p.wait_ns)) { ok = false; break; }
          fence_proxy_async_global();
        }
        const int nkb = t.l2 ? nkb2 : nkb1;
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          mbar_expect_tx(full0 + 8 * s, STAGE_BYTES);
          tma_load_2d(sa, mA, full0 + 8 * s, kb * BK, t.c.row0);
          tma_load_2d(sa + A_BYTES, mB, full0 + 8 * s, kb * BK, b0);
          tma_load_2d(sa + A_BYTES + B_BYTES / 2, mB, full0 + 8 * s, kb * BK, b1);
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
        if (!mbar_wait(qfull0 + 8 * q, qph, abort_flag, p.wait_ns)) { ok = false; break; }
        const int L = tail->queue[q];
        mbar_arrive(qempty0 + 8 * q);
        if (L < 0) break;
        const bool l2 = L >= T1;
        const int nkb = l2 ? nkb2 : nkb1;
        const uint32_t idesc = l2 ? kIdesc2 : kIdesc1;
        const int acc = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, p.wait_ns)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, p.wait_ns)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint64_t ad = sdesc(sa), bd = sdesc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb | kk) != 0);
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
    const int qw = warp & 3;             // TMEM lanes 32qw..32qw+31 belong to this warp
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * kStageWarpBytes);
    int tl = 0;
    bool ok = true;
    for (int n = 0;; ++n) {
      const int q = n % kQueue;
      const uint32_t qph = (uint32_t)(n / kQueue) & 1u;
      ok = mbar_wait(qfull0 + 8 * q, qph, abort_flag, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      const int L = tail->queue[q];
      __syncwarp();
      if (lane == 0) mbar_arrive(qempty0 + 8 * q);
      if (L < 0) break;
      const MlpTile t = mlp_tile<ACT, TM>(tail, p.E, T1, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, p.wait_ns);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(qw * 32) << 16) + (uint32_t)(acc * BN);
      const int wrow0 = t.c.row0 + qw * 32;
      bool over = false;
      if (!t.l2) {
        const int nrows = warp_rows(p1, wrow0, t.c.rows - qw * 32, lane);
        if (nrows > 0) store_tile<ACT, F16>(p1, tb, wrow0, nrows, t.c.n0, stg, lane, over);
        // this warp's h rows of the tile are written: count them for the m-tile
        // (__syncwarp orders the lanes' stores before lane 0's release, which
        // carries them to GPU scope)
        __syncwarp();
        if (lane == 0) red_release_gpu_add(p.dep + t.m, 1);
      } else {
        const int nrows = warp_rows(p2, wrow0, t.c.rows - qw * 32, lane);
        if (nrows > 0) store_tile<COMB ? kCombine : kPlain, F16>(p2, tb, wrow0, nrows, t.c.n0, stg, lane, over);
      }
      if (F16 && over) atomicOr(p.status, MOE_DEV_RANGE);
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

template <int ACT, bool F16, bool COMB, bool NARROW>
cudaError_t launch_t(const CUtensorMap (&maps)[4], const MlpParams& p, int grid, cudaStream_t s) {
  constexpr size_t smem = mlp_smem<NARROW>();
  cudaError_t err = set_smem_once<tc_expert_mlp<ACT, F16, COMB, NARROW>>(smem);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_expert_mlp<ACT, F16, COMB, NARROW>, dim3(grid), dim3(kThreads), smem, s, maps[0], maps[1],
                    maps[2], maps[3], p);
}
template <int ACT, bool F16, bool NARROW>
cudaError_t launch_n(const CUtensorMap (&maps)[4], const MlpParams& p, bool comb, int grid, cudaStream_t s) {
  return comb ? launch_t<ACT, F16, true, NARROW>(maps, p, grid, s) : launch_t<ACT, F16, false, NARROW>(maps, p, grid, s);
}
template <int ACT, bool F16>
cudaError_t launch_c(const CUtensorMap (&maps)[4], const MlpParams& p, bool comb, bool narrow, int grid,
                     cudaStream_t s) {
  return narrow ? launch_n<ACT, F16, true>(maps, p, comb, grid, s) : launch_n<ACT, F16, false>(maps, p, comb, grid, s);
}

std::atomic<unsigned long long> g_wait_ns{kWaitNs};
std::atomic<int> g_dep_extra{0};

}  // namespace

void set_expert_mlp_test_hooks(unsigned long long wait_ns, int dep_extra) {
  g_wait_ns.store(wait_ns != 0 ? wait_ns : kWaitNs);
  g_dep_extra.store(dep_extra);
}

size_t expert_mlp_counters(const moe_config& c) {
  const int tm = c.T <= kNarrowRows ? kNarrowRows : BM;   // the m-tile height the launch takes
  return 1 + (size_t)c.T * c.k / tm + (size_t)c.E + 1;
}

cudaError_t launch_expert_mlp(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                              const void* w2, void* h, const CombineOut* comb, float* yp, int* counters,
                              uint32_t* status, cudaStream_t s, int e_mod) {
  if (c.T == 0) return cudaSuccess;
  if (comb == nullptr && yp == nullptr) return cudaErrorInvalidValue;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const bool f16 = c.hidden_dtype == MOE_DTYPE_F16;
  const uint64_t rows = (uint64_t)c.T * (uint64_t)c.k;
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const int EW = e_mod > 0 ? e_mod : c.E;   // experts whose weights are given
  // narrow tiles where no routed expert can have more than 64 rows (any
  // segment stays correct: it is cut into 64-row m-tiles); the counters'
  // count (expert_mlp_counters) follows the same rule
  const bool narrow = c.T <= kNarrowRows;
  const uint32_t tm = narrow ? kNarrowRows : BM;
  CUtensorMap maps[4];
  if (!make_map(&maps[0], xp, rows, (uint64_t)c.d, false, tm) ||
      !make_map(&maps[1], w1, (uint64_t)EW * F1, (uint64_t)c.d, false) ||
      !make_map(&maps[2], h, rows, (uint64_t)c.F, f16, tm) ||
      !make_map(&maps[3], w2, (uint64_t)EW * c.d, (uint64_t)c.F, f16))
    return cudaErrorInvalidValue;
  MlpParams p{offsets, h, comb ? comb->out : yp, comb ? comb->src_tok : nullptr, comb ? comb->row_w : nullptr,
              c.E, c.d, c.F, F1, comb ? comb->T : 0, (int)rows, counters, counters + 1, status,
              g_wait_ns.load(), g_dep_extra.load(), EW};
  const bool cb = comb != nullptr;
  const long long mt_max = (long long)(rows / tm) + c.E;
  const long long nt = (c.act == MOE_ACT_SWIGLU ? (c.F + BN / 2 - 1) / (BN / 2) : (c.F + BN - 1) / BN) +
                       (c.d + BN - 1) / BN;
  const int grid = (int)std::min<long long>(mt_max * nt, di.sms);
  if (c.act == MOE_ACT_SWIGLU)
    return f16 ? launch_c<kSwiglu, true>(maps, p, cb, narrow, grid, s)
               : launch_c<kSwiglu, false>(maps, p, cb, narrow, grid, s);
  return f16 ? launch_c<kRelu, true>(maps, p, cb, narrow, grid, s) : launch_c<kRelu, false>(maps, p, cb, narrow, grid, s);
}

}  // namespace moe
