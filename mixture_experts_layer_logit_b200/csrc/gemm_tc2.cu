// Step 4 with 2-SM tiles: the experts' grouped GEMMs (Megatron-Core
// best-practice page, "Megatron-Core MoE的关键特性": GroupedGEMM), each tile
// computed by a pair of CTAs on two SMs of one cluster through
// tcgen05.mma.cta_group::2.
//
// A pair tile is 256 rows x 256 columns.  CTA r of the pair loads rows
// [128 r, 128 r + 128) of the A tile and weight rows [128 r, 128 r + 128) of
// the B tile (SwiGLU: r = 0 the gate rows, r = 1 the up rows) to the same
// shared-memory offsets; the even CTA issues the MMA (M = 256, N = 256,
// K = 16) and each CTA's TMEM receives its 128 rows x 256 columns.  Per SM and
// k-block this loads 32 KB for 128 x 256 x 64 multiply-adds where the 1-SM
// tile loads 48 KB, so the same bytes in flight feed 1.5x the math, and six
// stages fit in shared memory.
//
// Barriers (in both CTAs at the same offsets):
//   full[s]   used in the even CTA: both CTAs' loads of stage s complete on it
//             (its producer expects the bytes of both halves);
//   empty[s]  both: the MMA commit arrives on both once stage s has been read;
//   tfull[a]  both: accumulator a is ready (commit to both CTAs);
//   tempty[a] used in the even CTA: the pair's 8 epilogue warps free a.
// Every wait is bounded (~2 s).  A role that gives up sets MOE_DEV_TIMEOUT and
// the abort flags of both CTAs; both CTAs always meet at the closing cluster
// barrier, after the even CTA has waited for its MMAs and for the loads
// counted on its barriers, and only then free TMEM.
#include "gemm_common.cuh"

#include <algorithm>

namespace moe {
namespace {

using namespace tc;
using namespace gemm;

constexpr int PM = 256;                    // rows of a pair tile
constexpr int HM = PM / 2;                 // A rows per CTA
constexpr int HN = BN / 2;                 // B rows per CTA
constexpr int STAGES = 6;
constexpr int A_BYTES = HM * BK * 2;       // 16 KB
constexpr int B_BYTES = HN * BK * 2;       // 16 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

struct Tail {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];
};
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + kStagingBytes + sizeof(Tail);
static_assert(kSmemBytes <= 227 * 1024, "shared memory of one CTA");

template <int MODE, bool F16>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kThreads, 1)
tc_grouped_gemm_pair(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                     const Params p) {
  constexpr uint32_t kIdesc = idesc_f16kind(PM, BN, layer2(MODE) && F16);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;   // the same offset in both CTAs
  unsigned char* staging = smem_raw + (base - raw) + (size_t)STAGES * STAGE_BYTES;
  Tail* tail = reinterpret_cast<Tail*>(staging + kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_rank();
  const int pair = (int)cluster_id(), npairs = (int)cluster_count();
  const int nt = (MODE == kSwiglu) ? (p.Nout + BN / 2 - 1) / (BN / 2) : (p.Nout + BN - 1) / BN;
  const int nkb = (p.K + BK - 1) / BK;

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
      mbar_init(tempty0 + 8 * a, 8);
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
  pdl_wait();                  // offsets[] and the A rows come from earlier kernels
  pdl_launch_dependents();
  if (warp == 0) {
    if (!tile_table_warp(p.offsets, p.E, PM, nt, p.rows_alloc, tail->tstart, lane) && lane == 0 &&
        blockIdx.x == 0)
      atomicOr(p.status, MOE_DEV_BOUNDS);   // offsets[] unusable: no tile is scheduled
  }
  for (int e = threadIdx.x; e <= p.E; e += kThreads) tail->seg[e] = p.offsets[e];
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
        const TileCoord c = decode_tile<MODE, PM>(tail->tstart, tail->seg, p.E, L);
        const int arow = c.row0 + HM * (int)rank;
        const int brow =
            weight_block(p, c.e) * p.b_rows + c.n0 + (rank == 0 ? 0 : (MODE == kSwiglu ? p.up_off : HN));
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          if (rank == 0) mbar_expect_tx(full0 + 8 * s, 2 * STAGE_BYTES);   // both halves
          tma_load_2d_pair(sa, &tmA, full0_lead + 8 * s, kb * BK, arow);
          tma_load_2d_pair(sa + A_BYTES, &tmB, full0_lead + 8 * s, kb * BK, brow);
          ++it;
        }
      }
      if (!ok) give_up();
      if (rank == 0) {
        // the loads still in flight (of both CTAs) complete on these barriers
        for (int i = max(0, it - STAGES); i < it; ++i)
          mbar_wait(full0 + 8 * (i % STAGES), (uint32_t)(i / STAGES) & 1u, nullptr, kDrainNs);
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
        const int acc = tl & 1;
        const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
        if (!mbar_wait(tempty0 + 8 * acc, aph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
        tc_fence_after();
        const uint32_t d_tmem = tmem + (uint32_t)(acc * BN);
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kWaitNs)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          const uint64_t ad = sdesc(sa), bd = sdesc(sa + A_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk)
            tc_mma_pair(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), kIdesc, (kb | kk) != 0);
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
    const int q = warp & 3;              // TMEM lanes 32q..32q+31 belong to this warp
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * kStageWarpBytes);
    int tl = 0;
    bool ok = true;
    for (int L = pair; L < total; L += npairs, ++tl) {
      const TileCoord c = decode_tile<MODE, PM>(tail->tstart, tail->seg, p.E, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int wrow0 = c.row0 + HM * (int)rank + q * 32;
      const int nrows = warp_rows(p, wrow0, c.rows - HM * (int)rank - q * 32, lane);
      bool over = false;
      if (nrows > 0) store_tile<MODE, F16>(p, tb, wrow0, nrows, c.n0, stg, lane, over);
      if (F16 && over) atomicOr(p.status, MOE_DEV_RANGE);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(tempty0_lead + 8 * acc);   // accumulator free again
    }
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

template <int MODE, bool F16>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, int pairs, cudaStream_t s) {
  cudaError_t err = set_smem_once<tc_grouped_gemm_pair<MODE, F16>>(kSmemBytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_grouped_gemm_pair<MODE, F16>, dim3(2 * pairs), dim3(kThreads), kSmemBytes, s, ma, mb, p);
}

template <bool F16>
cudaError_t launch_layers(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                          const void* w2, void* h, void* yp, uint32_t* status, int sms, cudaStream_t s,
                          const CombineOut* comb, int e_mod) {
  const int EW = e_mod > 0 ? e_mod : c.E;   // experts whose weights are given
  const uint64_t rows = (uint64_t)c.T * (uint64_t)c.k;
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const long long mt_max = (long long)(rows / PM) + c.E;
  const int max_pairs = std::max(1, sms / 2);
  CUtensorMap ma, mb;
  cudaError_t err;

  // layer 1: h = act(xp W1[e]^T)
  if (!make_map(&ma, xp, rows, (uint64_t)c.d, false) || !make_map(&mb, w1, (uint64_t)EW * F1, (uint64_t)c.d, false))
    return cudaErrorInvalidValue;
  Params p1{offsets, h, c.E, c.d, c.F, F1, c.F, (int)rows, status};
  p1.e_mod = e_mod;
  if (c.act == MOE_ACT_SWIGLU) {
    const long long nt = (c.F + BN / 2 - 1) / (BN / 2);
    err = launch_one<kSwiglu, F16>(ma, mb, p1, (int)std::min<long long>(mt_max * nt, max_pairs), s);
  } else {
    const long long nt = (c.F + BN - 1) / BN;
    err = launch_one<kRelu, F16>(ma, mb, p1, (int)std::min<long long>(mt_max * nt, max_pairs), s);
  }
  if (err != cudaSuccess) return err;

  // layer 2: yp = h W2[e]^T in fp32
  if (!make_map(&ma, h, rows, (uint64_t)c.F, F16) || !make_map(&mb, w2, (uint64_t)EW * c.d, (uint64_t)c.F, F16))
    return cudaErrorInvalidValue;
  Params p2{offsets, yp, c.E, c.F, c.d, c.d, 0, (int)rows, status};
  p2.e_mod = e_mod;
  const long long nt2 = (c.d + BN - 1) / BN;
  const int g2 = (int)std::min<long long>(mt_max * nt2, max_pairs);
  if (comb != nullptr) {   // step 5 fused: gate-weighted sums into the token rows of out
    p2.out = comb->out;
    p2.src_tok = comb->src_tok;
    p2.row_w = comb->row_w;
    p2.out_rows = comb->T;
    return launch_one<kCombine, F16>(ma, mb, p2, g2, s);
  }
  return launch_one<kPlain, F16>(ma, mb, p2, g2, s);
}

}  // namespace

cudaError_t launch_grouped_plain_tc_pair(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
                                         const void* B, int K, int Nout, float* out, uint32_t* status, bool f16,
                                         cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  CUtensorMap ma, mb;
  if (!make_map(&ma, A, (uint64_t)rows_alloc, (uint64_t)K, f16) ||
      !make_map(&mb, B, (uint64_t)c.E * Nout, (uint64_t)K, f16))
    return cudaErrorInvalidValue;
  Params p{offsets, out, c.E, K, Nout, Nout, 0, rows_alloc, status};
  const long long tiles = ((long long)rows_alloc / PM + c.E) * ((Nout + BN - 1) / BN);
  const int pairs = (int)std::min<long long>(tiles, std::max(1, di.sms / 2));
  return f16 ? launch_one<kPlain, true>(ma, mb, p, pairs, s) : launch_one<kPlain, false>(ma, mb, p, pairs, s);
}

cudaError_t launch_expert_ffn_tc_pair(const moe_config& c, const void* xp, const int32_t* offsets,
                                      const void* w1, const void* w2, void* h, void* yp,
                                      uint32_t* status, cudaStream_t s, const CombineOut* comb, int e_mod) {
  if (c.T == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  if (c.hidden_dtype == MOE_DTYPE_F16)
    return launch_layers<true>(c, xp, offsets, w1, w2, h, yp, status, di.sms, s, comb, e_mod);
  return launch_layers<false>(c, xp, offsets, w1, w2, h, yp, status, di.sms, s, comb, e_mod);
}

}  // namespace moe
