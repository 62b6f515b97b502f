// Step 4 on the 5th-generation tensor cores (sm_100a): the experts' two
// layers as grouped GEMMs over the variable-length expert segments.
//
// Megatron-Core best-practice page, "Megatron-Core MoE的关键特性": GroupedGEMM
// merges the experts' many small GEMMs into one kernel to keep the SMs busy.
// Experts: two-layer ReLU MLP (FastMoE announcement, Transformer-XL
// experiment) or SwiGLU whose W1 holds the gate rows before the up rows
// (Megatron-Core page, "从HuggingFace到Megatron的权重转换要点").
//
// Design (one CTA per SM, persistent):
//   * A = expert-grouped rows (xp or h), B = one expert's weight rows; both
//     K-major 16-bit (bf16 for layer 1; the hidden type, fp16 or bf16, for
//     layer 2), staged by TMA (128-byte swizzle) into a STAGES-deep ring.
//   * warp 0 lane 0 issues the TMA loads, warp 1 lane 0 issues
//     tcgen05.mma.cta_group::1.kind::f16 (128 x 256 x 16, fp32 accumulators in
//     TMEM), warps 2-5 drain TMEM with tcgen05.ld and run the epilogue of
//     gemm_common.cuh: layer 1 applies the activation (ReLU, or
//     silu(gate) * up for SwiGLU) and stores h; layer 2 stores fp32 yp or
//     adds the gate-weighted rows into out (fused combine).
//   * two 256-column TMEM accumulators let the epilogue of one tile overlap
//     the main loop of the next.
//   * the tile table (ceil(M_e / 128) * n-tiles per expert) is built on the
//     device from offsets[], so nothing is read back to the host; within an
//     expert the m-tiles of one n-tile are consecutive, so the CTAs working at
//     the same time share the same weight tile in L2.
//   * a tile that runs past its expert's segment computes rows of the next
//     expert (or zero rows past the buffer) and masks them at the store.
//   * every mbarrier wait is bounded (~2 s); on timeout the kernel sets
//     MOE_DEV_TIMEOUT, tells the other roles to stop, waits for its own TMA
//     loads and MMAs, frees TMEM and returns.
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
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;

struct Tail {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];     // copy of offsets[]: tiles are decoded without global loads
};
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + kStagingBytes + sizeof(Tail);

// F16: the hidden activation (layer-1 output, layer-2 A operand) and W2 are
// fp16 instead of bf16.
template <int MODE, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const Params p) {
  constexpr uint32_t kIdesc = idesc_f16kind(BM, BN, layer2(MODE) && F16);
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* staging = smem_raw + (base - raw) + (size_t)STAGES * STAGE_BYTES;
  Tail* tail = reinterpret_cast<Tail*>(staging + kStagingBytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
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
      mbar_init(tempty0 + 8 * a, 4);
    }
    mbar_init(drain, 1);
    tail->abort_flag = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
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
  pdl_wait();                  // offsets[] and the A rows come from earlier kernels
  pdl_launch_dependents();
  if (warp == 0) {
    if (!tile_table_warp(p.offsets, p.E, BM, nt, p.rows_alloc, tail->tstart, lane) && lane == 0 &&
        blockIdx.x == 0)
      atomicOr(p.status, MOE_DEV_BOUNDS);   // offsets[] unusable: no tile is scheduled
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
        const TileCoord c = decode_tile<MODE, BM>(tail->tstart, tail->seg, p.E, L);
        const int b0 = weight_block(p, c.e) * p.b_rows + c.n0;
        const int b1 = (MODE == kSwiglu) ? b0 + p.up_off : b0 + BN / 2;
        for (int kb = 0; kb < nkb; ++kb) {
          const int s = it % STAGES;
          const uint32_t ph = (uint32_t)(it / STAGES) & 1u;
          if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) { ok = false; break; }
          const uint32_t sa = base + (uint32_t)(s * STAGE_BYTES);
          mbar_expect_tx(full0 + 8 * s, STAGE_BYTES);
          tma_load_2d(sa, &tmA, full0 + 8 * s, kb * BK, c.row0);
          tma_load_2d(sa + A_BYTES, &tmB, full0 + 8 * s, kb * BK, b0);
          tma_load_2d(sa + A_BYTES + B_BYTES / 2, &tmB, full0 + 8 * s, kb * BK, b1);
          ++it;
        }
      }
      if (!ok) {
        atomicOr(p.status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
      }
      // wait for the loads still in flight before the CTA may exit
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
            tc_mma(d_tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), kIdesc, (kb | kk) != 0);
          tc_commit(empty0 + 8 * s);   // frees the stage once these MMAs have read it
          ++it;
        }
        if (!ok) break;
        tc_commit(tfull0 + 8 * acc);   // accumulator ready for the epilogue
      }
      if (!ok) {
        atomicOr(p.status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
      }
      tc_commit(drain);                 // every MMA issued above has completed
      mbar_wait(drain, 0, nullptr, kDrainNs);
    }
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;              // TMEM lanes 32q..32q+31 belong to this warp
    uint4* stg = reinterpret_cast<uint4*>(staging + (size_t)(warp - 2) * kStageWarpBytes);
    int tl = 0;
    bool ok = true;
    for (int L = blockIdx.x; L < total; L += gridDim.x, ++tl) {
      const TileCoord c = decode_tile<MODE, BM>(tail->tstart, tail->seg, p.E, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      const int wrow0 = c.row0 + q * 32;
      const int nrows = warp_rows(p, wrow0, c.rows - q * 32, lane);
      bool over = false;
      if (nrows > 0) store_tile<MODE, F16>(p, tb, wrow0, nrows, c.n0, stg, lane, over);
      if (F16 && over) atomicOr(p.status, MOE_DEV_RANGE);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(tempty0 + 8 * acc);   // accumulator free again
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

// ------------------------------------------------------------------- host
template <int MODE, bool F16>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, int grid, cudaStream_t s) {
  cudaError_t err = set_smem_once<tc_grouped_gemm<MODE, F16>>(kSmemBytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_grouped_gemm<MODE, F16>, dim3(grid), dim3(kThreads), kSmemBytes, s, ma, mb, p);
}

template <bool F16>
cudaError_t launch_layers(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                          const void* w2, void* h, void* yp, uint32_t* status, int sms, cudaStream_t s,
                          const CombineOut* comb, int e_mod) {
  const int EW = e_mod > 0 ? e_mod : c.E;   // experts whose weights are given
  const uint64_t rows = (uint64_t)c.T * (uint64_t)c.k;
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const long long mt_max = (long long)(rows / BM) + c.E;
  CUtensorMap ma, mb;
  cudaError_t err;

  // layer 1: h = act(xp W1[e]^T)
  if (!make_map(&ma, xp, rows, (uint64_t)c.d, false) || !make_map(&mb, w1, (uint64_t)EW * F1, (uint64_t)c.d, false))
    return cudaErrorInvalidValue;
  Params p1{offsets, h, c.E, c.d, c.F, F1, c.F, (int)rows, status};
  p1.e_mod = e_mod;
  if (c.act == MOE_ACT_SWIGLU) {
    const long long nt = (c.F + BN / 2 - 1) / (BN / 2);
    err = launch_one<kSwiglu, F16>(ma, mb, p1, (int)std::min<long long>(mt_max * nt, sms), s);
  } else {
    const long long nt = (c.F + BN - 1) / BN;
    err = launch_one<kRelu, F16>(ma, mb, p1, (int)std::min<long long>(mt_max * nt, sms), s);
  }
  if (err != cudaSuccess) return err;

  // layer 2: yp = h W2[e]^T, kept in fp32 so that the combine adds unrounded
  // expert outputs
  if (!make_map(&ma, h, rows, (uint64_t)c.F, F16) || !make_map(&mb, w2, (uint64_t)EW * c.d, (uint64_t)c.F, F16))
    return cudaErrorInvalidValue;
  Params p2{offsets, yp, c.E, c.F, c.d, c.d, 0, (int)rows, status};
  p2.e_mod = e_mod;
  const long long nt2 = (c.d + BN - 1) / BN;
  const int g2 = (int)std::min<long long>(mt_max * nt2, sms);
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

cudaError_t launch_grouped_plain_tc(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
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
  const long long tiles = ((long long)rows_alloc / BM + c.E) * ((Nout + BN - 1) / BN);
  const int grid = (int)std::min<long long>(tiles, di.sms);
  // kPlain takes the hidden type's operands: fp16 when F16
  return f16 ? launch_one<kPlain, true>(ma, mb, p, grid, s) : launch_one<kPlain, false>(ma, mb, p, grid, s);
}

cudaError_t launch_expert_ffn_tc(const moe_config& c, const void* xp, const int32_t* offsets,
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
