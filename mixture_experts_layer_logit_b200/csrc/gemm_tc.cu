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
//     K-major bf16, staged by TMA (128-byte swizzle) into a STAGES-deep ring.
//   * warp 0 lane 0 issues the TMA loads, warp 1 lane 0 issues
//     tcgen05.mma.cta_group::1.kind::f16 (128 x 256 x 16, fp32 accumulators in
//     TMEM), warps 2-5 drain TMEM with tcgen05.ld, apply the activation
//     (ReLU, or silu(gate) * up for SwiGLU) and store bf16 rows.
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
#include "tc_ptx.cuh"

namespace moe {
namespace {

using namespace tc;

constexpr int BM = 128, BN = 256, BK = 64;
constexpr int STAGES = 4;
constexpr int A_BYTES = BM * BK * 2;              // 16 KB
constexpr int B_BYTES = BN * BK * 2;              // 32 KB
constexpr int STAGE_BYTES = A_BYTES + B_BYTES;    // 48 KB
constexpr int kThreads = 192;
constexpr uint32_t kTmemCols = 512;
enum { kPlain = 0, kRelu = 1, kSwiglu = 2 };


struct Tail {
  unsigned long long full[STAGES], empty[STAGES], tfull[2], tempty[2], drain;
  uint32_t tmem_base;
  int abort_flag;
  int tstart[kMaxExperts + 1];
  int seg[kMaxExperts + 1];     // copy of offsets[]: tiles are decoded without global loads
};
// Epilogue staging: each epilogue warp turns its 32 rows x 128 bytes of output
// around in shared memory so that the global stores write whole 128-byte lines.
constexpr int kStageWarpBytes = 32 * 128;
constexpr size_t kStagingBytes = 4 * kStageWarpBytes;
constexpr size_t kSmemBytes = 1024 + (size_t)STAGES * STAGE_BYTES + kStagingBytes + sizeof(Tail);

struct Params {
  const int32_t* offsets;
  void* out;            // [rows][Nout]: bf16 h (layer 1) or fp32 yp (layer 2)
  int E, K, Nout;
  int b_rows;           // B rows per expert
  int up_off;           // SwiGLU: first up row inside an expert's B block
  int rows_alloc;       // rows of the A and output buffers (T*k); stores stop there
  uint32_t* status;
};

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

template <int MODE>
__device__ __forceinline__ TileCoord decode_tile(const int* tstart, const int32_t* offsets, int E, int L) {
  TileCoord c;
  c.e = tile_expert(tstart, E, L);
  const int seg0 = offsets[c.e];
  const int M = offsets[c.e + 1] - seg0;
  const int mt = (M + BM - 1) / BM;
  const int local = L - tstart[c.e];
  const int nti = local / mt, mti = local - nti * mt;
  c.row0 = seg0 + mti * BM;
  c.rows = min(BM, M - mti * BM);
  c.n0 = nti * (MODE == kSwiglu ? BN / 2 : BN);
  return c;
}

// F16: the hidden activation (layer-1 output, layer-2 A operand) and W2 are
// fp16 instead of bf16.
template <int MODE, bool F16>
__global__ void __launch_bounds__(kThreads, 1)
tc_grouped_gemm(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
                const Params p) {
  constexpr uint32_t kIdesc = idesc_f16kind(BM, BN, MODE == kPlain && F16);
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
        const TileCoord c = decode_tile<MODE>(tail->tstart, tail->seg, p.E, L);
        const int b0 = c.e * p.b_rows + c.n0;
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
      const TileCoord c = decode_tile<MODE>(tail->tstart, tail->seg, p.E, L);
      const int acc = tl & 1;
      const uint32_t aph = (uint32_t)(tl >> 1) & 1u;
      ok = mbar_wait(tfull0 + 8 * acc, aph, abort_flag, kWaitNs);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16) + (uint32_t)(acc * BN);
      // rows of this warp that may be stored: inside the segment and the buffers
      const int wrow0 = c.row0 + q * 32;
      int nrows = min(32, c.rows - q * 32);
      if (nrows > 0 && wrow0 + nrows > p.rows_alloc) {   // offsets[] beyond the buffers: skip and flag
        if (lane == 0) atomicOr(p.status, MOE_DEV_BOUNDS);
        nrows = p.rows_alloc - wrow0;
      }
      bool over = false;
      // One block = 128 bytes of output per row: 32 fp32 columns (layer 2) or
      // 64 16-bit hidden columns (layer 1).  Thread `lane` owns TMEM row
      // wrow0 + lane; the block is turned around in shared memory (16-byte
      // chunk i of row r at slot i ^ (r & 7), conflict-free both ways) and
      // written as 4 rows x 128 contiguous bytes per store instruction.
      constexpr int kBlocks = (MODE == kPlain) ? BN / 32 : (MODE == kRelu ? BN / 64 : BN / 128);
      constexpr int kPer16 = (MODE == kPlain) ? 4 : 8;
#pragma unroll 1
      for (int blk = 0; blk < kBlocks; ++blk) {
        uint4 v[8];
        if (MODE == kPlain) {
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
                  a0 = a0 / (1.f + __expf(-a0)) * u0;
                  a1 = a1 / (1.f + __expf(-a1)) * u1;
                }
                pk[j] = pack_hidden<F16>(a0, a1, over);
              }
              v[hf * 4 + i] = make_uint4(pk[0], pk[1], pk[2], pk[3]);
            }
          }
        }
        __syncwarp();
#pragma unroll
        for (int i = 0; i < 8; ++i) stg[lane * 8 + (i ^ (lane & 7))] = v[i];
        __syncwarp();
        const int col0 = c.n0 + blk * 8 * kPer16;
#pragma unroll
        for (int it = 0; it < 8; ++it) {
          const int rr = it * 4 + (lane >> 3), cc = lane & 7;
          const uint4 val = stg[rr * 8 + (cc ^ (rr & 7))];
          const int col = col0 + cc * kPer16;
          if (rr < nrows && col < p.Nout) {
            const size_t off = (size_t)(wrow0 + rr) * p.Nout + col;
            if (MODE == kPlain) *reinterpret_cast<uint4*>(static_cast<float*>(p.out) + off) = val;
            else *reinterpret_cast<uint4*>(static_cast<uint16_t*>(p.out) + off) = val;
          }
        }
      }
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
PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(ptr);
  });
  return fn;
}

// 2-D tensor map over a row-major [rows, cols] matrix of 16-bit elements
// (bf16 or fp16); box = 64 columns (128 bytes) x 128 rows, 128-byte swizzle,
// zero fill outside.
bool make_map(CUtensorMap* m, const void* ptr, uint64_t rows, uint64_t cols, bool f16) {
  auto fn = encode_fn();
  if (fn == nullptr) return false;
  cuuint64_t dims[2] = {cols, rows};
  cuuint64_t strides[1] = {cols * 2};
  cuuint32_t box[2] = {BK, BM};
  cuuint32_t estr[2] = {1, 1};
  return fn(m, f16 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT16 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2,
            const_cast<void*>(ptr), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
            CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

template <int MODE, bool F16>
cudaError_t launch_one(const CUtensorMap& ma, const CUtensorMap& mb, const Params& p, int grid, cudaStream_t s) {
  cudaError_t err = set_smem_once<tc_grouped_gemm<MODE, F16>>(kSmemBytes);
  if (err != cudaSuccess) return err;
  return launch_pdl(tc_grouped_gemm<MODE, F16>, dim3(grid), dim3(kThreads), kSmemBytes, s, ma, mb, p);
}

template <bool F16>
cudaError_t launch_layers(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                          const void* w2, void* h, void* yp, uint32_t* status, int sms, cudaStream_t s) {
  const uint64_t rows = (uint64_t)c.T * (uint64_t)c.k;
  const int F1 = (c.act == MOE_ACT_SWIGLU) ? 2 * c.F : c.F;
  const long long mt_max = (long long)(rows / BM) + c.E;
  CUtensorMap ma, mb;
  cudaError_t err;

  // layer 1: h = act(xp W1[e]^T)
  if (!make_map(&ma, xp, rows, (uint64_t)c.d, false) || !make_map(&mb, w1, (uint64_t)c.E * F1, (uint64_t)c.d, false))
    return cudaErrorInvalidValue;
  Params p1{offsets, h, c.E, c.d, c.F, F1, c.F, (int)rows, status};
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
  if (!make_map(&ma, h, rows, (uint64_t)c.F, F16) || !make_map(&mb, w2, (uint64_t)c.E * c.d, (uint64_t)c.F, F16))
    return cudaErrorInvalidValue;
  Params p2{offsets, yp, c.E, c.F, c.d, c.d, 0, (int)rows, status};
  const long long nt2 = (c.d + BN - 1) / BN;
  return launch_one<kPlain, F16>(ma, mb, p2, (int)std::min<long long>(mt_max * nt2, sms), s);
}

}  // namespace

cudaError_t launch_expert_ffn_tc(const moe_config& c, const void* xp, const int32_t* offsets,
                                 const void* w1, const void* w2, void* h, void* yp,
                                 uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  if (c.hidden_dtype == MOE_DTYPE_F16)
    return launch_layers<true>(c, xp, offsets, w1, w2, h, yp, status, di.sms, s);
  return launch_layers<false>(c, xp, offsets, w1, w2, h, yp, status, di.sms, s);
}

}  // namespace moe
