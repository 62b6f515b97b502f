// Steps 1-2 on the tensor cores for the bf16 layer: the gate GEMM as one
// tcgen05 tile of 128 tokens x E experts per CTA, followed by the gating
// epilogue (normalisation, softmax, top-k, renormalised weights, near-tie
// gap) on the token rows of logits.
//
// Gate: one fully-connected layer z = x W_gate^T (+ b) (FastMoE announcement,
// "特色二"); the gating network activates the k best experts of each input
// (FastMoE announcement, "1. MoE 设计" and "图4").  Normalisation
// (Skywork-MoE release, "Gating Logits归一化操作"; slides, slide 6):
// z_hat = lambda (z - mean) / std over the experts, population std, zero
// spread -> 0.  Equal scores: the lower expert index wins; a NaN or -inf
// score is never selected (a token with NaN logits keeps empty slots).
//
// Layout: x [T, d] and W_gate [E, d] are K-major bf16 and go through TMA
// (128-byte swizzle) into a ring of up to 8 stages (enough for the whole
// d = 512 reduction to be in flight at once); tcgen05.mma kind::f16 with
// M = 128, N = E rounded up to 16 (rows of W_gate past E load as zeros)
// accumulates the 128 x N logits in fp32 in TMEM.  The epilogue copies them to
// shared memory and gives every token four threads, each owning a quarter
// of the experts: partial sums, maxima and top-(k+1) lists are merged through
// shared memory in quarter order.  Each routing chunk of 128 tokens (one
// CTA, or one cluster below) also writes the chunk's per-expert histogram,
// per-expert sum of softmax probabilities
// (summed in a fixed order), near-tie count and sum of squared
// log-partitions (the router z-loss, Megatron-Core best-practice page,
// "Megatron-Core MoE的关键特性") for the permutation step.
//
// A small batch would leave most SMs idle and each chunk's loads and gating
// to one SM (decode: one chunk, d = 2048).  There the model width is cut into
// up to 8 slices, one CTA each, and a chunk's slices run as one thread-block
// cluster: each keeps its partial logits in its own shared memory, and each
// CTA adds its share of the chunk's rows over the slices, in slice order,
// through distributed shared memory.  It then gates those rows itself, one
// warp per token: butterfly reductions for the row statistics and k + 1
// rounds of a warp-wide arg-max (shuffles) for the top-(k+1).  The CTAs'
// histograms and sums meet in CTA 0, added in slice order.  The CTAs of a
// cluster are co-scheduled, so the two cluster barriers cannot stall.
#include "tc_ptx.cuh"

#include <math.h>

namespace moe {
namespace {

using namespace tc;

constexpr int RM = 128;            // tokens per CTA = routing chunk
constexpr int RK = 64;             // model-width slice per stage (128 bytes of bf16)
constexpr int kMaxStages = 8;
constexpr int kRingBytes = 192 * 1024;
constexpr int kSplit = 4;          // threads per token in the epilogue, each owning a quarter of the experts
constexpr int kThreads = RM * kSplit;
constexpr int kMaxKeep = 9;        // top-(k+1) list length for k <= 8
constexpr int kMaxKSlices = 8;     // CTAs that may share one chunk's model width
constexpr int kKSliceMaxChunks = 74;           // only batches of at most this many chunks split
static_assert(RM == kChunk, "one CTA per routing chunk");

struct RTail {
  unsigned long long full[kMaxStages], empty[kMaxStages], done;
  uint32_t tmem_base;
  int abort_flag;
  int ntie;
  int hist[kMaxExperts];
  float bias[kMaxExperts];
  float part[kSplit][4][RM];       // per quarter: sum, squares, max, exp-sum of each row
  float zrow[RM];                  // squared log-partition of each row (router z-loss)
};

// The top lists of quarters 1..3 of each row: (score, expert) pairs.  They
// live in the stage ring after the logits when there is room (the ring is
// free by then), else after the tail.
struct RLists {
  float v[kSplit - 1][kMaxKeep][RM];
  int i[kSplit - 1][kMaxKeep][RM];
};

__host__ __device__ constexpr int stage_bytes(int EP) { return RM * RK * 2 + EP * RK * 2; }
inline int num_stages(int EP) { return std::min(kMaxStages, kRingBytes / stage_bytes(EP)); }
inline size_t logits_bytes(int E) { return ((size_t)RM * (size_t)(E | 1) * sizeof(float) + 15) & ~(size_t)15; }
inline bool lists_in_ring(int E, int EP) {
  return logits_bytes(E) + sizeof(RLists) <= (size_t)num_stages(EP) * stage_bytes(EP);
}
// byte offset of the lists from the 1024-aligned base of shared memory
inline size_t lists_offset(int E, int EP) {
  return lists_in_ring(E, EP) ? logits_bytes(E) : (size_t)num_stages(EP) * stage_bytes(EP) + sizeof(RTail);
}
inline size_t smem_bytes(int E, int EP) {
  return 1024 + (size_t)num_stages(EP) * stage_bytes(EP) + sizeof(RTail) + (lists_in_ring(E, EP) ? 0 : sizeof(RLists));
}
__host__ __device__ constexpr uint32_t tmem_cols(int EP) { return EP <= 32 ? 32 : EP <= 64 ? 64 : EP <= 128 ? 128 : 256; }

// Keeps the N <= KB + 1 best (score, expert) pairs, best first, in registers
// (every index is a compile-time constant).  Pairs arrive in ascending expert
// order, so a new pair goes behind every kept pair whose score is >= its own:
// equal scores stay in ascending index order.  Empty slots hold -inf, so a
// NaN or -inf score is never kept.  The insertion is branch-free: slot j only
// looks at the old contents of slots j - 1 and j.
template <int KB>
struct TopList {
  static constexpr int kEmpty = 0x7fffffff;
  float v[KB + 1];
  int i[KB + 1];
  __device__ __forceinline__ void init() {
#pragma unroll
    for (int j = 0; j <= KB; ++j) { v[j] = -INFINITY; i[j] = kEmpty; }
  }
  template <int N>
  __device__ __forceinline__ void insert(float s, int e) {
#pragma unroll
    for (int j = N - 1; j >= 1; --j) {
      const bool up = s > v[j - 1];            // s ranks above slot j - 1: slot j takes j - 1
      const bool here = !up && s > v[j];       // s lands in slot j
      v[j] = up ? v[j - 1] : (here ? s : v[j]);
      i[j] = up ? i[j - 1] : (here ? e : i[j]);
    }
    const bool top = s > v[0];
    v[0] = top ? s : v[0];
    i[0] = top ? e : i[0];
  }
};

// Top-N over the scores Z[lo, hi) of one row (and their maximum); a later
// quarter's list is merged in by inserting its pairs best first: its experts
// all have higher indices, so lowest-index-wins order is kept.
template <int N, int KB>
__device__ __forceinline__ float topk_range(TopList<KB>& top, const float* Z, int lo, int hi) {
  float mh = -INFINITY;
#pragma unroll 4
  for (int e = lo; e < hi; ++e) {
    const float sc = Z[e];
    mh = fmaxf(mh, sc);
    top.template insert<N>(sc, e);
  }
  return mh;
}
template <int N, int KB>
__device__ __forceinline__ void topk_merge(TopList<KB>& top, const float (*lv)[RM], const int (*li)[RM], int row) {
  // the later list is sorted best first and its experts all have higher
  // indices: once a pair fails to beat the kept N-th score (strictly), so do
  // all after it
#pragma unroll
  for (int j = 0; j < N; ++j) {
    const float sc = lv[j][row];
    if (!(sc > top.v[N - 1])) break;
    top.template insert<N>(sc, li[j][row]);
  }
}

// Score the top-k is taken on: the biased logit, or its normalised value
// (zero spread -> 0; a NaN spread, from a NaN logit, leaves NaN scores).
__device__ __forceinline__ float gate_score(float zb, float lam, float mu, float sd) {
  return lam > 0.f ? (sd == 0.f ? 0.f : lam * (zb - mu) / sd) : zb;
}

// The partial results of each CTA of a cluster, gathered in CTA 0 (they live
// where the quarter lists would: the split epilogue has none).
struct RSlots {
  float psum[kMaxKSlices][kMaxExperts];
  int hist[kMaxKSlices][kMaxExperts];
  int ntie[kMaxKSlices];
  float zsum[kMaxKSlices];
};
static_assert(sizeof(RSlots) <= sizeof(RLists), "the slots reuse the lists' space");

// One warp gates one token row Z[0, E) (biased logits, in shared memory) on
// its own: lane l owns experts l, l + 32, ...  Mean, spread and the softmax
// sum are butterfly reductions (every lane ends with the same value); the
// top-(k+1) comes from k + 1 rounds of a warp-wide arg-max over the lanes'
// sorted local lists, ordered by score and then by the lower index, so the
// lowest index wins equal scores, and the first round's winner is the row's
// maximum.  Afterwards Z holds the row's softmax probabilities (zeros for an
// invalid row); lane j < k writes slot j.
template <int KB>
__device__ __forceinline__ void gate_row_warp(float* Z, int E, float lam, int t, bool valid, int lane,
                                              int32_t* __restrict__ topk_idx, float* __restrict__ topk_w,
                                              float* __restrict__ gap_out, int* hist, int* ntie, float* zrow,
                                              uint32_t* status) {
  constexpr int k = KB;
  if (lam > 0.f) {   // z_hat = lambda (z - mean) / std, written over z
    float s = 0.f;
    for (int e = lane; e < E; e += 32) s += Z[e];
    const float mu = warp_sum(s) / (float)E;
    float qq = 0.f;
    for (int e = lane; e < E; e += 32) {
      const float dv = Z[e] - mu;
      qq += dv * dv;
    }
    const float sd = sqrtf(warp_sum(qq) / (float)E);
    for (int e = lane; e < E; e += 32) Z[e] = gate_score(Z[e], lam, mu, sd);
  }
  TopList<KB> top;
  top.init();
  for (int e = lane; e < E; e += 32) top.template insert<KB + 1>(Z[e], e);
  // k + 1 rounds: the best head of the 32 local lists, then its owner pops it
  float wv[KB + 1];
  int wi[KB + 1];
#pragma unroll
  for (int r = 0; r <= KB; ++r) {
    float cv = top.v[0];
    int ci = top.i[0];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float ov = __shfl_xor_sync(0xffffffffu, cv, o);
      const int oi = __shfl_xor_sync(0xffffffffu, ci, o);
      const bool take = ov > cv || (ov == cv && oi < ci);
      cv = take ? ov : cv;
      ci = take ? oi : ci;
    }
    wv[r] = cv;
    wi[r] = ci;
    const bool pop = top.i[0] == ci;
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      top.v[j] = pop ? top.v[j + 1] : top.v[j];
      top.i[j] = pop ? top.i[j + 1] : top.i[j];
    }
    top.v[KB] = pop ? -INFINITY : top.v[KB];
    top.i[KB] = pop ? TopList<KB>::kEmpty : top.i[KB];
  }
  // the first winner is the row's largest score (-inf when no score is a
  // number above -inf, as the maximum over the row would be)
  const float m = wv[0];
  float Sh = 0.f;
  for (int e = lane; e < E; e += 32) {   // unnormalised probabilities over the scores
    const float pe = __expf(Z[e] - m);
    Z[e] = pe;
    Sh += pe;
  }
  const float S = warp_sum(Sh);
  const float invS = 1.f / S;
  float psel[KB], sel = 0.f;
#pragma unroll
  for (int j = 0; j < KB; ++j) {
    psel[j] = __expf(wv[j] - m) * invS;
    sel += psel[j];                     // slot order
  }
  const float rs = 1.f / sel;
  const float gap = (k < E) ? wv[k - 1] - wv[k] : INFINITY;
  if (valid) {
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      if (lane == j) {
        topk_idx[(size_t)t * k + j] = wi[j];
        topk_w[(size_t)t * k + j] = psel[j] * rs;
        // a row with fewer than k scores above -inf (NaN logits) keeps empty
        // slots: out of range, dropped by the permutation, and flagged
        if ((unsigned)wi[j] < (unsigned)E) atomicAdd(&hist[wi[j]], 1);
        else atomicOr(status, MOE_DEV_BOUNDS);
      }
    }
    if (lane == 0) {
      gap_out[t] = gap;
      if (gap < MOE_NEAR_TIE_GAP) atomicAdd(ntie, 1);
    }
  }
  if (lane == 0) {
    const float lse = m + logf(S);   // log sum_e exp(score): the router z-loss term of this row
    *zrow = valid ? lse * lse : 0.f;
  }
  for (int e = lane; e < E; e += 32) Z[e] = valid ? Z[e] * invS : 0.f;
}

// KB is the exact number of experts per token, so that every index into the
// top-k registers is a compile-time constant.  SPLIT: the chunk's model width
// is cut over a cluster of nks > 1 CTAs (a separate instantiation, so the
// unsplit kernel carries none of the exchange's registers).
template <int KB, bool SPLIT>
__global__ void __launch_bounds__(kThreads, 1)
route_tc_kernel(const __grid_constant__ CUtensorMap tmX, const __grid_constant__ CUtensorMap tmW,
                const float* __restrict__ bg, int T, int d, int E, int EP, int nst, float lam,
                int32_t* __restrict__ topk_idx, float* __restrict__ topk_w, float* __restrict__ gap_out,
                int32_t* __restrict__ hist_out, float* __restrict__ psum_out, int32_t* __restrict__ ntie_out,
                float* __restrict__ zsum_out, int nch, uint32_t* __restrict__ status, int lists_off, int nks) {
  constexpr int k = KB;
  extern __shared__ __align__(1024) unsigned char smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  unsigned char* sbase = smem_raw + (base - raw);
  const int SB = stage_bytes(EP);
  RTail* tail = reinterpret_cast<RTail*>(sbase + (size_t)nst * SB);
  RLists* lists = reinterpret_cast<RLists*>(sbase + lists_off);
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int chunk = blockIdx.x / nks, ks = blockIdx.x - chunk * nks, t0 = chunk * RM;
  const int nkb_all = (d + RK - 1) / RK;   // the host keeps nks <= nkb_all
  const int kb0 = (nkb_all * ks) / nks, nkb = (nkb_all * (ks + 1)) / nks - kb0;
  const uint32_t full0 = smem_u32(&tail->full[0]), empty0 = smem_u32(&tail->empty[0]);
  const uint32_t done = smem_u32(&tail->done);
  const volatile int* abort_flag = &tail->abort_flag;
  const uint32_t ncols = tmem_cols(EP);

  if (tid == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(full0 + 8 * s, 1);
      mbar_init(empty0 + 8 * s, 1);
    }
    mbar_init(done, 1);
    tail->abort_flag = 0;
    tail->ntie = 0;
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  for (int e = tid; e < E; e += kThreads) tail->hist[e] = 0;
  if (warp == 1) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;"
                 ::"r"(smem_u32(&tail->tmem_base)), "r"(ncols) : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
  }
  if (warp == 0 && lane == 0) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmX)) : "memory");
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(&tmW)) : "memory");
  }
  pdl_wait();                  // x, W_gate and b may come from the previous kernel
  pdl_launch_dependents();
  for (int e = tid; e < E; e += kThreads) tail->bias[e] = (bg != nullptr) ? bg[e] : 0.f;
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = tail->tmem_base;

  // ------------------------------------------------- gate GEMM main loop
  if (warp == 0 && lane == 0) {
    int issued = 0;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % nst;
      const uint32_t ph = (uint32_t)(kb / nst) & 1u;
      if (!mbar_wait(empty0 + 8 * s, ph ^ 1u, abort_flag, kWaitNs)) {
        atomicOr(status, MOE_DEV_TIMEOUT);
        tail->abort_flag = 1;
        break;
      }
      const uint32_t sa = base + (uint32_t)(s * SB);
      mbar_expect_tx(full0 + 8 * s, (uint32_t)SB);
      tma_load_2d(sa, &tmX, full0 + 8 * s, (kb0 + kb) * RK, t0);
      tma_load_2d(sa + RM * RK * 2, &tmW, full0 + 8 * s, (kb0 + kb) * RK, 0);
      ++issued;
    }
    for (int i = max(0, issued - nst); i < issued; ++i)   // loads still in flight
      mbar_wait(full0 + 8 * (i % nst), (uint32_t)(i / nst) & 1u, nullptr, kDrainNs);
  } else if (warp == 1 && lane == 0) {
    const uint32_t idesc = idesc_f16kind(RM, EP, false);
    bool ok = true;
    for (int kb = 0; kb < nkb; ++kb) {
      const int s = kb % nst;
      const uint32_t ph = (uint32_t)(kb / nst) & 1u;
      if (!mbar_wait(full0 + 8 * s, ph, abort_flag, kWaitNs)) { ok = false; break; }
      tc_fence_after();
      const uint32_t sa = base + (uint32_t)(s * SB);
      const uint64_t ad = sdesc(sa), bd = sdesc(sa + RM * RK * 2);
#pragma unroll
      for (int kk = 0; kk < RK / 16; ++kk)
        tc_mma(tmem, ad + (uint64_t)(2 * kk), bd + (uint64_t)(2 * kk), idesc, (kb | kk) != 0);
      tc_commit(empty0 + 8 * s);
    }
    if (!ok) {
      atomicOr(status, MOE_DEV_TIMEOUT);
      tail->abort_flag = 1;
    }
    tc_commit(done);   // arrives once every MMA above has completed
  }
  __syncwarp();
  bool ok = mbar_wait(done, 0, nullptr, kWaitNs) && !*abort_flag;
  ok = __all_sync(0xffffffffu, ok);
  tc_fence_after();

  // ------------------------------------------------- gating epilogue
  // The logits of each row go from TMEM to a padded shared-memory row (the
  // stage ring is free now; the odd row stride keeps a warp's column accesses
  // conflict-free).  Warps q, q + 4, q + 8 and q + 12 read the same TMEM lanes
  // 32q..32q+31: quarter p (= warp / 4) owns experts [E p / 4, E (p + 1) / 4).
  // Partial sums, maxima and top lists of the four quarters meet in shared
  // memory, always combined in quarter order.
  const int q = warp & 3, qtr = warp >> 2;
  const int row = q * 32 + lane;
  const int t = t0 + row;
  const bool valid = ok && t < T;
  const uint32_t tb = tmem + ((uint32_t)(q * 32) << 16);
  const int ldz = E | 1;
  float* Zall = reinterpret_cast<float*>(sbase);   // [RM][ldz]
  float* Z = Zall + (size_t)row * ldz;
  const int nch32 = (E + 31) / 32;
  // a split chunk's rows past the batch are never read: their warps skip the copy
  const int ncopy = (!SPLIT || q * 32 < T - t0) ? nch32 : 0;
  for (int c = qtr; c < ncopy; c += kSplit) {
    uint32_t r[32];
    tmem_ld32(tb + c * 32, r);
    tmem_wait_ld();
#pragma unroll
    for (int i = 0; i < 32; ++i) {
      const int e = c * 32 + i;
      if (e < E) Z[e] = __uint_as_float(r[i]) + (SPLIT ? 0.f : tail->bias[e]);
    }
  }
  tc_fence_before();
  __syncthreads();
  if constexpr (SPLIT) {
    // The chunk's slices are one thread-block cluster, each slice's partial
    // logits in its own shared memory.  CTA ks sums rows [r0, r1) of the
    // chunk's real tokens over the slices, in slice order, adds the bias,
    // keeps them in its own rows and gates them, one warp per row.  Its
    // histogram, probability sums, near-tie count and z-loss sum go into CTA
    // 0's slots, which CTA 0 adds in slice order.
    cluster_sync();   // every slice's partials are written
    const int nrows = min(RM, T - t0);
    const int r0 = (nrows * ks) / nks, r1 = (nrows * (ks + 1)) / nks;
    uint32_t zsl[kMaxKSlices];   // Zall in each slice's shared memory
#pragma unroll
    for (int sl = 0; sl < kMaxKSlices; ++sl) zsl[sl] = sl < nks ? cluster_addr(smem_u32(Zall), (uint32_t)sl) : 0u;
    // up to four elements per pass, all their loads issued before the first sum
    constexpr int kU = 4;
    const int nel = (r1 - r0) * E;
    for (int i0 = tid; i0 < nel; i0 += kU * kThreads) {
      float v[kU][kMaxKSlices];
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * kThreads;
        const int rr = i / E, e = i - rr * E;
        const uint32_t off = (uint32_t)(((r0 + rr) * ldz + e) * 4);
#pragma unroll
        for (int sl = 0; sl < kMaxKSlices; ++sl) v[u][sl] = (sl < nks && i < nel) ? ld_cluster_f32(zsl[sl] + off) : 0.f;
      }
#pragma unroll
      for (int u = 0; u < kU; ++u) {
        const int i = i0 + u * kThreads;
        if (i >= nel) break;
        const int rr = i / E, e = i - rr * E;
        float z = 0.f;
#pragma unroll
        for (int sl = 0; sl < kMaxKSlices; ++sl)
          if (sl < nks) z += v[u][sl];
        Zall[(size_t)(r0 + rr) * ldz + e] = z + tail->bias[e];   // a row only this CTA reads
      }
    }
    __syncthreads();
    for (int r = r0 + warp; r < r1; r += kThreads / 32)
      gate_row_warp<KB>(Zall + (size_t)r * ldz, E, lam, t0 + r, ok, lane, topk_idx, topk_w, gap_out, tail->hist,
                        &tail->ntie, &tail->zrow[r], status);
    __syncthreads();
    // this CTA's probability sums over its rows: nG groups of rows, the group
    // partials added in group order
    float* colpart = &tail->part[0][0][0];
    const int nG = kThreads / E;
    const int R = (r1 - r0 + nG - 1) / nG;
    if (tid < nG * E) {
      const int e = tid % E, g = tid / E;
      float sum = 0.f;
      const int ra = r0 + g * R, rb = min(r1, ra + R);
      for (int rr = ra; rr < rb; ++rr) sum += Zall[(size_t)rr * ldz + e];
      colpart[g * E + e] = sum;
    }
    __syncthreads();
    RSlots* slots = reinterpret_cast<RSlots*>(lists);
    for (int e = tid; e < E; e += kThreads) {
      float sum = 0.f;
      for (int g = 0; g < nG; ++g) sum += colpart[g * E + e];
      st_cluster_f32(cluster_addr(smem_u32(&slots->psum[ks][e]), 0), sum);
      st_cluster_u32(cluster_addr(smem_u32(&slots->hist[ks][e]), 0), (uint32_t)tail->hist[e]);
    }
    if (warp == 0) {   // the z-loss sum of this CTA's rows, in a fixed order
      float z = 0.f;
      for (int r = r0 + lane; r < r1; r += 32) z += tail->zrow[r];
      z = warp_sum(z);
      if (lane == 0) {
        st_cluster_f32(cluster_addr(smem_u32(&slots->zsum[ks]), 0), z);
        st_cluster_u32(cluster_addr(smem_u32(&slots->ntie[ks]), 0), (uint32_t)tail->ntie);
      }
    }
    cluster_sync();   // the slots of CTA 0 are filled; no CTA touches a peer's memory any more
    if (ks == 0) {
      for (int e = tid; e < E; e += kThreads) {
        float ps = 0.f;
        int hs = 0;
        for (int sl = 0; sl < nks; ++sl) {
          ps += slots->psum[sl][e];
          hs += slots->hist[sl][e];
        }
        psum_out[(size_t)chunk * E + e] = ps;
        hist_out[(size_t)e * nch + chunk] = hs;
      }
      if (tid == 0) {
        float z = 0.f;
        int nt = 0;
        for (int sl = 0; sl < nks; ++sl) {
          z += slots->zsum[sl];
          nt += slots->ntie[sl];
        }
        zsum_out[chunk] = z;
        ntie_out[chunk] = nt;
      }
    }
  }
  constexpr bool lead = !SPLIT;   // the quarter epilogue: this CTA gates the whole chunk
  if (lead) {
    const int lo = (E * qtr) / kSplit, hi = (E * (qtr + 1)) / kSplit;
    float (*part)[4][RM] = tail->part;
    if (lam > 0.f) {   // z_hat = lambda (z - mean) / std, written over z
      float s = 0.f;
#pragma unroll 4
      for (int e = lo; e < hi; ++e) s += Z[e];
      part[qtr][0][row] = s;
      __syncthreads();
      const float mu = (((part[0][0][row] + part[1][0][row]) + part[2][0][row]) + part[3][0][row]) / (float)E;
      float qq = 0.f;
#pragma unroll 4
      for (int e = lo; e < hi; ++e) {
        const float dv = Z[e] - mu;
        qq += dv * dv;
      }
      part[qtr][1][row] = qq;
      __syncthreads();
      const float sd =
          sqrtf((((part[0][1][row] + part[1][1][row]) + part[2][1][row]) + part[3][1][row]) / (float)E);
#pragma unroll 4
      for (int e = lo; e < hi; ++e) Z[e] = gate_score(Z[e], lam, mu, sd);
    }
    // the (k+1)-th score is only needed for the gap, which does not exist when k == E
    TopList<KB> top;
    top.init();
    const float mh = (k < E) ? topk_range<KB + 1>(top, Z, lo, hi) : topk_range<KB>(top, Z, lo, hi);
    part[qtr][2][row] = mh;
    if (qtr > 0) {
#pragma unroll
      for (int j = 0; j <= KB; ++j) {
        lists->v[qtr - 1][j][row] = top.v[j];
        lists->i[qtr - 1][j][row] = top.i[j];
      }
    }
    __syncthreads();
    const float m = fmaxf(fmaxf(part[0][2][row], part[1][2][row]), fmaxf(part[2][2][row], part[3][2][row]));
    float Sh = 0.f;
#pragma unroll 4
    for (int e = lo; e < hi; ++e) {   // unnormalised probabilities over the scores
      const float pe = __expf(Z[e] - m);
      Z[e] = pe;
      Sh += pe;
    }
    part[qtr][3][row] = Sh;
    __syncthreads();
    const float S = ((part[0][3][row] + part[1][3][row]) + part[2][3][row]) + part[3][3][row];
    const float invS = 1.f / S;
    if (qtr == 0) {
      const float lse = m + logf(S);   // log sum_e exp(score): the router z-loss term of this row
      tail->zrow[row] = valid ? lse * lse : 0.f;
      // the other quarters' lists, in quarter order: their experts all have
      // higher indices, so inserting them keeps lowest-index-wins order
#pragma unroll
      for (int p = 0; p < kSplit - 1; ++p) {
        if (k < E) topk_merge<KB + 1>(top, lists->v[p], lists->i[p], row);
        else topk_merge<KB>(top, lists->v[p], lists->i[p], row);
      }
      float psel[KB], sel = 0.f;
#pragma unroll
      for (int j = 0; j < KB; ++j) {
        psel[j] = __expf(top.v[j] - m) * invS;
        sel += psel[j];                     // slot order
      }
      const float rs = 1.f / sel;
      const float gap = (k < E) ? top.v[k - 1] - top.v[k] : INFINITY;
      if (valid) {
#pragma unroll
        for (int j = 0; j < KB; ++j) {
          topk_idx[(size_t)t * k + j] = top.i[j];
          topk_w[(size_t)t * k + j] = psel[j] * rs;
          // a row with fewer than k scores above -inf (NaN logits) keeps empty
          // slots: out of range, dropped by the permutation, and flagged
          if ((unsigned)top.i[j] < (unsigned)E) atomicAdd(&tail->hist[top.i[j]], 1);
          else atomicOr(status, MOE_DEV_BOUNDS);
        }
        gap_out[t] = gap;
        if (gap < MOE_NEAR_TIE_GAP) atomicAdd(&tail->ntie, 1);
      }
    }

    // per-expert probability sums of the chunk: the probabilities of each row in
    // shared memory, columns summed by nG groups of threads over row ranges, the
    // group partials added in group order (fixed order, deterministic)
#pragma unroll 4
    for (int e = lo; e < hi; ++e) Z[e] = valid ? Z[e] * invS : 0.f;
    tc_fence_before();
    __syncthreads();
    float* colpart = &part[0][0][0];               // [nG][E]; part is free again
    const int nG = kThreads / E;                   // >= 1 since E <= 256 = kThreads
    const int R = (RM + nG - 1) / nG;
    if (tid < nG * E) {
      const int e = tid % E, g = tid / E;
      float s = 0.f;
      const int r1 = min(RM, (g + 1) * R);
      for (int rr = g * R; rr < r1; ++rr) s += Zall[(size_t)rr * ldz + e];
      colpart[g * E + e] = s;
    }
    __syncthreads();
    for (int e = tid; e < E; e += kThreads) {
      float s = 0.f;
      for (int g = 0; g < nG; ++g) s += colpart[g * E + e];
      psum_out[(size_t)chunk * E + e] = s;
      hist_out[(size_t)e * nch + chunk] = tail->hist[e];
    }
    if (tid == 0) ntie_out[chunk] = tail->ntie;
    if (warp == 0) {   // the chunk's z-loss sum, in a fixed order
      float z = ((tail->zrow[lane] + tail->zrow[lane + 32]) + tail->zrow[lane + 64]) + tail->zrow[lane + 96];
      z = warp_sum(z);
      if (lane == 0) zsum_out[chunk] = z;
    }
  }   // lead
  if (warp == 1) {
    tc_fence_after();
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(tmem), "r"(ncols) : "memory");
  }
}

// Slices of the model width per chunk: doubled while the reduction takes more
// than one round of the stage ring, each slice keeps at least half a ring of
// k-blocks and the grid stays within one CTA per SM; only batches of at most
// 74 chunks split.  A chunk's slices form one cluster of at most 8 CTAs, and
// each CTA gates its share of the chunk's rows.  (Splitting the FastMoE
// layer's one-ring reduction over pairs made its route 8 us slower and its
// forward 14 us slower.)
int kslices(const moe_config& c, long long sms) {
  const int EP = ((c.E + 15) / 16) * 16;
  const int nch = num_chunks(c.T), nkb = (c.d + RK - 1) / RK, nst = num_stages(EP);
  if (nkb <= nst || nch > kKSliceMaxChunks) return 1;
  int n = 1;
  while (n < kMaxKSlices && (long long)nch * n * 2 <= sms && nkb / (n * 2) >= nst / 2) n *= 2;
  return n;
}

template <int KB, bool SPLIT>
cudaError_t launch_ks(const moe_config& c, const CUtensorMap& mx, const CUtensorMap& mw, int EP, const float* bg,
                      int32_t* idx, float* w, float* gap, int32_t* hist, float* psum, int32_t* ntie,
                      float* zsum, uint32_t* status, int nks, cudaStream_t s) {
  // the most any E <= kMaxExperts needs, so one attribute serves every launch
  static const size_t kMaxSmem = [] {
    size_t m = 0;
    for (int e = 1; e <= kMaxExperts; ++e) m = std::max(m, smem_bytes(e, ((e + 15) / 16) * 16));
    return m;
  }();
  cudaError_t err = set_smem_once<route_tc_kernel<KB, SPLIT>>(kMaxSmem);
  if (err != cudaSuccess) return err;
  const int nch = num_chunks(c.T);
  // PDL, and a chunk's slices as one cluster (nks consecutive CTAs)
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(nch * nks);
  cfg.blockDim = dim3(kThreads);
  cfg.dynamicSmemBytes = smem_bytes(c.E, EP);
  cfg.stream = s;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = (unsigned)nks;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 2;
  return cudaLaunchKernelEx(&cfg, route_tc_kernel<KB, SPLIT>, mx, mw, bg, c.T, c.d, c.E, EP, num_stages(EP),
                            c.lambda, idx, w, gap, hist, psum, ntie, zsum, nch, status, (int)lists_offset(c.E, EP),
                            nks);
}

template <int KB>
cudaError_t launch_kb(const moe_config& c, const CUtensorMap& mx, const CUtensorMap& mw, int EP, const float* bg,
                      int32_t* idx, float* w, float* gap, int32_t* hist, float* psum, int32_t* ntie,
                      float* zsum, uint32_t* status, cudaStream_t s) {
  DeviceInfo di;
  cudaError_t err = device_info(&di);
  if (err != cudaSuccess) return err;
  const int nks = kslices(c, di.sms);
  return nks > 1 ? launch_ks<KB, true>(c, mx, mw, EP, bg, idx, w, gap, hist, psum, ntie, zsum, status, nks, s)
                 : launch_ks<KB, false>(c, mx, mw, EP, bg, idx, w, gap, hist, psum, ntie, zsum, status, 1, s);
}

}  // namespace

bool route_tc_supported(const moe_config& c) { return c.dtype == MOE_DTYPE_BF16 && c.k <= 8; }

cudaError_t launch_route_tc(const moe_config& c, const void* x, const void* wg, const float* bg,
                            int32_t* topk_idx, float* topk_w, float* gap, int32_t* hist, float* psum,
                            int32_t* ntie, float* zsum, uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  const int EP = ((c.E + 15) / 16) * 16;
  CUtensorMap mx, mw;
  if (!make_map(&mx, x, (uint64_t)c.T, (uint64_t)c.d, false, RM) ||
      !make_map(&mw, wg, (uint64_t)c.E, (uint64_t)c.d, false, (uint32_t)EP))
    return cudaErrorInvalidValue;
#define MOE_ROUTE_K(K) \
  case K: return launch_kb<K>(c, mx, mw, EP, bg, topk_idx, topk_w, gap, hist, psum, ntie, zsum, status, s)
  switch (c.k) {
    MOE_ROUTE_K(1); MOE_ROUTE_K(2); MOE_ROUTE_K(3); MOE_ROUTE_K(4);
    MOE_ROUTE_K(5); MOE_ROUTE_K(6); MOE_ROUTE_K(7); MOE_ROUTE_K(8);
    default: return cudaErrorInvalidValue;
  }
#undef MOE_ROUTE_K
}

}  // namespace moe
