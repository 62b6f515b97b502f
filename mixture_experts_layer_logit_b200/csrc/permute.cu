// Step 3 of the layer: group the (token, slot) assignments by expert.
//
// Megatron-Core best-practice page, "MoE负载均衡的挑战与应对": experts have a
// capacity; assignments beyond it are dropped and only the residual carries
// them; the dropless variant keeps every assignment.  Priority inside an
// expert is ascending token index, so the result is unique and deterministic:
// positions come from prefix sums, never from atomics (atomics only count).
//
//   hist    : per-chunk expert histogram                       (skipped when the
//             route kernel already wrote it)
//   scan    : one CTA; per-expert exclusive prefix over chunks, counts, kept,
//             offsets, drop statistics and the Switch aux loss
//   scatter : one CTA per chunk; stable rank of every assignment inside its
//             expert from warp ballots, the capacity test, row_of / src_tok,
//             and the 16-byte-vector gather xp[row] = x[token]
#include "tc_ptx.cuh"

#include <math.h>

#include <algorithm>

namespace moe {
namespace {

constexpr unsigned kFull = 0xffffffffu;

// --------------------------------------------------------------------- hist
__global__ void __launch_bounds__(kChunk)
hist_kernel(const int32_t* __restrict__ topk_idx, const float* __restrict__ gap, int T, int E, int k,
            int nch, int32_t* __restrict__ hist, int32_t* __restrict__ ntie, uint32_t* status) {
  __shared__ int sh[kMaxExperts];
  __shared__ int nt;
  for (int e = threadIdx.x; e < E; e += blockDim.x) sh[e] = 0;
  if (threadIdx.x == 0) nt = 0;
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();
  const int t = blockIdx.x * kChunk + threadIdx.x;
  if (t < T) {
    for (int j = 0; j < k; ++j) {
      const int e = topk_idx[(size_t)t * k + j];
      if (e < 0 || e >= E) {
        atomicOr(status, MOE_DEV_BOUNDS);
        continue;
      }
      atomicAdd(&sh[e], 1);
    }
    if (gap != nullptr && gap[t] < MOE_NEAR_TIE_GAP) atomicAdd(&nt, 1);
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += blockDim.x) hist[(size_t)e * nch + blockIdx.x] = sh[e];
  if (threadIdx.x == 0 && ntie != nullptr) ntie[blockIdx.x] = nt;
}

// --------------------------------------------------------------------- scan
constexpr int kScanThreads = 1024;

// Expert totals of one warp's experts: the total over all chunks and the
// prefix over the chunks before `chunk` (hist is expert-major, so a warp reads
// each expert's chunk counts coalesced; four 32-chunk loads are in flight at
// once), and optionally the exclusive chunk offsets.
__device__ __forceinline__ void expert_totals(const int32_t* __restrict__ hist, int e, int nch, int chunk,
                                              int32_t* __restrict__ choff, int lane, int* total, int* prefix) {
  constexpr int kBatch = 4;
  int running = 0, pre = 0;
  const int32_t* hrow = hist + (size_t)e * nch;
  for (int c0 = 0; c0 < nch; c0 += 32 * kBatch) {
    int v[kBatch];
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int c = c0 + 32 * b + lane;
      v[b] = (c < nch) ? hrow[c] : 0;
    }
#pragma unroll
    for (int b = 0; b < kBatch; ++b) {
      const int c = c0 + 32 * b + lane;
      int incl = v[b];
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const int u = __shfl_up_sync(kFull, incl, o);
        if (lane >= o) incl += u;
      }
      if (choff != nullptr && c < nch) choff[(size_t)e * nch + c] = running + incl - v[b];
      if (c < chunk) pre += v[b];
      running += __shfl_sync(kFull, incl, 31);
    }
  }
  *total = running;
  *prefix = warp_sum(pre);
}

// Sum of the per-chunk sums of squared log-partitions (the router z-loss
// numerator) in a fixed order: lanes stride over the chunks in double, then a
// butterfly.  NaN when the route left none.
__device__ __forceinline__ double chunk_zsum(const float* __restrict__ zsum, int nch, int lane) {
  if (zsum == nullptr) return (double)NAN;
  double s = 0.0;
  for (int c = lane; c < nch; c += 32) s += (double)zsum[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
  return s;
}

__device__ __forceinline__ int chunk_ties(const int32_t* __restrict__ ntie, int nch, int lane) {
  int s = 0;
  if (ntie != nullptr)
    for (int c = lane; c < nch; c += 32) s += ntie[c];
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
  return (ntie != nullptr) ? s : -1;
}

// Expert totals for the whole block at once: thread (e, s), s < 8, sums the
// counts of chunks c = s, s + 8, ... of expert e (all its loads independent,
// so one round trip to L2 serves the block), the total and the part before
// `chunk`; the 8 partials of an expert meet by shuffles in a fixed order.
// With want_p it also forms P_e the same way from the per-chunk probability
// sums (or takes prob_mean), so P does not depend on the block size.
constexpr int kTotGroup = 8;

template <int kBlock>
__device__ __forceinline__ void block_expert_totals(const int32_t* __restrict__ hist, const float* __restrict__ psum,
                                                    const float* __restrict__ prob_mean, int E, int nch, int chunk,
                                                    int T, bool want_p, int* s_counts, int* s_pre, float* s_p) {
  static_assert(kBlock % 32 == 0, "whole warps");
  for (int i0 = 0; i0 < E * kTotGroup; i0 += kBlock) {
    const int idx = i0 + (int)threadIdx.x;
    const bool active = idx < E * kTotGroup;
    const int e = idx / kTotGroup, sub = idx % kTotGroup;
    int tot = 0, pre = 0;
    float ps = 0.f;
    if (active) {
      const int32_t* h = hist + (size_t)e * nch;
#pragma unroll 8
      for (int c = sub; c < nch; c += kTotGroup) {
        const int v = h[c];
        tot += v;
        pre += (c < chunk) ? v : 0;
      }
      if (want_p && prob_mean == nullptr && psum != nullptr) {
#pragma unroll 8
        for (int c = sub; c < nch; c += kTotGroup) ps += psum[(size_t)c * E + e];
      }
    }
#pragma unroll
    for (int o = kTotGroup / 2; o > 0; o >>= 1) {
      tot += __shfl_xor_sync(kFull, tot, o);
      pre += __shfl_xor_sync(kFull, pre, o);
      ps += __shfl_xor_sync(kFull, ps, o);
    }
    if (active && sub == 0) {
      s_counts[e] = tot;
      if (s_pre != nullptr) s_pre[e] = pre;
      if (want_p) s_p[e] = (prob_mean != nullptr) ? prob_mean[e] : (psum != nullptr ? ps / (float)T : NAN);
    }
  }
}

// One warp: kept = min(count, C) (all in dropless mode), offsets = exclusive
// scan of kept over the experts (8 experts per lane), the drop count and the
// Switch aux loss E * sum_e (count_e / (T k)) * P_e in double (the sum of
// count_e * P_e is divided by T k once: double divisions are slow).  Writes the
// offsets to s_off when given and the global results when `out` is set.
__device__ __forceinline__ void expert_offsets(const int* s_counts, const float* s_p, int s_ntie, double s_z,
                                               int E, int T, int k, int capacity, int* s_off, bool out,
                                               int32_t* counts, int32_t* kept, int32_t* offsets, moe_stats* stats,
                                               int lane) {
  constexpr int PER = kMaxExperts / 32;
  int kv[PER];
  int local = 0, drop = 0;
  double aux = 0.0;
  const double A = (double)T * (double)k;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    int cnt = 0, kp = 0;
    if (e < E) {
      cnt = s_counts[e];
      kp = (capacity < 0) ? cnt : min(cnt, capacity);
      if (out) aux += (double)cnt * (double)s_p[e];   // divided by T k once, below
    }
    kv[i] = kp;
    local += kp;
    drop += cnt - kp;
  }
  int incl = local;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int u = __shfl_up_sync(kFull, incl, o);
    if (lane >= o) incl += u;
  }
  int run = incl - local;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    if (e < E) {
      if (s_off != nullptr) s_off[e] = run;
      if (out) {
        offsets[e] = run;
        counts[e] = s_counts[e];
        kept[e] = kv[i];
      }
    }
    run += kv[i];
  }
  if (!out) return;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    drop += __shfl_xor_sync(kFull, drop, o);
    aux += __shfl_xor_sync(kFull, aux, o);
  }
  const int total = __shfl_sync(kFull, incl, 31);
  if (lane == 0) {
    offsets[E] = total;
    stats->drop_count = drop;
    stats->rows_kept = total;
    stats->capacity = capacity;
    stats->near_tie_count = s_ntie;
    stats->drop_rate = (T > 0) ? (float)((double)drop / A) : 0.f;
    stats->aux_loss = (T > 0) ? (float)((double)E * aux / A) : NAN;
    stats->z_loss = (T > 0) ? (float)(s_z / (double)T) : NAN;
  }
}

// Standalone scan (one CTA): chunk offsets for the scatter, and the results.
__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const int32_t* __restrict__ hist, int32_t* __restrict__ choff, int nch, int T, int E, int k,
            int capacity, const float* __restrict__ prob_mean, const float* __restrict__ psum,
            const int32_t* __restrict__ ntie, const float* __restrict__ zsum, int32_t* __restrict__ counts,
            int32_t* __restrict__ kept, int32_t* __restrict__ offsets, moe_stats* __restrict__ stats) {
  __shared__ int s_counts[kMaxExperts];
  __shared__ float s_p[kMaxExperts];
  __shared__ int s_ntie;
  __shared__ double s_z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kScanThreads / 32;
  pdl_wait();
  pdl_launch_dependents();
  for (int e = warp; e < E; e += nwarps) {   // chunk offsets for the scatter
    int tot, pre;
    expert_totals(hist, e, nch, 0, choff, lane, &tot, &pre);
  }
  block_expert_totals<kScanThreads>(hist, psum, prob_mean, E, nch, 0, T, true, s_counts, nullptr, s_p);
  if (warp == nwarps - 1) {
    const int nt = chunk_ties(ntie, nch, lane);
    const double z = chunk_zsum(zsum, nch, lane);
    if (lane == 0) {
      s_ntie = nt;
      s_z = z;
    }
  }
  __syncthreads();
  if (warp == 0)
    expert_offsets(s_counts, s_p, s_ntie, s_z, E, T, k, capacity, nullptr, true, counts, kept, offsets, stats, lane);
}

// ------------------------------------------------------------------ scatter
constexpr int kScatterThreads = 512;   // 4 rank warps, then all 16 warps copy

template <typename TX>
__device__ __forceinline__ void copy_rows(const TX* __restrict__ x, TX* __restrict__ xp, int d,
                                          int t, const int* rows, int k, int lane) {
  const int nvec = d * (int)sizeof(TX) / 16;
  const uint4* src = reinterpret_cast<const uint4*>(x + (size_t)t * d);
  for (int v = lane; v < nvec; v += 32) {
    const uint4 val = __ldg(src + v);
    for (int j = 0; j < k; ++j) {
      const int r = rows[j];
      if (r >= 0) reinterpret_cast<uint4*>(xp + (size_t)r * d)[v] = val;
    }
  }
}

struct ScatterArgs {
  const int32_t* topk_idx;
  const int32_t* hist;        // FUSED: per-chunk histograms [E][nch]
  int32_t* choff;             // separate scan: chunk offsets [E][nch]
  const float* prob_mean;     // FUSED, statistics block: P_e given, or
  const float* psum;          //   summed from the per-chunk probability sums
  const int32_t* ntie;
  const float* zsum;          // per-chunk sums of squared log-partitions (z-loss), or NULL
  int32_t* counts;
  int32_t* kept;
  int32_t* offsets;           // read (separate scan) or written by the statistics block (FUSED)
  moe_stats* stats;
  int32_t* row_of;
  int32_t* src_tok;
  const float* topk_w;        // with row_w: the gate weight of each kept row is
  float* row_w;               //   copied to row_w[row] (fused combine)
  float* out;                 // fused combine: the layer output, zeroed here
  int* zero;                  // or NULL: nzero ints zeroed here (the next kernel's tile-queue counters)
  int nzero;
  uint32_t* status;           // device error bits (a bounded wait that gave up)
  int T, d, E, k, nch, capacity;
  int slice_vec;              // 16-byte vectors of a row per column slice (gridDim.y slices)
};

// Ranks with warp ballots (k <= KB <= 8).  Lane l of rank warp w owns token
// t = chunk*128 + 32 w + l.  For each slot j' the 9 ballots of the bits of
// the slot-j' expert ids let every lane count, for each of its own experts e,
// the lanes below it that also chose e (in any slot): that count is the rank
// of (t, e) inside the warp.  Expert ids are < 256, so bit 8 marks "no expert".
//
// FUSED: the block first derives its chunk's offsets from the histograms
// itself (every block reads all E x nch counts from L2 and scans them), so no
// separate scan kernel runs; one extra block, (nch, 0), writes counts, kept,
// offsets and the statistics.  The grid's y dimension splits each token row into
// column slices, so that layers with few chunks and wide rows still spread
// the gather over all SMs; the ranks are recomputed by every slice.
template <int KB, typename TX, bool FUSED, bool STAGED>
__global__ void __launch_bounds__(kScatterThreads)
scatter_kernel(const TX* __restrict__ x, TX* __restrict__ xp, const ScatterArgs a) {
  constexpr int kRankWarps = kChunk / 32;
  constexpr int kWarps = kScatterThreads / 32;
  static_assert(kRankWarps <= kWarps, "one rank warp per 32 tokens of a chunk");
  extern __shared__ __align__(128) uint4 xs[];    // [tokens][W]: this block's slice of the chunk's x rows
  __shared__ __align__(8) unsigned long long xbar;
  __shared__ int wcnt[kRankWarps][kMaxExperts];
  __shared__ int rows_sm[kChunk][KB];
  __shared__ int s_pre[kMaxExperts], s_off[kMaxExperts], s_counts[kMaxExperts];
  __shared__ float s_p[kMaxExperts];
  __shared__ int s_ntie;
  __shared__ double s_z;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  const int E = a.E, k = a.k, T = a.T;
  if (FUSED && chunk == a.nch) {
    // One extra block (x = nch, y = 0) writes the layer's counts, kept,
    // offsets and statistics, so that no chunk block carries that work.
    if (blockIdx.y != 0) return;
    pdl_wait();
    pdl_launch_dependents();
    block_expert_totals<kScatterThreads>(a.hist, a.psum, a.prob_mean, E, a.nch, a.nch, T, true, s_counts, nullptr,
                                         s_p);
    if (warp == kWarps - 1) {
      const int nt = chunk_ties(a.ntie, a.nch, lane);
      const double z = chunk_zsum(a.zsum, a.nch, lane);
      if (lane == 0) {
        s_ntie = nt;
        s_z = z;
      }
    }
    __syncthreads();
    if (warp == 0)
      expert_offsets(s_counts, s_p, s_ntie, s_z, E, T, k, a.capacity, nullptr, true, a.counts, a.kept, a.offsets,
                     a.stats, lane);
    return;
  }
  const int nvec = a.d * (int)sizeof(TX) / 16;
  const int v0 = blockIdx.y * a.slice_vec;
  const int W = max(0, min(nvec, v0 + a.slice_vec) - v0);
  const int t0 = chunk * kChunk;
  const int ntok = min(kChunk, T - t0);
  const uint32_t bar = tc::smem_u32(&xbar);
  for (int i = threadIdx.x; i < kRankWarps * kMaxExperts; i += kScatterThreads) (&wcnt[0][0])[i] = 0;
  if (threadIdx.x == 0) {
    tc::mbar_init(bar, 1);
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
  }
  __syncthreads();
  // Before the wait on the routing kernel: x and out are not touched by it
  // (it starts only after everything earlier on the stream has finished), so
  // the slice of the chunk's x rows is brought into shared memory by TMA bulk
  // copies and the fused-combine output rows are zeroed while it runs.
  if (STAGED && warp == 0 && W > 0) {
    if (lane == 0) tc::mbar_expect_tx(bar, (uint32_t)(ntok * W * 16));
    __syncwarp();
    const char* src = reinterpret_cast<const char*>(x) + ((size_t)t0 * nvec + v0) * 16;
    for (int i = lane; i < ntok; i += 32)
      tc::bulk_load(tc::smem_u32(xs + (size_t)i * W), src + (size_t)i * nvec * 16, (uint32_t)(W * 16), bar);
  }
  // the expert kernel's counters: nothing reads them before that kernel's
  // own wait on this grid, and nothing earlier on the stream still runs
  if (a.zero != nullptr && blockIdx.x == 0 && blockIdx.y == 0)
    for (int i = threadIdx.x; i < a.nzero; i += kScatterThreads) a.zero[i] = 0;
  if (a.out != nullptr) {
    constexpr int kOutVec = 16 / (int)sizeof(TX) / 4;   // float4 of out per 16-byte vector of x
    const int wo = W * kOutVec;
    for (int u = threadIdx.x; u < ntok * wo; u += kScatterThreads) {
      const int tok = u / wo;
      reinterpret_cast<float4*>(a.out + (size_t)(t0 + tok) * a.d)[v0 * kOutVec + (u - tok * wo)] =
          make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }
  pdl_wait();
  pdl_launch_dependents();
  // the rank warps' expert ids (and gate weights) first: their loads overlap
  // the histogram reads
  int val[KB], rank_w[KB];
  float wsel[KB];
  const int t = chunk * kChunk + warp * 32 + lane;
  if (warp < kRankWarps) {
    const bool tv = t < T;
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      int e = 0x1ff;
      wsel[j] = 0.f;
      if (tv && j < k) {
        e = a.topk_idx[(size_t)t * k + j];
        if (e < 0 || e >= E) e = 0x1ff;
        if (a.row_w != nullptr) wsel[j] = a.topk_w[(size_t)t * k + j];
      }
      val[j] = e;
    }
  }
  if (FUSED) {
    block_expert_totals<kScatterThreads>(a.hist, nullptr, nullptr, E, a.nch, chunk, T, false, s_counts, s_pre,
                                         nullptr);
    __syncthreads();
    if (warp == 0)
      expert_offsets(s_counts, nullptr, 0, 0.0, E, T, k, a.capacity, s_off, false, nullptr, nullptr, nullptr, nullptr,
                     lane);
  } else {
    for (int e = threadIdx.x; e < E; e += kScatterThreads) {
      s_pre[e] = a.choff[(size_t)e * a.nch + chunk];
      s_off[e] = a.offsets[e];
    }
  }
  __syncthreads();

  if (warp < kRankWarps) {
    unsigned B[KB][9];
#pragma unroll
    for (int j = 0; j < KB; ++j)
#pragma unroll
      for (int b = 0; b < 9; ++b) B[j][b] = __ballot_sync(kFull, (val[j] >> b) & 1);
    const unsigned lt = (1u << lane) - 1u;
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      const int e = val[j];
      int below = 0, all = 0;
#pragma unroll
      for (int jj = 0; jj < KB; ++jj) {
        unsigned m = kFull;
#pragma unroll
        for (int b = 0; b < 9; ++b) m &= ((e >> b) & 1) ? B[jj][b] : ~B[jj][b];
        below += __popc(m & lt);
        all += __popc(m);
        // a repeated expert inside one token (only possible for caller-made
        // indices) is ordered by slot, like the assignments of distinct tokens
        if (jj < j && val[jj] == e) ++below;
      }
      rank_w[j] = below;
      if (e < E && below == 0) wcnt[warp][e] = all;   // first occurrence writes the warp's count
    }
  }
  __syncthreads();
  if (warp < kRankWarps) {
    const bool writer = blockIdx.y == 0;   // one slice writes the index outputs
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      const int e = val[j];
      int row = -1;
      if (e < E) {
        int before = 0;   // assignments of expert e in the earlier warps of this chunk
        for (int w = 0; w < warp; ++w) before += wcnt[w][e];
        const int r = s_pre[e] + before + rank_w[j];
        if (a.capacity < 0 || r < a.capacity) {
          row = s_off[e] + r;
          if (writer) {
            a.src_tok[row] = t;
            if (a.row_w != nullptr) a.row_w[row] = wsel[j];
          }
        }
      }
      if (writer && t < T && j < k) a.row_of[(size_t)t * k + j] = row;
      rows_sm[warp * 32 + lane][j] = row;
    }
  }
  __syncthreads();

  // gather: the block's column slice [v0, v0 + W) of every token row of the
  // chunk to the kept destination rows, from shared memory (STAGED) or
  // straight from x with four 16-byte loads in flight per thread
  const int units = ntok * W;
  if (STAGED) {
    if (W > 0 && !tc::mbar_wait(bar, 0, nullptr, tc::kWaitNs)) {
      if (threadIdx.x == 0) atomicOr(a.status, MOE_DEV_TIMEOUT);
      return;
    }
    // one bulk copy of the slice per kept (token, slot), shared memory -> xp row
    bool issued = false;
    for (int u = threadIdx.x; u < ntok * KB && W > 0; u += kScatterThreads) {
      const int tok = u / KB, j = u - tok * KB;
      const int r = rows_sm[tok][j];
      if (r >= 0) {
        tc::bulk_store(reinterpret_cast<char*>(xp) + ((size_t)r * nvec + v0) * 16, tc::smem_u32(xs + (size_t)tok * W),
                       (uint32_t)(W * 16));
        issued = true;
      }
    }
    if (issued) tc::bulk_store_drain();
    return;
  }
  for (int u0 = threadIdx.x; u0 < units; u0 += 4 * kScatterThreads) {
    uint4 v[4];
    int tok[4], col[4];
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int u = u0 + q * kScatterThreads;
      tok[q] = -1;
      if (u < units) {
        tok[q] = u / W;
        col[q] = v0 + (u - tok[q] * W);
        v[q] = __ldg(reinterpret_cast<const uint4*>(x + (size_t)(t0 + tok[q]) * a.d) + col[q]);
      }
    }
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      if (tok[q] < 0) continue;
#pragma unroll
      for (int j = 0; j < KB; ++j) {
        const int r = rows_sm[tok[q]][j];
        if (r >= 0) reinterpret_cast<uint4*>(xp + (size_t)r * a.d)[col[q]] = v[q];
      }
    }
  }
}

// Generic ranks for k > 8: thread e walks the chunk's assignments in token
// order and numbers those of expert e.
template <typename TX>
__global__ void __launch_bounds__(kScatterThreads)
scatter_generic_kernel(const TX* __restrict__ x, const int32_t* __restrict__ topk_idx,
                       const int32_t* __restrict__ choff, const int32_t* __restrict__ offsets,
                       int T, int d, int E, int k, int nch, int capacity,
                       int32_t* __restrict__ row_of, int32_t* __restrict__ src_tok, TX* __restrict__ xp) {
  extern __shared__ int idx_sm[];     // [kChunk * k] expert of each assignment, -1 if invalid
  pdl_wait();
  pdl_launch_dependents();
  const int chunk = blockIdx.x;
  const int t0 = chunk * kChunk;
  const int n = min(kChunk, T - t0) * k;
  int32_t* rows = row_of + (size_t)t0 * k;
  for (int i = threadIdx.x; i < n; i += kScatterThreads) {
    int e = topk_idx[(size_t)t0 * k + i];
    idx_sm[i] = (e < 0 || e >= E) ? -1 : e;
    rows[i] = -1;
  }
  __syncthreads();
  for (int e = threadIdx.x; e < E; e += kScatterThreads) {
    int r = choff[(size_t)e * nch + chunk];
    for (int i = 0; i < n; ++i) {
      if (idx_sm[i] != e) continue;
      if (capacity < 0 || r < capacity) {
        const int row = offsets[e] + r;
        rows[i] = row;
        src_tok[row] = t0 + i / k;
      }
      ++r;
    }
  }
  __syncthreads();   // the row numbers written above are visible to the whole block
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  for (int i = warp; i < kChunk; i += kScatterThreads / 32) {
    const int tt = t0 + i;
    if (tt >= T) break;
    copy_rows<TX>(x, xp, d, tt, rows + (size_t)i * k, k, lane);
  }
}

// Column slices per chunk.  When the whole grid fits in about one wave (two
// blocks per SM), every block stages its slice of x in shared memory before
// it waits for the routing kernel (slices of up to kSliceVec 16-byte vectors,
// 64 KB for a 128-token chunk), so the reads overlap that kernel.  Otherwise
// blocks read x directly, and rows are cut into as many slices (of at least
// 32 vectors) as keep the grid within one wave of two blocks per SM: a
// second, partly filled wave cost more than the longer rows per block.
constexpr int kSliceVec = 32;

inline bool scatter_staged(int nch, int nvec, int sms) {
  return (long long)nch * ((nvec + kSliceVec - 1) / kSliceVec) <= 2LL * sms;
}

inline int scatter_slices(int nch, int nvec, bool staged, int sms, int* slice_vec) {
  int S;
  if (staged) {
    S = (nvec + kSliceVec - 1) / kSliceVec;
    // a decode-sized batch (one chunk) would run a handful of blocks: halve
    // the slices (the FP8 decode forward 111.6 -> 109.6 us; a 64-chunk
    // layer, where halving cost 2 us, keeps them)
    if ((long long)nch * S < 16) S = (nvec + kSliceVec / 2 - 1) / (kSliceVec / 2);
  } else {
    S = (2 * sms) / nch;
    S = std::min(S, nvec / 32);
  }
  S = std::max(S, 1);
  *slice_vec = (nvec + S - 1) / S;
  return (nvec + *slice_vec - 1) / *slice_vec;
}

template <typename TX, bool FUSED, bool STAGED, int KB>
cudaError_t launch_scatter_kb(const dim3& g, const TX* x, TX* xp, const ScatterArgs& b, cudaStream_t s) {
  size_t smem = 0;
  if (STAGED) {
    constexpr size_t kMaxSmem = (size_t)kChunk * kSliceVec * 16;
    cudaError_t err = set_smem_once<scatter_kernel<KB, TX, FUSED, STAGED>>(kMaxSmem);
    if (err != cudaSuccess) return err;
    smem = (size_t)kChunk * b.slice_vec * 16;
  }
  return launch_pdl(scatter_kernel<KB, TX, FUSED, STAGED>, g, dim3(kScatterThreads), smem, s, x, xp, b);
}

template <typename TX, bool FUSED, bool STAGED>
cudaError_t launch_scatter_s(const moe_config& c, const TX* x, TX* xp, ScatterArgs b, int sms, cudaStream_t s) {
  int slice_vec = 0;
  const int S = scatter_slices(b.nch, c.d * (int)sizeof(TX) / 16, STAGED, sms, &slice_vec);
  b.slice_vec = slice_vec;
  const dim3 g(b.nch + (FUSED ? 1 : 0), S);   // FUSED: one more block row for the statistics
  if (c.k <= 1) return launch_scatter_kb<TX, FUSED, STAGED, 1>(g, x, xp, b, s);
  if (c.k <= 2) return launch_scatter_kb<TX, FUSED, STAGED, 2>(g, x, xp, b, s);
  if (c.k <= 4) return launch_scatter_kb<TX, FUSED, STAGED, 4>(g, x, xp, b, s);
  return launch_scatter_kb<TX, FUSED, STAGED, 8>(g, x, xp, b, s);
}

template <typename TX, bool FUSED>
cudaError_t launch_scatter_t(const moe_config& c, const TX* x, TX* xp, const ScatterArgs& a, cudaStream_t s) {
  DeviceInfo di;
  const int sms = (device_info(&di) == cudaSuccess) ? di.sms : 148;
  if (scatter_staged(a.nch, c.d * (int)sizeof(TX) / 16, sms))
    return launch_scatter_s<TX, FUSED, true>(c, x, xp, a, sms, s);
  return launch_scatter_s<TX, FUSED, false>(c, x, xp, a, sms, s);
}

template <typename TX>
cudaError_t launch_generic_t(const moe_config& c, const TX* xx, TX* pp, const ScatterArgs& a, cudaStream_t s) {
  const dim3 g(a.nch), b(kScatterThreads);
  const size_t smem = sizeof(int) * kChunk * (size_t)c.k;
  cudaError_t err = set_smem_once<scatter_generic_kernel<TX>>(sizeof(int) * kChunk * kMaxExperts);
  if (err != cudaSuccess) return err;
  return launch_pdl(scatter_generic_kernel<TX>, g, b, smem, s, xx, a.topk_idx, a.choff, a.offsets, c.T, c.d, c.E,
                    c.k, a.nch, a.capacity, a.row_of, a.src_tok, pp);
}

// The scan is fused into the scatter while the histograms every block reads
// stay small (64 KB); otherwise, and for k > 8 or no tokens, one scan block
// runs first and the scatter reads its chunk offsets.
constexpr long long kFusedHistMax = 16384;

template <typename TX>
cudaError_t launch_permute_t(const moe_config& c, const void* x, void* xp, ScatterArgs a, cudaStream_t s) {
  const TX* xx = static_cast<const TX*>(x);
  TX* pp = static_cast<TX*>(xp);
  if (c.T > 0 && c.k <= 8 && (long long)c.E * a.nch <= kFusedHistMax)
    return launch_scatter_t<TX, true>(c, xx, pp, a, s);
  cudaError_t e = launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, s, a.hist, a.choff,
                             a.nch, c.T, c.E, c.k, a.capacity, a.prob_mean, a.psum, a.ntie, a.zsum, a.counts,
                             a.kept, a.offsets, a.stats);
  if (e != cudaSuccess || c.T == 0) return e;
  if (c.k <= 8) return launch_scatter_t<TX, false>(c, xx, pp, a, s);
  return launch_generic_t<TX>(c, xx, pp, a, s);
}

}  // namespace

cudaError_t launch_hist(const moe_config& c, const int32_t* topk_idx, const float* gap,
                        int32_t* hist, int32_t* ntie, uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  return launch_pdl(hist_kernel, dim3(num_chunks(c.T)), dim3(kChunk), 0, s, topk_idx, gap, c.T, c.E, c.k,
                    num_chunks(c.T), hist, gap != nullptr ? ntie : nullptr, status);
}

cudaError_t launch_permute(const moe_config& c, int capacity, const void* x, const int32_t* topk_idx,
                           const int32_t* hist, int32_t* choff, const float* prob_mean, const float* psum,
                           const int32_t* ntie, const float* zsum, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                           cudaStream_t s, const float* topk_w, float* row_w, float* out, int* zero, int nzero) {
  ScatterArgs a{};
  a.topk_idx = topk_idx;
  a.hist = hist;
  a.choff = choff;
  a.prob_mean = prob_mean;
  a.psum = psum;
  a.ntie = ntie;
  a.zsum = zsum;
  a.counts = counts;
  a.kept = kept;
  a.offsets = offsets;
  a.stats = stats;
  a.row_of = row_of;
  a.src_tok = src_tok;
  a.topk_w = topk_w;
  a.row_w = row_w;
  a.out = out;
  a.zero = zero;
  a.nzero = nzero;
  a.status = &stats->status;
  a.T = c.T;
  a.d = c.d;
  a.E = c.E;
  a.k = c.k;
  a.nch = num_chunks(c.T);
  a.capacity = capacity;
  if (c.dtype == MOE_DTYPE_BF16) return launch_permute_t<__nv_bfloat16>(c, x, xp, a, s);
  return launch_permute_t<float>(c, x, xp, a, s);
}

}  // namespace moe
