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
#include "internal.cuh"

#include <math.h>

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

__global__ void __launch_bounds__(kScanThreads)
scan_kernel(const int32_t* __restrict__ hist, int32_t* __restrict__ choff, int nch, int T, int E, int k,
            int capacity, const float* __restrict__ prob_mean, const float* __restrict__ psum,
            const int32_t* __restrict__ ntie, int32_t* __restrict__ counts, int32_t* __restrict__ kept,
            int32_t* __restrict__ offsets, moe_stats* __restrict__ stats) {
  __shared__ int s_counts[kMaxExperts];
  __shared__ float s_p[kMaxExperts];
  __shared__ int s_ntie;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int nwarps = kScanThreads / 32;
  pdl_wait();
  pdl_launch_dependents();

  // per-expert exclusive scan over chunks (expert-major hist, coalesced); the
  // loads of four 32-chunk groups are issued before any of them is scanned
  constexpr int kBatch = 4;
  for (int e = warp; e < E; e += nwarps) {
    int running = 0;
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
        if (c < nch) choff[(size_t)e * nch + c] = running + incl - v[b];
        running += __shfl_sync(kFull, incl, 31);
      }
    }
    // P_e for the aux loss
    float P = NAN;
    if (prob_mean != nullptr) {
      P = prob_mean[e];
    } else if (psum != nullptr) {
      float s = 0.f;
#pragma unroll 4
      for (int c = lane; c < nch; c += 32) s += psum[(size_t)c * E + e];
      P = warp_sum(s) / (float)T;
    }
    if (lane == 0) { s_counts[e] = running; s_p[e] = P; }
  }
  if (warp == nwarps - 1) {
    int s = 0;
    if (ntie != nullptr)
      for (int c = lane; c < nch; c += 32) s += ntie[c];
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) s += __shfl_xor_sync(kFull, s, o);
    if (lane == 0) s_ntie = (ntie != nullptr) ? s : -1;
  }
  __syncthreads();

  // offsets = exclusive scan of kept over experts (one warp, 8 experts per lane)
  if (warp == 0) {
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
        aux += ((double)cnt / A) * (double)s_p[e];
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
        offsets[e] = run;
        counts[e] = s_counts[e];
        kept[e] = kv[i];
      }
      run += kv[i];
    }
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
      stats->aux_loss = (T > 0) ? (float)((double)E * aux) : NAN;
    }
  }
}

// ------------------------------------------------------------------ scatter
constexpr int kScatterThreads = 512;   // 4 rank warps, then 16 warps copying rows

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

// Ranks with warp ballots (k <= KB <= 8).  Lane l of rank warp w owns token
// t = chunk*64 + 32 w + l.  For each slot j' the 9 ballots of the bits of the
// slot-j' expert ids let every lane count, for each of its own experts e, the
// lanes below it that also chose e (in any slot): that count is the rank of
// (t, e) inside the warp.  Expert ids are < 256, so bit 8 marks "no expert".
template <int KB, typename TX>
__global__ void __launch_bounds__(kScatterThreads)
scatter_kernel(const TX* __restrict__ x, const int32_t* __restrict__ topk_idx,
               const int32_t* __restrict__ choff, const int32_t* __restrict__ offsets,
               int T, int d, int E, int k, int nch, int capacity,
               int32_t* __restrict__ row_of, int32_t* __restrict__ src_tok, TX* __restrict__ xp) {
  constexpr int kRankWarps = kChunk / 32;
  static_assert(kRankWarps <= kScatterThreads / 32, "one rank warp per 32 tokens of a chunk");
  __shared__ int wcnt[kRankWarps][kMaxExperts];
  __shared__ int rows_sm[kChunk][KB];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int chunk = blockIdx.x;
  for (int i = threadIdx.x; i < kRankWarps * kMaxExperts; i += kScatterThreads) (&wcnt[0][0])[i] = 0;
  pdl_wait();
  pdl_launch_dependents();
  __syncthreads();

  int val[KB], rank_w[KB];
  const int t = chunk * kChunk + warp * 32 + lane;
  if (warp < kRankWarps) {
    const bool tv = t < T;
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      int e = 0x1ff;
      if (tv && j < k) {
        e = topk_idx[(size_t)t * k + j];
        if (e < 0 || e >= E) e = 0x1ff;
      }
      val[j] = e;
    }
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
#pragma unroll
    for (int j = 0; j < KB; ++j) {
      const int e = val[j];
      int row = -1;
      if (e < E) {
        int before = 0;   // assignments of expert e in the earlier warps of this chunk
        for (int w = 0; w < warp; ++w) before += wcnt[w][e];
        const int r = choff[(size_t)e * nch + chunk] + before + rank_w[j];
        if (capacity < 0 || r < capacity) {
          row = offsets[e] + r;
          src_tok[row] = t;
        }
      }
      if (t < T && j < k) row_of[(size_t)t * k + j] = row;
      rows_sm[warp * 32 + lane][j] = row;
    }
  }
  __syncthreads();
  // gather: each warp copies whole token rows to their kept destinations
  for (int i = warp; i < kChunk; i += kScatterThreads / 32) {
    const int tt = chunk * kChunk + i;
    if (tt >= T) break;
    copy_rows<TX>(x, xp, d, tt, rows_sm[i], k, lane);
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

template <typename TX>
cudaError_t launch_scatter_t(const moe_config& c, int cap, const void* x, const int32_t* idx,
                             const int32_t* choff, const int32_t* off, int32_t* row_of,
                             int32_t* src_tok, void* xp, cudaStream_t s) {
  const int nch = num_chunks(c.T);
  const TX* xx = static_cast<const TX*>(x);
  TX* pp = static_cast<TX*>(xp);
  const dim3 g(nch), b(kScatterThreads);
#define MOE_SCATTER(KB) \
  return launch_pdl(scatter_kernel<KB, TX>, g, b, 0, s, xx, idx, choff, off, c.T, c.d, c.E, c.k, nch, cap, \
                    row_of, src_tok, pp)
  if (c.k <= 1) MOE_SCATTER(1);
  if (c.k <= 2) MOE_SCATTER(2);
  if (c.k <= 4) MOE_SCATTER(4);
  if (c.k <= 8) MOE_SCATTER(8);
#undef MOE_SCATTER
  const size_t smem = sizeof(int) * kChunk * (size_t)c.k;
  cudaError_t err = set_smem_once<scatter_generic_kernel<TX>>(sizeof(int) * kChunk * kMaxExperts);
  if (err != cudaSuccess) return err;
  return launch_pdl(scatter_generic_kernel<TX>, g, b, smem, s, xx, idx, choff, off, c.T, c.d, c.E, c.k, nch, cap,
                    row_of, src_tok, pp);
}

}  // namespace

cudaError_t launch_hist(const moe_config& c, const int32_t* topk_idx, const float* gap,
                        int32_t* hist, int32_t* ntie, uint32_t* status, cudaStream_t s) {
  if (c.T == 0) return cudaSuccess;
  return launch_pdl(hist_kernel, dim3(num_chunks(c.T)), dim3(kChunk), 0, s, topk_idx, gap, c.T, c.E, c.k,
                    num_chunks(c.T), hist, gap != nullptr ? ntie : nullptr, status);
}

cudaError_t launch_scan(const moe_config& c, int capacity, const int32_t* hist, int32_t* choff,
                        const float* prob_mean, const float* psum, const int32_t* ntie,
                        int32_t* counts, int32_t* kept, int32_t* offsets, moe_stats* stats,
                        cudaStream_t s) {
  return launch_pdl(scan_kernel, dim3(1), dim3(kScanThreads), 0, s, hist, choff, num_chunks(c.T), c.T, c.E, c.k,
                    capacity, prob_mean, psum, ntie, counts, kept, offsets, stats);
}

cudaError_t launch_scatter(const moe_config& c, int capacity, const void* x, const int32_t* topk_idx,
                           const int32_t* choff, const int32_t* offsets, int32_t* row_of,
                           int32_t* src_tok, void* xp, uint32_t* status, cudaStream_t s) {
  (void)status;
  if (c.T == 0) return cudaSuccess;
  if (c.dtype == MOE_DTYPE_BF16)
    return launch_scatter_t<__nv_bfloat16>(c, capacity, x, topk_idx, choff, offsets, row_of, src_tok, xp, s);
  return launch_scatter_t<float>(c, capacity, x, topk_idx, choff, offsets, row_of, src_tok, xp, s);
}

}  // namespace moe
