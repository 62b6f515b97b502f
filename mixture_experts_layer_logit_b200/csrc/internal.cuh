// Internal declarations shared by the CUDA translation units of libmoe.
#pragma once

#include <cuda_runtime.h>
#include <cuda_bf16.h>
#include <cuda_fp16.h>
#include <stdint.h>
#include <stddef.h>

#include "moe.h"

namespace moe {

// Tokens per routing / permutation chunk.  The route kernel, the histogram and
// the scatter kernel all cut the token axis into chunks of this size, and the
// per-chunk histograms and prefix sums live in the scratch workspace.
constexpr int kChunk = 128;
constexpr int kMaxExperts = 256;

// Scratch layout (byte offsets into the step workspace).
struct Scratch {
  size_t hist;      // int32 [E][nchunks]   assignments per (expert, chunk)
  size_t choff;     // int32 [E][nchunks]   exclusive prefix over chunks
  size_t psum;      // float [nchunks][E]   per-chunk sums of softmax probabilities
  size_t ntie;      // int32 [nchunks]      near-tie tokens per chunk
  size_t zsum;      // float [nchunks]      per-chunk sums of squared log-partitions (router z-loss)
  size_t status;    // uint32               device error bits of a standalone moe_route
  size_t mlp;       // int32 [expert_mlp_counters] tile queue of the one-launch expert kernel (bf16)
  size_t total;
};

inline int num_chunks(int T) { return (T + kChunk - 1) / kChunk; }
Scratch scratch_layout(const moe_config& c);

inline size_t align256(size_t x) { return (x + 255) & ~size_t(255); }

// ------------------------------------------------------------------ launchers
// Every launcher enqueues on `s` and returns cudaGetLastError().

// Route: logits, normalisation, softmax, top-k; per-chunk histogram, probability
// sums, near-tie counts and z-loss sums into scratch.  TX = float or __nv_bfloat16.
cudaError_t launch_route(const moe_config& c, const void* x, const void* wg, const float* bg,
                         int32_t* topk_idx, float* topk_w, float* gap,
                         int32_t* hist, float* psum, int32_t* ntie, float* zsum, uint32_t* status,
                         cudaStream_t s);
// The same on tcgen05 tensor cores (bf16, k <= 8).
bool route_tc_supported(const moe_config& c);
cudaError_t launch_route_tc(const moe_config& c, const void* x, const void* wg, const float* bg,
                            int32_t* topk_idx, float* topk_w, float* gap, int32_t* hist, float* psum,
                            int32_t* ntie, float* zsum, uint32_t* status, cudaStream_t s);
// One launch: prob_mean[e] = sum over chunks of psum / T and *z_loss = sum over
// chunks of zsum / T, both in a fixed order; either output may be NULL.
cudaError_t launch_route_totals(const moe_config& c, const float* psum, const float* zsum, float* prob_mean,
                                float* z_loss, cudaStream_t s);
// seg[0] = 0, seg[1] = rows (the shared expert's single segment)
cudaError_t launch_fill_segment(int32_t* seg, int rows, cudaStream_t s);
// out[i] += add[i] for n floats (n a multiple of 4)
cudaError_t launch_add_rows(float* out, const float* add, size_t n, cudaStream_t s);
// *coef = beta * *coef + (1 - beta) * xi * stats->drop_rate (one thread).
cudaError_t launch_aux_coef_update(const moe_stats* stats, float* coef, float beta, float xi, cudaStream_t s);
// Histogram of topk_idx per chunk (+ near ties from gap when given).
cudaError_t launch_hist(const moe_config& c, const int32_t* topk_idx, const float* gap,
                        int32_t* hist, int32_t* ntie, uint32_t* status, cudaStream_t s);
// Step 3 after the histograms: counts, kept, offsets, statistics, stable
// ranks, the capacity test, row_of/src_tok and the gather xp[row] = x[t].
// Either prob_mean (standalone) or psum (fused forward) or neither supplies
// P_e for the aux loss; zsum (fused forward) or NULL (z_loss = NaN) the z-loss; choff is scratch for the chunk offsets when the scan
// runs as its own kernel.  With row_w and out (fused combine, k <= 8 path):
// row_w[row] = topk_w of each kept assignment and out is zeroed.
cudaError_t launch_permute(const moe_config& c, int capacity, const void* x, const int32_t* topk_idx,
                           const int32_t* hist, int32_t* choff, const float* prob_mean, const float* psum,
                           const int32_t* ntie, const float* zsum, int32_t* counts, int32_t* kept,
                           int32_t* offsets, int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                           cudaStream_t s, const float* topk_w = nullptr, float* row_w = nullptr,
                           float* out = nullptr, int* zero = nullptr, int nzero = 0);
// True when the permutation runs scatter_kernel, whose prologue can zero the
// `zero` ints of launch_permute (T > 0 and k <= 8); otherwise they are ignored.
inline bool scatter_zeroes(const moe_config& c) { return c.T > 0 && c.k <= 8; }
// Expert FFN on CUDA cores (fp32 path).
// e_mod > 0: c.E counts row segments, and segment e uses the weights of
// expert e % e_mod (of e_mod given); 0: segment e is expert e.
cudaError_t launch_expert_ffn_simt(const moe_config& c, const void* xp, const int32_t* offsets,
                                   const void* w1, const void* w2, void* h, void* yp, uint32_t* status,
                                   cudaStream_t s, int e_mod = 0);
// Fused step 5 for the bf16 path with k <= 2: layer 2 adds row_w[row] * y of
// every permuted row into out[src_tok[row]] (out zeroed beforehand) instead
// of writing yp.
struct CombineOut {
  const int32_t* src_tok;
  const float* row_w;
  float* out;
  int T;
};
// Expert FFN on tcgen05 tensor cores (bf16 path).
cudaError_t launch_expert_ffn_tc(const moe_config& c, const void* xp, const int32_t* offsets,
                                 const void* w1, const void* w2, void* h, void* yp,
                                 uint32_t* status, cudaStream_t s, const CombineOut* comb = nullptr,
                                 int e_mod = 0);
// Both expert layers in one launch on the bf16 path, from one dynamic tile
// queue: with comb (k <= 2) the second layer adds into comb->out (the fused
// step 5), else it writes fp32 yp.  `counters` holds expert_mlp_counters(c)
// ints, zeroed before the launch.
size_t expert_mlp_counters(const moe_config& c);
cudaError_t launch_expert_mlp(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                              const void* w2, void* h, const CombineOut* comb, float* yp, int* counters,
                              uint32_t* status, cudaStream_t s, int e_mod = 0);
// Test hooks of the one-launch expert kernel (see moe_testing_set_expert_wait):
// the limit of its bounded waits (0 = the default 2 s) and an amount added to
// the layer-2 dependency target (0 = none; > 0 makes that wait unreachable).
void set_expert_mlp_test_hooks(unsigned long long wait_ns, int dep_extra);
// The same with 2-SM pair tiles (tcgen05.mma.cta_group::2, 256 x 256).
cudaError_t launch_expert_ffn_tc_pair(const moe_config& c, const void* xp, const int32_t* offsets,
                                      const void* w1, const void* w2, void* h, void* yp,
                                      uint32_t* status, cudaStream_t s, const CombineOut* comb = nullptr,
                                      int e_mod = 0);
// ------------------------------------------------------------- backward
// Buffers of the layer's backward: the forward's discrete choices (read from
// its workspace) and the backward workspace.  Padded rows: every expert's
// kept rows, its segment padded with zero rows to a multiple of
// bwd_pad_rows(); rows_alloc bounds them.
struct BwdState {
  const int32_t* topk_idx;   // [T][k]   forward: selected experts
  const float* topk_w;       // [T][k]   forward: gate weights
  const int32_t* counts;     // [E]      forward: pre-drop counts
  const int32_t* offsets;    // [E+1]    forward: permuted row offsets
  const int32_t* row_of;     // [T][k]   forward: permuted row of a slot (-1 dropped)
  const int32_t* src_tok;    // [A]      forward: token of a permuted row
  int32_t* pad_offsets;      // [E+1]
  int rows_alloc;
  void* xp;                  // [rows][d]   x of each padded row (element type of the path)
  void* dout_perm;           // [rows][d]   dout of each padded row (element type of the path)
  float* wrow;               // [rows]      gate weight of each padded row
  float* u;                  // [rows][F1]  first-layer pre-activation
  void* du;                  // [rows][F1]  (element type of the path)
  void* hw;                  // [rows][F]   w * h (element type of the path)
  float* dwpart;             // [column tiles of F][rows]
  float* dxp;                // [rows][d]
  float* z;                  // [slices][T][E] partial logits (bwd_logit_slices)
  float* dz;                 // [T][E]
  float* dwg_part;           // [nsplit][E][d + 1]
  int nsplit, tok_per_split;
  uint32_t* status;
  // fp16 GEMM operands (bf16 path with an fp16 hidden type): dout is scaled
  // by a power of two s into the fp16 range, and every result linear in dout
  // is scaled back by 1/s where it is written
  bool f16;
  unsigned* amax;            // max |dout| as float bits (zeroed before the amax kernel)
  float* scale;              // [2]: s, 1/s (1, 1 without fp16 operands)
  void* w1h;                 // fp16 copy of W1 (f16), else unused
};
int bwd_pad_rows();
int bwd_logit_slices(const moe_config& c);
int bwd_tc_col_tile();     // columns of a tensor-core backward tile (the dw partials per row)
int bwd_simt_col_tile();
// bf16 -> fp16 (round to nearest even, saturating at +-65504)
cudaError_t launch_convert_bf16_f16(const void* src, void* dst, size_t n, cudaStream_t s);
// prep (padded offsets, the dout scale) and gather (x, dout, gate weight of every padded row)
cudaError_t launch_bwd_front(const moe_config& c, const void* x, const float* dout, const BwdState& st,
                             cudaStream_t s);
// the expert layers' gradients: dh with the activation backward, dxp, dW2, dW1
// pair: 2-SM pair tiles (256 x 256) for every GEMM, else 1-SM tiles (128 x 256)
cudaError_t launch_expert_backward_tc(const moe_config& c, const BwdState& st, const void* w1, const void* w2,
                                      float* dw1, float* dw2, bool pair, cudaStream_t s);
cudaError_t launch_expert_backward_simt(const moe_config& c, const BwdState& st, const void* w1, const void* w2,
                                        float* dw1, float* dw2, cudaStream_t s);
// out[rows][Nout] = A[rows][K] B_e[Nout][K]^T over the segments of offsets (E of them), fp32 out;
// f16: both operands fp16 (else bf16)
cudaError_t launch_grouped_plain_tc(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
                                    const void* B, int K, int Nout, float* out, uint32_t* status, bool f16,
                                    cudaStream_t s);
cudaError_t launch_grouped_plain_tc_pair(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
                                         const void* B, int K, int Nout, float* out, uint32_t* status, bool f16,
                                         cudaStream_t s);
cudaError_t launch_grouped_plain_simt(const moe_config& c, const void* A, const int32_t* offsets, int rows_alloc,
                                      const void* B, int K, int Nout, float* out, uint32_t* status, cudaStream_t s);
// the gate's gradient (logits recomputed), dx and dW_gate / db
cudaError_t launch_bwd_gate(const moe_config& c, const void* x, const void* wg, const float* bg, const BwdState& st,
                            float aux_coef, float z_coef, float* dx, float* dwg, float* dbg, float* dw_out,
                            cudaStream_t s);

// ------------------------------------------------------- MX FP8 experts
// Buffers of the FP8 expert step: kept offsets from the permutation, padded
// offsets (multiples of mx_pad_rows()), the padded E4M3 layer-1 input rows and
// hidden activation with their scale atoms.
struct MxBuffers {
  const int32_t* offsets;   // [E+1] kept
  int32_t* pad;             // [E+1]
  const void* xp;           // [rows][d] bf16 permuted rows (from the permutation)
  int rows_pad;
  void* xq;                 // [rows_pad][d] E4M3
  void* xs;                 // scale atoms of xq
  void* hq;                 // [rows_pad][F] E4M3
  void* hs;                 // scale atoms of hq
  int* ctr;                 // [1 + rows_pad / 128] the expert kernel's tile and dependency counters
};
int mx_pad_rows();
size_t mx_scale_bytes(size_t rows, size_t K);   // rows, K multiples of 128
cudaError_t launch_mx_prepare_weights(const moe_config& c, const void* w1, const void* w2, void* w1q, void* w1s,
                                      void* w2q, void* w2s, cudaStream_t s);
// steps 4 of the FP8 layer: padded offsets, the quantised input rows, both
// layers; yp [rows][d] fp32 at the kept rows
cudaError_t launch_mx_experts(const moe_config& c, const MxBuffers& b, const void* w1q, const void* w1s,
                              const void* w2q, const void* w2s, float* yp, uint32_t* status, cudaStream_t s);

// Combine.
cudaError_t launch_combine(const moe_config& c, const void* yp, const int32_t* row_of,
                           const float* topk_w, void* out, cudaStream_t s);

// One step of the layer-wise adaptive aux-loss coefficient (Skywork-MoE
// release, "2.自适应的Aux Loss"): an exponential moving average, smoothing
// beta, of xi times the drop rate.  The same expression on host and device.
__host__ __device__ inline float aux_coef_step(float coef, float drop_rate, float beta, float xi) {
  return beta * coef + (1.f - beta) * (xi * drop_rate);
}

// Device properties cached per device (SM count, compute capability).
struct DeviceInfo {
  int sms = 0;
  int major = 0, minor = 0;
  size_t smem_optin = 0;
};
cudaError_t device_info(DeviceInfo* out);

// Address of the library's fixed scratch array (MOE_STATIC_SCRATCH_BYTES) on
// the current device; looked up once per device.
cudaError_t static_scratch_address(void** out);

// ------------------------------------------------------------ device helpers
__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  return v;
}
__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, o));
  return v;
}

__device__ __forceinline__ float to_float(float v) { return v; }
__device__ __forceinline__ float to_float(__nv_bfloat16 v) { return __bfloat162float(v); }

}  // namespace moe

namespace moe {

// Tile table of a grouped GEMM over expert segments: expert e owns rows
// [offsets[e], offsets[e+1]) and ceil(M_e / BM) * nt tiles, numbered from
// tstart[e]; tstart[E] is the total.  Run by the 32 lanes of one warp
// (E <= 256, 8 experts per lane).  offsets[] must be non-decreasing inside
// [0, rows_alloc] with at most 2^30 tiles in all; otherwise the table is
// left empty (no tile runs, nothing is written) and false is returned.
__device__ __forceinline__ bool tile_table_warp(const int32_t* __restrict__ offsets, int E, int BM,
                                                int nt, int rows_alloc, int* tstart, int lane) {
  constexpr int PER = kMaxExperts / 32;
  int loc[PER];
  long long sum64 = 0;
  bool ok = true;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    const int e = lane * PER + i;
    long long m = 0;
    if (e < E) {
      const int a = offsets[e], b = offsets[e + 1];
      ok &= (a >= 0) && (b >= a) && (b <= rows_alloc);
      m = (long long)b - a;
    }
    const long long tiles = ((m + BM - 1) / BM) * (long long)nt;
    ok &= tiles <= (1LL << 30);
    loc[i] = (int)(tiles > (1LL << 30) ? 0 : tiles);
    sum64 += loc[i];
  }
  ok = __all_sync(0xffffffffu, ok);
  long long tot = sum64;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) tot += __shfl_xor_sync(0xffffffffu, tot, o);
  ok = ok && tot <= (1LL << 30);
  int sum = 0;
#pragma unroll
  for (int i = 0; i < PER; ++i) {
    if (!ok) loc[i] = 0;
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
    if (e < E) tstart[e] = run;
    run += loc[i];
  }
  if (lane == 31) tstart[E] = incl;
  return ok;
}

// Expert owning tile L: the largest e with tstart[e] <= L (empty experts have
// tstart[e] == tstart[e+1] and are skipped by taking the largest).
__device__ __forceinline__ int tile_expert(const int* tstart, int E, int L) {
  int lo = 0, hi = E - 1;
  while (lo < hi) {
    const int mid = (lo + hi + 1) >> 1;
    if (tstart[mid] <= L) lo = mid; else hi = mid - 1;
  }
  return lo;
}

}  // namespace moe

#include <atomic>
#include <utility>

namespace moe {

// Programmatic dependent launch.  Every kernel of the layer is launched with
// the programmatic-serialization attribute, so it may start while the kernel
// before it in the stream drains.  A kernel does only work that touches no
// global memory before pdl_wait() (barrier set-up, TMEM allocation,
// tensor-map prefetch); pdl_wait() returns once the previous grid has
// completed and its writes are visible, which by induction covers every
// earlier kernel.  Without a programmatic predecessor both calls are no-ops.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t s,
                       Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

// Raises a kernel's dynamic shared-memory limit once per device (the first
// call, made before any stream capture, does the work; later calls only read
// an atomic), so launches stay free of attribute calls.
template <auto Kernel>
cudaError_t set_smem_once(size_t bytes) {
  static std::atomic<unsigned long long> done{0};
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const unsigned long long bit = 1ull << (dev & 63);
  if (done.load(std::memory_order_acquire) & bit) return cudaSuccess;
  e = cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)bytes);
  if (e == cudaSuccess) done.fetch_or(bit, std::memory_order_acq_rel);
  else (void)cudaGetLastError();   // report it here, do not leave it for the next launch check
  return e;
}

}  // namespace moe
