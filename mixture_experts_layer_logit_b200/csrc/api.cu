// C ABI of libmoe: argument checks, workspace layout and the order of the
// kernels of each step.  See include/moe.h for the contract of every entry.
#include "internal.cuh"

#include <math.h>

#include <algorithm>
#include <mutex>

namespace moe {

cudaError_t device_info(DeviceInfo* out) {
  constexpr int kMaxDev = 64;
  static DeviceInfo cache[kMaxDev];
  static std::once_flag once[kMaxDev];
  int dev = 0;
  cudaError_t err = cudaGetDevice(&dev);
  if (err != cudaSuccess) return err;
  if (dev < 0 || dev >= kMaxDev) return cudaErrorInvalidDevice;
  cudaError_t res = cudaSuccess;
  std::call_once(once[dev], [&] {
    DeviceInfo d;
    int v = 0;
    if ((res = cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return;
    d.sms = v;
    if ((res = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMajor, dev)) != cudaSuccess) return;
    d.major = v;
    if ((res = cudaDeviceGetAttribute(&v, cudaDevAttrComputeCapabilityMinor, dev)) != cudaSuccess) return;
    d.minor = v;
    if ((res = cudaDeviceGetAttribute(&v, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess) return;
    d.smem_optin = (size_t)v;
    cache[dev] = d;
  });
  if (res != cudaSuccess) return res;
  if (cache[dev].sms == 0) return cudaErrorUnknown;
  *out = cache[dev];
  return cudaSuccess;
}

Scratch scratch_layout(const moe_config& c) {
  const size_t nch = (size_t)num_chunks(c.T);
  Scratch s;
  size_t off = 0;
  s.hist = off;  off = align256(off + sizeof(int32_t) * (size_t)c.E * nch);
  s.choff = off; off = align256(off + sizeof(int32_t) * (size_t)c.E * nch);
  s.psum = off;  off = align256(off + sizeof(float) * (size_t)c.E * nch);
  s.ntie = off;  off = align256(off + sizeof(int32_t) * nch);
  s.zsum = off;  off = align256(off + sizeof(float) * nch);
  s.status = off; off = align256(off + sizeof(uint32_t));
  s.mlp = off;    off = align256(off + (c.dtype == MOE_DTYPE_BF16 ? sizeof(int) * expert_mlp_counters(c) : 0));
  s.total = off > 0 ? off : 256;
  return s;
}

}  // namespace moe

using namespace moe;

namespace {

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

moe_status check_config(const moe_config* c) {
  if (c == nullptr) return MOE_ERR_ARG;
  if (c->T < 0 || c->d < 1 || c->E < 1 || c->F < 1 || c->k < 1) return MOE_ERR_ARG;
  if (c->k > c->E) return MOE_ERR_ARG;
  if (c->act != MOE_ACT_RELU && c->act != MOE_ACT_SWIGLU) return MOE_ERR_ARG;
  if (c->dtype != MOE_DTYPE_BF16 && c->dtype != MOE_DTYPE_F32) return MOE_ERR_ARG;
  if (c->dtype == MOE_DTYPE_BF16 && c->hidden_dtype != MOE_DTYPE_BF16 && c->hidden_dtype != MOE_DTYPE_F16)
    return MOE_ERR_ARG;
  if (c->dtype == MOE_DTYPE_F32 && c->hidden_dtype != MOE_DTYPE_F32) return MOE_ERR_ARG;
  if (!isfinite(c->capacity_factor) || !isfinite(c->lambda)) return MOE_ERR_ARG;
  if (c->E > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  const int mult = (c->dtype == MOE_DTYPE_BF16) ? 16 : 4;
  if (c->d % mult != 0 || c->F % mult != 0) return MOE_ERR_UNSUPPORTED;
  // index arithmetic stays in int32 for T*k rows and 64-bit for elements
  if ((long long)c->T * c->k > (1LL << 30)) return MOE_ERR_UNSUPPORTED;
  if ((long long)c->E * (c->act == MOE_ACT_SWIGLU ? 2 : 1) * c->F > (1LL << 31) - 1) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// Capacity in assignments; -1 in dropless mode.  Evaluated in double in the
// order the header states; saturates at INT32_MAX (any C >= T keeps everything).
int capacity_of(const moe_config& c) {
  if (!(c.capacity_factor > 0.f)) return -1;
  const double C = ceil((double)c.capacity_factor * (double)((long long)c.T * c.k) / (double)c.E);
  if (C >= 2147483647.0) return 2147483647;
  return (int)C;
}

moe_status check_ws(void* ws, size_t ws_bytes, size_t need) {
  if (ws == nullptr || (reinterpret_cast<uintptr_t>(ws) & 255u) != 0 || ws_bytes < need) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

moe_status check_device(bool need_tc) {
  // A non-sticky error left by an earlier, unrelated runtime call would
  // otherwise be picked up by the launch checks below and reported as ours.
  (void)cudaGetLastError();
  DeviceInfo di;
  if (device_info(&di) != cudaSuccess) return MOE_ERR_CUDA;
  if (need_tc && di.major != 10) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

inline moe_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MOE_OK : MOE_ERR_CUDA; }

size_t elem_size(const moe_config& c) { return c.dtype == MOE_DTYPE_BF16 ? 2 : 4; }

moe_ws_layout layout_of(const moe_config& c) {
  moe_ws_layout L{};
  const size_t T = (size_t)c.T, k = (size_t)c.k, E = (size_t)c.E, A = T * k, es = elem_size(c);
  size_t off = 0;
  L.topk_idx = off;  off = align256(off + 4 * A);
  L.topk_w = off;    off = align256(off + 4 * A);
  L.gap = off;       off = align256(off + 4 * T);
  L.counts = off;    off = align256(off + 4 * E);
  L.kept = off;      off = align256(off + 4 * E);
  L.offsets = off;   off = align256(off + 4 * (E + 1));
  L.row_of = off;    off = align256(off + 4 * A);
  L.src_tok = off;   off = align256(off + 4 * A);
  L.row_w = off;     off = align256(off + 4 * A);
  L.xp = off;        off = align256(off + es * A * (size_t)c.d);
  L.h = off;         off = align256(off + es * A * (size_t)c.F);
  L.yp = off;        off = align256(off + 4 * A * (size_t)c.d);   // fp32 for both element types
  L.scratch = off;   off = align256(off + scratch_layout(c).total);
  L.total = off;
  return L;
}

template <typename T>
T* at(void* base, size_t off) { return reinterpret_cast<T*>(static_cast<char*>(base) + off); }

// step 3 given the histogram already in scratch
moe_status permute_from_hist(const moe_config& c, const void* x, const int32_t* topk_idx,
                             const float* prob_mean, const float* psum, const int32_t* ntie, const float* zsum,
                             int32_t* counts, int32_t* kept, int32_t* offsets, int32_t* row_of,
                             int32_t* src_tok, void* xp, moe_stats* stats, const Scratch& sc, void* ws,
                             cudaStream_t s, const float* topk_w = nullptr, float* row_w = nullptr,
                             float* out = nullptr, int* zero = nullptr, int nzero = 0) {
  return cuda_status(launch_permute(c, capacity_of(c), x, topk_idx, at<int32_t>(ws, sc.hist),
                                    at<int32_t>(ws, sc.choff), prob_mean, psum, ntie, zsum, counts, kept,
                                    offsets, row_of, src_tok, xp, stats, s, topk_w, row_w, out, zero, nzero));
}

// Mean assignments per expert from which the expert GEMMs use 2-SM tiles.
constexpr long long kPairRowsPerExpert = 512;
bool pair_tiles(const moe_config& c) { return (long long)c.T * c.k >= kPairRowsPerExpert * c.E; }

moe_status expert_ffn(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                      const void* w2, void* h, void* yp, moe_stats* stats, cudaStream_t s,
                      const CombineOut* comb = nullptr, int e_mod = 0) {
  if (c.dtype == MOE_DTYPE_BF16) {
    // 2-SM pair tiles (256 rows) pay off once the expert segments hold a few
    // hundred rows on average; short segments waste half a pair tile.
    if (pair_tiles(c))
      return cuda_status(
          launch_expert_ffn_tc_pair(c, xp, offsets, w1, w2, h, yp, &stats->status, s, comb, e_mod));
    return cuda_status(launch_expert_ffn_tc(c, xp, offsets, w1, w2, h, yp, &stats->status, s, comb, e_mod));
  }
  return cuda_status(launch_expert_ffn_simt(c, xp, offsets, w1, w2, h, yp, &stats->status, s, e_mod));
}

// The forward fuses step 5 into the second expert GEMM when a token has at
// most two expert outputs to add (then the sum does not depend on the order
// the additions arrive in) and the tensor-core path runs.
bool fused_combine(const moe_config& c) { return c.dtype == MOE_DTYPE_BF16 && c.k <= 2 && c.T > 0; }

// On the 1-SM tiles both expert layers and the combine run as one launch
// with a dynamic tile queue; its counters use the yp region of the forward
// workspace, which the fused combine leaves unwritten.
bool one_launch(const moe_config& c) {
  return fused_combine(c) && !pair_tiles(c) &&
         sizeof(int) * expert_mlp_counters(c) <= sizeof(float) * (size_t)c.T * c.k * c.d;
}

// Without the fused combine, the two expert layers on 1-SM tiles still run as
// one launch that writes yp (the expert step on its own, and the forward when
// k > 2); the tile queue's counters live in scratch.
bool one_launch_plain(const moe_config& c) {
  return c.dtype == MOE_DTYPE_BF16 && c.T > 0 && !pair_tiles(c);
}
moe_status expert_mlp_plain(const moe_config& c, const void* xp, const int32_t* offsets, const void* w1,
                            const void* w2, void* h, void* yp, moe_stats* stats, int* counters,
                            bool counters_zeroed, cudaStream_t s, int e_mod = 0) {
  if (!counters_zeroed && cudaMemsetAsync(counters, 0, sizeof(int) * expert_mlp_counters(c), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return cuda_status(launch_expert_mlp(c, xp, offsets, w1, w2, h, nullptr, static_cast<float*>(yp), counters,
                                       &stats->status, s, e_mod));
}

// The configuration step 4 runs with over `nseg` caller-given segments of a
// `rows`-row buffer: one "assignment" per row, one tile-table entry per segment.
moe_config segments_config(const moe_config& c, int nseg, int rows) {
  moe_config cc = c;
  cc.T = rows;
  cc.k = 1;
  cc.E = nseg;
  cc.capacity_factor = 0.f;
  cc.lambda = 0.f;
  return cc;
}

// Steps 4-5 fused (out zeroed beforehand); counters: the yp region.
moe_status experts_combine(const moe_config& c, const void* xp, const int32_t* offsets, const int32_t* src_tok,
                           const float* row_w, const void* w1, const void* w2, void* h, float* out, int* counters,
                           void* yp, moe_stats* stats, bool counters_zeroed, cudaStream_t s) {
  const CombineOut comb{src_tok, row_w, out, c.T};
  if (one_launch(c)) {
    if (!counters_zeroed && cudaMemsetAsync(counters, 0, sizeof(int) * expert_mlp_counters(c), s) != cudaSuccess)
      return MOE_ERR_CUDA;
    return cuda_status(launch_expert_mlp(c, xp, offsets, w1, w2, h, &comb, nullptr, counters, &stats->status, s));
  }
  return expert_ffn(c, xp, offsets, w1, w2, h, yp, stats, s, &comb);
}

// Layout of the backward workspace (each region 256-byte aligned).
struct BwdLayout {
  int rows;
  int nsplit, tok_per_split, col_tiles;
  size_t pad_offsets, xp, dout_perm, wrow, u, du, hw, dwpart, dxp, z, dz, dwg_part, amax, scale, w1h, total;
};

// The backward's GEMM operands are fp16 when the forward's hidden type is
// fp16 (dout scaled into its range), else of the element type of x.
bool bwd_f16(const moe_config& c) { return c.dtype == MOE_DTYPE_BF16 && c.hidden_dtype == MOE_DTYPE_F16; }

BwdLayout bwd_layout(const moe_config& c) {
  BwdLayout L{};
  const size_t es = elem_size(c);
  const int F1 = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  const long long rows = (long long)c.T * c.k + (long long)(bwd_pad_rows() - 1) * c.E;
  L.rows = (int)((rows + 127) / 128 * 128);
  const int col = c.dtype == MOE_DTYPE_BF16 ? bwd_tc_col_tile() : bwd_simt_col_tile();
  L.col_tiles = (c.F + col - 1) / col;
  L.tok_per_split = std::max(256, (((c.T + 63) / 64) + 63) / 64 * 64);
  L.nsplit = std::max(1, (c.T + L.tok_per_split - 1) / L.tok_per_split);
  const size_t R = (size_t)L.rows, T = (size_t)c.T, E = (size_t)c.E, d = (size_t)c.d;
  size_t off = 0;
  L.pad_offsets = off; off = align256(off + 4 * (E + 1));
  L.xp = off;          off = align256(off + es * R * d);
  L.dout_perm = off;   off = align256(off + es * R * d);
  L.wrow = off;        off = align256(off + 4 * R);
  L.u = off;           off = align256(off + 4 * R * (size_t)F1);
  L.du = off;          off = align256(off + es * R * (size_t)F1);
  L.hw = off;          off = align256(off + es * R * (size_t)c.F);
  L.dwpart = off;      off = align256(off + 4 * R * (size_t)L.col_tiles);
  L.dxp = off;         off = align256(off + 4 * R * d);
  L.z = off;           off = align256(off + 4 * (size_t)bwd_logit_slices(c) * T * E);
  L.dz = off;          off = align256(off + 4 * T * E);
  L.dwg_part = off;    off = align256(off + 4 * (size_t)L.nsplit * E * (d + 1));
  L.amax = off;        off = align256(off + 4);
  L.scale = off;       off = align256(off + 8);
  L.w1h = off;         off = align256(off + (bwd_f16(c) ? 2 * E * (size_t)F1 * d : 0));
  L.total = off;
  return L;
}

// The FP8 (MX) layer: the forward workspace, then its own regions.
struct MxLayout {
  moe_ws_layout base;
  int rows_pad;
  size_t pad, xq, xs, hq, hs, ctr, total;
};

MxLayout mx_layout(const moe_config& c) {
  MxLayout L{};
  L.base = layout_of(c);
  const long long rows = (long long)c.T * c.k + (long long)(mx_pad_rows() - 1) * c.E;
  L.rows_pad = (int)((rows + 127) / 128 * 128);
  const size_t R = (size_t)L.rows_pad;
  size_t off = L.base.total;
  L.pad = off; off = align256(off + 4 * ((size_t)c.E + 1));
  L.xq = off;  off = align256(off + R * (size_t)c.d);
  L.xs = off;  off = align256(off + mx_scale_bytes(R, (size_t)c.d));
  L.hq = off;  off = align256(off + R * (size_t)c.F);
  L.hs = off;  off = align256(off + mx_scale_bytes(R, (size_t)c.F));
  L.ctr = off; off = align256(off + 4 * (1 + R / 128));
  L.total = off;
  return L;
}

moe_status check_mx_config(const moe_config* c) {
  moe_status st = check_config(c);
  if (st != MOE_OK) return st;
  if (c->dtype != MOE_DTYPE_BF16) return MOE_ERR_UNSUPPORTED;
  if (c->d % 128 != 0 || c->F % 128 != 0) return MOE_ERR_UNSUPPORTED;
  return MOE_OK;
}

// The layer with a shared expert: the forward workspace, then the shared
// expert's regions (its config is the layer's with one expert of width Fs
// over T rows, one row per token).
struct SharedLayout {
  moe_ws_layout base;
  moe_config sc;
  size_t seg, h, y, scratch, total;
};

SharedLayout shared_layout(const moe_config& c, int Fs) {
  SharedLayout L{};
  L.base = layout_of(c);
  moe_config one = c;
  one.E = 1;
  one.F = Fs;
  L.sc = segments_config(one, 1, c.T);
  const size_t hs = c.dtype == MOE_DTYPE_BF16 ? 2 : 4;
  size_t off = L.base.total;
  L.seg = off;     off = align256(off + 8);
  L.h = off;       off = align256(off + hs * (size_t)c.T * Fs);
  L.y = off;       off = align256(off + 4 * (size_t)c.T * c.d);
  L.scratch = off; off = align256(off + scratch_layout(L.sc).total);
  L.total = off;
  return L;
}

}  // namespace

extern "C" {

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "MOE_OK";
    case MOE_ERR_ARG: return "MOE_ERR_ARG: invalid argument";
    case MOE_ERR_UNSUPPORTED: return "MOE_ERR_UNSUPPORTED: shape or device not supported";
    case MOE_ERR_WORKSPACE: return "MOE_ERR_WORKSPACE: workspace missing, misaligned or too small";
    case MOE_ERR_CUDA: return "MOE_ERR_CUDA: a CUDA call failed";
  }
  return "unknown moe_status";
}

size_t moe_scratch_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return scratch_layout(*cfg).total;
}

size_t moe_workspace_size(const moe_config* cfg, moe_ws_layout* layout) {
  if (check_config(cfg) != MOE_OK) return 0;
  const moe_ws_layout L = layout_of(*cfg);
  if (layout != nullptr) *layout = L;
  return L.total;
}

moe_status moe_route(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                     int32_t* topk_idx, float* topk_w, float* gap, float* prob_mean, float* z_loss,
                     void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T > 0 && (x == nullptr || Wg == nullptr || topk_idx == nullptr || topk_w == nullptr || gap == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned4(bg) || !aligned4(topk_idx) || !aligned4(topk_w) ||
      !aligned4(gap) || !aligned4(prob_mean) || !aligned4(z_loss))
    return MOE_ERR_ARG;
  const Scratch sc = scratch_layout(c);
  if ((st = check_ws(ws, ws_bytes, sc.total)) != MOE_OK) return st;
  if ((st = check_device(false)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  cudaError_t e = launch_route(c, x, Wg, bg, topk_idx, topk_w, gap, at<int32_t>(ws, sc.hist),
                               at<float>(ws, sc.psum), at<int32_t>(ws, sc.ntie), at<float>(ws, sc.zsum),
                               at<uint32_t>(ws, sc.status), s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  if (c.T == 0) {   // empty batch: P_e and the z-loss are not defined
    if (prob_mean != nullptr && cudaMemsetAsync(prob_mean, 0xff, sizeof(float) * (size_t)c.E, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    if (z_loss != nullptr && cudaMemsetAsync(z_loss, 0xff, sizeof(float), s) != cudaSuccess) return MOE_ERR_CUDA;
    return MOE_OK;
  }
  return cuda_status(launch_route_totals(c, at<float>(ws, sc.psum), at<float>(ws, sc.zsum), prob_mean, z_loss, s));
}

moe_status moe_permute(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                       const float* gap, const float* prob_mean,
                       int32_t* counts, int32_t* kept, int32_t* offsets,
                       int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                       void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (counts == nullptr || kept == nullptr || offsets == nullptr || stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (x == nullptr || topk_idx == nullptr || row_of == nullptr || src_tok == nullptr || xp == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(xp) || !aligned4(topk_idx) || !aligned4(gap) || !aligned4(prob_mean) ||
      !aligned4(counts) || !aligned4(kept) || !aligned4(offsets) || !aligned4(row_of) || !aligned4(src_tok) ||
      !aligned4(stats))
    return MOE_ERR_ARG;
  const Scratch sc = scratch_layout(c);
  if ((st = check_ws(ws, ws_bytes, sc.total)) != MOE_OK) return st;
  if ((st = check_device(false)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(&stats->status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = launch_hist(c, topk_idx, gap, at<int32_t>(ws, sc.hist), at<int32_t>(ws, sc.ntie),
                              &stats->status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return permute_from_hist(c, x, topk_idx, prob_mean, nullptr,
                           (gap != nullptr && c.T > 0) ? at<int32_t>(ws, sc.ntie) : nullptr, nullptr, counts, kept,
                           offsets, row_of, src_tok, xp, stats, sc, ws, s);
}

moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const int32_t* offsets,
                          const void* W1, const void* W2, void* h, void* yp,
                          moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (offsets == nullptr || stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (xp == nullptr || W1 == nullptr || W2 == nullptr || h == nullptr || yp == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(xp) || !aligned16(W1) || !aligned16(W2) || !aligned16(h) || !aligned16(yp) ||
      !aligned4(offsets) || !aligned4(stats))
    return MOE_ERR_ARG;
  const Scratch sc = scratch_layout(c);
  if ((st = check_ws(ws, ws_bytes, sc.total)) != MOE_OK) return st;
  if ((st = check_device(c.dtype == MOE_DTYPE_BF16)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (one_launch_plain(c))
    return expert_mlp_plain(c, xp, offsets, W1, W2, h, yp, stats, at<int>(ws, sc.mlp), false, s);
  return expert_ffn(c, xp, offsets, W1, W2, h, yp, stats, s);
}

moe_status moe_expert_ffn_combine(const moe_config* cfg, const void* xp, const int32_t* offsets,
                                  const int32_t* src_tok, const float* row_w, const void* W1, const void* W2,
                                  void* h, void* out, moe_stats* stats, void* ws, size_t ws_bytes,
                                  moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.dtype != MOE_DTYPE_BF16 || c.k > 2) return MOE_ERR_UNSUPPORTED;
  if (offsets == nullptr || stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (xp == nullptr || src_tok == nullptr || row_w == nullptr || W1 == nullptr || W2 == nullptr ||
                  h == nullptr || out == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(xp) || !aligned16(W1) || !aligned16(W2) || !aligned16(h) || !aligned16(out) ||
      !aligned4(offsets) || !aligned4(src_tok) || !aligned4(row_w) || !aligned4(stats))
    return MOE_ERR_ARG;
  const moe_ws_layout L = layout_of(c);
  if ((st = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return st;
  if ((st = check_device(true)) != MOE_OK) return st;
  if (c.T == 0) return MOE_OK;
  return experts_combine(c, xp, offsets, src_tok, row_w, W1, W2, h, static_cast<float*>(out), at<int>(ws, L.yp),
                         at<char>(ws, L.yp), stats, false, reinterpret_cast<cudaStream_t>(stream));
}

moe_status moe_combine(const moe_config* cfg, const void* yp, const int32_t* row_of,
                       const float* topk_w, void* out, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (c.T > 0 && (yp == nullptr || row_of == nullptr || topk_w == nullptr || out == nullptr)) return MOE_ERR_ARG;
  if (!aligned16(yp) || !aligned16(out) || !aligned4(row_of) || !aligned4(topk_w)) return MOE_ERR_ARG;
  if ((st = check_device(false)) != MOE_OK) return st;
  return cuda_status(launch_combine(c, yp, row_of, topk_w, out, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_layer_forward(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                             const void* W1, const void* W2, void* out, moe_stats* stats,
                             void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (x == nullptr || Wg == nullptr || W1 == nullptr || W2 == nullptr || out == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned4(bg) || !aligned16(W1) || !aligned16(W2) ||
      !aligned16(out) || !aligned4(stats))
    return MOE_ERR_ARG;
  const moe_ws_layout L = layout_of(c);
  if ((st = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return st;
  if ((st = check_device(c.dtype == MOE_DTYPE_BF16)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scr = at<char>(ws, L.scratch);
  const Scratch sc = scratch_layout(c);
  int32_t* idx = at<int32_t>(ws, L.topk_idx);
  float* w = at<float>(ws, L.topk_w);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  void* yp = at<char>(ws, L.yp);

  const bool fuse = fused_combine(c);
  // the tile queue's counters: the yp region when step 5 is fused (yp is
  // then never written), else the scratch region
  const bool plain1 = !fuse && one_launch_plain(c);
  int* counters = plain1 ? at<int>(scr, sc.mlp) : at<int>(ws, L.yp);
  if (cudaMemsetAsync(&stats->status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  // the tile-queue counters are zeroed by the scatter's prologue when it runs
  // scatter_kernel (no memset node between kernels), else here, ahead of the
  // kernel chain
  const bool mlp1 = one_launch(c) || plain1;
  const bool zero_in_scatter = mlp1 && scatter_zeroes(c);
  if (mlp1 && !zero_in_scatter &&
      cudaMemsetAsync(counters, 0, sizeof(int) * expert_mlp_counters(c), s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // steps 1-2: the route kernel also leaves the histogram, probability sums and
  // near-tie counts of every chunk in scratch, so step 3 starts from the
  // histograms (the scatter scans them itself)
  cudaError_t e = launch_route(c, x, Wg, bg, idx, w, at<float>(ws, L.gap), at<int32_t>(scr, sc.hist),
                               at<float>(scr, sc.psum), at<int32_t>(scr, sc.ntie), at<float>(scr, sc.zsum),
                               &stats->status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  float* row_w = at<float>(ws, L.row_w);
  float* out_f = static_cast<float*>(out);
  st = permute_from_hist(c, x, idx, nullptr, c.T > 0 ? at<float>(scr, sc.psum) : nullptr,
                         c.T > 0 ? at<int32_t>(scr, sc.ntie) : nullptr, c.T > 0 ? at<float>(scr, sc.zsum) : nullptr,
                         at<int32_t>(ws, L.counts),
                         at<int32_t>(ws, L.kept), offsets, row_of, at<int32_t>(ws, L.src_tok),
                         at<char>(ws, L.xp), stats, sc, scr, s, fuse ? w : nullptr, fuse ? row_w : nullptr,
                         fuse ? out_f : nullptr, zero_in_scatter ? counters : nullptr,
                         zero_in_scatter ? (int)expert_mlp_counters(c) : 0);
  if (st != MOE_OK) return st;
  if (fuse)   // steps 4-5: the second layer adds the gate-weighted expert outputs into out
    return experts_combine(c, at<char>(ws, L.xp), offsets, at<int32_t>(ws, L.src_tok), row_w, W1, W2,
                           at<char>(ws, L.h), out_f, counters, yp, stats, true, s);
  if (plain1)
    st = expert_mlp_plain(c, at<char>(ws, L.xp), offsets, W1, W2, at<char>(ws, L.h), yp, stats, counters, true,
                          s);
  else
    st = expert_ffn(c, at<char>(ws, L.xp), offsets, W1, W2, at<char>(ws, L.h), yp, stats, s);
  if (st != MOE_OK) return st;
  return cuda_status(launch_combine(c, yp, row_of, w, out, s));
}

moe_status moe_permute_static(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                              const float* gap, const float* prob_mean,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                              moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (counts == nullptr || kept == nullptr || offsets == nullptr || stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (x == nullptr || topk_idx == nullptr || row_of == nullptr || src_tok == nullptr || xp == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(xp) || !aligned4(topk_idx) || !aligned4(gap) || !aligned4(prob_mean) ||
      !aligned4(counts) || !aligned4(kept) || !aligned4(offsets) || !aligned4(row_of) || !aligned4(src_tok) ||
      !aligned4(stats))
    return MOE_ERR_ARG;
  const Scratch sc = scratch_layout(c);
  if (sc.total > (size_t)MOE_STATIC_SCRATCH_BYTES) return MOE_ERR_UNSUPPORTED;   // beyond the fixed array
  if ((st = check_device(false)) != MOE_OK) return st;
  void* ws = nullptr;
  if (static_scratch_address(&ws) != cudaSuccess) return MOE_ERR_CUDA;
  // the kernels of moe_permute, in the same order, on the library's array
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (cudaMemsetAsync(&stats->status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t e = launch_hist(c, topk_idx, gap, at<int32_t>(ws, sc.hist), at<int32_t>(ws, sc.ntie),
                              &stats->status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  return permute_from_hist(c, x, topk_idx, prob_mean, nullptr,
                           (gap != nullptr && c.T > 0) ? at<int32_t>(ws, sc.ntie) : nullptr, nullptr, counts, kept,
                           offsets, row_of, src_tok, xp, stats, sc, ws, s);
}

moe_status moe_aux_coef_update(const moe_stats* stats, float* coef, float beta, float xi, moe_stream_t stream) {
  if (stats == nullptr || coef == nullptr || !aligned4(stats) || !aligned4(coef)) return MOE_ERR_ARG;
  if (!(beta >= 0.f && beta <= 1.f) || !(xi >= 0.f) || !isfinite(xi)) return MOE_ERR_ARG;
  moe_status st = check_device(false);
  if (st != MOE_OK) return st;
  return cuda_status(launch_aux_coef_update(stats, coef, beta, xi, reinterpret_cast<cudaStream_t>(stream)));
}

moe_status moe_aux_coef_next(float coef, float drop_rate, float beta, float xi, float* next) {
  if (next == nullptr || !isfinite(coef) || !(drop_rate >= 0.f && drop_rate <= 1.f)) return MOE_ERR_ARG;
  if (!(beta >= 0.f && beta <= 1.f) || !(xi >= 0.f) || !isfinite(xi)) return MOE_ERR_ARG;
  *next = aux_coef_step(coef, drop_rate, beta, xi);
  return MOE_OK;
}

size_t moe_segments_scratch_size(const moe_config* cfg, int32_t nseg, int32_t rows) {
  if (check_config(cfg) != MOE_OK || nseg < 1 || nseg > kMaxExperts || rows < 0) return 0;
  const moe_config cc = segments_config(*cfg, nseg, rows);
  if (check_config(&cc) != MOE_OK) return 0;
  return scratch_layout(cc).total;
}

moe_status moe_expert_ffn_segments(const moe_config* cfg, int32_t nseg, int32_t rows, const int32_t* seg_offsets,
                                   const void* xp, const void* W1, const void* W2, void* h, void* yp,
                                   moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  if (nseg < 1 || rows < 0) return MOE_ERR_ARG;
  if (nseg > kMaxExperts) return MOE_ERR_UNSUPPORTED;
  const moe_config cc = segments_config(*cfg, nseg, rows);
  if ((st = check_config(&cc)) != MOE_OK) return st;
  if (seg_offsets == nullptr || stats == nullptr) return MOE_ERR_ARG;
  if (rows > 0 && (xp == nullptr || W1 == nullptr || W2 == nullptr || h == nullptr || yp == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(xp) || !aligned16(W1) || !aligned16(W2) || !aligned16(h) || !aligned16(yp) ||
      !aligned4(seg_offsets) || !aligned4(stats))
    return MOE_ERR_ARG;
  const Scratch sc = scratch_layout(cc);
  if ((st = check_ws(ws, ws_bytes, sc.total)) != MOE_OK) return st;
  if ((st = check_device(cc.dtype == MOE_DTYPE_BF16)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  if (rows == 0) return MOE_OK;
  if (one_launch_plain(cc))
    return expert_mlp_plain(cc, xp, seg_offsets, W1, W2, h, yp, stats, at<int>(ws, sc.mlp), false, s, cfg->E);
  return expert_ffn(cc, xp, seg_offsets, W1, W2, h, yp, stats, s, nullptr, cfg->E);
}

size_t moe_backward_workspace_size(const moe_config* cfg) {
  if (check_config(cfg) != MOE_OK) return 0;
  return bwd_layout(*cfg).total;
}

moe_status moe_layer_backward(const moe_config* cfg, const void* x, const void* Wg, const float* bg, const void* W1,
                              const void* W2, const float* dout, float aux_coef, float z_coef, const void* fws,
                              size_t fws_bytes, float* dx, float* dWg, float* dbg, float* dW1, float* dW2,
                              float* dw, moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (stats == nullptr || Wg == nullptr || W1 == nullptr || W2 == nullptr || dWg == nullptr || dW1 == nullptr ||
      dW2 == nullptr)
    return MOE_ERR_ARG;
  if (c.T > 0 && (x == nullptr || dout == nullptr || dx == nullptr)) return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned4(bg) || !aligned16(W1) || !aligned16(W2) || !aligned16(dout) ||
      !aligned16(dx) || !aligned16(dWg) || !aligned4(dbg) || !aligned16(dW1) || !aligned16(dW2) || !aligned4(dw) ||
      !aligned4(stats))
    return MOE_ERR_ARG;
  if (!isfinite(aux_coef) || !isfinite(z_coef)) return MOE_ERR_ARG;
  const moe_ws_layout FL = layout_of(c);
  if ((st = check_ws(const_cast<void*>(fws), fws_bytes, FL.total)) != MOE_OK) return st;
  const BwdLayout BL = bwd_layout(c);
  if ((st = check_ws(ws, ws_bytes, BL.total)) != MOE_OK) return st;
  if ((st = check_device(c.dtype == MOE_DTYPE_BF16)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  const int F1 = c.act == MOE_ACT_SWIGLU ? 2 * c.F : c.F;
  if (c.T == 0) {   // no token: every weight gradient is zero
    if (cudaMemsetAsync(dW1, 0, sizeof(float) * (size_t)c.E * F1 * c.d, s) != cudaSuccess ||
        cudaMemsetAsync(dW2, 0, sizeof(float) * (size_t)c.E * c.d * c.F, s) != cudaSuccess ||
        cudaMemsetAsync(dWg, 0, sizeof(float) * (size_t)c.E * c.d, s) != cudaSuccess ||
        (dbg != nullptr && cudaMemsetAsync(dbg, 0, sizeof(float) * (size_t)c.E, s) != cudaSuccess))
      return MOE_ERR_CUDA;
    return MOE_OK;
  }
  void* f = const_cast<void*>(fws);
  BwdState b{};
  b.topk_idx = at<int32_t>(f, FL.topk_idx);
  b.topk_w = at<float>(f, FL.topk_w);
  b.counts = at<int32_t>(f, FL.counts);
  b.offsets = at<int32_t>(f, FL.offsets);
  b.row_of = at<int32_t>(f, FL.row_of);
  b.src_tok = at<int32_t>(f, FL.src_tok);
  b.pad_offsets = at<int32_t>(ws, BL.pad_offsets);
  b.rows_alloc = BL.rows;
  b.xp = at<char>(ws, BL.xp);
  b.dout_perm = at<char>(ws, BL.dout_perm);
  b.wrow = at<float>(ws, BL.wrow);
  b.u = at<float>(ws, BL.u);
  b.du = at<char>(ws, BL.du);
  b.hw = at<char>(ws, BL.hw);
  b.dwpart = at<float>(ws, BL.dwpart);
  b.dxp = at<float>(ws, BL.dxp);
  b.z = at<float>(ws, BL.z);
  b.dz = at<float>(ws, BL.dz);
  b.dwg_part = at<float>(ws, BL.dwg_part);
  b.nsplit = BL.nsplit;
  b.tok_per_split = BL.tok_per_split;
  b.status = &stats->status;
  b.f16 = bwd_f16(c);
  b.amax = at<unsigned>(ws, BL.amax);
  b.scale = at<float>(ws, BL.scale);
  b.w1h = at<char>(ws, BL.w1h);
  // padded rows: x, dout and the gate weight of every kept assignment
  if (launch_bwd_front(c, x, dout, b, s) != cudaSuccess) return MOE_ERR_CUDA;
  // the first layer's pre-activation u = xp W1[e]^T, then the expert layers' gradients
  cudaError_t e;
  if (c.dtype == MOE_DTYPE_BF16) {
    const void* w1 = W1;
    if (b.f16) {   // fp16 operands: W1 converted once per call (kind::f16 takes one type for A and B)
      if (launch_convert_bf16_f16(W1, b.w1h, (size_t)c.E * F1 * c.d, s) != cudaSuccess) return MOE_ERR_CUDA;
      w1 = b.w1h;
    }
    // the recomputed pre-activation on 2-SM pair tiles when the segments are long, as the forward's layer 1
    e = pair_tiles(c) ? launch_grouped_plain_tc_pair(c, b.xp, b.pad_offsets, b.rows_alloc, w1, c.d, F1, b.u,
                                                     b.status, b.f16, s)
                      : launch_grouped_plain_tc(c, b.xp, b.pad_offsets, b.rows_alloc, w1, c.d, F1, b.u, b.status,
                                                b.f16, s);
    if (e == cudaSuccess) e = launch_expert_backward_tc(c, b, w1, W2, dW1, dW2, pair_tiles(c), s);
  } else {
    e = launch_grouped_plain_simt(c, b.xp, b.pad_offsets, b.rows_alloc, W1, c.d, F1, b.u, b.status, s);
    if (e == cudaSuccess) e = launch_expert_backward_simt(c, b, W1, W2, dW1, dW2, s);
  }
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  // the gate: scores, logits, dx and dW_gate
  return cuda_status(launch_bwd_gate(c, x, Wg, bg, b, aux_coef, z_coef, dx, dWg, dbg, dw, s));
}

size_t moe_mxfp8_weight_bytes(const moe_config* cfg, size_t* w1q, size_t* w1s, size_t* w2q, size_t* w2s) {
  if (check_mx_config(cfg) != MOE_OK) return 0;
  const moe_config& c = *cfg;
  const size_t F1 = c.act == MOE_ACT_SWIGLU ? 2 * (size_t)c.F : (size_t)c.F;
  const size_t a = (size_t)c.E * F1 * c.d, b = mx_scale_bytes((size_t)c.E * F1, (size_t)c.d);
  const size_t cq = (size_t)c.E * c.d * c.F, d = mx_scale_bytes((size_t)c.E * c.d, (size_t)c.F);
  if (w1q) *w1q = a;
  if (w1s) *w1s = b;
  if (w2q) *w2q = cq;
  if (w2s) *w2s = d;
  return a + b + cq + d;
}

moe_status moe_prepare_mxfp8_weights(const moe_config* cfg, const void* W1, const void* W2, void* W1q, void* W1s,
                                     void* W2q, void* W2s, moe_stream_t stream) {
  moe_status st = check_mx_config(cfg);
  if (st != MOE_OK) return st;
  if (W1 == nullptr || W2 == nullptr || W1q == nullptr || W1s == nullptr || W2q == nullptr || W2s == nullptr)
    return MOE_ERR_ARG;
  if (!aligned16(W1) || !aligned16(W2) || !aligned16(W1q) || !aligned16(W1s) || !aligned16(W2q) || !aligned16(W2s))
    return MOE_ERR_ARG;
  if ((st = check_device(false)) != MOE_OK) return st;
  return cuda_status(launch_mx_prepare_weights(*cfg, W1, W2, W1q, W1s, W2q, W2s,
                                               reinterpret_cast<cudaStream_t>(stream)));
}

size_t moe_workspace_size_mxfp8(const moe_config* cfg) {
  if (check_mx_config(cfg) != MOE_OK) return 0;
  return mx_layout(*cfg).total;
}

moe_status moe_layer_forward_mxfp8(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                                   const void* W1q, const void* W1s, const void* W2q, const void* W2s, void* out,
                                   moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream) {
  moe_status st = check_mx_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (stats == nullptr) return MOE_ERR_ARG;
  if (c.T > 0 && (x == nullptr || Wg == nullptr || W1q == nullptr || W1s == nullptr || W2q == nullptr ||
                  W2s == nullptr || out == nullptr))
    return MOE_ERR_ARG;
  if (!aligned16(x) || !aligned16(Wg) || !aligned4(bg) || !aligned16(W1q) || !aligned16(W1s) ||
      !aligned16(W2q) || !aligned16(W2s) || !aligned16(out) || !aligned4(stats))
    return MOE_ERR_ARG;
  const MxLayout M = mx_layout(c);
  const moe_ws_layout& L = M.base;
  if ((st = check_ws(ws, ws_bytes, M.total)) != MOE_OK) return st;
  if ((st = check_device(true)) != MOE_OK) return st;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  void* scr = at<char>(ws, L.scratch);
  const Scratch sc = scratch_layout(c);
  int32_t* idx = at<int32_t>(ws, L.topk_idx);
  float* w = at<float>(ws, L.topk_w);
  int32_t* row_of = at<int32_t>(ws, L.row_of);
  int32_t* offsets = at<int32_t>(ws, L.offsets);
  if (cudaMemsetAsync(&stats->status, 0, sizeof(uint32_t), s) != cudaSuccess) return MOE_ERR_CUDA;
  // steps 1-3 as the bf16 layer (the permuted rows in bf16, no fused combine)
  cudaError_t e = launch_route(c, x, Wg, bg, idx, w, at<float>(ws, L.gap), at<int32_t>(scr, sc.hist),
                               at<float>(scr, sc.psum), at<int32_t>(scr, sc.ntie), at<float>(scr, sc.zsum),
                               &stats->status, s);
  if (e != cudaSuccess) return MOE_ERR_CUDA;
  st = permute_from_hist(c, x, idx, nullptr, c.T > 0 ? at<float>(scr, sc.psum) : nullptr,
                         c.T > 0 ? at<int32_t>(scr, sc.ntie) : nullptr, c.T > 0 ? at<float>(scr, sc.zsum) : nullptr,
                         at<int32_t>(ws, L.counts), at<int32_t>(ws, L.kept), offsets, row_of,
                         at<int32_t>(ws, L.src_tok), at<char>(ws, L.xp), stats, sc, scr, s);
  if (st != MOE_OK) return st;
  // step 4 on the MX FP8 tensor cores, then step 5
  MxBuffers b{offsets, at<int32_t>(ws, M.pad), at<char>(ws, L.xp), M.rows_pad, at<char>(ws, M.xq),
              at<char>(ws, M.xs), at<char>(ws, M.hq), at<char>(ws, M.hs), at<int>(ws, M.ctr)};
  float* yp = at<float>(ws, L.yp);
  if (launch_mx_experts(c, b, W1q, W1s, W2q, W2s, yp, &stats->status, s) != cudaSuccess) return MOE_ERR_CUDA;
  return cuda_status(launch_combine(c, yp, row_of, w, out, s));
}

size_t moe_workspace_size_shared(const moe_config* cfg, int32_t F_shared) {
  if (check_config(cfg) != MOE_OK || F_shared < 1) return 0;
  moe_config one = *cfg;
  one.E = 1;
  one.k = 1;
  one.F = F_shared;
  if (check_config(&one) != MOE_OK) return 0;
  return shared_layout(*cfg, F_shared).total;
}

moe_status moe_layer_forward_shared(const moe_config* cfg, int32_t F_shared, const void* x, const void* Wg,
                                    const float* bg, const void* W1, const void* W2, const void* W1_shared,
                                    const void* W2_shared, void* out, moe_stats* stats, void* ws, size_t ws_bytes,
                                    moe_stream_t stream) {
  moe_status st = check_config(cfg);
  if (st != MOE_OK) return st;
  const moe_config& c = *cfg;
  if (F_shared < 1) return MOE_ERR_ARG;
  moe_config one = c;
  one.E = 1;
  one.k = 1;
  one.F = F_shared;
  if ((st = check_config(&one)) != MOE_OK) return st;
  if (c.T > 0 && (W1_shared == nullptr || W2_shared == nullptr)) return MOE_ERR_ARG;
  if (!aligned16(W1_shared) || !aligned16(W2_shared)) return MOE_ERR_ARG;
  const SharedLayout L = shared_layout(c, F_shared);
  if ((st = check_ws(ws, ws_bytes, L.total)) != MOE_OK) return st;
  // the routed experts into out, on the front of the workspace
  if ((st = moe_layer_forward(cfg, x, Wg, bg, W1, W2, out, stats, ws, L.base.total, stream)) != MOE_OK) return st;
  if (c.T == 0) return MOE_OK;
  cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
  // the shared expert over every token (one segment of T rows, x as the rows), then out += its output
  int32_t* seg = at<int32_t>(ws, L.seg);
  if (launch_fill_segment(seg, c.T, s) != cudaSuccess) return MOE_ERR_CUDA;
  const moe_config& sc = L.sc;
  void* scr = at<char>(ws, L.scratch);
  if (one_launch_plain(sc))
    st = expert_mlp_plain(sc, x, seg, W1_shared, W2_shared, at<char>(ws, L.h), at<char>(ws, L.y), stats,
                          at<int>(scr, scratch_layout(sc).mlp), false, s, 1);
  else
    st = expert_ffn(sc, x, seg, W1_shared, W2_shared, at<char>(ws, L.h), at<char>(ws, L.y), stats, s, nullptr, 1);
  if (st != MOE_OK) return st;
  return cuda_status(launch_add_rows(static_cast<float*>(out), at<float>(ws, L.y), (size_t)c.T * c.d, s));
}

moe_status moe_testing_set_expert_wait(uint64_t wait_ns, int32_t extra_dependency) {
  if (wait_ns > 60000000000ull || extra_dependency < 0) return MOE_ERR_ARG;
  set_expert_mlp_test_hooks(wait_ns, extra_dependency);
  return MOE_OK;
}

}  // extern "C"
