/*
 * moe.h -- C ABI of the B200 (sm_100a) top-k gated Mixture-of-Experts FFN
 * layer, forward pass, on one GPU.
 *
 * The layer (FastMoE announcement "智源x清华开源FastMoE", section
 * "1. MoE 设计", Figure 1): a gating network scores E experts for each token,
 * the k best are activated, and the token's output is the gate-weighted sum of
 * those k experts' outputs.  Five steps, each a hand-written CUDA kernel:
 *
 *   1. gate GEMM            z = x W_gate^T (+ b)
 *   2. normalise + top-k    optional z_hat = lambda (z - mean_e z) / std_e z,
 *                           p = softmax, top-k (lowest expert index wins ties),
 *                           weights = p of the selected experts / their sum
 *   3. permute              per-expert histogram + prefix sums group the
 *                           (token, slot) assignments by expert in ascending
 *                           token order; each expert keeps its first C
 *                           assignments (capacity mode) or all (dropless)
 *   4. expert FFN           grouped GEMMs over the variable-length expert
 *                           segments: ReLU MLP or SwiGLU
 *   5. combine              out[t] = sum over kept slots of w * expert output
 *
 * Conventions shared by every entry point:
 *   - Every data pointer is a DEVICE pointer owned by the caller, 16-byte
 *     aligned.  The library allocates no memory and never synchronises: work
 *     is enqueued on `stream` (NULL = legacy default stream) and returns.
 *   - Row-major layouts.  Weights use the nn.Linear [out, in] layout:
 *     W_gate[E, d]; W1[E, F1, d] with F1 = F (ReLU) or 2F (SwiGLU: rows [0, F)
 *     are the gate projection, rows [F, 2F) the up projection -- the order of
 *     the merged pair matters, Megatron-Core best-practice page, section
 *     "从HuggingFace到Megatron的权重转换要点"); W2[E, d, F].
 *   - Element type of x, W_gate, W1 and xp: bf16 (MOE_DTYPE_BF16, fp32
 *     accumulation, tcgen05 tensor cores) or fp32 (MOE_DTYPE_F32, CUDA-core
 *     FFMA throughout).  On the bf16 path the expert hidden activation h and
 *     W2 share moe_config.hidden_dtype: bf16, or fp16 (10-bit mantissa, 8x
 *     finer rounding of h; W2 then has to be given in fp16, see
 *     moe_convert_bf16_to_f16).  The expert outputs yp and the layer output out
 *     are fp32 for both paths (rounding them to bf16 would by itself use up
 *     most of the output tolerance on the largest elements).  Gate bias, gate
 *     weights (topk_w), gap and prob_mean are fp32; indices are int32.
 *   - Errors a host can see (bad arguments, unsupported shapes, too small a
 *     workspace, a failed launch) are returned synchronously and nothing is
 *     enqueued.  Errors only the device can see (an index out of range, a
 *     bounded wait that gave up) are OR-ed into moe_stats.status (device
 *     memory), which the caller reads after synchronising.
 *   - A = T*k assignments.  Buffers indexed by permuted row (src_tok, xp, h,
 *     yp) are sized for A rows (the dropless worst case); the rows in use are
 *     [0, offsets[E]).
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t; declared here so that callers need no CUDA header. */
typedef struct CUstream_st* moe_stream_t;

typedef enum moe_status {
  MOE_OK = 0,
  MOE_ERR_ARG = 1,         /* null or misaligned pointer, negative size, k > E, bad enum */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside the supported set (see moe_config) or no sm_100 device */
  MOE_ERR_WORKSPACE = 3,   /* ws is NULL, misaligned (256 B) or smaller than required */
  MOE_ERR_CUDA = 4         /* a CUDA runtime/driver call failed (launch, tensor-map encoding) */
} moe_status;

enum { MOE_ACT_RELU = 0, MOE_ACT_SWIGLU = 1 };
enum { MOE_DTYPE_F32 = 0, MOE_DTYPE_BF16 = 1, MOE_DTYPE_F16 = 2 };

/* Device-detected error bits in moe_stats.status. */
#define MOE_DEV_TIMEOUT 1u   /* a bounded wait inside a kernel gave up (~2 s); the kernel returned early */
#define MOE_DEV_BOUNDS  2u   /* an expert index or a row outside its buffer was seen and skipped */
#define MOE_DEV_RANGE   4u   /* an fp16 hidden activation exceeded +-65504 and was saturated */

/* Near-tie threshold: tokens whose k-th and (k+1)-th scores differ by less
 * than this are counted in moe_stats.near_tie_count. */
#define MOE_NEAR_TIE_GAP 1e-4f

/*
 * Layer shape and mode.
 *   T >= 0 tokens, d >= 1 model width, 1 <= E <= 256 experts, F >= 1 expert
 *   hidden width, 1 <= k <= E experts per token.
 *   bf16: d and F multiples of 16.  fp32: d and F multiples of 4.
 *   capacity_factor <= 0: dropless.  Otherwise the per-expert capacity is
 *     C = ceil((double)capacity_factor * (double)(T*k) / (double)E), computed on
 *     the host in that order from the float32 factor (Switch/GShard capacity;
 *     Megatron-Core best-practice page, section "MoE负载均衡的挑战与应对";
 *     Skywork-MoE slides, slide 4 "Preliminaries": based on Switch).
 *   lambda <= 0: plain softmax gating.  lambda > 0: gating-logit
 *     normalisation z_hat = lambda * (z - mean) / std over the E logits of a
 *     token (population std; zero spread gives z_hat = 0) before softmax and
 *     top-k (Skywork-MoE release, section "Gating Logits归一化操作"; slides,
 *     slide 6, "lambda = 1 seems to be the best value").
 */
typedef struct moe_config {
  int32_t T, d, E, F, k;
  int32_t act;               /* MOE_ACT_RELU | MOE_ACT_SWIGLU */
  int32_t dtype;             /* MOE_DTYPE_BF16 | MOE_DTYPE_F32 */
  float capacity_factor;     /* <= 0: dropless */
  float lambda;              /* <= 0: plain softmax */
  int32_t hidden_dtype;      /* element type of h and W2: MOE_DTYPE_BF16 | MOE_DTYPE_F16 on the
                                bf16 path, MOE_DTYPE_F32 on the fp32 path */
} moe_config;

/* Per-forward statistics, in DEVICE memory, written by moe_permute (and by
 * moe_layer_forward).  Drop-token rate and load balance are the quantities the
 * Skywork-MoE adaptive aux-loss controller monitors (Skywork-MoE release,
 * section "2.自适应的Aux Loss"; see moe_aux_coef_update).  The router z-loss
 * is the Z-Loss the Megatron-Core best-practice page names among its
 * load-balancing methods (section "Megatron-Core MoE的关键特性"); the pages
 * give no formula, and the one above is the reading this library takes. */
typedef struct moe_stats {
  int32_t drop_count;        /* assignments dropped by the capacity */
  int32_t rows_kept;         /* offsets[E] = T*k - drop_count */
  int32_t capacity;          /* C, or -1 in dropless mode */
  int32_t near_tie_count;    /* tokens with gap < MOE_NEAR_TIE_GAP; -1 if gap was not given */
  float drop_rate;           /* drop_count / (T*k); 0 when T == 0 */
  float aux_loss;            /* E * sum_e (counts_e/(T*k)) * P_e (pre-drop counts); NaN if P not given or T == 0 */
  uint32_t status;           /* MOE_DEV_* bits; cleared by moe_permute, OR-ed by later steps */
  float z_loss;              /* router z-loss (1/T) sum_t (log sum_e exp s[t, e])^2 over the scores the
                                softmax takes (z_hat when lambda > 0, else z); written by
                                moe_layer_forward, NaN from a standalone moe_permute or when T == 0 */
} moe_stats;

/* Byte offsets of the intermediates inside a moe_layer_forward workspace
 * (each 256-byte aligned), so that a caller can read them after a forward.
 * row_w[A] fp32 holds the gate weight of each kept permuted row.  On the bf16
 * path with k <= 2 the forward fuses step 5 into the second expert GEMM: it
 * writes row_w and leaves yp unwritten; otherwise it writes yp and not row_w. */
typedef struct moe_ws_layout {
  size_t topk_idx, topk_w, gap, counts, kept, offsets, row_of, src_tok, row_w;
  size_t xp, h, yp, scratch, total;
} moe_ws_layout;

/* Human-readable name of a status code (static string, never NULL). */
const char* moe_status_string(moe_status s);

/* Scratch bytes the step calls (moe_route, moe_permute, moe_expert_ffn) need
 * in `ws`; 0 when cfg is invalid. */
size_t moe_scratch_size(const moe_config* cfg);

/* Workspace bytes moe_layer_forward needs (all intermediates + scratch); 0
 * when cfg is invalid.  Fills *layout when it is not NULL. */
size_t moe_workspace_size(const moe_config* cfg, moe_ws_layout* layout);

/*
 * Steps 1-2: gate GEMM, optional normalisation, softmax, top-k.
 * FastMoE announcement, "特色二" (the gate is one fully-connected layer) and
 * "图4" (top-2 gate: the two highest-scoring experts are activated).
 *   x[T, d], Wg[E, d] (cfg dtype); bg[E] fp32 or NULL (no bias).
 *   topk_idx[T, k] int32: selected experts, best first; equal scores resolve
 *     to the lower expert index.  A NaN or -inf score is never selected: a
 *     token with fewer than k scores above -inf (NaN logits) keeps 2^31 - 1
 *     in its remaining slots, which the permutation drops; in
 *     moe_layer_forward such a token sets MOE_DEV_BOUNDS and its output row
 *     is 0.
 *   topk_w[T, k] fp32: softmax probabilities of the selected experts divided
 *     by their sum (they sum to 1).
 *   gap[T] fp32: k-th minus (k+1)-th largest score (z_hat or z), +inf if k == E.
 *   prob_mean[E] fp32 or NULL: P_e = mean over tokens of the full softmax
 *     probability of expert e (input of the aux loss).
 *   z_loss fp32 scalar or NULL: the router z-loss of the batch (moe_stats.z_loss).
 *   ws: at least moe_scratch_size(cfg) bytes.
 */
moe_status moe_route(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                     int32_t* topk_idx, float* topk_w, float* gap, float* prob_mean, float* z_loss,
                     void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Step 3: histogram, prefix sums, stable ranks, capacity drop, gather.
 * Megatron-Core best-practice page, sections "MoE负载均衡的挑战与应对" (expert
 * capacity; overflow tokens are dropped and carried by the residual; dropless
 * alternative) and "Megatron-Core MoE的关键特性" (token permutation kernels).
 *   topk_idx[T, k] int32 (an index outside [0, E) sets MOE_DEV_BOUNDS and the
 *     slot is treated as dropped).
 *   gap[T] fp32 or NULL: only used for near_tie_count.
 *   prob_mean[E] fp32 or NULL: only used for aux_loss.
 *   counts[E]: assignments per expert; kept[E]: after the capacity;
 *   offsets[E+1]: exclusive prefix sum of kept (expert e owns permuted rows
 *     [offsets[e], offsets[e+1]) in ascending token order).
 *   row_of[T, k]: permuted row of slot (t, j), -1 if dropped.
 *   src_tok[A]: token of each permuted row (rows >= offsets[E] untouched).
 *   xp[A, d]: xp[row] = x[src_tok[row]].
 *   stats: device moe_stats (required).
 */
moe_status moe_permute(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                       const float* gap, const float* prob_mean,
                       int32_t* counts, int32_t* kept, int32_t* offsets,
                       int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                       void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Step 4: the experts over their row segments, one grouped GEMM per layer.
 * Megatron-Core best-practice page, "Megatron-Core MoE的关键特性"
 * (GroupedGEMM merges the experts' small GEMMs into one kernel); FastMoE
 * announcement, Transformer-XL experiment (two-layer ReLU MLP experts).
 *   ReLU:   h = relu(xp W1[e]^T);  SwiGLU: h = silu(xp Wg_e^T) * (xp Wu_e^T),
 *           silu(u) = u / (1 + exp(-u));   then yp = h W2[e]^T.
 *   xp[A, d], offsets[E+1] (device, from moe_permute), W1[E, F1, d],
 *   W2[E, d, F] (hidden_dtype); h[A, F] (hidden_dtype) and yp[A, d] fp32 are
 *   written for rows [0, offsets[E]).
 *   bf16 path: the activation is computed in fp32 from the fp32 accumulator and
 *   h is rounded once to hidden_dtype (it is the tensor-core operand of the
 *   second layer); fp16 h saturates at +-65504 and sets MOE_DEV_RANGE.
 *   stats: device moe_stats; a kernel timeout ORs MOE_DEV_TIMEOUT into status.
 *   ws: at least moe_scratch_size(cfg) bytes.
 */
moe_status moe_expert_ffn(const moe_config* cfg, const void* xp, const int32_t* offsets,
                          const void* W1, const void* W2, void* h, void* yp,
                          moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Steps 4-5 fused, as moe_layer_forward runs them on the bf16 path with
 * k <= 2: the expert FFNs of moe_expert_ffn, each kept row's output added,
 * times its gate weight, straight into the token's row of out.  No yp is
 * formed.  Megatron-Core best-practice page, "Megatron-Core MoE的关键特性"
 * (GroupedGEMM); FastMoE announcement, "1. MoE 设计" (the output is the
 * gate-weighted sum of the selected experts' outputs).
 *   xp[A, d], offsets[E+1], W1, W2, h: as moe_expert_ffn.
 *   src_tok[A]: token of each permuted row (from moe_permute).
 *   row_w[A] fp32: gate weight of each kept row (the row_w region of a
 *     moe_layer_forward workspace holds it after a forward).
 *   out[T, d] fp32: must hold zeros on entry; each element receives at most
 *     two additions (k <= 2) onto that exact zero, so the result does not
 *     depend on their order.
 *   ws: a moe_layer_forward workspace (moe_workspace_size bytes); its yp
 *     region is used for the tile scheduler's counters.
 *   MOE_ERR_UNSUPPORTED unless dtype is bf16 and k <= 2.
 */
moe_status moe_expert_ffn_combine(const moe_config* cfg, const void* xp, const int32_t* offsets,
                                  const int32_t* src_tok, const float* row_w, const void* W1, const void* W2,
                                  void* h, void* out, moe_stats* stats, void* ws, size_t ws_bytes,
                                  moe_stream_t stream);

/*
 * Step 4 over caller-given row segments that share the weights of E experts:
 * the expert-parallel form of the step.  With the experts partitioned over G
 * GPUs (FastMoE announcement, "特色四", Figure 6: each worker holds its own
 * experts and the inputs of an expert are sent to its worker), a GPU receives
 * from each of the G source ranks that rank's rows for its E local experts,
 * expert by expert; the G blocks of E segments are run as they arrived.
 * Segment i holds rows [seg_offsets[i], seg_offsets[i+1]) of xp and runs
 * through local expert i % E:
 *   cfg: d, F, act, dtype, hidden_dtype as for the layer; E = the experts
 *     whose weights W1[E, F1, d] and W2[E, d, F] are given; T, k,
 *     capacity_factor and lambda are ignored.
 *   nseg (1..256) segments over a buffer of `rows` rows: seg_offsets[nseg+1]
 *     device int32, non-decreasing inside [0, rows] (else MOE_DEV_BOUNDS and
 *     nothing is computed); xp[rows, d], h[rows, F] (hidden_dtype) and
 *     yp[rows, d] fp32 as in moe_expert_ffn, written for rows
 *     [0, seg_offsets[nseg]).
 *   ws: at least moe_segments_scratch_size(cfg, nseg, rows) bytes.
 */
size_t moe_segments_scratch_size(const moe_config* cfg, int32_t nseg, int32_t rows);
moe_status moe_expert_ffn_segments(const moe_config* cfg, int32_t nseg, int32_t rows, const int32_t* seg_offsets,
                                   const void* xp, const void* W1, const void* W2, void* h, void* yp,
                                   moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Step 5: un-permute and combine.  out[t] = sum over j = 0..k-1 with
 * row_of[t, j] >= 0 of topk_w[t, j] * yp[row_of[t, j]], accumulated in fp32 in
 * slot order; 0 for a token whose slots were all dropped (the residual path
 * outside the layer carries it: Megatron-Core best-practice page, section
 * "MoE负载均衡的挑战与应对").
 *   yp[A, d] fp32, row_of[T, k], topk_w[T, k] -> out[T, d] fp32.
 */
moe_status moe_combine(const moe_config* cfg, const void* yp, const int32_t* row_of,
                       const float* topk_w, void* out, moe_stream_t stream);

/*
 * The whole layer: steps 1-5 back to back on `stream`, intermediates inside
 * `ws` (layout from moe_workspace_size).  No host synchronisation and no
 * device-to-host copy, so it may be captured in a CUDA graph.
 *   x[T, d], Wg[E, d], bg[E] or NULL, W1[E, F1, d], W2[E, d, F] -> out[T, d] fp32;
 *   stats: device moe_stats (required).
 */
moe_status moe_layer_forward(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                             const void* W1, const void* W2, void* out, moe_stats* stats,
                             void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The backward of the layer: the gradients of
 *     L = sum_{t,i} dout[t, i] out[t, i] + aux_coef * aux_loss + z_coef * z_loss
 * with respect to x, W_gate, the gate bias, W1 and W2, for a forward already
 * run by moe_layer_forward on the same inputs.  The layer's figures on the
 * pages are training figures (FastMoE announcement, "特色三"; Skywork-MoE
 * release, "训练Infra"), and the aux loss (Switch form, pre-drop counts) and
 * its coefficient and the z-loss are those of moe_stats and moe_aux_coef_update.
 * The forward's discrete choices (selected experts, capacity drops, counts)
 * carry no gradient and are read from its workspace `fws`.
 *   x, Wg, bg (or NULL), W1, W2: as for the forward (W2 in hidden_dtype).
 *   dout[T, d] fp32: the gradient of L with respect to out.
 *   fws: the workspace of that forward (moe_workspace_size bytes), unchanged
 *     since.
 *   Outputs, all fp32 and fully written: dx[T, d], dWg[E, d], dbg[E] (or
 *     NULL), dW1[E, F1, d], dW2[E, d, F]; dw[T, k] (or NULL): the gradient of
 *     the gate weights topk_w (0 for a dropped slot).
 *   ws: at least moe_backward_workspace_size(cfg) bytes (256-byte aligned).
 *   stats: device moe_stats; device-detected errors are OR-ed into status
 *     (clear it before the call for a clean record).
 * The expert GEMMs run on the tensor cores on the bf16 path, with fp32
 * accumulation and operands of the hidden type: with fp16 (the default),
 * dout is scaled by a power of two s so that max|s dout| lies in [512, 1024),
 * x, W1, s dout, s du and w h are rounded to fp16 (saturating at +-65504, which
 * sets MOE_DEV_RANGE) and every result is scaled back by 1/s; with bf16 they
 * are bf16.  The fp32 path runs in fp32 FFMA.  The gate's gradient, dx and
 * dW_gate are fp32.  Gradients are written, never accumulated into.
 */
size_t moe_backward_workspace_size(const moe_config* cfg);
moe_status moe_layer_backward(const moe_config* cfg, const void* x, const void* Wg, const float* bg, const void* W1,
                              const void* W2, const float* dout, float aux_coef, float z_coef, const void* fws,
                              size_t fws_bytes, float* dx, float* dWg, float* dbg, float* dW1, float* dW2,
                              float* dw, moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * The layer with a shared expert: every token also goes, with weight 1 and
 * outside the routing, through one more expert whose output is added to the
 * routed experts' sum (the MoE survey page, "MoE未来重点研究方向", item 4:
 * DeepSeekMoE's shared experts).  Several shared experts are one shared expert
 * of their summed hidden width F_shared (W1 rows stacked -- for SwiGLU all the
 * gate rows, then all the up rows -- and W2 columns side by side).
 *   W1_shared[F1s, d] (F1s = F_shared or 2 F_shared) in the element type of x,
 *   W2_shared[d, F_shared] in hidden_dtype; everything else as
 *   moe_layer_forward, whose workspace layout the first moe_workspace_size(cfg)
 *   bytes of ws keep.  ws: at least moe_workspace_size_shared(cfg, F_shared)
 *   bytes (0 when F_shared is not a supported width).
 */
size_t moe_workspace_size_shared(const moe_config* cfg, int32_t F_shared);
moe_status moe_layer_forward_shared(const moe_config* cfg, int32_t F_shared, const void* x, const void* Wg,
                                    const float* bg, const void* W1, const void* W2, const void* W1_shared,
                                    const void* W2_shared, void* out, moe_stats* stats, void* ws, size_t ws_bytes,
                                    moe_stream_t stream);

/*
 * The layer with FP8 expert weights.  The Skywork-MoE release serves its model
 * with FP8 weights (inference section: 146 GB on an 8 x 4090 server); the
 * pages fix no FP8 format.  This library takes the microscaled (MX) form the
 * B200 tensor cores run natively (tcgen05.mma kind::mxf8f6f4): E4M3 elements
 * and one power-of-two scale (UE8M0) per 32 consecutive elements along the
 * reduction.  A block's scale 2^X is the least that brings every |v| / 2^X
 * within 448, and elements round to the nearest E4M3 value, ties to even.
 * Both expert layers run on it: the weights are quantised once by
 * moe_prepare_mxfp8_weights, the layer-1 input rows and the hidden activation
 * on every call.  Routing, permutation and combine are the bf16 layer's.
 *   Shapes: the bf16 path with d and F multiples of 128 (else
 *     MOE_ERR_UNSUPPORTED); cfg.hidden_dtype is not used.
 *   moe_mxfp8_weight_bytes: bytes of the four prepared arrays (returned
 *     through the pointers that are not NULL) and their sum; 0 for an
 *     unsupported cfg.
 *   moe_prepare_mxfp8_weights: W1[E, F1, d] and W2[E, d, F] bf16 (device) ->
 *     W1q, W1s, W2q, W2s (device, 16-byte aligned, sizes from
 *     moe_mxfp8_weight_bytes).  Their layout is the kernels' own (scales in
 *     512-byte atoms of 128 rows x 4 blocks; a SwiGLU expert's W1 rows
 *     interleaved gate/up by 64) and is read only by this library.
 *   moe_layer_forward_mxfp8: as moe_layer_forward with the prepared weights;
 *     ws: at least moe_workspace_size_mxfp8(cfg) bytes, whose first
 *     moe_workspace_size(cfg) bytes have the moe_ws_layout of the bf16 forward
 *     (yp holds the fp32 expert outputs; the fused combine is not used).
 */
size_t moe_mxfp8_weight_bytes(const moe_config* cfg, size_t* w1q, size_t* w1s, size_t* w2q, size_t* w2s);
moe_status moe_prepare_mxfp8_weights(const moe_config* cfg, const void* W1, const void* W2, void* W1q, void* W1s,
                                     void* W2q, void* W2s, moe_stream_t stream);
size_t moe_workspace_size_mxfp8(const moe_config* cfg);
moe_status moe_layer_forward_mxfp8(const moe_config* cfg, const void* x, const void* Wg, const float* bg,
                                   const void* W1q, const void* W1s, const void* W2q, const void* W2s, void* out,
                                   moe_stats* stats, void* ws, size_t ws_bytes, moe_stream_t stream);

/*
 * Weight preparation (run once when the weights are loaded, not per forward):
 * dst[i] = fp16(src[i]) for n bf16 values, round to nearest even; values
 * beyond the fp16 range saturate to +-65504.  Every bf16 value of magnitude in
 * [2^-17, 65504] converts exactly; smaller ones round to fp16 subnormals.
 * Used to give W2 to the layer when hidden_dtype is MOE_DTYPE_F16.
 * src and dst: device, 16-byte aligned, not overlapping.  No counterpart on
 * the pages: it prepares the storage format of the second expert layer.
 */
moe_status moe_convert_bf16_to_f16(const void* src, void* dst, size_t n, moe_stream_t stream);

/*
 * Layer-wise adaptive aux-loss coefficient (Skywork-MoE release, section
 * "2.自适应的Aux Loss"; slides, slide 7: each layer's coefficient is raised
 * when its token drop rate rises and lowered when it falls, to keep the drop
 * rate in a suitable band).  The pages give no formula; the reading taken is
 * an exponential moving average of a target proportional to the drop rate:
 *     coef <- beta * coef + (1 - beta) * xi * drop_rate
 * with smoothing 0 <= beta <= 1 and sensitivity xi >= 0 (both finite).
 *
 * moe_aux_coef_update: on the device, after a forward: reads stats->drop_rate
 *   (device moe_stats of that layer) and updates *coef (device fp32) in place,
 *   one thread on `stream`, no host synchronisation.  MOE_ERR_ARG for a NULL
 *   or misaligned pointer or beta / xi out of range.
 * moe_aux_coef_next: the same step on the host: *next = the updated value of
 *   coef given drop_rate (0 <= drop_rate <= 1).  MOE_ERR_ARG on a bad value.
 */
moe_status moe_aux_coef_update(const moe_stats* stats, float* coef, float beta, float xi, moe_stream_t stream);
moe_status moe_aux_coef_next(float coef, float drop_rate, float beta, float xi, float* next);

/*
 * Test hook for the failure path of the bounded waits.  No counterpart on the
 * pages.  Every wait inside the kernels gives up after a limit (2 s by
 * default), sets MOE_DEV_TIMEOUT in moe_stats.status, stops the kernel's other
 * roles, waits for its own copies and MMAs in flight, frees its tensor memory
 * and returns, so that the context stays usable.  This call lets a test reach
 * that path without a GPU fault, in the one-launch expert kernel (bf16 path,
 * 1-SM tiles, the kernel moe_layer_forward and moe_expert_ffn run on layers
 * with T*k < 512*E):
 *   wait_ns: limit of that kernel's waits in ns (0 = the default 2 s; at most
 *     60 s);
 *   extra_dependency: added to the number of layer-1 releases a layer-2 tile
 *     waits for (0 = none; > 0 makes that wait unreachable, so it runs out).
 * The setting is process-wide and applies to launches made after the call;
 * MOE_ERR_ARG for wait_ns > 60 s or extra_dependency < 0.  Not for use
 * outside tests.
 */
moe_status moe_testing_set_expert_wait(uint64_t wait_ns, int32_t extra_dependency);

/* Size of the library's fixed device scratch array used by moe_permute_static. */
#define MOE_STATIC_SCRATCH_BYTES (2u << 20)

/*
 * moe_permute without a caller workspace: the same kernels and results, with
 * their scratch (per-chunk histograms, chunk offsets, near-tie counts) in one
 * fixed device array of MOE_STATIC_SCRATCH_BYTES bytes that the library owns,
 * one per device.  It allocates nothing: no cudaMalloc, no cudaFree, no
 * allocating library routine.  No counterpart on the pages: it is a calling
 * convention for users that cannot hand out device memory.
 *   Arguments, layout, ownership and results: as moe_permute, minus ws.
 *   Limit: moe_scratch_size(cfg) <= MOE_STATIC_SCRATCH_BYTES, else
 *     MOE_ERR_UNSUPPORTED before any device work (e.g. E = 64 experts, k = 2
 *     allows T up to about 342k tokens on the bf16 path, 345k on fp32).
 *   The first call on a device looks up the array's address (that device
 *     must be current; make this first call before any stream capture) and
 *     returns MOE_ERR_CUDA if the lookup fails; a failed lookup is retried by
 *     the next call, a successful one is kept for the life of the process.
 *     cudaDeviceReset destroys the array, and the kept address with it: do
 *     not call this entry point on a device after resetting it.
 *   Every scratch word the kernels read is written earlier in the same call;
 *     the one value that must start at zero, stats->status, is cleared by the
 *     call on `stream`.
 *   Calls that overlap in time on one device (several streams or host
 *     threads) share the array and race: the caller must serialise them.
 */
moe_status moe_permute_static(const moe_config* cfg, const void* x, const int32_t* topk_idx,
                              const float* gap, const float* prob_mean,
                              int32_t* counts, int32_t* kept, int32_t* offsets,
                              int32_t* row_of, int32_t* src_tok, void* xp, moe_stats* stats,
                              moe_stream_t stream);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
