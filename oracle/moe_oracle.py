"""Float64 CPU oracle for the forward pass of a top-k gated MoE FFN layer.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline / reference legs of ``bench.py`` may import this module.  The
CUDA product path never imports, calls or links it, and it shares no code,
tables or helpers with that path.  The only module both sides use is the
seeded input generator ``moe_workloads``, which holds none of this arithmetic.

Everything here is plain NumPy in float64 (the stored bf16/fp32 inputs are
upcast exactly), written to be checked against the pages by eye:

* The layer (FastMoE announcement, "1. MoE 设计" and Figure 1): a gating
  network scores the n experts for each input and activates the k best; the
  output is the gate-weighted sum of the k activated experts' outputs.
* The gate is one fully-connected layer (FastMoE announcement, "特色二").
* Gating-logit normalisation (Skywork-MoE release, "技术创新 1. Gating Logits
  归一化操作"; Skywork-MoE slides, slide 6 "Gating Logit Normalization",
  "lambda = 1 seems to be the best value").  The formula itself did not survive
  on the page; the reading used is: standardise the logits over the experts
  (population standard deviation), multiply by lambda, then softmax.
* Top-k with the lowest expert index winning equal scores.
* Expert capacity and token dropping: tokens beyond an expert's capacity are
  dropped and only the residual path carries them (Megatron-Core best-practice
  page, "MoE负载均衡的挑战与应对" and its Q&A); dropless mode keeps all
  (Skywork-MoE slides, slide 10 "Discussion").  Capacity is the Switch/GShard
  form C = ceil(cf * T * k / E) (the slides' slide 4 "Preliminaries": the
  architecture is based on Switch Transformers); priority is by ascending
  token index within each expert.
* Load-balancing auxiliary loss (Megatron-Core page, same section; the
  Skywork slides' slide 7 formula is blank): Switch form
  aux = E * sum_e f_e * P_e with f_e the fraction of pre-drop assignments to
  expert e and P_e the mean full-softmax probability of expert e.
* Router z-loss (Megatron-Core page, "Megatron-Core MoE的关键特性", which
  names Z-Loss among the load-balancing methods without a formula).  Reading:
  the mean over tokens of the squared log-partition function of the scores the
  softmax takes (z_hat when lambda > 0, else z).
* Adaptive aux-loss coefficient (Skywork-MoE release, "2.自适应的Aux Loss";
  slides, slide 7: layer-wise coefficients, raised when the token drop rate
  rises and lowered when it falls; the formula itself is not on the pages).
  Reading: per layer, alpha <- beta * alpha + (1 - beta) * xi * drop_rate, an
  exponential moving average of a target proportional to the drop rate.
* Experts: two-layer MLP with ReLU (FastMoE announcement, Transformer-XL
  experiment: 512->1024->512) or the gated SwiGLU pair whose gate and up
  projections are stored concatenated, gate first (Megatron-Core page,
  "从HuggingFace到Megatron的权重转换要点": the order of gate_proj/up_proj
  in dense_h_to_4h matters).

Parity pins: every function here is checked in ``tests/test_oracle_pins.py``
against brute force, closed forms, invariants and textbook special cases.  The
numeric form of the normalisation and of the aux loss is pinned to the
readings above, not to the pages (whose formulas are missing).
"""
from __future__ import annotations

import dataclasses
import math
from typing import Optional, Sequence

import numpy as np

RELU = "relu"
SWIGLU = "swiglu"


@dataclasses.dataclass(frozen=True)
class LayerConfig:
    """Shape and mode of one MoE layer.

    capacity_factor <= 0 selects dropless mode; lam <= 0 selects plain softmax
    gating.  capacity_factor is held as the float32 value the C ABI receives.
    """

    T: int
    d: int
    E: int
    F: int
    k: int
    act: str = RELU
    capacity_factor: float = 0.0
    lam: float = 0.0

    @classmethod
    def from_workload(cls, w, T: Optional[int] = None) -> "LayerConfig":
        return cls(T=w.T if T is None else T, d=w.d, E=w.E, F=w.F, k=w.k, act=w.act,
                   capacity_factor=w.capacity_factor, lam=w.lam)


# ---------------------------------------------------------------- step 1: gate
def gate_logits(x: np.ndarray, wg: np.ndarray, bias: Optional[np.ndarray] = None) -> np.ndarray:
    """z[t, e] = sum_i x[t, i] * W_gate[e, i] (+ b[e]).

    FastMoE announcement, "特色二": the gate is a single fully-connected layer.
    """
    z = np.asarray(x, np.float64) @ np.asarray(wg, np.float64).T
    if bias is not None:
        z = z + np.asarray(bias, np.float64)[None, :]
    return z


# ------------------------------------------------------- step 2: normalise/top-k
def normalise_logits(z: np.ndarray, lam: float) -> np.ndarray:
    """Gating-logit normalisation over the expert axis.

    Skywork-MoE release, "Gating Logits归一化操作" / slides, slide 6.  Reading:
    z_hat = lam * (z - mean_e z) / std_e z with the population standard deviation
    (divide by E).  A row with zero spread maps to all zeros.  lam <= 0 returns z
    unchanged (plain softmax gating).
    """
    if lam <= 0:
        return np.array(z, dtype=np.float64, copy=True)
    mu = z.mean(axis=1, keepdims=True)
    sd = np.sqrt(((z - mu) ** 2).mean(axis=1, keepdims=True))
    out = np.zeros_like(z)
    nz = sd[:, 0] > 0
    out[nz] = lam * (z[nz] - mu[nz]) / sd[nz]
    return out


def softmax(s: np.ndarray) -> np.ndarray:
    """Row softmax over experts, max subtracted first."""
    m = s.max(axis=1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=1, keepdims=True)


def top_k(s: np.ndarray, k: int):
    """Indices of the k largest scores per row, largest first; equal scores are
    ordered by ascending expert index (a stable sort on -s).

    Returns (idx[T, k], gap[T]) with gap = k-th largest - (k+1)-th largest score
    (+inf when k == E), the margin that decides the selected set.
    """
    order = np.argsort(-s, axis=1, kind="stable")
    idx = order[:, :k]
    T, E = s.shape
    rows = np.arange(T)
    if k < E:
        gap = s[rows, order[:, k - 1]] - s[rows, order[:, k]]
    else:
        gap = np.full(T, np.inf)
    return idx.astype(np.int64), gap


@dataclasses.dataclass
class Routing:
    s: np.ndarray        # scores the top-k is taken on: z_hat (lam > 0) or z   [T, E]
    p: np.ndarray        # full softmax probabilities                          [T, E]
    idx: np.ndarray      # selected experts, best first                         [T, k]
    w: np.ndarray        # renormalised gate weights of the selected experts    [T, k]
    gap: np.ndarray      # k-th minus (k+1)-th score                            [T]
    prob_mean: np.ndarray  # P_e = mean_t p[t, e]                               [E]
    z_loss: float = float("nan")  # mean_t (log sum_e exp s[t, e])^2 (NaN when T == 0)


def route(x, wg, bias, cfg: LayerConfig, forced_mask: Optional[np.ndarray] = None,
          forced_idx: Optional[np.ndarray] = None) -> Routing:
    """Steps 1-2: logits, optional normalisation, softmax, top-k, weights.

    The k selected experts' weights are their softmax probabilities divided by
    the probabilities' sum over the selected set (so they sum to 1).

    ``forced_mask`` / ``forced_idx`` replace the selection of the masked tokens
    by a given one (used where the device took the other side of a near-tie);
    their weights are then recomputed from this oracle's own probabilities.
    """
    z = gate_logits(x, wg, bias)
    s = normalise_logits(z, cfg.lam)
    p = softmax(s)
    idx, gap = top_k(s, cfg.k)
    if forced_mask is not None:
        idx = idx.copy()
        idx[forced_mask] = np.asarray(forced_idx)[forced_mask]
    psel = np.take_along_axis(p, idx, axis=1)
    w = psel / psel.sum(axis=1, keepdims=True)
    return Routing(s=s, p=p, idx=idx, w=w, gap=gap, prob_mean=p.mean(axis=0), z_loss=z_loss(s))


def log_partition(s: np.ndarray) -> np.ndarray:
    """lse[t] = log sum_e exp(s[t, e]), the row maximum taken out first."""
    m = s.max(axis=1)
    return m + np.log(np.exp(s - m[:, None]).sum(axis=1))


def z_loss(s: np.ndarray) -> float:
    """Router z-loss: (1/T) sum_t (log sum_e exp s[t, e])^2 over the scores the
    softmax takes (Megatron-Core page, "Megatron-Core MoE的关键特性": Z-Loss; the
    formula is this reading).  NaN for an empty batch."""
    if s.shape[0] == 0:
        return float("nan")
    return float(np.mean(log_partition(s) ** 2))


def adaptive_aux_coef(alpha: float, drop_rate: float, beta: float, xi: float) -> float:
    """One step of the layer-wise adaptive aux-loss coefficient (Skywork-MoE
    release, "2.自适应的Aux Loss"; slides, slide 7: raise the coefficient when
    the drop rate rises, lower it when it falls).  Reading: the coefficient is
    an exponential moving average, with smoothing beta, of xi times the drop
    rate of the step just taken."""
    return beta * alpha + (1.0 - beta) * xi * drop_rate


# ---------------------------------------------------- step 3: capacity/permute
def capacity(cfg: LayerConfig) -> Optional[int]:
    """Expert capacity in assignments, C = ceil(cf * (T*k) / E), evaluated in
    double precision in that order; None in dropless mode (cf <= 0)."""
    cf = float(np.float32(cfg.capacity_factor))
    if cf <= 0:
        return None
    return int(math.ceil(cf * float(cfg.T * cfg.k) / float(cfg.E)))


@dataclasses.dataclass
class Dispatch:
    C: Optional[int]
    counts: np.ndarray    # assignments per expert before dropping      [E]
    kept: np.ndarray      # assignments per expert after dropping       [E]
    offsets: np.ndarray   # exclusive prefix sum of kept                [E+1]
    row_of: np.ndarray    # permuted row of assignment (t, j), -1 if dropped  [T, k]
    src_tok: np.ndarray   # token of each permuted row                  [A_kept]
    drop_count: int
    drop_rate: float
    aux: float


def dispatch(idx: np.ndarray, cfg: LayerConfig, prob_mean: Optional[np.ndarray] = None) -> Dispatch:
    """Step 3: group assignments by expert, ascending token index inside each
    expert; keep the first C of each expert (all in dropless mode).

    Per-expert counts, drop rate (dropped / (T*k)) and the Switch-style
    auxiliary loss E * sum_e (counts_e / (T*k)) * P_e are reported alongside.
    """
    T, k, E = cfg.T, cfg.k, cfg.E
    C = capacity(cfg)
    counts = np.bincount(idx.ravel(), minlength=E).astype(np.int64)
    kept = counts.copy() if C is None else np.minimum(counts, C)
    offsets = np.zeros(E + 1, dtype=np.int64)
    offsets[1:] = np.cumsum(kept)
    row_of = np.full((T, k), -1, dtype=np.int64)
    src_tok = np.zeros(int(offsets[E]), dtype=np.int64)
    for e in range(E):
        tt, jj = np.nonzero(idx == e)       # row-major order: ascending token index
        n = int(kept[e])
        rows = offsets[e] + np.arange(n)
        row_of[tt[:n], jj[:n]] = rows
        src_tok[rows] = tt[:n]
    drop_count = int((counts - kept).sum())
    A = T * k
    aux = float("nan")
    if prob_mean is not None:
        aux = float(E * np.sum((counts / A) * prob_mean))
    return Dispatch(C=C, counts=counts, kept=kept, offsets=offsets, row_of=row_of,
                    src_tok=src_tok, drop_count=drop_count, drop_rate=drop_count / A, aux=aux)


# ------------------------------------------------------------ step 4: experts
def expert_hidden(xe: np.ndarray, w1e: np.ndarray, act: str, F: int) -> np.ndarray:
    """First layer plus activation of one expert on rows xe[m, d].

    ReLU: h = max(xe W1^T, 0) (FastMoE Transformer-XL experts).  SwiGLU: with
    W1 = [W_gate; W_up] (gate rows first), h = silu(xe W_gate^T) * (xe W_up^T),
    silu(u) = u / (1 + exp(-u)).
    """
    u = np.asarray(xe, np.float64) @ np.asarray(w1e, np.float64).T
    if act == RELU:
        return np.maximum(u, 0.0)
    g, up = u[:, :F], u[:, F:2 * F]
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g)) * up


def expert_ffn(xe, w1e, w2e, act: str, F: int) -> np.ndarray:
    """One expert's two-layer MLP: y = h W2^T."""
    return expert_hidden(xe, w1e, act, F) @ np.asarray(w2e, np.float64).T


def expert_segments(xp: np.ndarray, offsets: np.ndarray, w1, w2, cfg: LayerConfig,
                    want_hidden: bool = False):
    """Step 4 over the expert-grouped rows: rows [offsets[e], offsets[e+1]) of xp
    go through expert e.  Returns (h or None, yp)."""
    n = int(offsets[-1])
    yp = np.zeros((n, cfg.d))
    h = np.zeros((n, cfg.F)) if want_hidden else None
    for e in range(cfg.E):
        a, b = int(offsets[e]), int(offsets[e + 1])
        if a == b:
            continue
        he = expert_hidden(xp[a:b], w1[e], cfg.act, cfg.F)
        if want_hidden:
            h[a:b] = he
        yp[a:b] = he @ np.asarray(w2[e], np.float64).T
    return h, yp


# ------------------------------------------------------------ step 5: combine
def combine(yp: np.ndarray, row_of: np.ndarray, w: np.ndarray, T: int, d: int) -> np.ndarray:
    """out[t] = sum over kept slots j (in slot order) of w[t, j] * yp[row_of[t, j]];
    a token whose slots were all dropped gets 0 (the residual carries it)."""
    out = np.zeros((T, d))
    for j in range(row_of.shape[1]):
        keep = row_of[:, j] >= 0
        out[keep] += w[keep, j, None] * np.asarray(yp, np.float64)[row_of[keep, j]]
    return out


# ------------------------------------------------------------- whole layer
@dataclasses.dataclass
class Forward:
    routing: Routing
    dispatch: Dispatch
    out: np.ndarray
    yp: Optional[np.ndarray] = None
    h: Optional[np.ndarray] = None


def forward(x, wg, bias, w1, w2, cfg: LayerConfig, forced_mask=None, forced_idx=None,
            want_hidden: bool = False) -> Forward:
    """The full layer: route -> dispatch -> experts -> combine.

    x[T, d], wg[E, d], bias[E] or None, w1[e] -> [F1, d], w2[e] -> [d, F]
    (any indexable of per-expert float64-convertible matrices)."""
    x = np.asarray(x, np.float64)
    r = route(x, wg, bias, cfg, forced_mask, forced_idx)
    dsp = dispatch(r.idx, cfg, r.prob_mean)
    xp = x[dsp.src_tok]
    h, yp = expert_segments(xp, dsp.offsets, w1, w2, cfg, want_hidden)
    out = combine(yp, dsp.row_of, r.w, cfg.T, cfg.d)
    return Forward(routing=r, dispatch=dsp, out=out, yp=yp, h=h)


def forward_tokens(x, w1, w2, cfg: LayerConfig, r: Routing, dsp: Dispatch,
                   tokens: Sequence[int]) -> np.ndarray:
    """Layer output for selected tokens only, given the full routing and dispatch
    (for sampled checks at sizes where the full float64 forward is too slow).
    Each expert's weights are converted once for all sampled tokens it serves."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x = np.asarray(x)
    out = np.zeros((len(tokens), cfg.d))
    by_expert = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.k):
            if dsp.row_of[t, j] >= 0:
                by_expert.setdefault(int(r.idx[t, j]), []).append((i, t, j))
    for e, lst in by_expert.items():
        xs = np.asarray(x[[t for _, t, _ in lst]], np.float64)
        ys = expert_ffn(xs, w1[e], w2[e], cfg.act, cfg.F)
        for (i, t, j), y in zip(lst, ys):
            out[i] += r.w[t, j] * y
    return out


# ------------------------------------------------------------ shared expert
def shared_expert(x, w1s, w2s, act: str, F_shared: int) -> np.ndarray:
    """A shared expert (the MoE survey page, "MoE未来重点研究方向", item 4:
    DeepSeekMoE's shared experts): an expert every token goes through with
    weight 1, outside the routing.  Several shared experts are one expert of
    their summed hidden width (their W1 rows stacked -- for SwiGLU all gate
    rows, then all up rows -- and their W2 columns side by side)."""
    return expert_ffn(np.asarray(x, np.float64), w1s, w2s, act, F_shared)


def forward_with_shared(x, wg, bias, w1, w2, w1s, w2s, F_shared: int, cfg: LayerConfig, forced_mask=None,
                        forced_idx=None) -> Forward:
    """The layer plus a shared expert: out = routed combine + shared_expert(x)."""
    fw = forward(x, wg, bias, w1, w2, cfg, forced_mask, forced_idx)
    fw.out = fw.out + shared_expert(x, w1s, w2s, cfg.act, F_shared)
    return fw


# ------------------------------------------------------------- brute force
def brute_force(x, wg, bias, w1, w2, cfg: LayerConfig) -> np.ndarray:
    """Dense check of the whole layer for tiny inputs, written independently of
    the functions above: every expert runs on every token, then a mask built
    from the top-k selection and the capacity keeps the selected, non-dropped
    pairs.

    * the score spread uses sqrt(E[z^2] - E[z]^2) instead of E[(z - mu)^2];
    * top-k is k rounds of argmax (first maximum = lowest index), masking each
      winner;
    * weights are a softmax taken over the selected scores only;
    * capacity ranks come from a running count down the token axis.
    """
    x = np.asarray(x, np.float64)
    T, E, k = cfg.T, cfg.E, cfg.k
    z = x @ np.asarray(wg, np.float64).T
    if bias is not None:
        z = z + np.asarray(bias, np.float64)
    if cfg.lam > 0:
        mu = z.sum(axis=1, keepdims=True) / E
        var = np.maximum((z * z).sum(axis=1, keepdims=True) / E - mu * mu, 0.0)
        sd = np.sqrt(var)
        s = np.where(sd > 0, cfg.lam * (z - mu) / np.where(sd > 0, sd, 1.0), 0.0)
    else:
        s = z
    sel = np.zeros((T, E), dtype=bool)
    work = s.copy()
    for _ in range(k):
        a = np.argmax(work, axis=1)
        sel[np.arange(T), a] = True
        work[np.arange(T), a] = -np.inf
    ssel = np.where(sel, s, -np.inf)
    ex = np.where(sel, np.exp(ssel - ssel.max(axis=1, keepdims=True)), 0.0)
    wfull = ex / ex.sum(axis=1, keepdims=True)
    cf = float(np.float32(cfg.capacity_factor))
    if cf > 0:
        C = math.ceil(cf * T * k / E)
        rank = np.cumsum(sel, axis=0) - 1
        keep = sel & (rank < C)
    else:
        keep = sel
    out = np.zeros((T, cfg.d))
    F = cfg.F
    for e in range(E):
        w1e = np.asarray(w1[e], np.float64)
        if cfg.act == RELU:
            hid = np.clip(x @ w1e.T, 0.0, None)
        else:
            gate = x @ w1e[:F].T
            with np.errstate(over="ignore"):
                hid = gate * (1.0 / (1.0 + np.exp(-gate))) * (x @ w1e[F:2 * F].T)
        ye = hid @ np.asarray(w2[e], np.float64).T
        out += (keep[:, e] * wfull[:, e])[:, None] * ye
    return out
