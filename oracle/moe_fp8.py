"""Float64 CPU oracle of the MoE layer with FP8 expert weights (MX format).

TEST INFRASTRUCTURE, like ``moe_oracle``: only ``tests/``,
``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may import it.

The Skywork-MoE release serves the model with FP8 weights (its inference
section: the FP8-quantised weights take 146 GB on an 8 x 4090 server), and
the MoE survey page lists FP8 among the ways to cut the layer's memory and
bandwidth.  The pages fix no FP8 format.  Reading (DESIGN C19): the
microscaled form B200 tensor cores take natively -- E4M3 elements with one
power-of-two scale per 32 consecutive elements along the reduction
dimension -- applied to both expert layers:

* every expert weight row is quantised in blocks of 32 along its reduction
  axis (W1 rows along d, W2 rows along F);
* the layer-1 input rows (xp) are quantised the same way along d, and the
  hidden activation h along F, before the next GEMM;
* a block's scale is 2^X with X the least integer such that every |v| / 2^X
  <= 448 (the largest E4M3 value), so no element saturates; an all-zero block
  has X = -127;
* an element is v / 2^X rounded to the nearest E4M3 value, ties to even.

The gate GEMM, the routing, the permutation and the combine are those of
``moe_oracle``; only the expert MLP reads the dequantised values.
"""
from __future__ import annotations

import math

import numpy as np

from . import moe_oracle as om

E4M3_MAX = 448.0
BLOCK = 32


def e4m3_round(y: np.ndarray) -> np.ndarray:
    """Nearest E4M3 value (4 exponent bits, bias 7, 3 mantissa bits, largest
    finite 448, subnormal step 2^-9), ties to even; saturates at +-448."""
    y = np.asarray(y, np.float64)
    a = np.minimum(np.abs(y), E4M3_MAX)
    out = np.zeros_like(a)
    nz = a > 0
    e = np.floor(np.log2(np.where(nz, a, 1.0)))
    e = np.maximum(e, -6.0)                  # below 2^-6: the subnormal grid, step 2^-9
    step = np.exp2(e - 3.0)
    q = np.round(a / step) * step            # numpy rounds halves to even
    out[nz] = q[nz]
    return np.copysign(np.minimum(out, E4M3_MAX), y)


def mx_scale_exponent(amax: float) -> int:
    """Least integer X with amax <= 448 * 2^X (-127 for amax == 0)."""
    if amax == 0.0:
        return -127
    m, e = math.frexp(amax)                  # amax = m 2^e, m in [0.5, 1)
    X = e - 9 if 2.0 * m <= 1.75 else e - 8  # 448 = 1.75 * 2^8
    return int(min(max(X, -127), 127))


def mx_quantize(a: np.ndarray):
    """Blocks of 32 along the last axis: returns (dequantised values, X[..., n/32])."""
    a = np.asarray(a, np.float64)
    n = a.shape[-1]
    assert n % BLOCK == 0, "the quantised axis is a multiple of 32"
    blocks = a.reshape(a.shape[:-1] + (n // BLOCK, BLOCK))
    amax = np.max(np.abs(blocks), axis=-1)
    X = np.vectorize(mx_scale_exponent, otypes=[np.int64])(amax) if amax.size else amax.astype(np.int64)
    sc = np.exp2(X.astype(np.float64))[..., None]
    q = e4m3_round(blocks / sc) * sc
    return q.reshape(a.shape), X


def mxq(a: np.ndarray) -> np.ndarray:
    """Quantise and dequantise (blocks of 32 along the last axis)."""
    return mx_quantize(a)[0]


def hidden_window(xq: np.ndarray, w1q: np.ndarray, act: str, F: int, rel: float) -> np.ndarray:
    """How far a finite-precision evaluation of one expert's hidden activation
    may sit from the exact one, per element, when each pre-activation carries
    an absolute error of at most rel * sum_i |xq_i w1q_i| (a dot product
    accumulated in floating point) and the activation itself a relative one
    of rel.  ReLU is 1-Lipschitz; for SwiGLU h = silu(g) up, |silu'| <= 1.1,
    so |dh| <= 1.1 dg (|up| + dup) + |silu(g)| dup (expert_hidden gives the
    two activations)."""
    xq = np.asarray(xq, np.float64)
    w1q = np.asarray(w1q, np.float64)
    u = xq @ w1q.T
    du = rel * (np.abs(xq) @ np.abs(w1q).T)
    h = om.expert_hidden(xq, w1q, act, F)
    if act == om.RELU:
        return du + rel * np.abs(h)
    g, up = u[:, :F], u[:, F:2 * F]
    dg, dup = du[:, :F], du[:, F:2 * F]
    with np.errstate(over="ignore"):
        s = g / (1.0 + np.exp(-g))
    return 1.1 * dg * (np.abs(up) + dup) + np.abs(s) * dup + rel * np.abs(h)


def admits(hd: np.ndarray, Xd: np.ndarray, h: np.ndarray, window: np.ndarray):
    """Whether the MX values hd (blocks of 32 along the last axis, block
    exponents Xd) are the quantisation of SOME h' with |h' - h| <= window
    element-wise.  Both decisions are monotone in the value: the block
    exponent in the block maximum, the E4M3 rounding in the element, so h'
    ranges over an interval and hd must lie between the quantisations of its
    ends.  Returns (admitted, differs): per element, whether hd is admitted
    and whether it differs from the quantisation of h itself."""
    hd = np.asarray(hd, np.float64)
    h = np.asarray(h, np.float64)
    w = np.asarray(window, np.float64)
    R, n = h.shape
    nb = n // BLOCK
    hb, wb, db = (a.reshape(R, nb, BLOCK) for a in (h, w, hd))
    lo = np.max(np.maximum(np.abs(hb) - wb, 0.0), axis=-1)
    hi = np.max(np.abs(hb) + wb, axis=-1)
    Xs = np.vectorize(mx_scale_exponent, otypes=[np.int64])
    Xd = np.asarray(Xd, np.int64).reshape(R, nb)
    block_ok = (Xs(lo) <= Xd) & (Xd <= Xs(hi))
    sc = np.exp2(Xd.astype(np.float64))[..., None]
    q = db / sc
    el_ok = (e4m3_round((hb - wb) / sc) <= q) & (q <= e4m3_round((hb + wb) / sc))
    admitted = (el_ok & block_ok[..., None]).reshape(R, n)
    return admitted, hd != mxq(h)


class MXExperts:
    """Lazy dequantised view of stacked expert weights (each row quantised
    along its last axis): ``a[e]`` is expert e's matrix after the round trip."""

    def __init__(self, experts):
        self.experts = experts

    def __len__(self):
        return len(self.experts)

    def __getitem__(self, e):
        return mxq(np.asarray(self.experts[e], np.float64))


def expert_ffn_mx(xe, w1qe, w2qe, act: str, F: int) -> np.ndarray:
    """One expert on rows xe with dequantised weights: the input rows and the
    hidden activation are quantised before their GEMMs."""
    h = om.expert_hidden(mxq(xe), w1qe, act, F)
    return mxq(h) @ np.asarray(w2qe, np.float64).T


def forward(x, wg, bias, w1, w2, cfg: om.LayerConfig, forced_mask=None, forced_idx=None) -> om.Forward:
    """The layer with MX FP8 expert weights: routing and permutation as the
    bf16 layer; each expert's MLP on quantised inputs, weights and hidden.
    The returned Forward's ``h`` holds, per permuted row, the hidden
    activation before its quantisation."""
    x = np.asarray(x, np.float64)
    r = om.route(x, wg, bias, cfg, forced_mask, forced_idx)
    dsp = om.dispatch(r.idx, cfg, r.prob_mean)
    yp = np.zeros((int(dsp.offsets[-1]), cfg.d))
    hid = np.zeros((int(dsp.offsets[-1]), cfg.F))
    w1q, w2q = MXExperts(w1), MXExperts(w2)
    for e in range(cfg.E):
        a, b = int(dsp.offsets[e]), int(dsp.offsets[e + 1])
        if a < b:
            h = om.expert_hidden(mxq(x[dsp.src_tok[a:b]]), w1q[e], cfg.act, cfg.F)
            hid[a:b] = h
            yp[a:b] = mxq(h) @ np.asarray(w2q[e], np.float64).T
    out = om.combine(yp, dsp.row_of, r.w, cfg.T, cfg.d)
    return om.Forward(routing=r, dispatch=dsp, out=out, yp=yp, h=hid)


def hidden_windows(x, w1, cfg: om.LayerConfig, dsp: om.Dispatch, rel: float) -> np.ndarray:
    """hidden_window for every permuted row of the layer (rows grouped by
    expert as dsp orders them)."""
    x = np.asarray(x, np.float64)
    out = np.zeros((int(dsp.offsets[-1]), cfg.F))
    w1q = MXExperts(w1)
    for e in range(cfg.E):
        a, b = int(dsp.offsets[e]), int(dsp.offsets[e + 1])
        if a < b:
            out[a:b] = hidden_window(mxq(x[dsp.src_tok[a:b]]), w1q[e], cfg.act, cfg.F, rel)
    return out


def forward_tokens(x, w1, w2, cfg: om.LayerConfig, r: om.Routing, dsp: om.Dispatch, tokens) -> np.ndarray:
    """The MX layer's output for selected tokens only (sampled checks)."""
    tokens = np.asarray(tokens, dtype=np.int64)
    x = np.asarray(x)
    out = np.zeros((len(tokens), cfg.d))
    by_expert = {}
    for i, t in enumerate(tokens):
        for j in range(cfg.k):
            if dsp.row_of[t, j] >= 0:
                by_expert.setdefault(int(r.idx[t, j]), []).append((i, t, j))
    w1q, w2q = MXExperts(w1), MXExperts(w2)
    for e, lst in by_expert.items():
        xs = np.asarray(x[[t for _, t, _ in lst]], np.float64)
        ys = expert_ffn_mx(xs, w1q[e], w2q[e], cfg.act, cfg.F)
        for (i, t, j), y in zip(lst, ys):
            out[i] += r.w[t, j] * y
    return out
