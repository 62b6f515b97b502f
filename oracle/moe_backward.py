"""Float64 CPU oracle of the backward pass of the top-k gated MoE FFN layer.

TEST INFRASTRUCTURE, like ``moe_oracle`` (the forward it differentiates):
only ``tests/``, ``__graft_entry__.smoke()`` and ``bench.py``'s CPU legs may
import it; the CUDA path never does.

The pages' figures for the layer are training figures (FastMoE announcement,
"特色三": up to 47x faster training than a plain PyTorch MoE on one GPU;
Skywork-MoE release, "训练Infra": 38 % MFU in training), so the layer is also
differentiated.  The scalar differentiated is

    L = sum_{t, i} dout[t, i] * out[t, i]  +  aux_coef * aux  +  z_coef * z_loss

with dout the gradient arriving from above, aux the Switch-form balance loss
and z_loss the router z-loss of the forward (moe_oracle: readings C7 and the
z-loss reading).  The expert choice, the capacity drops and the counts in aux
are discrete: they carry no gradient and stay as the forward decided them.
The steps below run the forward's in reverse, in its notation:

* combine: dy[row] = w[t, j] * dout[t] and dw[t, j] = <dout[t], y[row]> for
  every kept slot (a dropped slot has neither);
* second expert layer: dW2[e] = dy_e^T h_e, dh = dy W2[e];
* activation: ReLU du = dh * [u > 0] (0 at u = 0); SwiGLU with u = [g, v]:
  dg = dh * v * silu'(g), dv = dh * silu(g), silu'(g) = s(g) (1 + g (1 - s(g))),
  s the logistic function;
* first expert layer: dW1[e] = du_e^T xp_e, dxp = du W1[e], and dx[t] sums
  dxp over the token's kept slots;
* gate weights: w = p_sel / S with S the sum of the selected probabilities,
  so dp[t, i] = (dw_i - sum_j w_j dw_j) / S for the selected i;
* aux: P_e is the mean over tokens of p[t, e], so dp[t, e] += aux_coef * E *
  f_e / T with f_e = counts_e / (T k);
* softmax: ds = p * (dp - <dp, p>); z-loss: ds += z_coef * (2 / T) * lse_t * p;
* normalisation (lambda > 0): s = lambda * n, n = (z - mean) / std (population
  std, over the experts): dz = (lambda / std) (ds - mean(ds) - n mean(ds n));
  a row with zero spread has s = 0 whatever z is, so dz = 0 there;
* gate: dW_gate = dz^T x, db = sum_t dz, dx += dz W_gate.

Pins (tests/test_oracle_backward_pins.py): central finite differences of L
through the forward oracle on tiny layers, closed forms, and planted mistakes.
"""
from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np

from . import moe_oracle as om


@dataclasses.dataclass
class Grads:
    dx: np.ndarray      # [T, d]
    dwg: np.ndarray     # [E, d]
    dbias: np.ndarray   # [E]
    dw1: np.ndarray     # [E, F1, d]
    dw2: np.ndarray     # [E, d, F]
    dw: np.ndarray      # [T, k]  gradient of the gate weights (0 for dropped slots)
    ds: np.ndarray      # [T, E]  gradient of the scores the softmax takes
    dz: np.ndarray      # [T, E]  gradient of the logits
    abs_dw1: Optional[np.ndarray] = None   # [E, F1, d]  expert_abs_contractions, when asked for
    abs_dw2: Optional[np.ndarray] = None   # [E, d, F]


def loss(fw: om.Forward, dout: np.ndarray, aux_coef: float = 0.0, z_coef: float = 0.0) -> float:
    """The scalar the backward differentiates (see the module text)."""
    L = float(np.sum(np.asarray(dout, np.float64) * fw.out))
    if aux_coef != 0.0:
        L += aux_coef * fw.dispatch.aux
    if z_coef != 0.0:
        L += z_coef * fw.routing.z_loss
    return L


def silu_grad(g: np.ndarray) -> np.ndarray:
    """d/dg of g * s(g): s(g) (1 + g (1 - s(g)))."""
    sg = 1.0 / (1.0 + np.exp(-g))
    return sg * (1.0 + g * (1.0 - sg))


def expert_backward(xe, w1e, w2e, dye, act: str, F: int):
    """One expert's two layers in reverse on rows xe[m, d] with output
    gradient dye[m, d]: returns (dxe, dw1e, dw2e)."""
    xe = np.asarray(xe, np.float64)
    w1e = np.asarray(w1e, np.float64)
    w2e = np.asarray(w2e, np.float64)
    u = xe @ w1e.T
    if act == om.RELU:
        h = np.maximum(u, 0.0)
    else:
        g, v = u[:, :F], u[:, F:2 * F]
        with np.errstate(over="ignore"):
            h = g / (1.0 + np.exp(-g)) * v
    dw2e = dye.T @ h
    dh = dye @ w2e
    if act == om.RELU:
        du = dh * (u > 0.0)
    else:
        with np.errstate(over="ignore"):
            sg = 1.0 / (1.0 + np.exp(-g))
            du = np.concatenate([dh * v * silu_grad(g), dh * g * sg], axis=1)
    dw1e = du.T @ xe
    dxe = du @ w1e
    return dxe, dw1e, dw2e


def expert_abs_contractions(xe, w1e, w2e, dye, act: str, F: int):
    """The weight-gradient contractions of one expert taken over absolute
    values: A2 = |dy|^T |h| and A1 = |du|_abs^T |x| with |du|_abs =
    (|dy| |W2[e]|) * |act'(u)| (SwiGLU: |v silu'(g)| for the gate columns,
    |silu(g)| for the up columns).  A rounding of relative size eps in every
    product of a contraction moves its result by at most eps times the same
    contraction over absolute values; these are the scales the bf16-path
    weight gradients are compared against."""
    xe = np.asarray(xe, np.float64)
    w1e = np.asarray(w1e, np.float64)
    w2e = np.asarray(w2e, np.float64)
    u = xe @ w1e.T
    if act == om.RELU:
        h = np.maximum(u, 0.0)
        dact = (u > 0.0).astype(np.float64)
    else:
        g, v = u[:, :F], u[:, F:2 * F]
        with np.errstate(over="ignore"):
            sg = 1.0 / (1.0 + np.exp(-g))
        h = g * sg * v
    ady = np.abs(dye)
    A2 = ady.T @ np.abs(h)
    adh = ady @ np.abs(w2e)
    if act == om.RELU:
        adu = adh * dact
    else:
        adu = np.concatenate([adh * np.abs(v * silu_grad(g)), adh * np.abs(g * sg)], axis=1)
    A1 = adu.T @ np.abs(xe)
    return A1, A2


def normalise_backward(z: np.ndarray, ds: np.ndarray, lam: float) -> np.ndarray:
    """dz from ds through z_hat = lam (z - mean) / std (population std); rows
    with zero spread get 0.  lam <= 0: the identity."""
    if lam <= 0:
        return np.array(ds, copy=True)
    mu = z.mean(axis=1, keepdims=True)
    sd = np.sqrt(((z - mu) ** 2).mean(axis=1, keepdims=True))
    dz = np.zeros_like(z)
    nz = sd[:, 0] > 0
    n = (z[nz] - mu[nz]) / sd[nz]
    g = ds[nz]
    dz[nz] = (lam / sd[nz]) * (g - g.mean(axis=1, keepdims=True) - n * (g * n).mean(axis=1, keepdims=True))
    return dz


def gate_weight_backward(p: np.ndarray, idx: np.ndarray, w: np.ndarray, dw: np.ndarray) -> np.ndarray:
    """dp[T, E] from dw[T, k] through w = p_sel / sum(p_sel) (renormalised
    top-k): dp_i = (dw_i - sum_j w_j dw_j) / sum(p_sel) for the selected i."""
    T, E = p.shape
    dp = np.zeros((T, E))
    if T == 0:
        return dp
    psel = np.take_along_axis(p, idx, axis=1)
    S = psel.sum(axis=1, keepdims=True)
    np.put_along_axis(dp, idx, (dw - np.sum(w * dw, axis=1, keepdims=True)) / S, axis=1)
    return dp


def aux_prob_grad(counts: np.ndarray, T: int, k: int, aux_coef: float) -> np.ndarray:
    """d(aux_coef * aux)/dp[t, e] = aux_coef * E * f_e / T, f_e = counts_e / (T k)
    (the same for every token); shape [E]."""
    E = counts.shape[0]
    if T == 0 or aux_coef == 0.0:
        return np.zeros(E)
    return aux_coef * E * (counts / float(T * k)) / T


def softmax_backward(p: np.ndarray, dp: np.ndarray) -> np.ndarray:
    """ds from dp through p = softmax(s): p * (dp - <dp, p>)."""
    return p * (dp - np.sum(dp * p, axis=1, keepdims=True))


def z_loss_score_grad(s: np.ndarray, p: np.ndarray, z_coef: float) -> np.ndarray:
    """d(z_coef * z_loss)/ds = z_coef * (2 / T) * lse_t * p[t, e]."""
    T = s.shape[0]
    if T == 0 or z_coef == 0.0:
        return np.zeros_like(s)
    return z_coef * (2.0 / T) * om.log_partition(s)[:, None] * p


def backward(x, wg, bias, w1, w2, cfg: om.LayerConfig, dout, aux_coef: float = 0.0, z_coef: float = 0.0,
             fw: Optional[om.Forward] = None, want_abs: bool = False) -> Grads:
    """All gradients of L (module text) for one layer.  fw: the forward of the
    same inputs (computed here when not given; a forced routing in it is kept)."""
    x = np.asarray(x, np.float64)
    wg = np.asarray(wg, np.float64)
    dout = np.asarray(dout, np.float64)
    if fw is None:
        fw = om.forward(x, wg, bias, w1, w2, cfg)
    r, dsp = fw.routing, fw.dispatch
    T, d, E, F, k = cfg.T, cfg.d, cfg.E, cfg.F, cfg.k
    F1 = F if cfg.act == om.RELU else 2 * F

    # ---- combine and the experts
    dx = np.zeros((T, d))
    dw = np.zeros((T, k))
    dw1 = np.zeros((E, F1, d))
    dw2 = np.zeros((E, d, F))
    abs1 = np.zeros((E, F1, d)) if want_abs else None
    abs2 = np.zeros((E, d, F)) if want_abs else None
    rows_t = dsp.src_tok
    for e in range(E):
        a, b = int(dsp.offsets[e]), int(dsp.offsets[e + 1])
        if a == b:
            continue
        toks = rows_t[a:b]
        # slot of each row: the j with row_of[t, j] == row
        rows = np.arange(a, b)
        slot = np.array([int(np.nonzero(dsp.row_of[t] == rr)[0][0]) for t, rr in zip(toks, rows)])
        ye = om.expert_ffn(x[toks], w1[e], w2[e], cfg.act, F)
        dw[toks, slot] = np.sum(dout[toks] * ye, axis=1)
        dye = r.w[toks, slot][:, None] * dout[toks]
        dxe, dw1[e], dw2[e] = expert_backward(x[toks], w1[e], w2[e], dye, cfg.act, F)
        np.add.at(dx, toks, dxe)
        if want_abs:
            abs1[e], abs2[e] = expert_abs_contractions(x[toks], w1[e], w2[e], dye, cfg.act, F)

    # ---- gate weights, aux, softmax, z-loss
    dp = gate_weight_backward(r.p, r.idx, r.w, dw) + aux_prob_grad(dsp.counts, T, k, aux_coef)[None, :]
    ds = softmax_backward(r.p, dp) + z_loss_score_grad(r.s, r.p, z_coef)

    # ---- normalisation and the gate
    z = om.gate_logits(x, wg, bias)
    dz = normalise_backward(z, ds, cfg.lam)
    dwg = dz.T @ x
    dbias = dz.sum(axis=0)
    dx += dz @ wg
    return Grads(dx=dx, dwg=dwg, dbias=dbias, dw1=dw1, dw2=dw2, dw=dw, ds=ds, dz=dz, abs_dw1=abs1, abs_dw2=abs2)
