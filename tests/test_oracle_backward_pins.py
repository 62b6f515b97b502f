"""Pins of the float64 backward oracle.

The backward is the derivative of the forward oracle (itself pinned in
test_oracle_pins.py), so it is pinned by central finite differences of the
scalar L = <dout, out> + aux_coef * aux + z_coef * z_loss through the forward,
on tiny layers whose top-k gaps and capacity ranks are far from a switch
(the selection and the drops are discrete and stay fixed under the small
perturbations), plus closed forms of single steps.  The last block plants
plausible mistakes in the backward oracle (on the CPU) and checks that a pin
catches each."""
import math

import numpy as np
import pytest

import oracle
from oracle import moe_oracle as om
from oracle import moe_backward as ob

EPS = 1e-6
GRID = [
    # (T, d, E, F, k, act, cf, lam, bias, aux_coef, z_coef)
    (12, 6, 4, 5, 2, om.SWIGLU, 0.75, 1.0, True, 0.3, 0.2),
    (10, 5, 3, 4, 1, om.RELU, 0.0, 0.0, False, 0.0, 0.0),
    (14, 4, 5, 3, 3, om.RELU, 1.0, 0.5, True, 1.0, 0.0),
    (9, 6, 4, 4, 4, om.SWIGLU, 0.0, 2.0, False, 0.0, 0.5),
    (16, 5, 6, 3, 2, om.SWIGLU, 0.5, 0.0, True, 0.7, 0.1),
]


def _layer(seed, T, d, E, F, k, act, cf, lam, bias):
    rng = np.random.default_rng(seed)
    cfg = oracle.LayerConfig(T=T, d=d, E=E, F=F, k=k, act=act, capacity_factor=cf, lam=lam)
    F1 = F if act == om.RELU else 2 * F
    return (cfg, rng.standard_normal((T, d)), rng.standard_normal((E, d)),
            rng.standard_normal(E) if bias else None, rng.standard_normal((E, F1, d)) / 2,
            rng.standard_normal((E, d, F)) / 2, rng.standard_normal((T, d)))


def check_finite_differences():
    """Worst |analytic - central difference| / max(1, |analytic|) per tensor
    and grid point, as failure strings."""
    bad = []
    for gi, (T, d, E, F, k, act, cf, lam, bias, ac, zc) in enumerate(GRID):
        cfg, x, wg, b, w1, w2, dout = _layer(100 + gi, T, d, E, F, k, act, cf, lam, bias)
        fw = om.forward(x, wg, b, w1, w2, cfg)
        # the pins need decided selections: skip grids with a near tie
        assert np.all(fw.routing.gap > 1e-3), f"grid {gi}: near tie in the pin layer"
        g = ob.backward(x, wg, b, w1, w2, cfg, dout, ac, zc)
        args = {"x": x, "wg": wg, "b": b, "w1": w1, "w2": w2}

        def L(**kw):
            a = dict(args)
            a.update(kw)
            return ob.loss(om.forward(a["x"], a["wg"], a["b"], a["w1"], a["w2"], cfg), dout, ac, zc)

        for name, ana in [("x", g.dx), ("wg", g.dwg), ("b", g.dbias), ("w1", g.dw1), ("w2", g.dw2)]:
            if args[name] is None:
                continue
            worst = 0.0
            for i in np.ndindex(args[name].shape):
                a = args[name].copy()
                a[i] += EPS
                lp = L(**{name: a})
                a[i] -= 2 * EPS
                lm = L(**{name: a})
                num = (lp - lm) / (2 * EPS)
                worst = max(worst, abs(num - ana[i]) / max(1.0, abs(ana[i])))
            if worst > 1e-7:
                bad.append(f"grid {gi} d{name}: {worst:.2e}")
    return bad


def check_closed_forms():
    bad = []
    # softmax backward of a uniform row with dp = e_0: ds = p (e_0 - p_0) = (1/E)(e_0 - 1/E)
    E = 4
    p = np.full((1, E), 0.25)
    dp = np.zeros((1, E)); dp[0, 0] = 1.0
    ds = ob.softmax_backward(p, dp)
    if not np.allclose(ds, 0.25 * (np.eye(E)[0] - 0.25), atol=1e-15):
        bad.append(f"softmax_backward {ds}")
    # renormalised top-2 of probabilities (0.5, 0.3): w = (5/8, 3/8); dw = (1, 0)
    # dp_0 = (1 - 5/8) / 0.8, dp_1 = (0 - 5/8) / 0.8
    dpw = ob.gate_weight_backward(np.array([[0.5, 0.3, 0.2]]), np.array([[0, 1]]), np.array([[0.625, 0.375]]),
                                  np.array([[1.0, 0.0]]))
    if not np.allclose(dpw, [[0.375 / 0.8, -0.625 / 0.8, 0.0]], atol=1e-15):
        bad.append(f"gate_weight_backward {dpw}")
    # silu'(0) = 1/2; silu'(g) -> 1 for large g
    if abs(ob.silu_grad(np.array([0.0]))[0] - 0.5) > 1e-15 or abs(ob.silu_grad(np.array([40.0]))[0] - 1.0) > 1e-12:
        bad.append("silu_grad")
    # aux: counts (2, 0, 2) of T = 2, k = 2, E = 3: d aux / dp = E f / T = 3 * (0.5, 0, 0.5) / 2
    if not np.allclose(ob.aux_prob_grad(np.array([2, 0, 2]), 2, 2, 1.0), [0.75, 0.0, 0.75], atol=1e-15):
        bad.append("aux_prob_grad")
    # z-loss on a uniform row of T = 1, E = 2, scores 0: lse = ln 2, ds = 2 ln 2 * 1/2 each
    if not np.allclose(ob.z_loss_score_grad(np.zeros((1, 2)), np.full((1, 2), 0.5), 1.0), math.log(2.0),
                       atol=1e-15):
        bad.append("z_loss_score_grad")
    # normalisation of a row with zero spread passes no gradient
    if np.any(ob.normalise_backward(np.full((1, 3), 2.0), np.ones((1, 3)), 1.0) != 0.0):
        bad.append("normalise_backward zero spread")
    return bad


def test_finite_differences():
    assert check_finite_differences() == []


def test_closed_forms():
    assert check_closed_forms() == []


def test_abs_contractions_bound_the_weight_gradients():
    """expert_abs_contractions: on positive inputs (and a ReLU that passes them
    all) they equal the weight gradients; in general they bound them."""
    rng = np.random.default_rng(3)
    x, w1, w2, dy = (np.abs(rng.standard_normal(s)) for s in [(6, 4), (5, 4), (4, 5), (6, 4)])
    A1, A2 = ob.expert_abs_contractions(x, w1, w2, dy, om.RELU, 5)
    _, dw1, dw2 = ob.expert_backward(x, w1, w2, dy, om.RELU, 5)
    assert np.allclose(A1, dw1, rtol=1e-14) and np.allclose(A2, dw2, rtol=1e-14)
    x, w1, w2, dy = (rng.standard_normal(s) for s in [(6, 4), (10, 4), (4, 5), (6, 4)])
    A1, A2 = ob.expert_abs_contractions(x, w1, w2, dy, om.SWIGLU, 5)
    _, dw1, dw2 = ob.expert_backward(x, w1, w2, dy, om.SWIGLU, 5)
    assert np.all(np.abs(dw1) <= A1 * (1 + 1e-12)) and np.all(np.abs(dw2) <= A2 * (1 + 1e-12))


def test_dropped_slots_carry_no_gradient():
    cfg, x, wg, b, w1, w2, dout = _layer(7, 20, 4, 2, 3, 1, om.RELU, 0.3, 0.0, False)
    fw = om.forward(x, wg, b, w1, w2, cfg)
    g = ob.backward(x, wg, b, w1, w2, cfg, dout)
    dropped = fw.dispatch.row_of < 0
    assert dropped.any()
    assert np.all(g.dw[dropped] == 0.0)


# -------------------------------------------------- planted mistakes (CPU)
def _all():
    return check_finite_differences() + check_closed_forms()


def _mut_no_renorm(p, idx, w, dw):
    T, E = p.shape
    dp = np.zeros((T, E))
    S = np.take_along_axis(p, idx, axis=1).sum(axis=1, keepdims=True)
    np.put_along_axis(dp, idx, dw / S, axis=1)
    return dp


def _mut_no_aux(counts, T, k, aux_coef):
    return np.zeros(counts.shape[0])


def _mut_z_sign(s, p, z_coef):
    return -ob._orig_z(s, p, z_coef)


def _mut_silu_grad_is_sigmoid(g):
    return 1.0 / (1.0 + np.exp(-g))


def _mut_norm_missing_term(z, ds, lam):
    if lam <= 0:
        return np.array(ds, copy=True)
    mu = z.mean(axis=1, keepdims=True)
    sd = np.sqrt(((z - mu) ** 2).mean(axis=1, keepdims=True))
    return (lam / sd) * (ds - ds.mean(axis=1, keepdims=True))


def _mut_softmax_no_centering(p, dp):
    return p * dp


ob._orig_z = ob.z_loss_score_grad
MUTATIONS = {
    "weights_not_renormalised": ("gate_weight_backward", _mut_no_renorm),
    "aux_gradient_dropped": ("aux_prob_grad", _mut_no_aux),
    "z_loss_gradient_sign": ("z_loss_score_grad", _mut_z_sign),
    "silu_grad_is_the_sigmoid": ("silu_grad", _mut_silu_grad_is_sigmoid),
    "normalisation_missing_term": ("normalise_backward", _mut_norm_missing_term),
    "softmax_backward_not_centred": ("softmax_backward", _mut_softmax_no_centering),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(ob, attr, fn)
    assert _all() != [], f"planted mistake '{name}' went unnoticed by every pin"
