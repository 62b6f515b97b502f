"""Pins of the float64 oracle against things other than itself.

The pages print no worked numeric example, so the oracle is pinned by:
brute force on tiny inputs (dense evaluation of every expert, masked by the
top-k selection and the capacity), hand-derived closed forms
(``tests/golden/closed_form_cases.json``), invariants, and special cases that
reduce to textbook formulas written out here with numpy.  The last block plants
plausible mistakes in the oracle (on the CPU) and checks that the pins catch
each of them.
"""
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import moe_oracle as om

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "closed_form_cases.json")


def _rand_layer(rng, T, d, E, F, k, act, cf=0.0, lam=0.0, bias=False):
    cfg = oracle.LayerConfig(T=T, d=d, E=E, F=F, k=k, act=act, capacity_factor=cf, lam=lam)
    x = rng.standard_normal((T, d))
    wg = rng.standard_normal((E, d)) / math.sqrt(d)
    b = (-1.2 * np.log(np.arange(E) + 1.0)) if bias else None
    F1 = F if act == oracle.RELU else 2 * F
    w1 = rng.standard_normal((E, F1, d)) / math.sqrt(d)
    w2 = rng.standard_normal((E, d, F)) / math.sqrt(F)
    return cfg, x, wg, b, w1, w2


# ------------------------------------------------------------ closed forms
def _cases():
    with open(GOLDEN) as f:
        return {c["name"]: c for c in json.load(f)["cases"]}


def check_closed_forms():
    """Returns a list of failure strings (empty when every closed form holds)."""
    bad = []
    c = _cases()

    for name in ["two_experts_lambda1_top2", "two_experts_plain_top1", "four_experts_tie_lowest_index"]:
        cs = c[name]
        x = np.array(cs["x"]); wg = np.array(cs["wg"])
        cfg = oracle.LayerConfig(T=x.shape[0], d=x.shape[1], E=wg.shape[0], F=1, k=cs["k"],
                                 lam=cs["lam"])
        r = om.route(x, wg, None, cfg)
        if not np.array_equal(r.idx, np.array(cs["expected_idx"])):
            bad.append(f"{name}: idx {r.idx.tolist()}")
        if not np.allclose(r.w, np.array(cs["expected_w"]), rtol=0, atol=1e-14):
            bad.append(f"{name}: w {r.w.tolist()}")
        eg = np.array(cs["expected_gap"], dtype=np.float64)
        if not (np.array_equal(np.isinf(eg), np.isinf(r.gap)) and
                np.allclose(r.gap[~np.isinf(eg)], eg[~np.isinf(eg)], atol=1e-14)):
            bad.append(f"{name}: gap {r.gap.tolist()}")
        if "expected_p1" in cs and abs(r.p[0, 1] - cs["expected_p1"]) > 1e-14:
            bad.append(f"{name}: p1 {r.p[0, 1]}")
        if "top1_idx" in cs:
            r1 = om.route(x, wg, None, dataclass_replace(cfg, k=1))
            if not np.array_equal(r1.idx, np.array(cs["top1_idx"])) or abs(r1.gap[0] - cs["top1_gap"][0]) > 0:
                bad.append(f"{name}: top1 {r1.idx.tolist()} {r1.gap.tolist()}")

    cs = c["capacity_first_tokens_win"]
    T, E, k = cs["T"], cs["E"], cs["k"]
    cfg = oracle.LayerConfig(T=T, d=1, E=E, F=1, k=k, capacity_factor=cs["capacity_factor"])
    x = np.ones((T, 1)); wg = np.zeros((E, 1)); b = np.array(cs["bias"])
    r = om.route(x, wg, b, cfg)
    dsp = om.dispatch(r.idx, cfg, r.prob_mean)
    if dsp.C != cs["expected_C"]:
        bad.append(f"capacity: C={dsp.C}")
    if dsp.counts.tolist() != cs["expected_counts"] or dsp.kept.tolist() != cs["expected_kept"]:
        bad.append(f"capacity: counts {dsp.counts} kept {dsp.kept}")
    if dsp.row_of.tolist() != cs["expected_row_of"]:
        bad.append(f"capacity: row_of {dsp.row_of.tolist()}")
    if abs(dsp.drop_rate - cs["expected_drop_rate"]) > 1e-15 or abs(dsp.aux - cs["expected_aux"]) > 1e-13:
        bad.append(f"capacity: drop {dsp.drop_rate} aux {dsp.aux}")
    w1 = np.ones((E, 1, 1)); w2 = np.ones((E, 1, 1))
    fw = om.forward(x, wg, b, w1, w2, cfg)
    if not np.allclose(fw.out[:, 0], [1, 1, 0, 0, 0], atol=1e-15):
        bad.append(f"capacity: out {fw.out[:, 0]}")

    for name, act in [("relu_expert_identity", oracle.RELU), ("swiglu_expert_gate_first", oracle.SWIGLU)]:
        cs = c[name]
        x = np.array(cs["x"]); w1 = np.array(cs["w1"]); w2 = np.array(cs["w2"])
        F = w2.shape[2]
        cfg = oracle.LayerConfig(T=x.shape[0], d=x.shape[1], E=1, F=F, k=1, act=act)
        fw = om.forward(x, np.zeros((1, x.shape[1])), None, w1, w2, cfg)
        if not np.allclose(fw.out, np.array(cs["expected_out"]), rtol=0, atol=1e-13):
            bad.append(f"{name}: out {fw.out.tolist()}")
    return bad


def check_losses():
    """Closed forms of the router z-loss and of the adaptive aux coefficient."""
    bad = []
    c = _cases()
    for name in ["z_loss_constant_scores", "z_loss_two_tokens"]:
        cs = c[name]
        got = om.z_loss(np.array(cs["scores"], dtype=np.float64))
        if not abs(got - cs["expected_z_loss"]) <= 1e-12 * max(1.0, abs(cs["expected_z_loss"])):
            bad.append(f"{name}: {got}")
    cs = c["z_loss_after_normalisation"]
    x = np.array(cs["x"]); wg = np.array(cs["wg"])
    cfg = oracle.LayerConfig(T=1, d=2, E=2, F=1, k=cs["k"], lam=cs["lam"])
    got = om.route(x, wg, None, cfg).z_loss
    if not abs(got - cs["expected_z_loss"]) <= 1e-13:
        bad.append(f"z_loss_after_normalisation: {got}")
    if not math.isnan(om.z_loss(np.zeros((0, 3)))):
        bad.append("z_loss of an empty batch")
    cs = c["adaptive_aux_coef_constant_drop_rate"]
    a = cs["alpha0"]
    for _ in range(cs["steps"]):
        a = om.adaptive_aux_coef(a, cs["drop_rate"], cs["beta"], cs["xi"])
    if not abs(a - cs["expected_alpha"]) <= 1e-15:
        bad.append(f"adaptive_aux_coef: {a}")
    # the coefficient rises with the drop rate and falls with it
    up = om.adaptive_aux_coef(0.05, 0.3, 0.8, 1.0)
    down = om.adaptive_aux_coef(0.05, 0.01, 0.8, 1.0)
    if not (down < 0.05 < up):
        bad.append(f"adaptive_aux_coef direction: {down} {up}")
    return bad


def dataclass_replace(cfg, **kw):
    import dataclasses
    return dataclasses.replace(cfg, **kw)


# ------------------------------------------------------------- brute force
BRUTE_GRID = [
    # (T, d, E, F, k, act, cf, lam, bias)
    (40, 16, 4, 24, 1, oracle.RELU, 0.0, 0.0, False),
    (40, 16, 4, 24, 2, oracle.RELU, 0.0, 1.0, False),
    (64, 8, 8, 16, 2, oracle.SWIGLU, 1.0, 0.0, True),
    (64, 8, 8, 16, 3, oracle.RELU, 1.25, 1.0, False),
    (33, 12, 5, 8, 5, oracle.SWIGLU, 0.0, 0.5, False),
    (50, 8, 6, 8, 4, oracle.RELU, 0.7, 2.0, True),
    (17, 4, 1, 4, 1, oracle.RELU, 0.0, 0.0, False),
    (64, 16, 8, 8, 8, oracle.SWIGLU, 0.0, 1.0, True),
    (64, 16, 8, 8, 2, oracle.SWIGLU, 0.3, 0.0, True),
]


def check_brute_force(seed=0):
    bad = []
    rng = np.random.default_rng(seed)
    for (T, d, E, F, k, act, cf, lam, bias) in BRUTE_GRID:
        cfg, x, wg, b, w1, w2 = _rand_layer(rng, T, d, E, F, k, act, cf, lam, bias)
        fw = om.forward(x, wg, b, w1, w2, cfg)
        bf = om.brute_force(x, wg, b, w1, w2, cfg)
        err = np.max(np.abs(fw.out - bf)) if fw.out.size else 0.0
        if not err <= 1e-12 * max(1.0, np.max(np.abs(bf))):
            bad.append(f"brute force {T,d,E,F,k,act,cf,lam,bias}: max err {err}")
    return bad


# ---------------------------------------------------------------- invariants
def check_invariants(seed=1):
    bad = []
    rng = np.random.default_rng(seed)
    for (T, d, E, F, k, act, cf, lam, bias) in BRUTE_GRID:
        cfg, x, wg, b, w1, w2 = _rand_layer(rng, T, d, E, F, k, act, cf, lam, bias)
        r = om.route(x, wg, b, cfg)
        dsp = om.dispatch(r.idx, cfg, r.prob_mean)
        A = T * k
        if not np.allclose(r.w.sum(axis=1), 1.0, atol=1e-14):
            bad.append("weights do not sum to 1")
        if int(dsp.counts.sum()) != A:
            bad.append("sum counts != T*k")
        if int(dsp.kept.sum()) != A - dsp.drop_count:
            bad.append("sum kept != T*k - drops")
        if dsp.C is not None and np.any(dsp.kept > dsp.C):
            bad.append("kept above capacity")
        # each row of each expert is used exactly once and maps back to its token
        rows = dsp.row_of[dsp.row_of >= 0]
        if sorted(rows.tolist()) != list(range(int(dsp.offsets[-1]))):
            bad.append("row_of is not a bijection onto kept rows")
        tt, jj = np.nonzero(dsp.row_of >= 0)
        if not np.array_equal(dsp.src_tok[dsp.row_of[tt, jj]], tt):
            bad.append("src_tok does not invert row_of")
        if not np.array_equal(r.idx[tt, jj], np.searchsorted(dsp.offsets, dsp.row_of[tt, jj], side="right") - 1):
            bad.append("row lies outside its expert's segment")
        for e in range(E):
            seg = dsp.src_tok[dsp.offsets[e]:dsp.offsets[e + 1]]
            if np.any(np.diff(seg) <= 0):
                bad.append("segment not in ascending token order")
        # tokens dropped from an expert come after every kept token of it
        for e in range(E):
            tok_sel = np.nonzero((r.idx == e).any(axis=1))[0]
            kept_tok = set(dsp.src_tok[dsp.offsets[e]:dsp.offsets[e + 1]].tolist())
            dropped = [t for t in tok_sel if t not in kept_tok]
            if dropped and kept_tok and min(dropped) < max(kept_tok):
                bad.append("drop priority is not by ascending token index")
        if lam > 0:
            zh = om.normalise_logits(om.gate_logits(x, wg, b), lam)
            if not np.allclose(zh.mean(axis=1), 0.0, atol=1e-12):
                bad.append("normalised logits mean != 0")
            if not np.allclose(zh.std(axis=1), lam, atol=1e-12):
                bad.append("normalised logits std != lambda")
            # the normalisation is a per-row increasing affine map: same top-k as raw logits
            r_raw = om.route(x, wg, b, dataclass_replace(cfg, lam=0.0))
            if not np.array_equal(np.sort(r_raw.idx, 1), np.sort(r.idx, 1)):
                bad.append("lambda normalisation changed the top-k set")
        # dropless output is invariant under a permutation of the tokens
        if cf <= 0:
            perm = rng.permutation(T)
            fw = om.forward(x, wg, b, w1, w2, cfg)
            fwp = om.forward(x[perm], wg, b, w1, w2, cfg)
            if not np.allclose(fwp.out, fw.out[perm], atol=1e-12):
                bad.append("dropless output depends on token order")
    return bad


# ----------------------------------------------------------- special cases
def check_special_cases(seed=2):
    bad = []
    rng = np.random.default_rng(seed)
    # E=1, k=1: the textbook dense FFN, written out with numpy here.
    for act in (oracle.RELU, oracle.SWIGLU):
        cfg, x, wg, b, w1, w2 = _rand_layer(rng, 24, 16, 1, 12, 1, act)
        fw = om.forward(x, wg, b, w1, w2, cfg)
        if act == oracle.RELU:
            dense = np.maximum(x @ w1[0].T, 0) @ w2[0].T
        else:
            g = x @ w1[0][:12].T
            dense = (g * (1 / (1 + np.exp(-g))) * (x @ w1[0][12:].T)) @ w2[0].T
        if not np.allclose(fw.out, dense, atol=1e-12):
            bad.append(f"E=1 {act} differs from dense FFN")
    # k=E, dropless: every expert used, weights are the full softmax of the scores.
    cfg, x, wg, b, w1, w2 = _rand_layer(rng, 20, 8, 4, 8, 4, oracle.RELU, lam=1.0)
    fw = om.forward(x, wg, b, w1, w2, cfg)
    z = x @ wg.T
    zh = (z - z.mean(1, keepdims=True)) / z.std(1, keepdims=True)
    pfull = np.exp(zh) / np.exp(zh).sum(1, keepdims=True)
    mix = sum(pfull[:, e:e + 1] * (np.maximum(x @ w1[e].T, 0) @ w2[e].T) for e in range(4))
    if not np.allclose(fw.out, mix, atol=1e-12):
        bad.append("k=E is not the softmax-weighted mixture")
    if not np.all(fw.dispatch.counts == 20):
        bad.append("k=E does not use every expert for every token")
    # capacity >= T equals dropless
    cfg, x, wg, b, w1, w2 = _rand_layer(rng, 30, 8, 4, 8, 2, oracle.SWIGLU)
    big = dataclass_replace(cfg, capacity_factor=4.0)   # C = ceil(4*30*2/4) = 60 >= 30
    f1 = om.forward(x, wg, b, w1, w2, cfg)
    f2 = om.forward(x, wg, b, w1, w2, big)
    if f2.dispatch.drop_count != 0 or not np.array_equal(f1.out, f2.out):
        bad.append("capacity >= T differs from dropless")
    # aux: uniform routing gives exactly 1; collapse onto one expert with k=1 gives E
    E = 8
    cfgu = oracle.LayerConfig(T=16, d=1, E=E, F=1, k=1, capacity_factor=0.0)
    idx = (np.arange(16) % E)[:, None]
    if abs(om.dispatch(idx, cfgu, np.full(E, 1.0 / E)).aux - 1.0) > 1e-15:
        bad.append("uniform aux != 1")
    pm = np.zeros(E); pm[3] = 1.0
    if abs(om.dispatch(np.full((16, 1), 3), cfgu, pm).aux - E) > 1e-12:
        bad.append("collapsed aux != E")
    # zero-spread logits normalise to zeros (uniform softmax)
    zero = om.normalise_logits(np.full((2, 4), 0.7), 1.0)
    if not np.array_equal(zero, np.zeros((2, 4))):
        bad.append("zero-spread normalisation")
    return bad


# ------------------------------------------------------------------ tests
def test_closed_forms():
    assert check_closed_forms() == []


def test_brute_force_agreement():
    assert check_brute_force() == []


def test_invariants():
    assert check_invariants() == []


def test_special_cases():
    assert check_special_cases() == []


def check_shared():
    """Shared expert: every token through it with weight 1.  E = 1, k = 1 and
    the shared expert equal to the routed one gives twice the routed output;
    two shared experts stacked into one wide expert equal their sum."""
    bad = []
    rng = np.random.default_rng(11)
    T, d, F = 12, 8, 6
    x = rng.standard_normal((T, d))
    w1 = rng.standard_normal((1, 2 * F, d)) / 3
    w2 = rng.standard_normal((1, d, F)) / 3
    cfg = oracle.LayerConfig(T=T, d=d, E=1, F=F, k=1, act=oracle.SWIGLU)
    fw = om.forward_with_shared(x, np.zeros((1, d)), None, w1, w2, w1[0], w2[0], F, cfg)
    dense = om.forward(x, np.zeros((1, d)), None, w1, w2, cfg).out
    if not np.allclose(fw.out, 2 * dense, rtol=0, atol=1e-12):
        bad.append("shared == routed expert: out != 2 * routed")
    a1, a2 = rng.standard_normal((2 * F, d)), rng.standard_normal((d, F))
    b1, b2 = rng.standard_normal((2 * F, d)), rng.standard_normal((d, F))
    wide1 = np.concatenate([a1[:F], b1[:F], a1[F:], b1[F:]])      # gate rows, then up rows
    wide2 = np.concatenate([a2, b2], axis=1)
    two = om.shared_expert(x, a1, a2, oracle.SWIGLU, F) + om.shared_expert(x, b1, b2, oracle.SWIGLU, F)
    if not np.allclose(om.shared_expert(x, wide1, wide2, oracle.SWIGLU, 2 * F), two, rtol=0, atol=1e-12):
        bad.append("two shared experts != one wide shared expert")
    return bad


def test_shared_expert():
    assert check_shared() == []


def test_losses_closed_forms():
    assert check_losses() == []


def test_capacity_formula_values():
    # the capacities of the workloads: ceil(cf * T * k / E)
    cases = [((8192, 2, 64, 1.25), 320), ((4096, 2, 16, 1.0), 512), ((64, 6, 64, 1.0), 6),
             ((32768, 6, 64, 1.0), 3072), ((5, 1, 2, 0.75), 2), ((5, 1, 2, 0.8), 3), ((7, 2, 3, 1.0), 5)]
    for (T, k, E, cf), C in cases:
        assert om.capacity(oracle.LayerConfig(T=T, d=1, E=E, F=1, k=k, capacity_factor=cf)) == C
    assert om.capacity(oracle.LayerConfig(T=8, d=1, E=2, F=1, k=1, capacity_factor=0.0)) is None


def test_forward_tokens_matches_full_forward():
    rng = np.random.default_rng(5)
    cfg, x, wg, b, w1, w2 = _rand_layer(rng, 48, 16, 6, 8, 2, oracle.SWIGLU, cf=0.8, lam=1.0, bias=True)
    fw = om.forward(x, wg, b, w1, w2, cfg)
    toks = [0, 5, 17, 47, 30]
    sub = om.forward_tokens(x, w1, w2, cfg, fw.routing, fw.dispatch, toks)
    assert np.allclose(sub, fw.out[toks], atol=1e-13)


def test_forced_routing_replaces_selection():
    rng = np.random.default_rng(6)
    cfg, x, wg, b, w1, w2 = _rand_layer(rng, 20, 8, 5, 8, 2, oracle.RELU, cf=1.0)
    base = om.route(x, wg, b, cfg)
    mask = np.zeros(20, bool); mask[[3, 7]] = True
    forced = base.idx.copy(); forced[3] = [4, 0]; forced[7] = [1, 2]
    r = om.route(x, wg, b, cfg, mask, forced)
    assert r.idx[3].tolist() == [4, 0] and r.idx[7].tolist() == [1, 2]
    assert np.array_equal(r.idx[~mask], base.idx[~mask])
    assert np.allclose(r.w[3], r.p[3, [4, 0]] / r.p[3, [4, 0]].sum())


def test_workload_generator_is_seeded_and_bf16_exact():
    import moe_workloads as mw
    w = mw.WORKLOADS["fastmoe_txl"].replace(T=16, E=4, d=64, F=64)
    a, b = mw.gen_x(w), mw.gen_x(w)
    assert a.dtype == np.uint16 and np.array_equal(a, b)
    assert not np.array_equal(mw.gen_x(w, shard=1), a)
    f = mw.to_f64(a)
    # bf16 values have at most 8 significant bits
    m, _ = np.frexp(f[f != 0])
    assert np.all(np.abs(m * 256 - np.round(m * 256)) == 0)
    # round-to-nearest-even on hand-picked bit patterns
    vals = np.array([1.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -2.5, 1.0 + 2 ** -7 + 2 ** -9], np.float32)
    got = mw.bf16_bits_to_f32(mw.round_to_bf16_bits(vals))
    assert got.tolist() == [1.0, 1.0, 1.0 + 2 ** -6, -2.5, 1.0 + 2 ** -7]
    bias = mw.gen_bias(mw.WORKLOADS["fine_decode_cap"])
    assert bias[0] == 0.0 and np.all(np.diff(bias) < 0)


# -------------------------------------------------- planted mistakes (CPU)
def _all_pins():
    return (check_closed_forms() + check_brute_force() + check_invariants() + check_special_cases() +
            check_losses() + check_shared())


def _mut_sample_std(z, lam):
    if lam <= 0:
        return np.array(z, copy=True)
    mu = z.mean(axis=1, keepdims=True)
    return lam * (z - mu) / z.std(axis=1, ddof=1, keepdims=True)


def _mut_no_scale(z, lam):
    if lam <= 0:
        return np.array(z, copy=True)
    mu = z.mean(axis=1, keepdims=True)
    return (z - mu) / z.std(axis=1, keepdims=True)


def _mut_topk_highest_index_on_ties(s, k):
    order = np.argsort(-s[:, ::-1], axis=1, kind="stable")
    order = s.shape[1] - 1 - order
    idx = order[:, :k]
    T, E = s.shape
    rows = np.arange(T)
    gap = s[rows, order[:, k - 1]] - s[rows, order[:, k]] if k < E else np.full(T, np.inf)
    return idx, gap


def _mut_swapped_gate_up(xe, w1e, act, F):
    u = np.asarray(xe, np.float64) @ np.asarray(w1e, np.float64).T
    if act == om.RELU:
        return np.maximum(u, 0.0)
    up, g = u[:, :F], u[:, F:2 * F]
    return g / (1.0 + np.exp(-g)) * up


def _mut_combine_drops_weights(yp, row_of, w, T, d):
    out = np.zeros((T, d))
    for j in range(row_of.shape[1]):
        keep = row_of[:, j] >= 0
        out[keep] += np.asarray(yp)[row_of[keep, j]]
    return out


def _mut_softmax_no_renorm_route(x, wg, bias, cfg, forced_mask=None, forced_idx=None):
    r = _orig_route(x, wg, bias, cfg, forced_mask, forced_idx)
    r.w = np.take_along_axis(r.p, r.idx, axis=1)
    return r


_orig_route = om.route
_orig_dispatch = om.dispatch


def _mut_capacity_latest_first(idx, cfg, prob_mean=None):
    # keeps the LAST C tokens of each expert instead of the first C
    rev = idx[::-1].copy()
    d = _orig_dispatch(rev, cfg, prob_mean)
    T = cfg.T
    row_of = d.row_of[::-1].copy()
    d.row_of = row_of
    d.src_tok = T - 1 - d.src_tok
    return d


def _mut_capacity_floor(cfg):
    cf = float(np.float32(cfg.capacity_factor))
    if cf <= 0:
        return None
    return int(math.floor(cf * cfg.T * cfg.k / cfg.E))


def _mut_aux_postdrop(idx, cfg, prob_mean=None):
    d = _orig_dispatch(idx, cfg, prob_mean)
    if prob_mean is not None:
        d.aux = float(cfg.E * np.sum((d.kept / (cfg.T * cfg.k)) * prob_mean))
    return d


def _mut_gate_transposed_bias_sign(x, wg, bias=None):
    z = np.asarray(x, np.float64) @ np.asarray(wg, np.float64).T
    if bias is not None:
        z = z - np.asarray(bias, np.float64)[None, :]
    return z


def _mut_z_loss_not_squared(s):
    if s.shape[0] == 0:
        return float("nan")
    return float(np.mean(om.log_partition(s)))


def _mut_z_loss_summed(s):
    if s.shape[0] == 0:
        return float("nan")
    return float(np.sum(om.log_partition(s) ** 2))


def _mut_log_partition_is_max(s):
    return s.max(axis=1)


def _mut_coef_beta_swapped(alpha, drop_rate, beta, xi):
    return (1.0 - beta) * alpha + beta * xi * drop_rate


def _mut_shared_gate_weighted(x, w1s, w2s, act, F_shared):
    return 0.5 * om.expert_ffn(np.asarray(x, np.float64), w1s, w2s, act, F_shared)


MUTATIONS = {
    "sample_std": ("normalise_logits", _mut_sample_std),
    "lambda_ignored": ("normalise_logits", _mut_no_scale),
    "ties_to_highest_index": ("top_k", _mut_topk_highest_index_on_ties),
    "swapped_gate_up": ("expert_hidden", _mut_swapped_gate_up),
    "combine_ignores_weights": ("combine", _mut_combine_drops_weights),
    "weights_not_renormalised": ("route", _mut_softmax_no_renorm_route),
    "drop_earliest_tokens": ("dispatch", _mut_capacity_latest_first),
    "capacity_floor": ("capacity", _mut_capacity_floor),
    "aux_uses_kept_counts": ("dispatch", _mut_aux_postdrop),
    "bias_sign_flipped": ("gate_logits", _mut_gate_transposed_bias_sign),
    "z_loss_not_squared": ("z_loss", _mut_z_loss_not_squared),
    "z_loss_summed_over_tokens": ("z_loss", _mut_z_loss_summed),
    "log_partition_is_the_max": ("log_partition", _mut_log_partition_is_max),
    "coef_smoothing_swapped": ("adaptive_aux_coef", _mut_coef_beta_swapped),
    "shared_expert_weighted": ("shared_expert", _mut_shared_gate_weighted),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(om, attr, fn)
    assert _all_pins() != [], f"planted mistake '{name}' went unnoticed by every pin"
