"""Pins of the MX FP8 oracle (oracle/moe_fp8.py).

* The E4M3 grid, decoded here from its bit fields (independently of the
  rounding code): every finite code rounds to itself, and every midpoint
  between neighbours rounds to the neighbour with the even mantissa.
* Block scales: closed forms of the least X with amax <= 448 * 2^X.
* Blocks are independent and lie along the last axis; a block already on
  the grid (times a power of two) survives the round trip exactly; the error
  of any element is at most half a grid step of its block.
* A layer whose inputs and weights are small integers, so that every
  quantised tensor is exactly representable, gives the bf16 oracle's output
  exactly.
* The parity tests' admission of a device quantisation (admits): a value
  just off a rounding midpoint admits both neighbours only when the window
  covers the midpoint, never a value two steps away, and likewise the block
  exponent at the 448 * 2^X edge; hidden_window bounds sampled perturbations
  of the pre-activations and is reached to within a factor ~3.
* Planted mistakes (ties away from zero, the saturating floor-based scale,
  blocks along the wrong axis) each fail a pin."""
import math

import numpy as np
import pytest

import oracle
from oracle import moe_oracle as om
from oracle import moe_fp8 as mf


def e4m3_grid():
    vals = []
    for code in range(256):
        s, e, m = code >> 7, (code >> 3) & 15, code & 7
        if e == 15 and m == 7:
            continue          # NaN
        v = (m / 8.0) * 2.0 ** -6 if e == 0 else (1.0 + m / 8.0) * 2.0 ** (e - 7)
        vals.append((-v if s else v, m))
    return vals


def check_grid():
    bad = []
    grid = e4m3_grid()
    v = np.array([g for g, _ in grid])
    if not np.array_equal(mf.e4m3_round(v), v):
        bad.append("grid values do not round to themselves")
    pos = sorted({(abs(g), m) for g, m in grid})
    for (a, ma), (b, mb) in zip(pos[:-1], pos[1:]):
        if a == b:
            continue
        mid = (a + b) / 2
        want = a if ma % 2 == 0 else b
        got = float(mf.e4m3_round(np.array([mid]))[0])
        if got != want:
            bad.append(f"midpoint {mid}: {got}, want {want}")
            break
    if float(mf.e4m3_round(np.array([1e6]))[0]) != 448.0:
        bad.append("no saturation")
    return bad


def check_scales():
    bad = []
    cases = [(1.0, -8), (1.75, -8), (1.76, -7), (448.0, 0), (449.0, 1), (0.0, -127), (1.9, -7), (3.5, -7),
             (3.6, -6), (2.0 ** -20, -28)]
    for amax, X in cases:
        if mf.mx_scale_exponent(amax) != X:
            bad.append(f"scale of {amax}: {mf.mx_scale_exponent(amax)}, want {X}")
    return bad


def check_blocks():
    bad = []
    rng = np.random.default_rng(0)
    R = 64                       # rows: a multiple of 32, so that blocks along columns would also fit
    a = rng.standard_normal((R, 96)) * np.exp2(rng.integers(-20, 6, size=R))[:, None]
    q, X = mf.mx_quantize(a)
    if X.shape != (R, 3):
        bad.append(f"scale shape {X.shape}")
    for i in range(R):           # rows are independent
        if not np.array_equal(mf.mx_quantize(a[i:i + 1])[0][0], q[i]):
            bad.append(f"row {i} depends on other rows")
            break
    for i in range(0, R, 7):     # blocks of 32 along the row are independent
        for j in range(3):
            blk = a[i, 32 * j:32 * j + 32]
            if not np.array_equal(mf.mx_quantize(blk[None])[0][0], q[i, 32 * j:32 * j + 32]):
                bad.append(f"block ({i},{j}) depends on other blocks")
    # error at most half a step of the block's top binade (3 mantissa bits: 1/16 of it)
    err = np.abs(q - a).reshape(R, 3, 32)
    top = np.exp2(np.floor(np.log2(np.maximum(np.max(np.abs(a.reshape(R, 3, 32)), -1), 1e-300))))
    if np.any(err > (top / 16.0 + 1e-300)[..., None] + 1e-300):
        bad.append("error above half a step")
    # a block on the grid times 2^5 survives exactly
    g = np.array([v for v, _ in e4m3_grid() if abs(v) <= 448.0])
    blk = (rng.choice(g, 32) * 32.0)[None]
    blk[0, 0] = 448.0 * 32.0
    if not np.array_equal(mf.mxq(blk), blk):
        bad.append("grid block not exact")
    return bad


def check_exact_layer():
    """Small integers: every quantised tensor is exact, so the MX layer equals
    the bf16-valued oracle layer."""
    bad = []
    rng = np.random.default_rng(1)
    T, d, E, F, k = 24, 32, 3, 32, 2
    cfg = oracle.LayerConfig(T=T, d=d, E=E, F=F, k=k, act=om.RELU)
    x = rng.integers(-1, 2, size=(T, d)).astype(np.float64)
    wg = rng.standard_normal((E, d))
    w1 = (rng.integers(-1, 2, size=(E, F, d)) * (rng.random((E, F, d)) < 0.15)).astype(np.float64)
    w2 = rng.integers(-2, 3, size=(E, d, F)).astype(np.float64)
    fw_mx = mf.forward(x, wg, None, w1, w2, cfg)
    fw = om.forward(x, wg, None, w1, w2, cfg)
    h = np.concatenate([np.maximum(x @ w1[e].T, 0) for e in range(E)])
    if np.max(np.abs(h)) > 16:
        bad.append("exact-layer construction: h leaves the exact integer range")
    if not np.allclose(fw_mx.out, fw.out, rtol=0, atol=1e-12):
        bad.append("MX layer differs on exactly representable inputs")
    return bad


def check_admits():
    """The admission check of a device quantisation (admits): in a block with
    maximum 1.75 (X = -8 exactly, 1.75 = 448 * 2^-8), 1.0625 is the midpoint
    of the grid neighbours 1.0 and 1.125.  Just above it, a zero window admits
    only 1.125; a window that covers the midpoint admits both, never a value
    two steps away.  A block maximum just above 1.75 takes X = -7; a zero
    window rejects X = -8, one that reaches below 1.75 admits it.  Signs are
    symmetric."""
    bad = []
    h = np.full((1, 32), 0.5)
    h[0, 0] = 1.75
    h[0, 1] = 1.0625 * (1 + 1e-6)
    h[0, 2] = -1.0625 * (1 + 1e-6)
    q, X = mf.mx_quantize(h)
    if X.tolist() != [[-8]] or q[0, 1] != 1.125 or q[0, 2] != -1.125:
        bad.append(f"admits setup {X.tolist()} {q[0, :3].tolist()}")
    zero, wide = np.zeros_like(h), np.full_like(h, 1e-5)
    ok, diff = mf.admits(q, X, h, zero)
    if not ok.all() or diff.any():
        bad.append("admits: the quantisation of h itself")
    for col, alt in ((1, 1.0), (2, -1.0)):
        other = q.copy()
        other[0, col] = alt
        ok0, _ = mf.admits(other, X, h, zero)
        okw, dw = mf.admits(other, X, h, wide)
        if ok0[0, col] or not okw[0, col] or not dw[0, col] or dw.sum() != 1:
            bad.append(f"admits: other neighbour of the midpoint (col {col})")
        far = q.copy()
        far[0, col] = 1.25 if alt > 0 else -1.25
        if mf.admits(far, X, h, wide)[0][0, col]:
            bad.append(f"admits: two steps away (col {col})")
    hb = h.copy()
    hb[0, 0] = 1.75 * (1 + 1e-6)
    qb, Xb = mf.mx_quantize(hb)
    if Xb.tolist() != [[-7]]:
        bad.append(f"admits: X just above the edge {Xb.tolist()}")
    if not mf.admits(qb, Xb, hb, zero)[0].all():
        bad.append("admits: X = -7 with a zero window")
    q8 = np.clip(hb, -1.75, 1.75)
    q8 = mf.e4m3_round(q8 / 2.0 ** -8) * 2.0 ** -8
    if mf.admits(q8, np.array([[-8]]), hb, zero)[0].any():
        bad.append("admits: X = -8 with a zero window")
    if not mf.admits(q8, np.array([[-8]]), hb, wide)[0].all():
        bad.append("admits: X = -8 with a window below the edge")
    return bad


def check_hidden_window():
    """hidden_window bounds the hidden activation of every perturbation of
    the pre-activations within rel * sum |x w| (sampled at the corners, where
    the bound is approached), for ReLU and SwiGLU; with rel = 0 it is 0."""
    bad = []
    rng = np.random.default_rng(7)
    x = mf.mxq(rng.standard_normal((6, 64)))
    for act, F1 in ((om.RELU, 32), (om.SWIGLU, 64)):
        F = 32
        w = mf.mxq(rng.standard_normal((F1, 64)) / 4)
        rel = 1e-3
        win = mf.hidden_window(x, w, act, F, rel)
        if np.any(mf.hidden_window(x, w, act, F, 0.0) != 0):
            bad.append(f"hidden_window {act}: rel = 0")
        u = x @ w.T
        du = rel * (np.abs(x) @ np.abs(w).T)
        h = om.expert_hidden(x, w, act, F)
        worst = 0.0
        for _ in range(64):
            sgn = rng.choice([-1.0, 1.0], size=u.shape)
            up = u + sgn * du
            hp = np.maximum(up, 0) if act == om.RELU else \
                up[:, :F] / (1 + np.exp(-up[:, :F])) * up[:, F:]
            worst = max(worst, float(np.max(np.abs(hp - h) / np.maximum(win, 1e-300))))
        # the perturbation reaches a good part of the bound, never past it
        if not 0.3 < worst <= 1.0:
            bad.append(f"hidden_window {act}: worst ratio {worst:.3f}")
    return bad


def test_admits():
    assert check_admits() == []


def test_hidden_window():
    assert check_hidden_window() == []


def _all():
    return check_grid() + check_scales() + check_blocks() + check_exact_layer() + check_admits()


def test_grid():
    assert check_grid() == []


def test_scales():
    assert check_scales() == []


def test_blocks():
    assert check_blocks() == []


def test_exact_layer():
    assert check_exact_layer() == []


def test_mx_forward_close_to_bf16_forward():
    """Sanity of the reading: on a random layer the MX output stays near the
    unquantised one.  With 3 mantissa bits per operand the element-wise
    difference is large (tens of percent of RMS at the worst element), which
    is why the FP8 path is compared with this MX oracle, not the bf16 one."""
    rng = np.random.default_rng(2)
    cfg = oracle.LayerConfig(T=40, d=64, E=4, F=64, k=2, act=om.SWIGLU)
    x = rng.standard_normal((40, 64))
    wg = rng.standard_normal((4, 64)) / 8
    w1 = rng.standard_normal((4, 128, 64)) / 8
    w2 = rng.standard_normal((4, 64, 64)) / 8
    a = mf.forward(x, wg, None, w1, w2, cfg).out
    b = om.forward(x, wg, None, w1, w2, cfg).out
    rms = np.sqrt(np.mean(b ** 2))
    assert 0 < np.max(np.abs(a - b)) < 0.5 * rms


# -------------------------------------------------- planted mistakes (CPU)
def _mut_ties_away(y):
    y = np.asarray(y, np.float64)
    a = np.minimum(np.abs(y), 448.0)
    e = np.maximum(np.floor(np.log2(np.where(a > 0, a, 1.0))), -6.0)
    step = np.exp2(e - 3.0)
    q = np.floor(a / step + 0.5) * step
    return np.copysign(np.where(a > 0, np.minimum(q, 448.0), 0.0), y)


def _mut_floor_scale(amax):
    if amax == 0.0:
        return -127
    return int(math.floor(math.log2(amax))) - 8


_orig_mxq = mf.mx_quantize


def _mut_wrong_axis(a):
    a = np.asarray(a, np.float64)
    if a.ndim < 2 or a.shape[-2] % 32:
        return _orig_mxq(a)
    q, X = _orig_mxq(np.swapaxes(a, -1, -2))
    return np.swapaxes(q, -1, -2), X


MUTATIONS = {
    "ties_away_from_zero": ("e4m3_round", _mut_ties_away),
    "saturating_floor_scale": ("mx_scale_exponent", _mut_floor_scale),
    "blocks_along_columns": ("mx_quantize", _mut_wrong_axis),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistake_is_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(mf, attr, fn)
    assert _all() != [], f"planted mistake '{name}' went unnoticed"
