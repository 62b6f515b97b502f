"""The layer with MX FP8 expert weights (moe_prepare_mxfp8_weights,
moe_layer_forward_mxfp8) against the float64 MX oracle (oracle/moe_fp8.py).

* The prepared weights, decoded here from their bytes (E4M3 bit fields and
  the UE8M0 scale atoms, SwiGLU rows de-interleaved), equal the oracle's
  quantisation of the same bf16 weights exactly (both take the same integer
  decisions: the block exponent and round-to-nearest-even to the E4M3 grid).
* The forward, read back from its workspace: the quantised input rows equal
  the oracle's bit for bit (the same integer decisions on bf16 values).  The
  quantised hidden activation is an admissible MX quantisation of the exact
  one -- equal to the oracle's except where the exact value lies within the
  fp32 evaluation's error window of a decision (a rounding midpoint, a block
  maximum at 448 * 2^X), where the other neighbour is equally correct; such
  values are counted and held to 1e-3 of all.  The output equals the second
  layer applied to the device's own hidden activation within 1e-4 * RMS
  (fp32 accumulation of exact products), and the oracle's output within
  1e-4 * RMS on every token none of whose hidden values took the other
  decision.  These are the FP8 path's near ties, as near-tie scores are the
  routing's.
* Routing, permutation and statistics are the bf16 layer's, compared exactly
  off near ties."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
import oracle
from oracle import moe_oracle as om
from oracle import moe_fp8 as mf
from tests.gpu_harness import check_routing, to_np64

pytestmark = pytest.mark.gpu

W = mw.Workload


def e4m3_decode(b: np.ndarray) -> np.ndarray:
    b = b.astype(np.int64)
    s, e, m = b >> 7, (b >> 3) & 15, b & 7
    v = np.where(e == 0, (m / 8.0) * 2.0 ** -6, (1.0 + m / 8.0) * np.exp2(e - 7.0))
    return np.where(s == 1, -v, v)


def decode_matrix(q: np.ndarray, sf: np.ndarray, rows: int, K: int) -> np.ndarray:
    """Dequantised [rows][K] from E4M3 bytes and the scale atoms."""
    vals = e4m3_decode(q.reshape(rows, K))
    r = np.arange(rows)[:, None]
    kb = np.arange(K // 32)[None, :]
    off = ((r // 128) * (K // 128) + kb // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + kb % 4
    X = sf[off].astype(np.int64) - 127
    return vals * np.repeat(np.exp2(X.astype(np.float64)), 32, axis=1)


LAYERS = [
    W("mx_decode_like", T=64, d=256, E=16, F=256, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True, seed=81),
    W("mx_relu_cap", T=500, d=256, E=8, F=384, k=2, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.0, seed=82),
    W("mx_swiglu_lam", T=700, d=384, E=6, F=256, k=2, act=mw.SWIGLU, dtype=mw.BF16, lam=1.0, zipf_bias=True,
      seed=83),
    W("mx_E1", T=130, d=128, E=1, F=128, k=1, act=mw.RELU, dtype=mw.BF16, seed=84),
    W("mx_many_rows", T=1500, d=256, E=4, F=256, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=85),
    # at most 64 tokens with ReLU: the narrow stage layout's other activation,
    # and one expert holding every token (k = E = 2)
    W("mx_relu_narrow", T=40, d=256, E=2, F=384, k=2, act=mw.RELU, dtype=mw.BF16, seed=86),
]


def _prepare(w, inp):
    cfg = moe.make_config(w.T, w.d, w.E, w.F, w.k, w.act, w.dtype, w.capacity_factor, w.lam)
    w1, w2 = mw.to_device(inp.w1), mw.to_device(inp.w2)
    return cfg, moe.prepare_mxfp8(cfg, w1, w2)


@pytest.mark.parametrize("w", [LAYERS[0], LAYERS[1]], ids=["swiglu", "relu"])
def test_prepared_weights_equal_the_oracle_quantisation(w):
    inp = mw.generate(w)
    cfg, (w1q, w1s, w2q, w2s) = _prepare(w, inp)
    torch.cuda.synchronize()
    F1 = w.F1
    W1 = decode_matrix(w1q.cpu().numpy(), w1s.cpu().numpy(), w.E * F1, w.d).reshape(w.E, F1, w.d)
    W2 = decode_matrix(w2q.cpu().numpy(), w2s.cpu().numpy(), w.E * w.d, w.F).reshape(w.E, w.d, w.F)
    if w.act == mw.SWIGLU:   # undo the interleave: rows [128 b, +64) gate 64 b.., the next 64 up 64 b..
        F = w.F
        perm = np.empty(F1, dtype=np.int64)
        for b in range(F // 64):
            perm[128 * b:128 * b + 64] = np.arange(64 * b, 64 * b + 64)
            perm[128 * b + 64:128 * b + 128] = F + np.arange(64 * b, 64 * b + 64)
        W1u = np.empty_like(W1)
        W1u[:, perm, :] = W1
        W1 = W1u
    for e in range(w.E):
        assert np.array_equal(W1[e], mf.mxq(mw.to_f64(inp.w1[e]))), f"W1[{e}]"
        assert np.array_equal(W2[e], mf.mxq(mw.to_f64(inp.w2[e]))), f"W2[{e}]"


# The kernel accumulates the exact E4M3 products in fp32 and evaluates the
# activation in fp32: each pre-activation within REL * sum|x w| of the exact
# one and the activation within REL relative -- a reading with margin (fp32
# accumulation over d <= 4096 in blocks of 32 keeps well below it).
REL = 2.0 ** -16


def _align256(n):
    return (n + 255) // 256 * 256


def mx_regions(cfg, w):
    """Byte offsets of the MX forward's own workspace regions, which follow
    the bf16 forward's: padded offsets, xq, xs, hq, hs and the expert
    kernel's counters (the layout of moe_workspace_size_mxfp8, checked
    against its total)."""
    _, lay = moe.moe_workspace_size(cfg)
    rows = w.T * w.k + 127 * w.E
    R = (rows + 127) // 128 * 128
    sb = lambda K: (R // 128) * (K // 128) * 512
    off = lay.total
    reg = {}
    for name, n in (("pad", 4 * (w.E + 1)), ("xq", R * w.d), ("xs", sb(w.d)), ("hq", R * w.F), ("hs", sb(w.F)),
                    ("ctr", 4 * (1 + R // 128))):
        reg[name] = off
        off = _align256(off + n)
    assert off == moe.moe_workspace_size_mxfp8(cfg)
    return reg, R


def decode_rows(q, sf, R, K, rows):
    """Dequantised rows `rows` of an [R][K] MX matrix, and their block exponents."""
    vals = e4m3_decode(q.reshape(R, K)[rows])
    r = rows[:, None]
    kb = np.arange(K // 32)[None, :]
    off = ((r // 128) * (K // 128) + kb // 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) // 32) + kb % 4
    X = sf[off].astype(np.int64) - 127
    return vals * np.repeat(np.exp2(X.astype(np.float64)), 32, axis=1), X


def run_mx(w):
    """One MX forward checked in three parts against the oracle: the
    quantised input rows bit for bit; the quantised hidden activation as an
    admissible quantisation of the exact one (equal except at decisions the
    fp32 evaluation may take either way, counted); the output from the
    device's own hidden activation to fp32 accumulation, and end to end on
    every token none of whose hidden values took such a decision."""
    inp = mw.generate(w)
    cfg, (w1q, w1s, w2q, w2s) = _prepare(w, inp)
    x, wg, bias = mw.to_device(inp.x), mw.to_device(inp.wg), mw.to_device(inp.bias)
    T = w.T
    ws = torch.empty(moe.moe_workspace_size_mxfp8(cfg), dtype=torch.uint8, device="cuda")
    ws.fill_(0xFF)
    out = torch.empty((T, w.d), dtype=torch.float32, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_mxfp8(cfg, x, wg, bias, w1q, w1s, w2q, w2s, out, stats, ws)
    torch.cuda.synchronize()
    st = moe.read_stats(stats)
    assert st["status"] == 0, st
    n, lay = moe.moe_workspace_size(cfg)
    idx = ws[lay.topk_idx:lay.topk_idx + 4 * T * w.k].view(torch.int32).view(T, w.k).cpu().numpy()
    lc = oracle.LayerConfig.from_workload(w)
    xx, wgg = mw.to_f64(inp.x), mw.to_f64(inp.wg)
    r0 = om.route(xx, wgg, inp.bias, lc)
    forced, n_tie = check_routing(idx, r0)
    r = om.route(xx, wgg, inp.bias, lc, forced, idx) if n_tie else r0
    d = om.dispatch(r.idx, lc, r.prob_mean)
    assert st["drop_count"] == d.drop_count and st["rows_kept"] == int(d.offsets[-1])
    w1, w2 = mw.F64Experts(inp.w1), mw.F64Experts(inp.w2)
    fw = mf.forward(xx, wgg, inp.bias, w1, w2, lc, forced if n_tie else None, idx if n_tie else None)
    dsp = fw.dispatch
    nrow = int(dsp.offsets[-1])
    # the device's padded row of every kept row: expert segments start at multiples of 128
    reg, R = mx_regions(cfg, w)
    host = ws.cpu().numpy()
    pad = host[reg["pad"]:reg["pad"] + 4 * (w.E + 1)].view(np.int32)
    cnt = np.diff(dsp.offsets)
    assert np.array_equal(pad, np.concatenate([[0], np.cumsum((cnt + 127) // 128 * 128)]))
    e_of = np.repeat(np.arange(w.E), cnt)
    prow = pad[e_of] + np.arange(nrow) - dsp.offsets[e_of]
    # 1. the quantised input rows: exact (the same integer decisions on bf16 values)
    xd, _ = decode_rows(host[reg["xq"]:reg["xq"] + R * w.d], host[reg["xs"]:], R, w.d, prow)
    assert np.array_equal(xd, mf.mxq(xx[dsp.src_tok])), "quantised input rows"
    # 2. the quantised hidden activation
    hd, Xd = decode_rows(host[reg["hq"]:reg["hq"] + R * w.F], host[reg["hs"]:], R, w.F, prow)
    win = mf.hidden_windows(xx, w1, lc, dsp, REL)
    ok, diff = mf.admits(hd, Xd, fw.h, win)
    assert ok.all(), f"{(~ok).sum()} hidden values not a quantisation within the window, rows {np.nonzero(~ok)[0][:8]}"
    nflip = int(diff.sum())
    assert nflip <= 1e-3 * diff.size + 2, f"{nflip} of {diff.size} hidden values took the other decision"
    # 3a. the output from the device's own hidden activation
    w2q = mf.MXExperts(w2)
    yp = np.zeros((nrow, w.d))
    for e in range(w.E):
        a, b = int(dsp.offsets[e]), int(dsp.offsets[e + 1])
        if a < b:
            yp[a:b] = hd[a:b] @ w2q[e].T
    ref = om.combine(yp, dsp.row_of, r.w, T, w.d)
    o = to_np64(out)
    rms = float(np.sqrt(np.mean(fw.out ** 2))) if T else 1.0
    err2 = float(np.max(np.abs(o - ref))) if T else 0.0
    assert err2 <= 1e-4 * rms, f"layer 2 from the device's h: max|err| {err2:.3e} > 1e-4 * RMS {rms:.3e}"
    # 3b. end to end on the tokens whose hidden values all took the oracle's decisions
    flip_row = diff.any(axis=1)
    flip_tok = np.zeros(T, dtype=bool)
    for j in range(w.k):
        r_ = dsp.row_of[:, j]
        flip_tok |= (r_ >= 0) & flip_row[np.maximum(r_, 0)]
    keep = ~flip_tok
    err = float(np.max(np.abs(o[keep] - fw.out[keep]))) if keep.any() else 0.0
    assert err <= 1e-4 * rms, f"max|err| {err:.3e} > 1e-4 * RMS {rms:.3e} ({flip_tok.sum()} tokens apart)"
    return err / rms, nflip, int(flip_tok.sum())


@pytest.mark.parametrize("w", LAYERS, ids=[w.name for w in LAYERS])
def test_mxfp8_forward_matches_mx_oracle(w):
    rel, nflip, ntok = run_mx(w)
    print(w.name, f"max|err|/RMS {rel:.2e}, {nflip} hidden values on the other side ({ntok} tokens)")


@pytest.mark.parametrize("name", ["fine_decode_dropless", "fine_decode_cap"])
def test_mxfp8_decode_layer(name):
    rel, nflip, ntok = run_mx(mw.WORKLOADS[name])
    print(name, f"max|err|/RMS {rel:.2e}, {nflip} hidden values on the other side ({ntok} tokens)")


@pytest.mark.parametrize("name", ["mixtral_8x7b"])
def test_mxfp8_full_size_sampled(name):
    """The FP8 layer at a full bench size (Mixtral-8x7B shape: 32,768 rows
    over 8 experts, long segments): routing exact off near ties, drops and
    kept rows as the oracle's, and the output on 64 sampled tokens within
    2e-2 * RMS of the MX oracle.  At F = 14336 a hidden value that took the
    other rounding side moves an output element by about 1e-3 of RMS, so the
    bar holds without reading the hidden activation back."""
    w = mw.WORKLOADS[name]
    inp = mw.generate(w)
    cfg, (w1q, w1s, w2q, w2s) = _prepare(w, inp)
    x, wg, bias = mw.to_device(inp.x), mw.to_device(inp.wg), mw.to_device(inp.bias)
    T = w.T
    ws = torch.empty(moe.moe_workspace_size_mxfp8(cfg), dtype=torch.uint8, device="cuda")
    out = torch.empty((T, w.d), dtype=torch.float32, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_mxfp8(cfg, x, wg, bias, w1q, w1s, w2q, w2s, out, stats, ws)
    torch.cuda.synchronize()
    st = moe.read_stats(stats)
    assert st["status"] == 0, st
    _, lay = moe.moe_workspace_size(cfg)
    idx = ws[lay.topk_idx:lay.topk_idx + 4 * T * w.k].view(torch.int32).view(T, w.k).cpu().numpy()
    lc = oracle.LayerConfig.from_workload(w)
    xx, wgg = mw.to_f64(inp.x), mw.to_f64(inp.wg)
    r0 = om.route(xx, wgg, inp.bias, lc)
    forced, n_tie = check_routing(idx, r0)
    r = om.route(xx, wgg, inp.bias, lc, forced, idx) if n_tie else r0
    d = om.dispatch(r.idx, lc, r.prob_mean)
    assert st["drop_count"] == d.drop_count and st["rows_kept"] == int(d.offsets[-1])
    toks = np.sort(np.random.default_rng(3).choice(T, size=64, replace=False))
    toks = np.unique(np.concatenate([toks, [0, T - 1]]))
    ref = mf.forward_tokens(xx, mw.F64Experts(inp.w1), mw.F64Experts(inp.w2), lc, r, d, toks)
    o = to_np64(out[torch.from_numpy(toks).cuda()])
    rms = float(np.sqrt(np.mean(ref ** 2)))
    err = float(np.max(np.abs(o - ref)))
    print(name, f"FP8 max|err|/RMS {err / rms:.3e} on {len(toks)} tokens, {n_tie} near-tie tokens")
    assert err <= 2e-2 * rms
    del ws, out, w1q, w1s, w2q, w2s
    torch.cuda.empty_cache()
