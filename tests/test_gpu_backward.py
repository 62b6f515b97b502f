"""Parity of the layer's backward (moe_layer_backward, through the C ABI)
against the float64 backward oracle, which is itself pinned by finite
differences of the forward oracle.

For each layer: the forward runs (moe_layer_forward), then the backward of
L = <dout, out> + aux_coef * aux + z_coef * z_loss on the forward's workspace.
Every gradient is compared element by element with the oracle's:

* fp32 path: max|err| <= 1e-4 * max|ref| for every tensor;
* bf16 path with the default fp16 hidden type (fp16 GEMM operands, dout
  scaled by a power of two): every gradient within 2e-2 * RMS(ref);
* bf16 path, the expert weight gradients dW1 and dW2, in addition: each is a
  contraction over the expert's rows of operands rounded once each (dout and
  w*h for dW2; du, which carries the rounding of dout and its own, for dW1),
  so each product is off by at most 2u relative (u = 2^-11 for fp16 operands,
  2^-9 for bf16).  The bound is element by element:
  |err| <= 4u * (the same contraction over absolute values) + 1e-6 max|ref|
  (a factor 2 over the rounding model, for the fp32 accumulation).  A wrong
  row, column or expert gives an error of the size of the gradient itself and
  fails it.  With a bf16 hidden type (bf16 operands) this bound is the bar for
  dW1 and dW2: on layers whose weight gradients have heavy tails the bf16
  roundings alone put max|err| above 2e-2 RMS (reported, not asserted), and
  the other gradients are held to 4e-2 RMS (two bf16 roundings, of dout and
  of du, feed them: 8x those of the fp16 default, which meets 2e-2).

Near-tie tokens take the device's selection in the oracle (both selections are
correct there)."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
import oracle
from oracle import moe_oracle as om
from oracle import moe_backward as ob
from tests.gpu_harness import DeviceLayer, to_np64

pytestmark = pytest.mark.gpu

W = mw.Workload
LAYERS = [
    W("b_relu_cap", T=777, d=256, E=12, F=320, k=3, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.1, seed=71),
    W("b_swiglu_lam_bias", T=1000, d=192, E=8, F=208, k=2, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=0.9,
      lam=1.0, zipf_bias=True, seed=72),
    W("b_fine_top6", T=500, d=128, E=64, F=176, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True, seed=73),
    W("b_wide", T=600, d=512, E=4, F=544, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=74),
    W("b_E1", T=130, d=64, E=1, F=64, k=1, act=mw.RELU, dtype=mw.BF16, seed=75),
    W("b_fp32_relu", T=300, d=64, E=5, F=96, k=2, act=mw.RELU, dtype=mw.F32, capacity_factor=1.0, seed=76),
    W("b_fp32_swiglu", T=257, d=32, E=6, F=40, k=3, act=mw.SWIGLU, dtype=mw.F32, lam=0.5, seed=77),
    # T*k >= 512*E: every expert GEMM of the backward on 2-SM pair tiles
    # (ragged: F and F1 not multiples of 256, segments not multiples of 256)
    W("b_pair_swiglu", T=1300, d=256, E=4, F=320, k=2, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True, seed=78),
    W("b_pair_relu_cap", T=2600, d=192, E=8, F=448, k=2, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.1,
      seed=79),
]
AUX, ZC = 0.05, 0.01


def _close(got, ref, dtype, name, bar=2e-2):
    if ref.size == 0:
        return 0.0
    err = float(np.max(np.abs(got - ref)))
    if dtype == mw.BF16:
        rms = float(np.sqrt(np.mean(ref ** 2)))
        assert err <= bar * rms, f"{name}: max|err| {err:.3e} > {bar} * RMS {rms:.3e}"
        return err / rms
    scale = float(np.max(np.abs(ref)))
    assert err <= 1e-4 * scale, f"{name}: max|err| {err:.3e} > 1e-4 * max|ref| {scale:.3e}"
    return err / scale


def run_backward(L: DeviceLayer, seed: int):
    w, cfg = L.w, L.cfg
    # bf16 operands (a bf16 hidden type) round dout and du 8x coarser than fp16:
    # their bar for the non-weight gradients is 4e-2 RMS (weight gradients: the rounding bound)
    bar = 4e-2 if L.hidden == "bf16" else 2e-2
    res = L.forward()
    T, d, E, F, k = L.T, w.d, w.E, w.F, w.k
    F1 = F if w.act == mw.RELU else 2 * F
    rng = np.random.default_rng(seed)
    dout = rng.standard_normal((T, d)).astype(np.float32)
    w2_bwd = L.w2                         # W2 in the hidden type, as the forward took it
    dev = "cuda"
    dx = torch.empty((max(T, 1), d), dtype=torch.float32, device=dev)
    dwg = torch.empty((E, d), dtype=torch.float32, device=dev)
    dbg = torch.empty((E,), dtype=torch.float32, device=dev)
    dw1 = torch.full((E, F1, d), float("nan"), dtype=torch.float32, device=dev)
    dw2 = torch.full((E, d, F), float("nan"), dtype=torch.float32, device=dev)
    dw = torch.empty((max(T, 1), k), dtype=torch.float32, device=dev)
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device=dev)
    ws = torch.empty(moe.moe_backward_workspace_size(cfg), dtype=torch.uint8, device=dev)
    ws.fill_(0xA5)   # stale contents must not leak into any gradient
    moe.moe_layer_backward(cfg, L.x, L.wg, L.bias, L.w1, w2_bwd, torch.from_numpy(dout).cuda(), AUX, ZC, res["ws"],
                           dx, dwg, dbg, dw1, dw2, dw, stats, ws)
    torch.cuda.synchronize()
    st = moe.read_stats(stats)
    assert st["status"] == 0, st
    # the oracle, with the device's selection on near-tie tokens
    lc = oracle.LayerConfig.from_workload(w, T)
    x, wg = mw.to_f64(L.inp.x), mw.to_f64(L.inp.wg)
    w1, w2 = mw.F64Experts(L.inp.w1), mw.F64Experts(L.inp.w2)
    r0 = om.route(x, wg, L.inp.bias, lc)
    forced = r0.gap < 1e-4
    fw = om.forward(x, wg, L.inp.bias, w1, w2, lc, forced if forced.any() else None,
                    res["topk_idx"] if forced.any() else None)
    g = ob.backward(x, wg, L.inp.bias, w1, w2, lc, dout.astype(np.float64), AUX, ZC, fw=fw,
                    want_abs=w.dtype == mw.BF16)
    out = {}
    out["dw"] = _close(dw.cpu().numpy().astype(np.float64)[:T], g.dw, w.dtype, "dw", bar)
    if w.dtype == mw.BF16:
        f16 = L.hidden == "f16"
        u = 2.0 ** -11 if f16 else 2.0 ** -9
        for name, got, ref, A in [("dW2", dw2, g.dw2, g.abs_dw2), ("dW1", dw1, g.dw1, g.abs_dw1)]:
            got = to_np64(got)
            err = np.abs(got - ref)
            bound = 4 * u * A + 1e-6 * float(np.max(np.abs(ref)))
            worst = float(np.max(err / bound))
            assert worst <= 1.0, f"{name}: |err| exceeds the rounding bound by {worst:.2f}x"
            rms = float(np.sqrt(np.mean(ref ** 2)))
            out[name] = float(np.max(err)) / rms
            out[name + "_of_bound"] = worst
            if f16:
                assert out[name] <= 2e-2, f"{name}: max|err| {out[name]:.3e} RMS > 2e-2"
    else:
        out["dW2"] = _close(to_np64(dw2), g.dw2, w.dtype, "dW2")
        out["dW1"] = _close(to_np64(dw1), g.dw1, w.dtype, "dW1")
    out["dx"] = _close(to_np64(dx[:T]), g.dx, w.dtype, "dx", bar)
    out["dWg"] = _close(to_np64(dwg), g.dwg, w.dtype, "dWg", bar)
    if L.inp.bias is not None:
        out["db"] = _close(to_np64(dbg), g.dbias, w.dtype, "db", bar)
    return out


@pytest.mark.parametrize("w", LAYERS, ids=[w.name for w in LAYERS])
def test_backward_matches_oracle(w):
    rel = run_backward(DeviceLayer(w), w.seed + 1000)
    print(w.name, {k: f"{v:.2e}" for k, v in rel.items()})


@pytest.mark.parametrize("name", ["b_relu_cap", "b_wide", "b_fine_top6", "b_pair_swiglu"])
def test_backward_bf16_hidden(name):
    """A bf16 hidden type: the backward's GEMM operands are bf16 (no dout
    scale); the weight gradients meet the bf16 rounding bound."""
    w = next(x for x in LAYERS if x.name == name)
    rel = run_backward(DeviceLayer(w, hidden="bf16"), 5)
    print(name, "bf16 operands", {k: f"{v:.2e}" for k, v in rel.items()})


def test_backward_scale_invariance():
    """dout scaled by 2^-20 (far below the fp16 range) gives gradients scaled
    by 2^-20 to within the same tolerance: the power-of-two scale of the fp16
    operands follows dout's magnitude."""
    w = LAYERS[0]
    L = DeviceLayer(w)
    res = L.forward()
    T, d, E, F, k = L.T, w.d, w.E, w.F, w.k
    F1 = F if w.act == mw.RELU else 2 * F
    g0 = np.random.default_rng(9).standard_normal((T, d)).astype(np.float32)
    outs = []
    for sc in (1.0, 2.0 ** -20):
        dx = torch.empty((T, d), dtype=torch.float32, device="cuda")
        dwg = torch.empty((E, d), dtype=torch.float32, device="cuda")
        dw1 = torch.empty((E, F1, d), dtype=torch.float32, device="cuda")
        dw2 = torch.empty((E, d, F), dtype=torch.float32, device="cuda")
        stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
        ws = torch.empty(moe.moe_backward_workspace_size(L.cfg), dtype=torch.uint8, device="cuda")
        moe.moe_layer_backward(L.cfg, L.x, L.wg, L.bias, L.w1, L.w2, torch.from_numpy(g0 * np.float32(sc)).cuda(),
                               0.0, 0.0, res["ws"], dx, dwg, None, dw1, dw2, None, stats, ws)
        torch.cuda.synchronize()
        assert moe.read_stats(stats)["status"] == 0
        outs.append([t.double().cpu().numpy() / sc for t in (dx, dwg, dw1, dw2)])
    for a, b in zip(*outs):
        assert np.array_equal(a, b), "the power-of-two scale must cancel exactly"


def test_backward_no_tokens():
    w = W("b_empty", T=0, d=64, E=4, F=64, k=2, act=mw.RELU, dtype=mw.BF16)
    L = DeviceLayer(w)
    res = L.forward()
    cfg = L.cfg
    dwg = torch.full((4, 64), 7.0, device="cuda")
    dw1 = torch.full((4, 64, 64), 7.0, device="cuda")
    dw2 = torch.full((4, 64, 64), 7.0, device="cuda")
    dbg = torch.full((4,), 7.0, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    ws = torch.empty(max(moe.moe_backward_workspace_size(cfg), 256), dtype=torch.uint8, device="cuda")
    moe.moe_layer_backward(cfg, None, L.wg, None, L.w1, mw.to_device(L.inp.w2), None, 0.0, 0.0, res["ws"], None,
                           dwg, dbg, dw1, dw2, None, stats, ws)
    torch.cuda.synchronize()
    assert torch.all(dwg == 0) and torch.all(dw1 == 0) and torch.all(dw2 == 0) and torch.all(dbg == 0)
