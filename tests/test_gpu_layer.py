"""Whole-layer parity of moe_layer_forward against the float64 oracle.

* small/medium layers and the decode-sized workloads: every output element;
* the full-size workloads (FastMoE 8192 x 512, Skywork 4096 x 4096, Mixtral
  16384 x 4096, fine-grained 32768 x 2048): routing, counts, permutation and
  drop mask over all tokens, outputs on sampled tokens the oracle evaluates one
  by one (the FastMoE layer is small enough to check in full);
* edge cases: no tokens, one token, k = E, one expert, determinism."""
import dataclasses

import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
from oracle import moe_oracle as om
from tests import gpu_harness as gh
from tests.gpu_harness import DeviceLayer, check_routing, check_dispatch_exact, check_out, lcfg_of, to_np64

pytestmark = pytest.mark.gpu

W = mw.Workload


def run_and_check(L: DeviceLayer, sample: int = 0, seed: int = 0, tol=gh.BF16_TOL, want_ref: bool = False):
    res = L.forward()
    x = mw.to_f64(L.inp.x)
    wg = mw.to_f64(L.inp.wg)
    w1, w2 = mw.F64Experts(L.inp.w1), mw.F64Experts(L.inp.w2)
    cfg = lcfg_of(L.w, L.T)
    r0 = om.route(x, wg, L.inp.bias, cfg)
    forced, n_tie = check_routing(res["topk_idx"], r0)
    # near-tie tokens take the device's selection; everything downstream exact
    r = om.route(x, wg, L.inp.bias, cfg, forced, res["topk_idx"]) if n_tie else r0
    d = om.dispatch(r.idx, cfg, r.prob_mean)
    check_dispatch_exact(res, d, r, res["topk_idx"])
    st = res["stats"]
    assert st["status"] == 0
    assert st["drop_count"] == d.drop_count and st["rows_kept"] == int(d.offsets[-1])
    assert st["capacity"] == (-1 if d.C is None else d.C)
    if L.T > 0:
        assert abs(st["aux_loss"] - d.aux) <= 1e-4 * max(1.0, abs(d.aux))
        assert abs(st["drop_rate"] - d.drop_rate) <= 1e-6
        # router z-loss over every token (it does not depend on the selection)
        assert abs(st["z_loss"] - r0.z_loss) <= 1e-4 * abs(r0.z_loss), (st["z_loss"], r0.z_loss)
    else:
        assert np.isnan(st["z_loss"]) and np.isnan(st["aux_loss"])
    out = res["out"]
    if sample and sample < L.T:
        toks = np.sort(np.random.default_rng(seed).choice(L.T, size=sample, replace=False))
        toks = np.unique(np.concatenate([toks, [0, L.T - 1]]))
        ref = om.forward_tokens(x, w1, w2, cfg, r, d, toks)
        dev = to_np64(out[torch.from_numpy(toks).cuda()])
    else:
        toks = np.arange(L.T)
        ref = om.combine(om.expert_segments(x[d.src_tok], d.offsets, w1, w2, cfg)[1], d.row_of, r.w, L.T, L.w.d)
        dev = to_np64(out)
    rel = check_out(dev, ref, L.w.dtype, tol)
    if want_ref:
        return res, rel, n_tie, (toks, dev, ref, r, d)
    return res, rel, n_tie


MEDIUM = [
    W("m_relu_cap", T=777, d=256, E=12, F=320, k=3, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.1, seed=21),
    W("m_swiglu_lam", T=1000, d=192, E=8, F=208, k=2, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=0.9, lam=1.0,
      zipf_bias=True, seed=22),
    W("m_fp32", T=300, d=64, E=5, F=96, k=2, act=mw.RELU, dtype=mw.F32, seed=23),
    W("m_fine", T=700, d=128, E=64, F=176, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True, capacity_factor=1.0,
      seed=24),
    W("m_kE", T=150, d=64, E=4, F=64, k=4, act=mw.SWIGLU, dtype=mw.BF16, lam=1.0, seed=25),
    W("m_one", T=1, d=64, E=8, F=64, k=2, act=mw.RELU, dtype=mw.BF16, seed=26),
    W("m_E1", T=200, d=64, E=1, F=128, k=1, act=mw.SWIGLU, dtype=mw.BF16, seed=27),
    W("m_long_k", T=333, d=64, E=40, F=48, k=12, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.2, seed=28),
    W("m_multi_tile", T=3000, d=512, E=4, F=640, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=29),   # 2-SM tiles
    W("m_pair_relu_cap", T=2600, d=128, E=8, F=192, k=2, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.1,
      seed=30),                                                                                  # 2-SM tiles
    # one-launch expert kernel with the largest expert count: 256 tile-table
    # entries and dependency counters, many experts with no rows
    W("m_E256_k2", T=900, d=64, E=256, F=64, k=2, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=1.5, lam=1.0,
      zipf_bias=True, seed=32),
    # gate GEMM cut over the model width (2 chunks x 4 slices of 6 k-blocks)
    W("m_ksplit", T=200, d=1536, E=32, F=96, k=4, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=1.25, lam=1.0,
      seed=35),
]


@pytest.mark.parametrize("w", MEDIUM, ids=[w.name for w in MEDIUM])
def test_layer_medium(w):
    run_and_check(DeviceLayer(w))


def test_layer_empty_tokens():
    w = W("empty", T=0, d=64, E=4, F=64, k=2, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.0)
    L = DeviceLayer(w)
    res = L.forward()
    assert res["out"].numel() == 0
    assert res["stats"]["rows_kept"] == 0 and res["stats"]["drop_count"] == 0
    assert np.all(res["offsets"] == 0) and np.all(res["counts"] == 0)
    assert res["stats"]["drop_rate"] == 0.0 and np.isnan(res["stats"]["aux_loss"])
    assert np.isnan(res["stats"]["z_loss"])


@pytest.mark.parametrize("name", ["fastmoe_txl", "m_relu_cap", "m_multi_tile"])
def test_layer_bf16_hidden(name):
    """The bf16 hidden activation (h and W2 in bf16) also meets the output
    tolerance on these layers; on the capacity-mode fine-grained layers its
    single rounding of h reaches ~0.026 RMS, above 2e-2, which is why fp16 is
    the default hidden type."""
    w = mw.WORKLOADS.get(name) or next(m for m in MEDIUM if m.name == name)
    L = DeviceLayer(w, hidden="bf16")
    assert L.hidden == "bf16"
    run_and_check(L)


def hidden_rounding_bound(x, w1, w2, cfg, r, d, toks) -> np.ndarray:
    """Element-wise bound on what rounding h to bf16 (relative error <= 2^-9)
    can move the output: per kept slot, w * 2^-9 * |h| |W2[e]|^T, doubled as
    margin for the fp32 accumulations around it (which may also flip a
    rounding)."""
    bound = np.zeros((len(toks), cfg.d))
    by_expert = {}
    for i, t in enumerate(toks):
        for j in range(cfg.k):
            if d.row_of[t, j] >= 0:
                by_expert.setdefault(int(r.idx[t, j]), []).append((i, int(t), j))
    for e, lst in by_expert.items():
        h = om.expert_hidden(x[[t for _, t, _ in lst]], w1[e], cfg.act, cfg.F)
        b = np.abs(h) @ np.abs(np.asarray(w2[e], np.float64)).T
        for row, (i, t, j) in zip(b, lst):
            bound[i] += r.w[t, j] * row
    return 2.0 ** -8 * bound


# Whether the bf16 hidden activation's output stays within 2e-2 * RMS(out) on
# each named bf16 layer (the fp16 default meets it on all of them).
BF16_HIDDEN_MEETS_RMS_BAR = {
    "fastmoe_txl": True,
    "skywork_lambda1": True,
    "mixtral_8x7b": True,
    "fine_decode_dropless": True,
    "fine_decode_cap": False,
    "fine_large_dropless": True,
    "fine_large_cap": False,
}


@pytest.mark.parametrize("name", sorted(BF16_HIDDEN_MEETS_RMS_BAR))
def test_bf16_hidden_every_layer(name):
    """hidden_dtype bf16 on every named bf16 layer: routing and permutation
    exact as always; the output within the element-wise bound of h's one
    bf16 rounding (hidden_rounding_bound) everywhere checked, and against the
    2e-2 RMS bar as BF16_HIDDEN_MEETS_RMS_BAR records."""
    w = mw.WORKLOADS[name]
    L = DeviceLayer(w, hidden="bf16")
    assert L.hidden == "bf16"
    sample = 0 if w.T <= 8192 else 192
    _, rel, _, (toks, dev, ref, r, d) = run_and_check(L, sample=sample, seed=1, tol=None, want_ref=True)
    x = mw.to_f64(L.inp.x)
    w1, w2 = mw.F64Experts(L.inp.w1), mw.F64Experts(L.inp.w2)
    bound = hidden_rounding_bound(x, w1, w2, lcfg_of(L.w, L.T), r, d, toks)
    rms = float(np.sqrt(np.mean(ref ** 2)))
    excess = np.abs(dev - ref) - (bound + 1e-5 * rms)
    assert np.all(excess <= 0), f"{int((excess > 0).sum())} elements past the bf16 rounding bound"
    print(name, f"bf16 hidden: max|err|/RMS {rel:.3e}, max|err|/bound {float(np.max(np.abs(dev - ref) / (bound + 1e-5 * rms))):.3f}")
    assert (rel <= gh.BF16_TOL) == BF16_HIDDEN_MEETS_RMS_BAR[name], f"max|err|/RMS {rel:.3e}"
    del L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["m_swiglu_lam", "m_relu_cap", "m_ksplit"])
def test_layer_poisoned_workspace(name):
    """Every workspace word the forward reads is written earlier in the same
    call, so a workspace and output filled with 0xFF bytes give the same
    result.  This covers the expert kernel's tile-queue counters, which the
    scatter zeroes (in the yp region for k <= 2, in scratch for k > 2), and the
    route's arrival counters on a model-width split (m_ksplit)."""
    w = next(m for m in MEDIUM if m.name == name)
    L = DeviceLayer(w)
    a = L.forward()
    b = L.forward(poison=0xFF)
    assert b["stats"]["status"] == 0
    assert torch.equal(a["out"], b["out"])
    assert a["stats"] == b["stats"]


def test_layer_deterministic():
    L = DeviceLayer(MEDIUM[1])
    a = L.forward()
    b = L.forward()
    assert torch.equal(a["out"], b["out"])
    assert a["stats"] == b["stats"]


@pytest.mark.parametrize("name", ["m_ksplit", "fine_decode_dropless"])
def test_layer_deterministic_split_route(name):
    """The width-split route (partial logits summed over a cluster, rows gated
    per CTA, the chunk's sums gathered in CTA 0) and, on the decode layer, the
    narrow expert tiles give bit-identical results run to run."""
    w = next((m for m in MEDIUM if m.name == name), None) or mw.WORKLOADS[name]
    L = DeviceLayer(w)
    a = L.forward()
    b = L.forward()
    for key in ("topk_idx", "topk_w", "gap", "counts", "row_of"):
        assert np.array_equal(a[key], b[key]), key
    assert torch.equal(a["out"], b["out"])
    assert a["stats"] == b["stats"]


# dropless layers for a token with a NaN in its row: the tensor-core route with
# four threads per token (and the fused combine), the same route cut over the
# model width (one cluster of 4 slices per chunk, a warp per token), top-6
# with the separate combine, and the fp32 route on CUDA cores
NAN_LAYERS = {
    "nan_quarter": W("nan_quarter", T=300, d=256, E=16, F=64, k=2, act=mw.RELU, dtype=mw.BF16, seed=41),
    "nan_split": W("nan_split", T=200, d=1024, E=16, F=64, k=2, act=mw.SWIGLU, dtype=mw.BF16, lam=1.0, seed=42),
    "nan_k6": W("nan_k6", T=500, d=128, E=64, F=176, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True, seed=43),
    "nan_fp32": W("nan_fp32", T=300, d=64, E=5, F=96, k=2, act=mw.RELU, dtype=mw.F32, seed=44),
}


@pytest.mark.parametrize("name", sorted(NAN_LAYERS))
def test_nan_token_is_dropped_and_flagged(name):
    """A token whose row of x holds a NaN has no score above -inf: its k slots
    stay empty (outside [0, E)), it adds nothing to the histogram, the forward
    sets MOE_DEV_BOUNDS and the token's output row is zero.  Every other
    token's selection, gate weights and output are bit-identical to those of
    the same forward without the NaN (routing is per token, and a row's
    expert outputs do not depend on its position in the segment)."""
    w = NAN_LAYERS[name]
    inp = mw.generate(w)
    clean = DeviceLayer(w, inp).forward()
    assert clean["stats"]["status"] == 0
    bad = 37
    x = inp.x.copy()
    x[bad, 3] = 0x7FC0 if w.dtype == mw.BF16 else np.float32(np.nan)   # bf16 bits of a quiet NaN
    r = DeviceLayer(w, dataclasses.replace(inp, x=x)).forward()
    assert r["stats"]["status"] == moe.MOE_DEV_BOUNDS
    assert np.all((r["topk_idx"][bad] < 0) | (r["topk_idx"][bad] >= w.E))
    assert np.all(r["row_of"][bad] == -1)
    others = np.arange(w.T) != bad
    assert np.array_equal(r["topk_idx"][others], clean["topk_idx"][others])
    assert np.array_equal(r["topk_w"][others].view(np.uint32), clean["topk_w"][others].view(np.uint32))
    assert np.array_equal(r["counts"], np.bincount(clean["topk_idx"][others].ravel(), minlength=w.E))
    assert r["stats"]["rows_kept"] == (w.T - 1) * w.k
    out, ref = r["out"].cpu(), clean["out"].cpu()
    assert torch.all(out[bad] == 0)
    assert torch.equal(out[torch.from_numpy(others)], ref[torch.from_numpy(others)])


@pytest.mark.parametrize("name", ["tiny_fp32", "fastmoe_txl", "fine_decode_dropless", "fine_decode_cap"])
def test_layer_named_full(name):
    _, rel, _ = run_and_check(DeviceLayer(mw.WORKLOADS[name]))
    print(name, f"max|err| over the bar's scale {rel:.3e}")
    assert rel < 1.0


@pytest.mark.parametrize("name", ["skywork_lambda1", "mixtral_8x7b", "fine_large_dropless", "fine_large_cap"])
def test_layer_named_full_size_sampled(name):
    L = DeviceLayer(mw.WORKLOADS[name])
    _, rel, n_tie = run_and_check(L, sample=192, seed=1)
    print(name, f"max|err|/RMS {rel:.3e} (192 sampled tokens), {n_tie} near-tie tokens")
    assert rel < 1.0
    del L
    torch.cuda.empty_cache()


@pytest.mark.parametrize("name", ["m_swiglu_lam", "m_E1", "m_one", "m_pair_relu_cap", "m_E256_k2", "fastmoe_txl"])
def test_fused_combine_matches_the_steps(name):
    """bf16 layers with k <= 2: the forward adds the gate-weighted expert
    outputs inside the second GEMM (out zeroed by the permutation) instead of
    writing yp and running the combine kernel.  It must agree with the four
    step calls to fp32 rounding (w*y rounded, then one addition, against one
    fused multiply-add), and it must leave a token whose slots were all
    dropped at exactly zero."""
    w = mw.WORKLOADS.get(name) or next(m for m in MEDIUM if m.name == name)
    assert w.dtype == mw.BF16 and w.k <= 2
    L = DeviceLayer(w)
    fused = L.forward()["out"]
    idx, wt, gap, pm = L.route()
    perm = L.permute(idx, gap, pm)
    _, yp, _ = L.expert_ffn(perm["xp"], perm["offsets"])
    steps = L.combine(yp, perm["row_of"], wt)
    torch.cuda.synchronize()
    scale = float(steps.abs().max())
    assert float((fused - steps).abs().max()) <= 1e-6 * max(scale, 1e-30)
    dropped = (perm["row_of"] < 0).all(dim=1)
    assert torch.equal(fused[dropped], torch.zeros_like(fused[dropped]))


@pytest.mark.parametrize("name", ["fastmoe_txl", "m_swiglu_lam", "m_pair_relu_cap", "m_one", "m_E1"])
def test_expert_ffn_combine_entry_matches_forward(name):
    """moe_expert_ffn_combine runs steps 4-5 exactly as the forward does
    (one-launch kernel on 1-SM tiles, pair tiles otherwise): given the
    forward's permuted rows, tokens and row weights, and a zeroed out, it
    must reproduce the forward's output bit for bit, on two calls in a row."""
    w = mw.WORKLOADS.get(name) or next(m for m in MEDIUM if m.name == name)
    L = DeviceLayer(w)
    res = L.forward()
    ws, lay = res["ws"], res["layout"]
    T, k, d, F, E = L.T, w.k, w.d, w.F, w.E
    A = T * k

    def v(off, n, dt):
        return ws[off:off + n * torch.tensor([], dtype=dt).element_size()].view(dt)

    xp = v(lay.xp, A * d, L.tdt)
    offsets, src_tok, row_w = v(lay.offsets, E + 1, torch.int32), v(lay.src_tok, A, torch.int32), v(lay.row_w, A, torch.float32)
    h = torch.empty((A, F), dtype=L.hdt, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        out = torch.zeros((T, d), dtype=torch.float32, device="cuda")
        moe.moe_expert_ffn_combine(L.cfg, xp, offsets, src_tok, row_w, L.w1, L.w2, h, out, stats, ws)
        torch.cuda.synchronize()
        assert torch.equal(out, res["out"]), name
    assert moe.read_stats(stats)["status"] == 0
