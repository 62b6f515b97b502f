"""Per-step parity of the CUDA path (through the C ABI) against the float64
oracle, at sizes the oracle runs in seconds that still span several tiles and
leave ragged tails (T not a multiple of the 64-token chunk, segments not a
multiple of the 128-row tile, F not a multiple of the 128/256-column tile)."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
from oracle import moe_oracle as om
from tests.gpu_harness import (DeviceLayer, check_routing, check_dispatch_exact, check_out, lcfg_of, to_np64,
                               NEAR_TIE)

pytestmark = pytest.mark.gpu

W = mw.Workload
MEDIUM = {
    "relu_cap_ragged": W("relu_cap_ragged", T=777, d=256, E=12, F=320, k=3, act=mw.RELU, dtype=mw.BF16,
                         capacity_factor=1.1, seed=11),
    "swiglu_lambda_bias": W("swiglu_lambda_bias", T=1000, d=192, E=8, F=208, k=2, act=mw.SWIGLU, dtype=mw.BF16,
                            capacity_factor=0.9, lam=1.0, zipf_bias=True, seed=12),
    "fp32_relu": W("fp32_relu", T=300, d=64, E=5, F=96, k=2, act=mw.RELU, dtype=mw.F32, seed=13),
    "fp32_swiglu_cap": W("fp32_swiglu_cap", T=257, d=32, E=6, F=40, k=3, act=mw.SWIGLU, dtype=mw.F32,
                         capacity_factor=1.0, lam=0.5, seed=14),
    "fine_top6": W("fine_top6", T=500, d=128, E=64, F=176, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True,
                   seed=15),
    "dense_E1": W("dense_E1", T=130, d=64, E=1, F=64, k=1, act=mw.RELU, dtype=mw.BF16, seed=16),
    "big_k10": W("big_k10", T=200, d=64, E=16, F=64, k=10, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.0,
                 seed=17),
    "E256": W("E256", T=300, d=64, E=256, F=32, k=4, act=mw.RELU, dtype=mw.BF16, seed=18),
    # T*k >= 512*E: the expert GEMMs run on 2-SM pair tiles (256 rows); ragged
    # segment ends, a ragged last n-tile (F = 320) and both activations
    "pair_relu_ragged": W("pair_relu_ragged", T=1100, d=256, E=4, F=320, k=2, act=mw.RELU, dtype=mw.BF16,
                          capacity_factor=1.25, seed=19),
    "pair_swiglu_lambda": W("pair_swiglu_lambda", T=1500, d=192, E=3, F=208, k=2, act=mw.SWIGLU, dtype=mw.BF16,
                            lam=1.0, seed=20),
    # model widths of more than one ring of gate loads on few chunks: the gate
    # GEMM is cut over the model width (4 slices here, the last one 5 k-blocks
    # with a zero-filled tail, d = 1072), one cluster per chunk whose CTAs each
    # sum and gate a share of the rows; E = 24 is not a multiple of 16, with
    # normalisation and a gate bias
    "ksplit_lambda_bias": W("ksplit_lambda_bias", T=300, d=1072, E=24, F=64, k=3, act=mw.SWIGLU, dtype=mw.BF16,
                            capacity_factor=1.0, lam=1.0, zipf_bias=True, seed=33),
    # one chunk, the largest expert count and k (4 slices of 2 k-blocks)
    "ksplit_E256_k8": W("ksplit_E256_k8", T=64, d=512, E=256, F=32, k=8, act=mw.RELU, dtype=mw.BF16, seed=34),
    # 8 slices of one chunk that holds fewer tokens than slices: one token
    # (seven CTAs gate no row), and nine (one or two rows per CTA)
    "ksplit_T1": W("ksplit_T1", T=1, d=2048, E=64, F=64, k=6, act=mw.SWIGLU, dtype=mw.BF16, zipf_bias=True,
                   seed=37),
    "ksplit_T9": W("ksplit_T9", T=9, d=2048, E=40, F=64, k=4, act=mw.RELU, dtype=mw.BF16, lam=1.0, seed=38),
}


@pytest.fixture(scope="module", params=sorted(MEDIUM))
def layer(request):
    w = MEDIUM[request.param]
    return DeviceLayer(w)


def oracle_inputs(L: DeviceLayer):
    x = mw.to_f64(L.inp.x)
    return x, mw.to_f64(L.inp.wg), L.inp.bias, mw.F64Experts(L.inp.w1), mw.F64Experts(L.inp.w2)


def test_route(layer):
    L = layer
    idx, wt, gap, pm, zl = L.route(want_z_loss=True)
    torch.cuda.synchronize()
    x, wg, b, _, _ = oracle_inputs(L)
    r = om.route(x, wg, b, lcfg_of(L.w, L.T))
    di = idx.cpu().numpy()
    nt, _ = check_routing(di, r)
    # weights / gaps / probability means against float64
    dw = wt.cpu().numpy()
    ok = ~nt
    ref_w = np.take_along_axis(r.p, di, axis=1)
    ref_w = ref_w / ref_w.sum(axis=1, keepdims=True)
    assert np.max(np.abs(dw[ok] - ref_w[ok])) < 2e-5
    assert np.allclose(dw.sum(axis=1), 1.0, atol=1e-5)
    dg = gap.cpu().numpy()
    fin = np.isfinite(r.gap)
    assert np.array_equal(np.isfinite(dg), fin)
    assert np.max(np.abs(dg[fin] - r.gap[fin]), initial=0.0) < 1e-4
    assert np.allclose(pm.cpu().numpy(), r.prob_mean, rtol=1e-5, atol=1e-7)
    # router z-loss: mean over tokens of the squared log-partition of the scores
    assert abs(float(zl.item()) - r.z_loss) <= 1e-4 * abs(r.z_loss), (float(zl.item()), r.z_loss)


def test_permute_exact(layer):
    """Permutation from the oracle's own selection: everything bit-exact."""
    L = layer
    x, wg, b, _, _ = oracle_inputs(L)
    cfg = lcfg_of(L.w, L.T)
    r = om.route(x, wg, b, cfg)
    d = om.dispatch(r.idx, cfg, r.prob_mean)
    idx = torch.from_numpy(r.idx.astype(np.int32)).cuda()
    gap = torch.from_numpy(r.gap.astype(np.float32)).cuda()
    pm = torch.from_numpy(r.prob_mean.astype(np.float32)).cuda()
    res = L.permute(idx, gap, pm)
    torch.cuda.synchronize()
    dev = {k: v.cpu().numpy() for k, v in res.items() if k not in ("xp", "stats")}
    check_dispatch_exact(dev, d, r, r.idx)
    assert np.array_equal(dev["row_of"], d.row_of)
    n = int(d.offsets[-1])
    # the gather is a bit copy of x rows
    xp = res["xp"][:n].cpu()
    ref = L.x.cpu()[torch.from_numpy(d.src_tok)]
    assert torch.equal(xp.view(torch.int16) if xp.dtype == torch.bfloat16 else xp,
                       ref.view(torch.int16) if ref.dtype == torch.bfloat16 else ref)
    st = moe.read_stats(res["stats"])
    assert st["drop_count"] == d.drop_count and st["rows_kept"] == n
    assert st["capacity"] == (-1 if d.C is None else d.C)
    assert st["status"] == 0
    assert abs(st["drop_rate"] - d.drop_rate) <= 1e-7
    assert abs(st["aux_loss"] - d.aux) <= 1e-5 * max(1.0, abs(d.aux))
    assert st["near_tie_count"] == int(np.sum(r.gap.astype(np.float32) < np.float32(NEAR_TIE)))


def test_expert_ffn(layer):
    """Grouped GEMMs on the oracle's permuted rows."""
    L = layer
    x, wg, b, w1, w2 = oracle_inputs(L)
    cfg = lcfg_of(L.w, L.T)
    r = om.route(x, wg, b, cfg)
    d = om.dispatch(r.idx, cfg, r.prob_mean)
    n = int(d.offsets[-1])
    A = max(L.T * L.w.k, 1)
    xp = torch.zeros((A, L.w.d), dtype=L.tdt, device="cuda")
    xp[:n] = L.x[torch.from_numpy(d.src_tok).cuda()]
    # poison the unused rows: results must not depend on them
    if n < A:
        xp[n:] = float("nan")
    off = torch.from_numpy(d.offsets.astype(np.int32)).cuda()
    h, yp, stats = L.expert_ffn(xp, off)
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] == 0
    h_ref, yp_ref = om.expert_segments(x[d.src_tok], d.offsets, w1, w2, cfg, want_hidden=True)
    # h is rounded once to its storage type: half an ulp is at most 2^-8 (bf16)
    # or 2^-11 (fp16) of the value; fp32 accumulation adds far less
    hd = to_np64(h[:n])
    rel = {"bf16": 2.0 ** -8, "f16": 2.0 ** -11, "f32": 2.0 ** -20}[L.hidden]
    scale = float(np.sqrt(np.mean(h_ref ** 2))) if h_ref.size else 1.0
    assert np.all(np.abs(hd - h_ref) <= rel * np.abs(h_ref) + 1e-4 * scale)
    check_out(to_np64(yp[:n]), yp_ref, L.w.dtype)


def test_combine(layer):
    L = layer
    x, wg, b, w1, w2 = oracle_inputs(L)
    cfg = lcfg_of(L.w, L.T)
    r = om.route(x, wg, b, cfg)
    d = om.dispatch(r.idx, cfg, r.prob_mean)
    n = int(d.offsets[-1])
    A = max(L.T * L.w.k, 1)
    g = torch.Generator().manual_seed(5)
    yp = torch.randn((A, L.w.d), generator=g).cuda()
    row_of = torch.from_numpy(d.row_of.astype(np.int32)).cuda()
    tw = torch.from_numpy(r.w.astype(np.float32)).cuda()
    out = L.combine(yp, row_of, tw)
    torch.cuda.synchronize()
    ref = om.combine(to_np64(yp[:max(n, 1)]), d.row_of, r.w.astype(np.float32).astype(np.float64), L.T, L.w.d)
    o = to_np64(out)
    # fp32 fused multiply-adds over at most k slots, fp32 output
    bound = np.zeros_like(ref)
    for j in range(L.w.k):
        keep = d.row_of[:, j] >= 0
        bound[keep] += np.abs(r.w[keep, j, None]) * np.abs(to_np64(yp)[d.row_of[keep, j]])
    assert np.all(np.abs(o - ref) <= 4 * L.w.k * 2.0 ** -24 * bound + 1e-30)


# ------------------------------------------------------ adversarial permutes
def _small(T, E, k, cf, dtype=mw.BF16, d=32):
    return DeviceLayer(W("adv", T=T, d=d, E=E, F=32, k=k, act=mw.RELU, dtype=dtype, capacity_factor=cf, seed=3))


def _run_permute(L, idx_np, cf_cfg):
    idx = torch.from_numpy(idx_np.astype(np.int32)).cuda()
    res = L.permute(idx)
    torch.cuda.synchronize()
    return {k: (v.cpu().numpy() if k != "stats" else moe.read_stats(v)) for k, v in res.items() if k != "xp"}


@pytest.mark.parametrize("T,E,k,cf", [(300, 4, 2, 0.5), (129, 8, 1, 0.1), (1000, 16, 8, 1.0), (64, 3, 3, 0.0),
                                       (333, 20, 10, 0.7)])
def test_permute_all_to_few_experts(T, E, k, cf):
    """Every token picks experts 0..k-1 (maximal imbalance, heavy dropping)."""
    L = _small(T, E, k, cf)
    idx = np.tile(np.arange(k), (T, 1))
    idx[1::2] = idx[1::2, ::-1]    # vary slot order
    got = _run_permute(L, idx, cf)
    cfg = lcfg_of(L.w, T)
    d = om.dispatch(idx, cfg, None)
    assert np.array_equal(got["counts"], d.counts) and np.array_equal(got["kept"], d.kept)
    assert np.array_equal(got["offsets"], d.offsets) and np.array_equal(got["row_of"], d.row_of)
    assert np.array_equal(got["src_tok"][:int(d.offsets[-1])], d.src_tok)
    assert got["stats"]["drop_count"] == d.drop_count


def test_permute_random_indices_exact():
    """Uniformly random (distinct per token) selections over many chunks."""
    rng = np.random.default_rng(9)
    T, E, k = 4097, 37, 5
    L = _small(T, E, k, 1.3)
    idx = np.stack([rng.choice(E, size=k, replace=False) for _ in range(T)])
    got = _run_permute(L, idx, 1.3)
    d = om.dispatch(idx, lcfg_of(L.w, T), None)
    assert np.array_equal(got["row_of"], d.row_of) and np.array_equal(got["offsets"], d.offsets)
    assert np.array_equal(got["src_tok"][:int(d.offsets[-1])], d.src_tok)


def test_permute_repeated_expert_in_token():
    """A caller-made selection naming one expert twice is ordered by slot."""
    T, E, k = 70, 4, 2
    L = _small(T, E, k, 0.0)
    idx = np.array([[t % E, t % E] if t % 3 == 0 else [t % E, (t + 1) % E] for t in range(T)])
    got = _run_permute(L, idx, 0.0)
    d = om.dispatch(idx, lcfg_of(L.w, T), None)
    assert np.array_equal(got["row_of"], d.row_of)
    assert np.array_equal(got["src_tok"][:int(d.offsets[-1])], d.src_tok)


def test_permute_out_of_range_index_flags_and_drops():
    T, E, k = 40, 4, 2
    L = _small(T, E, k, 0.0)
    idx = np.array([[t % E, (t + 1) % E] for t in range(T)])
    idx[5, 1] = 9
    idx[17, 0] = -1
    got = _run_permute(L, idx, 0.0)
    assert got["stats"]["status"] & moe.MOE_DEV_BOUNDS
    assert got["row_of"][5, 1] == -1 and got["row_of"][17, 0] == -1
    # the valid slots are grouped exactly as if the bad slots did not exist
    valid = (idx >= 0) & (idx < E)
    assert int(got["offsets"][-1]) == int(valid.sum())
    for e in range(E):
        toks = np.nonzero((idx == e).any(axis=1))[0]
        seg = got["src_tok"][got["offsets"][e]:got["offsets"][e + 1]]
        assert np.array_equal(seg, toks)


def test_bad_arguments_rejected_on_gpu():
    L = _small(64, 4, 2, 0.0)
    idx, wt, gap, pm = L.route()
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_route(L.cfg, L.x, L.wg, None, idx, wt, gap, pm, torch.empty(16, dtype=torch.uint8, device="cuda"))
    assert ei.value.code == 3
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_combine(L.cfg, None, idx, wt, torch.empty_like(L.x))
    assert ei.value.code == 1


# ------------------------------------------------------- weight preparation
def test_convert_bf16_to_f16_matches_numpy():
    rng = np.random.default_rng(4)
    n = 100003                                     # not a multiple of the 8-wide vectors
    bits = rng.integers(0, 1 << 16, size=n, dtype=np.uint16)
    f = mw.bf16_bits_to_f32(bits)
    bits[~np.isfinite(f)] = 0                      # finite values only
    f = mw.bf16_bits_to_f32(bits)
    ref = np.clip(f, -65504, 65504).astype(np.float16)   # round to nearest even, saturated
    src = mw.to_device(bits)
    dst = torch.empty(n, dtype=torch.float16, device="cuda")
    moe.moe_convert_bf16_to_f16(src, dst)
    torch.cuda.synchronize()
    got = dst.cpu().numpy()
    assert np.array_equal(got.view(np.uint16), ref.view(np.uint16))
    # every value in [2^-17, 65504] survives exactly
    exact = (np.abs(f) >= 2.0 ** -17) & (np.abs(f) <= 65504)
    assert np.array_equal(got[exact].astype(np.float32), f[exact])


@pytest.mark.parametrize("dtype", [mw.BF16, mw.F32])
@pytest.mark.parametrize("case", ["negative", "decreasing", "past_buffer"])
def test_expert_ffn_rejects_corrupt_offsets(dtype, case):
    """offsets[] that are not a non-decreasing sequence inside [0, T*k] make the
    grouped GEMMs schedule no tile: nothing is written and MOE_DEV_BOUNDS is set."""
    w = W("corrupt", T=200, d=64, E=4, F=64, k=2, act=mw.SWIGLU, dtype=dtype, seed=5)
    L = DeviceLayer(w)
    A = L.T * w.k
    off = {"negative": [-256, 0, 100, 200, 400], "decreasing": [0, 150, 90, 300, 400],
           "past_buffer": [0, 100, 200, 300, A + 128]}[case]
    xp = torch.zeros((A, w.d), dtype=L.tdt, device="cuda")
    h0 = torch.full((A, w.F), 7.0, dtype=L.hdt, device="cuda")
    yp0 = torch.full((A, w.d), 7.0, dtype=torch.float32, device="cuda")
    h, yp = h0.clone(), yp0.clone()
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    moe.moe_expert_ffn(L.cfg, xp, torch.tensor(off, dtype=torch.int32, device="cuda"), L.w1, L.w2, h, yp, stats,
                       L.scratch())
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] & moe.MOE_DEV_BOUNDS
    assert torch.equal(h, h0) and torch.equal(yp, yp0)


def test_fp16_hidden_saturates_and_flags():
    """fp16 hidden activations beyond +-65504 saturate and set MOE_DEV_RANGE;
    rows that are computed but not stored never raise it (the rows past the
    kept ones hold NaN here)."""
    w = W("sat", T=256, d=64, E=4, F=64, k=2, act=mw.RELU, dtype=mw.BF16, seed=31)
    L = DeviceLayer(w)
    assert L.hidden == "f16"
    idx, _, gap, pm = L.route()
    perm = L.permute(idx, gap, pm)
    torch.cuda.synchronize()
    n = int(perm["offsets"][w.E].item())
    xp = perm["xp"].clone()
    xp[n:] = float("nan")
    _, _, st0 = L.expert_ffn(xp, perm["offsets"])
    torch.cuda.synchronize()
    assert moe.read_stats(st0)["status"] == 0
    L.w1.mul_(2.0 ** 17)                 # exact in bf16: pre-activations of ~1e5
    h, yp, st = L.expert_ffn(xp, perm["offsets"])
    torch.cuda.synchronize()
    assert moe.read_stats(st)["status"] & moe.MOE_DEV_RANGE
    hk = h[:n].float()
    assert torch.isfinite(hk).all()
    assert float(hk.abs().max()) == 65504.0
    assert bool((hk >= 0).all())         # ReLU, saturated to +65504, never wrapped


@pytest.mark.parametrize("offsets", [[0, 100, 130, 150, 160], [0, 0, 64, 65, 65], [0, 63, 64, 128, 160]])
def test_expert_ffn_short_layer_any_segment(offsets):
    """Caller-made expert segments on a small layer: longer than the layer's
    token count (an expert repeated inside a token), empty, or ending on and
    just past tile edges; every row must match the oracle's experts."""
    w = W("short", T=40, d=64, E=4, F=64, k=4, act=mw.SWIGLU, dtype=mw.BF16, seed=33)
    L = DeviceLayer(w)
    _, _, _, w1, w2 = oracle_inputs(L)
    cfg = lcfg_of(w, L.T)
    A = L.T * w.k
    g = torch.Generator().manual_seed(7)
    xp = torch.randn((A, w.d), generator=g).to(torch.bfloat16).cuda()
    off = torch.tensor(offsets, dtype=torch.int32).cuda()
    h, yp, stats = L.expert_ffn(xp, off)
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] == 0
    n = offsets[-1]
    xp64 = xp.float().cpu().numpy().astype(np.float64)
    _, yp_ref = om.expert_segments(xp64[:n], np.array(offsets), w1, w2, cfg)
    check_out(to_np64(yp[:n]), yp_ref, w.dtype)


def test_expert_ffn_small_batch_long_segment():
    """A batch of at most 64 tokens takes 64-row m-tiles (the narrow stage
    layout); a caller-made segment of 700 rows then spans 11 of them, more
    than one group of the second layer's tile order, next to a ragged short
    segment and empty ones."""
    w = W("narrow_long", T=64, d=64, E=16, F=96, k=12, act=mw.SWIGLU, dtype=mw.BF16, seed=36)
    L = DeviceLayer(w)
    _, _, _, w1, w2 = oracle_inputs(L)
    cfg = lcfg_of(w, L.T)
    A = L.T * w.k
    offsets = [0, 0, 700, 700, 733] + [733] * 11 + [768]
    assert len(offsets) == w.E + 1 and offsets[-1] == A
    g = torch.Generator().manual_seed(9)
    xp = torch.randn((A, w.d), generator=g).to(torch.bfloat16).cuda()
    h, yp, stats = L.expert_ffn(xp, torch.tensor(offsets, dtype=torch.int32).cuda())
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] == 0
    xp64 = xp.float().cpu().numpy().astype(np.float64)
    _, yp_ref = om.expert_segments(xp64, np.array(offsets), w1, w2, cfg)
    check_out(to_np64(yp), yp_ref, w.dtype)


def test_adaptive_aux_coef_on_the_device_follows_the_oracle():
    """moe_aux_coef_update, chained on the stream over scripted drop rates
    written into a device moe_stats, against the oracle's coefficient step."""
    import ctypes
    from oracle import moe_oracle as om
    beta, xi = 0.8, 0.25
    rates = [0.4, 0.4, 0.3, 0.1, 0.0, 0.0, 0.05, 0.5]
    coef = torch.full((1,), 0.02, dtype=torch.float32, device="cuda")
    ref = 0.02
    got = []
    for d in rates:
        st = moe.moe_stats()
        st.drop_rate = d
        stats = torch.frombuffer(bytearray(bytes(st)), dtype=torch.uint8).cuda()
        moe.moe_aux_coef_update(stats, coef, beta, xi)
        ref = om.adaptive_aux_coef(ref, d, beta, xi)
        got.append((float(coef.item()), ref))
    for g, r in got:
        assert abs(g - r) <= 1e-6 * max(1.0, abs(r)), got
    assert ctypes.sizeof(moe.moe_stats) == moe.STATS_BYTES
