"""The layer with a shared expert (moe_layer_forward_shared) against the
float64 oracle's forward_with_shared: every token through the shared expert
with weight 1, added to the routed combine.  Layers with the 1-SM and the
2-SM expert kernels, both activations, the fp32 path and the fine-grained
decode layer with a shared expert two fine experts wide (DeepSeekMoE's
layout)."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
import oracle
from oracle import moe_oracle as om
from tests.gpu_harness import check_routing, check_out, to_np64

pytestmark = pytest.mark.gpu

W = mw.Workload
CASES = [
    (W("sh_relu_cap", T=400, d=128, E=8, F=192, k=2, act=mw.RELU, dtype=mw.BF16, capacity_factor=1.0, seed=91), 256),
    (W("sh_swiglu_lam", T=700, d=256, E=6, F=128, k=2, act=mw.SWIGLU, dtype=mw.BF16, lam=1.0, seed=92), 384),
    (W("sh_pair", T=1300, d=128, E=2, F=128, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=93), 128),
    (W("sh_fp32", T=200, d=64, E=4, F=64, k=2, act=mw.SWIGLU, dtype=mw.F32, seed=94), 96),
    (mw.WORKLOADS["fine_decode_dropless"], 2 * 1408),
]


def _shared_weights(w, Fs, seed):
    rng = np.random.default_rng([seed, 77])
    F1s = Fs if w.act == mw.RELU else 2 * Fs
    a = (rng.standard_normal((F1s, w.d)) / np.sqrt(w.d)).astype(np.float32)
    b = (rng.standard_normal((w.d, Fs)) / np.sqrt(Fs)).astype(np.float32)
    if w.dtype == mw.BF16:
        return mw.round_to_bf16_bits(a), mw.round_to_bf16_bits(b)
    return a, b


@pytest.mark.parametrize("w,Fs", CASES, ids=[c[0].name for c in CASES])
def test_shared_expert_forward(w, Fs):
    inp = mw.generate(w)
    cfg = moe.make_config(w.T, w.d, w.E, w.F, w.k, w.act, w.dtype, w.capacity_factor, w.lam)
    x, wg, bias = mw.to_device(inp.x), mw.to_device(inp.wg), mw.to_device(inp.bias)
    w1 = mw.to_device(inp.w1)
    w2 = moe.prepare_w2(cfg, mw.to_device(inp.w2))
    a, b = _shared_weights(w, Fs, w.seed)
    w1s = mw.to_device(a)
    w2s = moe.prepare_w2(cfg, mw.to_device(b))
    n = moe.moe_workspace_size_shared(cfg, Fs)
    assert n > 0
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    out = torch.empty((w.T, w.d), dtype=torch.float32, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    moe.moe_layer_forward_shared(cfg, Fs, x, wg, bias, w1, w2, w1s, w2s, out, stats, ws)
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] == 0
    _, lay = moe.moe_workspace_size(cfg)
    idx = ws[lay.topk_idx:lay.topk_idx + 4 * w.T * w.k].view(torch.int32).view(w.T, w.k).cpu().numpy()
    lc = oracle.LayerConfig.from_workload(w)
    xx, wgg = mw.to_f64(inp.x), mw.to_f64(inp.wg)
    r0 = om.route(xx, wgg, inp.bias, lc)
    forced, n_tie = check_routing(idx, r0)
    fw = om.forward_with_shared(xx, wgg, inp.bias, mw.F64Experts(inp.w1), mw.F64Experts(inp.w2), mw.to_f64(a),
                                mw.to_f64(b), Fs, lc, forced if n_tie else None, idx if n_tie else None)
    rel = check_out(to_np64(out), fw.out, w.dtype)
    print(w.name, f"max|err| relative {rel:.2e}")
