"""Expert parallelism on one GPU through the C ABI.

* moe_expert_ffn_segments against the float64 oracle: the rows of G source
  ranks arrive as G blocks of E_local expert segments, segment i running
  through local expert i mod E_local (1-SM one-launch tiles, 2-SM pair tiles
  and the fp32 path, with empty and ragged segments);
* the expert-parallel forward with world size 1 (the exchanges are copies)
  through ``ExpertParallelLayer`` and ``LibmoeBackend``;
* G = 2 and 4 ranks emulated on the one GPU: every rank's steps 1-3, the
  row exchange done by hand in rank order, step 4 on each rank's received
  segments, the rows sent back, and the combine; each rank's output matches
  the oracle forward of its token shard with all E experts."""
import numpy as np
import pytest
import torch

import moe_workloads as mw
import mixture_experts_layer_logit_b200 as moe
from mixture_experts_layer_logit_b200 import expert_parallel as ep
import oracle
from oracle import moe_oracle as om
from tests.gpu_harness import check_out, to_np64

pytestmark = pytest.mark.gpu

W = mw.Workload


def _segments_case(w, G, seed):
    """Rows of G sources for E_local experts, source-major; random segment
    lengths (some empty)."""
    rng = np.random.default_rng(seed)
    n = w.E
    lens = rng.integers(0, 2 * max(1, w.T * w.k // (G * n)) + 1, size=G * n)
    lens[rng.integers(0, G * n)] = 0
    offs = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    return offs


@pytest.mark.parametrize("w,G", [
    (W("seg_relu", T=600, d=128, E=4, F=192, k=2, act=mw.RELU, dtype=mw.BF16, seed=51), 2),
    (W("seg_swiglu", T=500, d=192, E=3, F=208, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=52), 4),
    (W("seg_pair", T=4096, d=256, E=2, F=320, k=2, act=mw.SWIGLU, dtype=mw.BF16, seed=53), 2),
    (W("seg_fp32", T=300, d=64, E=3, F=96, k=2, act=mw.SWIGLU, dtype=mw.F32, seed=54), 2),
], ids=["relu_G2", "swiglu_G4", "pair_G2", "fp32_G2"])
def test_expert_ffn_segments(w, G):
    offs = _segments_case(w, G, w.seed)
    rows = int(offs[-1])
    nseg = G * w.E
    cfg = moe.make_config(w.T, w.d, w.E, w.F, w.k, w.act, w.dtype)
    if w.name == "seg_pair":
        assert rows >= 512 * nseg, "the pair-tile path needs long segments"
    rng = np.random.default_rng(w.seed + 100)
    xs = rng.standard_normal((rows + 7, w.d)).astype(np.float32)   # 7 spare rows past the segments
    xst = mw.round_to_bf16_bits(xs) if w.dtype == mw.BF16 else xs
    inp = mw.generate(w.replace(T=1))
    tdt = torch.bfloat16 if w.dtype == mw.BF16 else torch.float32
    xp = mw.to_device(xst)
    w1 = mw.to_device(inp.w1)
    w2 = moe.prepare_w2(cfg, mw.to_device(inp.w2))
    hdt = torch.float16 if w.dtype == mw.BF16 else torch.float32
    R = rows + 7
    h = torch.empty((R, w.F), dtype=hdt, device="cuda")
    yp = torch.full((R, w.d), 7.0, dtype=torch.float32, device="cuda")
    stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device="cuda")
    ws = torch.empty(moe.moe_segments_scratch_size(cfg, nseg, R), dtype=torch.uint8, device="cuda")
    moe.moe_expert_ffn_segments(cfg, nseg, R, torch.from_numpy(offs).cuda(), xp, w1, w2, h, yp, stats, ws)
    torch.cuda.synchronize()
    assert moe.read_stats(stats)["status"] == 0
    x64 = mw.to_f64(xst)
    ref = np.zeros((rows, w.d))
    for i in range(nseg):
        a, b = int(offs[i]), int(offs[i + 1])
        if b > a:
            e = i % w.E
            ref[a:b] = om.expert_ffn(x64[a:b], mw.to_f64(inp.w1[e]), mw.to_f64(inp.w2[e]), w.act, w.F)
    got = to_np64(yp[:rows])
    check_out(got, ref, w.dtype)
    assert torch.all(yp[rows:] == 7.0), "rows past the last segment are not written"


def _oracle_shard(w, inp, dev_idx):
    """The oracle forward of one shard; tokens whose k-th/(k+1)-th score gap
    is below 1e-4 take the device's selection (both are correct there)."""
    cfg = oracle.LayerConfig.from_workload(w)
    x, wg = mw.to_f64(inp.x), mw.to_f64(inp.wg)
    r0 = om.route(x, wg, inp.bias, cfg)
    forced = r0.gap < 1e-4
    return om.forward(x, wg, inp.bias, mw.F64Experts(inp.w1), mw.F64Experts(inp.w2), cfg,
                      forced if forced.any() else None, dev_idx if forced.any() else None)


def _backend(w, inp, G, rank):
    cfg = moe.make_config(w.T, w.d, w.E, w.F, w.k, w.act, w.dtype, w.capacity_factor, w.lam)
    local = ep.experts_of_rank(w.E, G, rank)
    w1 = mw.to_device(np.ascontiguousarray(inp.w1[local.start:local.stop]))
    w2 = moe.prepare_w2(cfg, mw.to_device(np.ascontiguousarray(inp.w2[local.start:local.stop])))
    return ep.LibmoeBackend(cfg, mw.to_device(inp.wg), mw.to_device(inp.bias), w1, w2, len(local))


EPW = W("ep_gpu", T=700, d=128, E=8, F=176, k=2, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=1.0, lam=1.0,
        zipf_bias=True, seed=61)


def test_expert_parallel_layer_world_one():
    inp = mw.generate(EPW)
    layer = ep.ExpertParallelLayer(_backend(EPW, inp, 1, 0), EPW.E, 0, 1)
    out, r = layer.forward(mw.to_device(inp.x))
    torch.cuda.synchronize()
    ref = _oracle_shard(EPW, inp, r["topk_idx"].cpu().numpy())
    check_out(to_np64(out), ref.out, EPW.dtype)


@pytest.mark.parametrize("G,w", [(2, EPW), (4, EPW), (2, EPW.replace(name="ep_gpu_k6", k=6, E=8, capacity_factor=0.0,
                                                                        act=mw.RELU))],
                         ids=["G2", "G4", "G2_top6_dropless"])
def test_expert_parallel_emulated_ranks(G, w):
    inps = [mw.generate(w, shard=r) for r in range(G)]
    # every rank's weights are the same draw (the generator is seeded per tensor, not per shard)
    bks = [_backend(w, inps[r], G, r) for r in range(G)]
    rs = [bks[r].route_permute(mw.to_device(inps[r].x)) for r in range(G)]
    n = w.E // G
    send = [ep.send_rows_per_rank(r["offsets"], w.E, G) for r in rs]
    kept = [[r["offsets"][e + 1] - r["offsets"][e] for e in range(w.E)] for r in rs]
    # the row all-to-all by hand: rank g receives, in source order, each source's block for g's experts
    outs_back = [[None] * G for _ in range(G)]   # [source][dest]: rows dest returns to source
    for g in range(G):
        blocks = [rs[s]["xp"][rs[s]["offsets"][g * n]:rs[s]["offsets"][(g + 1) * n]] for s in range(G)]
        xr = torch.cat(blocks, 0)
        recv_kept = [kept[s][g * n:(g + 1) * n] for s in range(G)]
        yr = bks[g].experts(xr, ep.segment_offsets(recv_kept), G * n)
        pos = 0
        for s in range(G):
            outs_back[s][g] = yr[pos:pos + send[s][g]]
            pos += send[s][g]
    for s in range(G):
        yp = torch.cat(outs_back[s], 0)
        out = bks[s].combine(yp, rs[s])
        torch.cuda.synchronize()
        ref = _oracle_shard(w, inps[s], rs[s]["topk_idx"].cpu().numpy())
        check_out(to_np64(out), ref.out, w.dtype)
    assert len({tuple(x) for x in send}) > 1 or G == 1
