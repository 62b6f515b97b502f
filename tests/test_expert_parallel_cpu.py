"""Expert parallelism across ranks, on CPU with gloo (world sizes 2 and 4).

Each rank holds E/G experts and its own token shard.  The exchange logic of
``mixture_experts_layer_logit_b200.expert_parallel`` (count all-to-all, row
all-to-all out and back, source-major segments on the receiving rank) runs
with gloo collectives; the compute steps are stood in for by the float64
oracle (route, dispatch, one expert MLP per received segment, combine).  Each
rank's output must equal the single-process oracle forward of its shard with
all E experts: capacity is applied per rank, to the rank's own tokens."""
import datetime
import os
import socket

import numpy as np
import pytest
import torch
import torch.multiprocessing as mp

import moe_workloads as mw

W = mw.Workload("ep_tiny", T=80, d=16, E=8, F=24, k=2, act=mw.SWIGLU, dtype=mw.F32, capacity_factor=0.75,
                lam=1.0, zipf_bias=True, seed=5)
W_DROPLESS = W.replace(name="ep_tiny_dropless", capacity_factor=0.0, act=mw.RELU, k=3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


class OracleBackend:
    """The compute steps in float64 (oracle), with the buffer conventions of
    the GPU backend: permuted rows grouped by global expert, the received
    segments run through local expert i % E_local."""

    def __init__(self, w, inp, local):
        import oracle
        from oracle import moe_oracle as om
        self.om = om
        self.w = w
        self.cfg = oracle.LayerConfig.from_workload(w)
        self.wg, self.bias = mw.to_f64(inp.wg), inp.bias
        self.w1 = [mw.to_f64(inp.w1[e]) for e in local]
        self.w2 = [mw.to_f64(inp.w2[e]) for e in local]

    def route_permute(self, x):
        xn = x.numpy()
        r = self.om.route(xn, self.wg, self.bias, self.cfg)
        d = self.om.dispatch(r.idx, self.cfg, r.prob_mean)
        return {"offsets": d.offsets.tolist(), "xp": torch.from_numpy(xn[d.src_tok]), "row_of": d.row_of,
                "w": r.w, "T": xn.shape[0]}

    def experts(self, xr, seg_offsets, nseg):
        xn = xr.numpy()
        y = np.zeros((xn.shape[0], self.w.d))
        for i in range(nseg):
            a, b = seg_offsets[i], seg_offsets[i + 1]
            if b > a:
                e = i % len(self.w1)
                y[a:b] = self.om.expert_ffn(xn[a:b], self.w1[e], self.w2[e], self.w.act, self.w.F)
        return torch.from_numpy(y)

    def combine(self, yp, r):
        return self.om.combine(yp.numpy(), r["row_of"], r["w"], r["T"], self.w.d)


def _worker(rank, world, port, w, q):
    import torch.distributed as dist
    from mixture_experts_layer_logit_b200 import expert_parallel as ep
    import oracle
    from oracle import moe_oracle as om
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = mw.generate(w, shard=rank)
        local = ep.experts_of_rank(w.E, world, rank)
        layer = ep.ExpertParallelLayer(OracleBackend(w, inp, local), w.E, rank, world)
        x = torch.from_numpy(mw.to_f64(inp.x))
        out, r = layer.forward(x)
        ref = om.forward(mw.to_f64(inp.x), mw.to_f64(inp.wg), inp.bias, mw.F64Experts(inp.w1),
                         mw.F64Experts(inp.w2), oracle.LayerConfig.from_workload(w))
        sent = ep.send_rows_per_rank(r["offsets"], w.E, world)
        q.put((rank, float(np.max(np.abs(out - ref.out))), float(np.max(np.abs(ref.out))), sent,
               ref.dispatch.drop_count))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,w", [(2, W), (4, W), (2, W_DROPLESS)], ids=["G2_cap", "G4_cap", "G2_dropless"])
def test_expert_parallel_matches_per_shard_oracle(world, w):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, w, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = [q.get(timeout=240) for _ in range(world)]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, err, scale, sent, drops in res:
        assert err <= 1e-12 * max(scale, 1.0), (rank, err)
        assert sum(sent) > 0
    if w.capacity_factor > 0:
        assert any(d > 0 for *_, d in res), "the capacity case should drop some tokens"
    # the Zipf bias makes the exchange uneven: ranks do not all send alike
    assert len({tuple(s) for _, _, _, s, _ in res}) > 1


def test_bookkeeping():
    from mixture_experts_layer_logit_b200 import expert_parallel as ep
    assert list(ep.experts_of_rank(8, 4, 2)) == [4, 5]
    with pytest.raises(ValueError):
        ep.experts_of_rank(6, 4, 0)
    offs = [0, 3, 3, 7, 10, 10, 12, 15, 15]          # 8 experts, kept 3,0,4,3,0,2,3,0
    assert ep.send_rows_per_rank(offs, 8, 2) == [10, 5]
    assert ep.send_rows_per_rank(offs, 8, 4) == [3, 7, 2, 3]
    assert ep.segment_offsets([[1, 0], [2, 5]]) == [0, 1, 1, 3, 8]
