"""The data-parallel (replica) path across ranks, on CPU with gloo, world size 2.

The layer shards over tokens: every rank holds the same weights and routes
its own tokens; no collective is on the data path.  The only collective of
`bench.py --gpus N` is the max over ranks of the step time.  These tests run
two gloo ranks that build their replica inputs and evaluate the layer with the
float64 oracle (standing in for the device step), and check that the shards
differ while the weights agree, that each rank's result equals a single-process
evaluation of its shard, and that the reported time is the slowest rank's."""
import datetime
import hashlib
import os
import socket

import numpy as np
import torch.multiprocessing as mp

import bench
import moe_workloads as mw

W = mw.Workload("dp_tiny", T=96, d=32, E=6, F=48, k=2, act=mw.SWIGLU, dtype=mw.BF16, capacity_factor=1.0, seed=3)


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    p = s.getsockname()[1]
    s.close()
    return p


def _digest(a):
    return hashlib.sha256(np.ascontiguousarray(a).tobytes()).hexdigest()


def _forward(inp):
    import oracle
    from oracle import moe_oracle as om
    cfg = oracle.LayerConfig.from_workload(W)
    return om.forward(mw.to_f64(inp.x), mw.to_f64(inp.wg), inp.bias, mw.F64Experts(inp.w1),
                      mw.F64Experts(inp.w2), cfg).out


def _worker(rank, world, port, q):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    try:
        inp = bench.replica_inputs(W, rank)
        out = _forward(inp)
        step_ms = 1.0 + rank            # the ranks' own step times
        slowest = bench.reduce_max_over_ranks(step_ms, world, "cpu")
        info = [None] * world
        dist.all_gather_object(info, (_digest(inp.w1), _digest(inp.w2), _digest(inp.wg), _digest(inp.x)))
        q.put((rank, slowest, info, out))
    finally:
        dist.destroy_process_group()


def test_two_replicas_with_gloo():
    world = 2
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, world, port, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = {}
    for _ in range(world):
        r, slowest, info, out = q.get(timeout=120)
        res[r] = (slowest, info, out)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for r in range(world):
        slowest, info, out = res[r]
        assert slowest == float(world)                 # max over ranks of 1.0, 2.0
        assert len({i[0] for i in info}) == 1 and len({i[1] for i in info}) == 1 and len({i[2] for i in info}) == 1
        assert len({i[3] for i in info}) == world       # every rank routes its own tokens
        ref = _forward(bench.replica_inputs(W, r))      # a single process on the same shard
        assert np.array_equal(out, ref)
    assert not np.array_equal(res[0][2], res[1][2])
    # whole-job throughput: all ranks' tokens over the slowest rank's time
    assert bench.job_tokens_per_second(world, W.T, 2.0) == world * W.T / 2e-3


def test_single_rank_reduction_is_identity():
    assert bench.reduce_max_over_ranks(3.5, 1, "cpu") == 3.5
    assert bench.job_tokens_per_second(1, 8192, 0.1) == 8192 / 1e-4
