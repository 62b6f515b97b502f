"""Expert parallelism for the MoE layer forward: the E experts are split
over G GPUs, E/G each, and tokens travel to the GPU of their expert and back.

FastMoE announcement, "特色四：支持大规模并行训练" and Figure 6 (the
model-parallel mode: every worker holds its own experts, and the inputs of
an expert are sent to its worker and the outputs returned); the all-to-all
of GShard in the same announcement's history of the method.

One forward on rank r (G ranks, rank g owning global experts
[g E/G, (g+1) E/G)):

1. steps 1-3 on the rank's own tokens over all E experts (route, then the
   permutation): the kept rows come out grouped by expert, and since the
   experts are numbered by owner, rank g's rows are one contiguous block;
2. count exchange: each rank sends every other rank the kept-row count of
   each of that rank's experts (an all-to-all of G x E/G integers), so every
   rank knows how many rows it sends and receives;
3. row exchange: an all-to-all of the permuted rows;
4. step 4 on the received rows: they arrive as G source blocks of E/G
   expert segments, run in that order by ``moe_expert_ffn_segments``
   (segment i uses local expert i mod E/G);
5. the expert outputs travel back by the reverse all-to-all and land in the
   rank's own permuted row order;
6. step 5 (combine) on the rank's own tokens.

Capacity is applied per rank to its own tokens, before any exchange: each
rank's batch is one group in the GShard sense, so a rank's output equals the
single-GPU forward of its token shard with all E experts.

The compute steps are a backend's (``LibmoeBackend``: the CUDA kernels of
libmoe through the C ABI); the exchanges use ``torch.distributed`` collectives
(NCCL on GPUs).  This module holds only the bookkeeping between them.
"""
from __future__ import annotations

from typing import List, Sequence

import mixture_experts_layer_logit_b200 as moe


def experts_of_rank(E: int, world: int, rank: int) -> range:
    """Global experts owned by `rank`: a contiguous block of E / world."""
    if E % world != 0:
        raise ValueError(f"E = {E} experts do not split evenly over {world} ranks")
    n = E // world
    return range(rank * n, (rank + 1) * n)


def send_rows_per_rank(offsets: Sequence[int], E: int, world: int) -> List[int]:
    """Rows of the local permuted buffer bound for each rank: the kept rows of
    that rank's experts (offsets[E+1] is the exclusive scan of kept)."""
    n = E // world
    return [int(offsets[(g + 1) * n]) - int(offsets[g * n]) for g in range(world)]


def segment_offsets(recv_kept: Sequence[Sequence[int]]) -> List[int]:
    """Exclusive scan of the received kept counts in arrival order: source
    rank major, local expert minor (recv_kept[s][e])."""
    out = [0]
    for row in recv_kept:
        for c in row:
            out.append(out[-1] + int(c))
    return out


def exchange_counts(kept: Sequence[int], world: int, group=None, device=None) -> List[List[int]]:
    """All-to-all of the per-expert kept counts: rank r sends to rank g the
    counts of g's experts and receives, from every source rank s, the counts
    of its own experts.  Returns recv_kept[s][e_local]."""
    import torch
    import torch.distributed as dist
    E = len(kept)
    n = E // world
    send = torch.tensor([int(c) for c in kept], dtype=torch.int64, device=device)
    if world == 1:
        return [send.tolist()]
    recv = torch.empty_like(send)
    dist.all_to_all_single(recv, send, group=group)
    return recv.view(world, n).tolist()


def exchange_rows(send, send_rows: Sequence[int], recv_rows: Sequence[int], group=None):
    """All-to-all of row blocks: send[sum(send_rows), ...] is split by
    destination rank, the result holds the blocks of every source rank in
    rank order."""
    import torch
    import torch.distributed as dist
    n_recv = int(sum(recv_rows))
    recv = torch.empty((n_recv,) + tuple(send.shape[1:]), dtype=send.dtype, device=send.device)
    if len(send_rows) == 1:
        recv.copy_(send[:n_recv])
        return recv
    dist.all_to_all_single(recv, send[:int(sum(send_rows))].contiguous(), [int(r) for r in recv_rows],
                           [int(r) for r in send_rows], group=group)
    return recv


class ExpertParallelLayer:
    """The forward of one MoE layer with its experts split over the ranks of
    `group` (world ranks).  `backend` runs the compute steps."""

    def __init__(self, backend, E: int, rank: int, world: int, group=None, device=None):
        self.backend = backend
        self.E = E
        self.rank = rank
        self.world = world
        self.group = group
        self.device = device
        self.local = experts_of_rank(E, world, rank)

    def forward(self, x):
        b = self.backend
        # 1. steps 1-3 on this rank's tokens, over all E experts
        r = b.route_permute(x)
        offsets = [int(v) for v in r["offsets"]]
        kept = [offsets[e + 1] - offsets[e] for e in range(self.E)]
        # 2. counts: what this rank sends to and receives from every rank
        send_rows = send_rows_per_rank(offsets, self.E, self.world)
        recv_kept = exchange_counts(kept, self.world, self.group, self.device)
        recv_rows = [sum(row) for row in recv_kept]
        # 3. rows out
        xr = exchange_rows(r["xp"], send_rows, recv_rows, self.group)
        # 4. the local experts over the received segments
        yr = b.experts(xr, segment_offsets(recv_kept), self.world * len(self.local))
        # 5. outputs back, into this rank's permuted row order
        yp = exchange_rows(yr, recv_rows, send_rows, self.group)
        # 6. combine on this rank's tokens
        return b.combine(yp, r), r


class LibmoeBackend:
    """Compute steps of the expert-parallel forward on the GPU, through the
    C ABI of libmoe: moe_route and moe_permute on the local tokens (all E
    experts), moe_expert_ffn_segments with the local experts' weights, and
    moe_combine."""

    def __init__(self, cfg, Wg, bg, W1_local, W2_local, E_local: int):
        import ctypes
        import torch
        self.cfg = cfg                                   # the layer: T = local tokens, all E experts
        self.cfg_local = moe.moe_config.from_buffer_copy(bytes(cfg))
        self.cfg_local.E = E_local
        self.cfg_local.k = min(self.cfg_local.k, E_local)
        self.Wg, self.bg, self.W1, self.W2 = Wg, bg, W1_local, W2_local
        self.device = Wg.device
        self.torch = torch
        self.ctypes = ctypes

    def route_permute(self, x):
        torch = self.torch
        c = self.cfg
        T, k, E, d = x.shape[0], c.k, c.E, c.d
        A = max(T * k, 1)
        dev = self.device
        cfg = moe.moe_config.from_buffer_copy(bytes(c))
        cfg.T = T
        ws = torch.empty(max(moe.moe_scratch_size(cfg), 256), dtype=torch.uint8, device=dev)
        r = {"T": T, "cfg": cfg}
        r["topk_idx"] = torch.empty((T, k), dtype=torch.int32, device=dev)
        r["topk_w"] = torch.empty((T, k), dtype=torch.float32, device=dev)
        gap = torch.empty((max(T, 1),), dtype=torch.float32, device=dev)
        pm = torch.empty((E,), dtype=torch.float32, device=dev)
        moe.moe_route(cfg, x, self.Wg, self.bg, r["topk_idx"], r["topk_w"], gap, pm, ws)
        counts = torch.empty(E, dtype=torch.int32, device=dev)
        keptd = torch.empty(E, dtype=torch.int32, device=dev)
        offs = torch.empty(E + 1, dtype=torch.int32, device=dev)
        r["row_of"] = torch.empty((T, k), dtype=torch.int32, device=dev)
        src_tok = torch.empty((A,), dtype=torch.int32, device=dev)
        r["xp"] = torch.empty((A, d), dtype=x.dtype, device=dev)
        r["stats"] = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device=dev)
        moe.moe_permute(cfg, x, r["topk_idx"], gap, pm, counts, keptd, offs, r["row_of"], src_tok, r["xp"],
                        r["stats"], ws)
        r["offsets"] = offs.cpu().tolist()        # the exchange needs the counts on the host
        return r

    def experts(self, xr, seg_offsets, nseg):
        torch = self.torch
        c = self.cfg_local
        rows = xr.shape[0]
        dev = self.device
        hdt = {moe.MOE_DTYPE_F16: torch.float16, moe.MOE_DTYPE_BF16: torch.bfloat16}.get(c.hidden_dtype,
                                                                                          torch.float32)
        h = torch.empty((max(rows, 1), c.F), dtype=hdt, device=dev)
        yp = torch.empty((max(rows, 1), c.d), dtype=torch.float32, device=dev)
        offs = torch.tensor(seg_offsets, dtype=torch.int32, device=dev)
        stats = torch.zeros(moe.STATS_BYTES, dtype=torch.uint8, device=dev)
        ws = torch.empty(max(moe.moe_segments_scratch_size(c, nseg, rows), 256), dtype=torch.uint8, device=dev)
        xin = xr if rows > 0 else torch.empty((1, c.d), dtype=xr.dtype, device=dev)
        moe.moe_expert_ffn_segments(c, nseg, rows, offs, xin, self.W1, self.W2, h, yp, stats, ws)
        st = moe.read_stats(stats)
        if st["status"] != 0:
            raise RuntimeError(f"expert step reported device status {st['status']}")
        return yp[:rows]

    def combine(self, yp, r):
        torch = self.torch
        cfg = r["cfg"]
        out = torch.empty((r["T"], cfg.d), dtype=torch.float32, device=self.device)
        ypin = yp if yp.shape[0] > 0 else torch.zeros((1, cfg.d), dtype=torch.float32, device=self.device)
        moe.moe_combine(cfg, ypin.contiguous(), r["row_of"], r["topk_w"], out)
        return out
