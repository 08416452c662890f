"""Expert parallelism for the routed-expert decode.

The routed block's experts are partitioned into contiguous ranges, one per
rank (one process per GPU). Each rank keeps only its range's streams and runs
``iqk_moe_decode_shard`` over the call's global routing: the slots routed to
its experts give a float32 partial of y. One all-reduce (sum) over the
process group joins the partials, and ``iqk_f32_to_bf16`` rounds the sum:
y = bf16_rn(sum over ranks of partial_r), the same block as
``iqk_moe_decode`` on one GPU, up to float32 summation order. The exchange is
[T, hidden] float32 per call (16 KB for one token at hidden 4096), latency-
bound on NVLink; NCCL carries it (gloo on CPU for the host-side tests).
"""
from __future__ import annotations

import contextlib
from typing import Tuple

from . import binding as B


def shard_range(experts: int, world: int, rank: int) -> Tuple[int, int]:
    """Experts [lo, hi) of `rank`: contiguous ranges whose sizes differ by at
    most one, covering 0 .. experts - 1 once."""
    if world < 1 or not 0 <= rank < world or experts < world:
        raise ValueError(f"cannot split {experts} experts over {world} ranks (rank {rank})")
    base, extra = divmod(experts, world)
    lo = rank * base + min(rank, extra)
    return lo, lo + base + (1 if rank < extra else 0)


def shard_streams(streams, lo: int, hi: int):
    """Host streams of experts [lo, hi) (views of the stacked planes; any
    object with fmt, experts, rows, cols and the five planes)."""
    if not 0 <= lo < hi <= streams.experts:
        raise ValueError(f"expert range [{lo}, {hi}) outside 0 .. {streams.experts}")
    cut = (lambda a: None if a is None else a[lo:hi])
    kind = type(streams)
    out = kind.__new__(kind)
    out.__dict__.update(streams.__dict__)
    out.experts = hi - lo
    for name in ("qs", "scl", "sch", "sex", "dv"):
        setattr(out, name, cut(getattr(streams, name)))
    return out


class ExpertParallelDecode:
    """The routed block's decode with its experts spread over a process group.

    gate, up, down: host streams of ALL experts (each rank uploads only its
    range); values: the 8-entry table. A call takes the global x [T, hidden]
    (bf16), ids [T, topk] (int32, global expert ids) and p [T, topk] (float32),
    identical on every rank, and returns y [T, hidden] (bf16) on every rank.
    Every rank must call it with the same shapes, in the same order.
    """

    def __init__(self, gate, up, down, values, group=None, device="cuda"):
        import torch.distributed as dist
        self.dist, self.group = dist, group
        world = dist.get_world_size(group) if dist.is_initialized() else 1
        rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.lo, self.hi = shard_range(gate.experts, world, rank)
        self.weights = [B.Weights.from_host(shard_streams(w, self.lo, self.hi), device) for w in (gate, up, down)]
        self.values = values
        self.world = world
        self.reduce = dist.is_initialized()  # one rank in a group still runs the collective
        self._ws = {}

    def __call__(self, x, ids, p, stream=None):
        """y for one call; the kernels and the all-reduce run on `stream`
        (torch's current stream when None)."""
        import torch
        T, topk = ids.shape
        g, u, d = self.weights
        ws = self._ws.get((T, topk))
        if ws is None:
            ws = self._ws[(T, topk)] = B.workspace(B.iqk_moe_workspace_bytes(0, T, topk, g.experts, g.cols, g.rows),
                                                   x.device)
        ctx = torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext()
        with ctx:
            part = B.iqk_moe_decode_shard(g, u, d, self.values, x, ids, p, self.lo, ws=ws)
            if self.reduce:
                self.dist.all_reduce(part, op=self.dist.ReduceOp.SUM, group=self.group)
            return B.iqk_f32_to_bf16(part)
