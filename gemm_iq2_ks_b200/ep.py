"""Expert parallelism for the routed-expert block (decode and prefill).

The routed block's experts are partitioned into contiguous ranges, one per
rank (one process per GPU). Each rank keeps only its range's streams and runs
``iqk_moe_decode_shard`` over the call's global routing: the slots routed to
its experts give a float32 partial of y. One all-reduce (sum) over the
process group joins the partials, and ``iqk_f32_to_bf16`` rounds the sum:
y = bf16_rn(sum over ranks of partial_r), the same block as
``iqk_moe_decode`` on one GPU, up to float32 summation order. The exchange is
[T, hidden] float32 per call (16 KB for one token at hidden 4096), latency-
bound on NVLink; NCCL carries it (gloo on CPU for the host-side tests).

Prefill (``ExpertParallelPrefill``) splits the tokens as well: each rank
holds its own tokens, and every (token, slot) pair travels to the rank that
owns its expert (all-to-all dispatch of the token rows), is computed there as
one float32 row (``iqk_moe_prefill_shard`` with one slot of weight 1), and
travels back (all-to-all combine), where ``iqk_moe_combine`` forms
y = bf16_rn(sum over slots in order of p * row): the same arithmetic as the
single-GPU prefill's combine.
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


class ExpertParallelPrefill:
    """The routed block's prefill with experts and tokens spread over a
    process group: all-to-all dispatch of each (token, slot) pair's row to
    the rank that owns its expert, the expert's block there, all-to-all
    combine back to the token's rank.

    gate, up, down: host streams of ALL experts (each rank uploads only its
    range); values: the 8-entry table. A call takes this rank's own tokens:
    x [T, hidden] (bf16), ids [T, topk] (int32, global expert ids in
    [0, experts)), p [T, topk] (float32); T may differ between ranks. It
    returns this rank's y [T, hidden] (bf16). Every rank must call it, in the
    same order. ``compute`` and ``combine`` replace the two device steps
    (for host-side tests): compute(rows bf16 [m, hidden], ids int32 [m]) ->
    float32 [m, hidden], one pair per row; combine(rows float32 [T*topk,
    hidden] in pair order, p) -> y.
    """

    def __init__(self, gate, up, down, values, group=None, device="cuda", compute=None, combine=None):
        import torch
        import torch.distributed as dist
        self.torch, self.dist, self.group = torch, dist, group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.rank = dist.get_rank(group) if dist.is_initialized() else 0
        self.experts = gate.experts
        self.bounds = [shard_range(gate.experts, self.world, r) for r in range(self.world)]
        self.lo, self.hi = self.bounds[self.rank]
        self.values = values
        self.device = device
        self.compute = compute
        self.combine = combine
        if compute is None:
            self.weights = [B.Weights.from_host(shard_streams(w, self.lo, self.hi), device) for w in (gate, up, down)]
            self.compute = self._compute_device
        if combine is None:
            self.combine = lambda rows, p: B.iqk_moe_combine(rows, p)
        self._starts = torch.tensor([lo for lo, _ in self.bounds], dtype=torch.int64)

    def _compute_device(self, rows, ids):
        torch = self.torch
        m = rows.shape[0]
        if m == 0:
            return torch.empty((0, rows.shape[1]), dtype=torch.float32, device=rows.device)
        g, u, d = self.weights
        one = torch.ones((m, 1), dtype=torch.float32, device=rows.device)
        return B.iqk_moe_prefill_shard(g, u, d, self.values, rows, ids.reshape(m, 1).contiguous(), one, self.lo)

    def plan(self, ids):
        """Pairs in dispatch order (grouped by owner rank, pair order within)
        and the number going to each rank."""
        torch = self.torch
        flat = ids.reshape(-1).to(torch.int64).cpu()
        if flat.numel() and (int(flat.min()) < 0 or int(flat.max()) >= self.experts):
            raise ValueError("expert id out of range")
        owner = torch.searchsorted(self._starts, flat, right=True) - 1
        order = torch.argsort(owner, stable=True)
        counts = torch.bincount(owner, minlength=self.world)
        return order, counts

    def _a2a(self, out, inp, out_splits, in_splits):
        if self.world == 1 and not self.dist.is_initialized():
            out.copy_(inp)
        else:
            self.dist.all_to_all_single(out, inp, out_splits, in_splits, group=self.group)

    def __call__(self, x, ids, p):
        torch = self.torch
        T, topk = ids.shape
        H = x.shape[1]
        dev = x.device
        order, send = self.plan(ids)
        send = send.to(dev)
        recv = torch.empty_like(send)
        self._a2a(recv, send, [1] * self.world, [1] * self.world)
        send_l, recv_l = send.tolist(), recv.tolist()
        order_d = order.to(dev)
        # dispatch: each pair's token row (bf16, moved as 32-bit words) and its expert id
        rows_out = x.contiguous().view(torch.int16).view(torch.int32)[order_d // topk]
        rows_in = torch.empty((sum(recv_l), H // 2), dtype=torch.int32, device=dev)
        self._a2a(rows_in, rows_out.contiguous(), recv_l, send_l)
        ids_out = ids.reshape(-1).to(torch.int32)[order_d].contiguous()
        ids_in = torch.empty((sum(recv_l),), dtype=torch.int32, device=dev)
        self._a2a(ids_in, ids_out, recv_l, send_l)
        # the owned experts' rows, one pair each, in float32
        res = self.compute(rows_in.view(torch.int16).view(-1, H).view(torch.bfloat16), ids_in)
        # combine: the rows travel back and land in pair order
        back = torch.empty((T * topk, H), dtype=torch.float32, device=dev)
        self._a2a(back, res.contiguous(), send_l, recv_l)
        pair_rows = torch.empty_like(back)
        pair_rows[order_d] = back
        return self.combine(pair_rows, p)
