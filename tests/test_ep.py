"""Expert parallelism, host side (no GPU): the expert partition, the stream
slices each rank keeps, and the decomposition of the routed block into
per-rank parts that an all-reduce joins -- on two gloo ranks."""
import os
import socket
import sys

import numpy as np
import pytest

import iqk_synth as S
from gemm_iq2_ks_b200 import ep
from oracle import oracle as O

torch = pytest.importorskip("torch")
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_shard_ranges_partition_the_experts():
    for E in (1, 2, 7, 8, 256, 257):
        for world in range(1, min(E, 9) + 1):
            ranges = [ep.shard_range(E, world, r) for r in range(world)]
            assert ranges[0][0] == 0 and ranges[-1][1] == E
            assert all(a[1] == b[0] for a, b in zip(ranges, ranges[1:]))
            sizes = [hi - lo for lo, hi in ranges]
            assert max(sizes) - min(sizes) <= 1 and min(sizes) >= 1
    for bad in [(4, 5, 0), (8, 2, 2), (8, 0, 0)]:
        with pytest.raises(ValueError):
            ep.shard_range(*bad)


def test_shard_streams_are_the_global_experts():
    w = S.random_streams(S.rng_for(5), "iq2_k", 6, 32, 512)
    s = ep.shard_streams(w, 2, 5)
    assert (s.fmt, s.experts, s.rows, s.cols) == ("iq2_k", 3, 32, 512)
    vals = S.value_table("int", 1)
    for e in range(3):
        assert np.array_equal(O.dequant_expert(s, e, vals), O.dequant_expert(w, e + 2, vals))
    with pytest.raises(ValueError):
        ep.shard_streams(w, 4, 7)


def _case():
    rng = S.rng_for(61)
    E, H, F, T, k = 10, 256, 256, 3, 4
    gate = S.random_streams(rng, "iq2_ks", E, F, H)
    up = S.random_streams(rng, "iq2_ks", E, F, H)
    down = S.random_streams(rng, "iq2_k", E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, k)
    return gate, up, down, S.value_table("dyadic", 2), x, ids, p


def test_shard_parts_sum_to_the_block():
    """The block's weighted sum over slots, regrouped by owner: for every
    partition of the experts the parts add up to the unsharded y and S."""
    gate, up, down, vals, x, ids, p = _case()
    full = O.moe(gate, up, down, vals, x, ids, p)
    for world in (2, 3, 10):
        parts = [O.moe_shard(gate, up, down, vals, x, ids, p, *ep.shard_range(10, world, r)) for r in range(world)]
        y = sum(pt["y"] for pt in parts)
        assert np.allclose(y, full["y"], rtol=1e-12, atol=1e-12 * np.abs(full["y"]).max())
        assert np.allclose(sum(pt["S"] for pt in parts), full["S"], rtol=1e-12)
    # a shard that owns none of the routed experts contributes exactly zero
    none = O.moe_shard(gate, up, down, vals, x, ids, p, 0, 0)
    assert not none["y"].any()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port):
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        gate, up, down, vals, x, ids, p = _case()
        lo, hi = ep.shard_range(gate.experts, world, rank)
        part = O.moe_shard(gate, up, down, vals, x, ids, p, lo, hi)["y"]
        t = torch.from_numpy(part.copy())
        dist.all_reduce(t, op=dist.ReduceOp.SUM)
        full = O.moe(gate, up, down, vals, x, ids, p)["y"]
        assert np.allclose(t.numpy(), full, rtol=1e-12, atol=1e-12 * np.abs(full).max())
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_all_reduce_their_parts_to_the_block():
    torch.multiprocessing.spawn(_rank, args=(2, _free_port()), nprocs=2, join=True)


def _prefill_rank(rank, world, port, E):
    """One gloo rank of the expert-parallel prefill: its own tokens, the
    dispatch / combine of the module, the expert step computed by the oracle
    (one pair per row), the result checked against the oracle's block."""
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    from tests.util import check_y
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rng = S.rng_for(90)
        H, F, k = 256, 256, 4
        gate = S.random_streams(rng, "iq2_ks", E, F, H)
        up = S.random_streams(rng, "iq2_k", E, F, H)
        down = S.random_streams(rng, "iq2_ks", E, H, F)
        vals = S.value_table("f16", 3)
        r2 = S.rng_for(91 + rank)
        T = 5 + 4 * rank  # ranks hold different token counts
        x = S.random_bf16(r2, (T, H))
        ids, p = S.routing(r2, T, E, k)
        lo, hi = ep.shard_range(E, world, rank)
        seen = []

        def compute(rows, rid):
            bits = rows.view(torch.int16).numpy().view(np.uint16)
            rid = rid.numpy()
            seen.append(rid.copy())
            if len(rid) == 0:
                return torch.empty((0, H), dtype=torch.float32)
            out = O.moe(gate, up, down, vals, bits, rid[:, None], np.ones((len(rid), 1), np.float32))
            return torch.from_numpy(out["y"].astype(np.float32))

        def combine(rows, pw):
            r = rows.numpy().reshape(T, k, H)
            acc = np.zeros((T, H), np.float32)
            for j in range(k):  # slot order, float32, as the device combine
                acc = acc + pw.numpy()[:, j:j + 1] * r[:, j]
            return O.bf16_round(acc)

        mod = ep.ExpertParallelPrefill(gate, up, down, vals, compute=compute, combine=combine)
        y = mod(torch.from_numpy(x.view(np.int16)).view(torch.bfloat16), torch.from_numpy(ids), torch.from_numpy(p))
        got = np.concatenate(seen) if seen else np.zeros(0, np.int32)
        assert np.all((got >= lo) & (got < hi)), "a pair reached a rank that does not own its expert"
        # every pair routed to this rank's experts, from every rank's tokens, arrived here
        owned = [ep.shard_range(E, world, r) for r in range(world)]
        routed = torch.tensor([int(np.sum((ids >= a) & (ids < b))) for a, b in owned])
        dist.all_reduce(routed)
        assert len(got) == int(routed[rank])
        check_y(y, O.moe(gate, up, down, vals, x, ids, p), None, f"rank {rank}")
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world", [2, 3])
def test_gloo_ranks_dispatch_and_combine_the_prefill(world):
    """All-to-all dispatch of every (token, slot) pair to its expert's owner
    and the combine back, over gloo ranks with different token counts."""
    torch.multiprocessing.spawn(_prefill_rank, args=(world, _free_port(), 10), nprocs=world, join=True)


def test_prefill_plan_groups_pairs_by_owner():
    mod = ep.ExpertParallelPrefill.__new__(ep.ExpertParallelPrefill)
    mod.torch, mod.world, mod.experts = torch, 3, 10
    mod.bounds = [ep.shard_range(10, 3, r) for r in range(3)]
    mod._starts = torch.tensor([lo for lo, _ in mod.bounds])
    ids = torch.tensor([[9, 0, 4], [3, 3, 7], [5, 1, 8]], dtype=torch.int32)
    order, counts = mod.plan(ids)
    owner = [next(r for r, (lo, hi) in enumerate(mod.bounds) if lo <= e < hi) for e in ids.reshape(-1).tolist()]
    assert counts.tolist() == [owner.count(r) for r in range(3)]
    assert order.tolist() == sorted(range(9), key=lambda i: (owner[i], i))
    with pytest.raises(ValueError):
        mod.plan(torch.tensor([[10]], dtype=torch.int32))
