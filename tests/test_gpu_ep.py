"""Expert parallelism on the GPU: each shard's float32 partial against the
oracle's part, the partials summed and rounded against the whole block, and
the module with one rank (plain and over a one-rank NCCL group) bit for bit
against the single-GPU decode."""
import os
import socket

import numpy as np
import pytest

import iqk_synth as S
from gemm_iq2_ks_b200 import ep
from oracle import oracle as O
from util import check_block, flat_stats, from_dev_bf16, read_h, to_dev_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def _case(seed, T, E=16, H=512, F=768, topk=6):
    rng = S.rng_for(seed)
    gate = S.random_streams(rng, "iq2_ks", E, F, H)
    up = S.random_streams(rng, "iq2_ks", E, F, H)
    down = S.random_streams(rng, "iq2_k", E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, topk)
    return gate, up, down, S.value_table("int", 4), x, ids, p


@pytest.mark.parametrize("T,world", [(1, 2), (4, 2), (16, 3)])
def test_shards_sum_to_the_block(B, T, world, parity_report):
    """Each shard's float32 partial against the oracle's part (its h read from
    the shard's workspace, its y with no output rounding); the partials summed
    and rounded against the whole block (the h of every pair comes from the
    shard that owns its expert)."""
    gate, up, down, vals, x, ids, p = _case(700 + T, T)
    xd, idd, pd = to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    total = torch.zeros((T, down.rows), dtype=torch.float32, device="cuda")
    h_all = np.full((T, ids.shape[1], gate.rows), np.nan)
    H, F, k = gate.cols, gate.rows, ids.shape[1]
    for r in range(world):
        lo, hi = ep.shard_range(gate.experts, world, r)
        wsr = [B.Weights.from_host(ep.shard_streams(w, lo, hi)) for w in (gate, up, down)]
        ws = B.workspace(B.iqk_moe_workspace_bytes(0, T, k, hi - lo, H, F))
        part = B.iqk_moe_decode_shard(*wsr, vals, xd, idd, pd, lo, ws=ws)
        torch.cuda.synchronize()
        mine = (ids >= lo) & (ids < hi)
        h = read_h(B, ws, 0, T, k, hi - lo, H, F)
        h_all[mine] = h[mine]
        ref = O.moe_shard(gate, up, down, vals, x, ids, p, lo, hi)
        out = check_block(part.cpu().numpy(), h, ref, down, vals, ids, np.where(mine, p, 0), f"shard {r}/{world} T={T}",
                          pairs=mine, y_f32=True)
        parity_report(f"shard {r}/{world} T={T}", flat_stats(out))
        total += part
    y = from_dev_bf16(B.iqk_f32_to_bf16(total))
    out = check_block(y, h_all, O.moe(gate, up, down, vals, x, ids, p), down, vals, ids, p,
                      f"sum of {world} shards T={T}")
    parity_report(f"sum of {world} shards T={T}", flat_stats(out))


def test_f32_to_bf16_rounds_to_nearest_even(B):
    rng = np.random.default_rng(3)
    v = np.concatenate([rng.standard_normal(4096).astype(np.float32) * 1e3,
                        np.array([0.0, -0.0, 1.0 + 2.0 ** -8, 1.0 + 3 * 2.0 ** -8, 3.0e38, -1e-40], np.float32)])
    out = B.iqk_f32_to_bf16(torch.from_numpy(v).cuda())
    got = out.view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_round(v))


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def test_module_with_one_rank_equals_the_single_gpu_decode(B):
    """With one rank the shard holds every expert: the module's y equals
    iqk_moe_decode's bit for bit, alone and over a one-rank NCCL group."""
    import torch.distributed as dist
    gate, up, down, vals, x, ids, p = _case(720, 3)
    xd, idd, pd = to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    ref = B.iqk_moe_decode(dg, du, dd, vals, xd, idd, pd)
    mod = ep.ExpertParallelDecode(gate, up, down, vals)
    assert torch.equal(mod(xd, idd, pd).view(torch.int16), ref.view(torch.int16))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    import datetime
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    try:
        mod1 = ep.ExpertParallelDecode(gate, up, down, vals)
        assert torch.equal(mod1(xd, idd, pd).view(torch.int16), ref.view(torch.int16))
        torch.cuda.synchronize()
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("T,world", [(37, 2), (300, 3)])
def test_prefill_shards_sum_to_the_block(B, T, world, parity_report):
    """iqk_moe_prefill_shard: each rank's float32 partial against the
    oracle's part (h from the shard's workspace), the partials summed and
    rounded against the whole block."""
    gate, up, down, vals, x, ids, p = _case(760 + T, T)
    xd, idd, pd = to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    H, F, k = gate.cols, gate.rows, ids.shape[1]
    total = torch.zeros((T, down.rows), dtype=torch.float32, device="cuda")
    h_all = np.full((T, k, F), np.nan)
    for r in range(world):
        lo, hi = ep.shard_range(gate.experts, world, r)
        wsr = [B.Weights.from_host(ep.shard_streams(w, lo, hi)) for w in (gate, up, down)]
        ws = B.workspace(B.iqk_moe_workspace_bytes(1, T, k, hi - lo, H, F))
        part = B.iqk_moe_prefill_shard(*wsr, vals, xd, idd, pd, lo, ws=ws)
        torch.cuda.synchronize()
        assert B.iqk_moe_status(ws) == B.IQK_OK  # other ranks' ids are not errors
        mine = (ids >= lo) & (ids < hi)
        h = read_h(B, ws, 1, T, k, hi - lo, H, F, valid_pairs=int(mine.sum()))
        h_all[mine] = h[mine]
        out = check_block(part.cpu().numpy(), h, O.moe_shard(gate, up, down, vals, x, ids, p, lo, hi), down, vals,
                          ids, np.where(mine, p, 0), f"prefill shard {r}/{world} T={T}", pairs=mine, y_f32=True)
        parity_report(f"prefill shard {r}/{world} T={T}", flat_stats(out))
        total += part
    y = from_dev_bf16(B.iqk_f32_to_bf16(total))
    out = check_block(y, h_all, O.moe(gate, up, down, vals, x, ids, p), down, vals, ids, p,
                      f"sum of {world} prefill shards T={T}")
    parity_report(f"sum of {world} prefill shards T={T}", flat_stats(out))


def test_combine_is_the_slot_order_weighted_sum(B):
    """iqk_moe_combine: y[t] = bf16(sum over slots in order of p * row), within
    one bf16 spacing of the exact sum (the rounding of float32 partial sums)."""
    rng = np.random.default_rng(5)
    T, k, H = 33, 6, 512
    rows = rng.standard_normal((T * k, H)).astype(np.float32)
    p = rng.random((T, k)).astype(np.float32)
    y = from_dev_bf16(B.iqk_moe_combine(torch.from_numpy(rows).cuda(), torch.from_numpy(p).cuda()))
    exact = np.einsum("tj,tjh->th", p.astype(np.float64), rows.reshape(T, k, H).astype(np.float64))
    got = (y.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    spac = 2.0 ** (np.floor(np.log2(np.maximum(np.abs(exact), 2.0 ** -126))) - 7)
    assert np.all(np.abs(got - exact) <= spac + 1e-6 * np.abs(rows).max())


def test_prefill_module_with_one_rank_equals_the_single_gpu_prefill(B, parity_report):
    """The all-to-all prefill with one rank (no group, then a one-rank NCCL
    group): every pair is dispatched to itself, computed as one float32 row
    and combined; against the oracle, and compared with iqk_moe_prefill."""
    import torch.distributed as dist
    gate, up, down, vals, x, ids, p = _case(730, 40)
    xd, idd, pd = to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    ref_dev = from_dev_bf16(B.iqk_moe_prefill(dg, du, dd, vals, xd, idd, pd))
    ref = O.moe(gate, up, down, vals, x, ids, p)
    mod = ep.ExpertParallelPrefill(gate, up, down, vals)
    y = from_dev_bf16(mod(xd, idd, pd))
    out = check_block(y, None, ref, down, vals, ids, p, "one-rank prefill module")
    parity_report("one-rank prefill module", dict(flat_stats(out), equal_to_single_gpu=bool(np.array_equal(y, ref_dev))))
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(_free_port())
    import datetime
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=torch.device("cuda:0"),
                            timeout=datetime.timedelta(seconds=60))
    try:
        mod1 = ep.ExpertParallelPrefill(gate, up, down, vals)
        y1 = from_dev_bf16(mod1(xd, idd, pd))
        torch.cuda.synchronize()
        assert np.array_equal(y1, y)
    finally:
        dist.destroy_process_group()
