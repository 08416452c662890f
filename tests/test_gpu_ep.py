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
from util import TOL, check_moe, from_dev_bf16, to_dev_bf16

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


def _check_partial(y, ref, what):
    """float32 partial: |y - y_ref| <= 2e-3 (S + S_prop) + S_round (no output rounding)."""
    err = np.abs(np.asarray(y, np.float64) - ref["y"])
    bound = TOL * (ref["S"] + ref["S_prop"]) + ref["S_round"] + 1e-30
    assert (err <= bound).all(), f"{what}: worst err/bound {float(np.max(err / bound)):.3f}"


@pytest.mark.parametrize("T,world", [(1, 2), (4, 2), (16, 3)])
def test_shards_sum_to_the_block(B, T, world):
    gate, up, down, vals, x, ids, p = _case(700 + T, T)
    xd, idd, pd = to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    total = torch.zeros((T, down.rows), dtype=torch.float32, device="cuda")
    for r in range(world):
        lo, hi = ep.shard_range(gate.experts, world, r)
        ws = [B.Weights.from_host(ep.shard_streams(w, lo, hi)) for w in (gate, up, down)]
        part = B.iqk_moe_decode_shard(*ws, vals, xd, idd, pd, lo)
        _check_partial(part.cpu().numpy(), O.moe_shard(gate, up, down, vals, x, ids, p, lo, hi),
                       f"shard {r}/{world} T={T}")
        total += part
    y = from_dev_bf16(B.iqk_f32_to_bf16(total))
    check_moe(y, O.moe(gate, up, down, vals, x, ids, p), f"sum of {world} shards T={T}")


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
