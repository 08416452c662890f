"""GPU parity of the tcgen05 prefill path against the CPU oracle (the prefill
reference is the decode reference applied per token)."""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.util import check_moe, from_dev_bf16, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def _case(seed, fmts, E, H, F, T, topk, skew=None):
    rng = S.rng_for(seed)
    gate = S.random_streams(rng, fmts[0], E, F, H)
    up = S.random_streams(rng, fmts[1], E, F, H)
    down = S.random_streams(rng, fmts[2], E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, topk)
    if skew is not None:  # route every token's first slot to one expert
        for t in range(T):
            if skew not in ids[t]:
                ids[t, 0] = skew
    return gate, up, down, x, ids, p


def _prefill(B, gate, up, down, values, x, ids, p, ws=None):
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    y = B.iqk_moe_prefill(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(ids).cuda(),
                          torch.from_numpy(p).cuda(), ws=ws)
    torch.cuda.synchronize()
    return from_dev_bf16(y)


@pytest.mark.parametrize("fmts", [("iq2_ks",) * 3, ("iq2_k",) * 3, ("iq2_ks", "iq2_k", "iq2_k"),
                                  ("iq2_k", "iq2_ks", "iq2_ks")])
@pytest.mark.parametrize("T", [1, 37, 300])
def test_prefill_small(B, fmts, T):
    gate, up, down, x, ids, p = _case(200 + T, fmts, E=8, H=512, F=512, T=T, topk=6)
    values = S.value_table("int", 5)
    y = _prefill(B, gate, up, down, values, x, ids, p)
    ref = O.moe(gate, up, down, values, x, ids, p)
    check_moe(y, ref, f"prefill {fmts} T={T}")


def test_prefill_many_pairs_per_expert(B):
    """One expert receives every token (> 128 pairs: several N tiles);
    ragged pair counts on the others; f16 table."""
    gate, up, down, x, ids, p = _case(300, ("iq2_ks",) * 3, E=6, H=768, F=512, T=333, topk=2, skew=3)
    values = S.value_table("f16", 6)
    y = _prefill(B, gate, up, down, values, x, ids, p)
    ref = O.moe(gate, up, down, values, x, ids, p)
    check_moe(y, ref, "prefill skewed")


def test_prefill_matches_decode_math(B):
    """Decode and prefill compute the same block: both within tolerance of
    the oracle on the same inputs (T=16, 64 experts)."""
    gate, up, down, x, ids, p = _case(301, ("iq2_k",) * 3, E=64, H=1024, F=512, T=16, topk=6)
    values = S.value_table("int", 7)
    ref = O.moe(gate, up, down, values, x, ids, p)
    y_pf = _prefill(B, gate, up, down, values, x, ids, p)
    check_moe(y_pf, ref, "prefill")
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    y_dec = B.iqk_moe_decode(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(ids).cuda(),
                             torch.from_numpy(p).cuda())
    check_moe(from_dev_bf16(y_dec), ref, "decode")


def test_prefill_bad_ids(B):
    gate, up, down, x, ids, p = _case(302, ("iq2_ks",) * 3, E=8, H=256, F=256, T=5, topk=3)
    values = S.value_table("int", 0)
    bad = ids.copy()
    bad[2, 1] = 99
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    ws = B.workspace(B.iqk_moe_workspace_bytes(1, 5, 3, 8, 256, 256))
    y = B.iqk_moe_prefill(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(bad).cuda(),
                          torch.from_numpy(p).cuda(), ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_EINVAL
    pv = p.copy()
    pv[2, 1] = 0
    fixed = ids.copy()
    fixed[2, 1] = 0
    ref = O.moe(gate, up, down, values, x, fixed, pv)
    check_moe(from_dev_bf16(y), ref, "prefill bad ids")


def test_prefill_full_iq2_ks_e256_top6_2048_sampled(B):
    """The prefill workload at full size (2048 tokens, 256 experts, top-6, IQ2_KS);
    sampled tokens checked against the oracle one by one, every output finite."""
    rng = S.rng_for(4)
    gate, up, down = S.moe_weights(rng, "iq2_ks", S.EXPERTS, S.HIDDEN, S.INTER)
    x = S.random_bf16(rng, (2048, S.HIDDEN))
    ids, p = S.routing(rng, 2048, S.EXPERTS, S.TOPK)
    values = S.value_table("int", 4)
    y = _prefill(B, gate, up, down, values, x, ids, p)
    yf = (y.astype(np.uint32) << 16).view(np.float32)
    assert np.all(np.isfinite(yf))
    sample = np.random.default_rng(0).choice(2048, size=12, replace=False)
    ref = O.moe(gate, up, down, values, x, ids, p, tokens=sample)
    check_moe(y[sample], ref, "prefill 2048 tokens, sampled")
