"""GPU parity of the tcgen05 prefill path against the CPU oracle (the prefill
reference is the decode reference applied per token). Both stages of the
block are checked: the SwiGLU output h read back from the workspace, and y."""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.util import check_block, flat_stats, from_dev_bf16, read_h, run_block, to_dev_bf16

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


def _check(B, gate, up, down, values, x, ids, p, what, report, prefill=True):
    y, h = run_block(B, gate, up, down, values, x, ids, p, prefill=prefill)
    out = check_block(y, h, O.moe(gate, up, down, values, x, ids, p), down, values, ids, p, what)
    report(what, flat_stats(out))
    return y


@pytest.mark.parametrize("fmts", [("iq2_ks",) * 3, ("iq2_k",) * 3, ("iq2_ks", "iq2_k", "iq2_k"),
                                  ("iq2_k", "iq2_ks", "iq2_ks")])
@pytest.mark.parametrize("T", [1, 37, 300])
def test_prefill_small(B, fmts, T, parity_report):
    gate, up, down, x, ids, p = _case(200 + T, fmts, E=8, H=512, F=512, T=T, topk=6)
    _check(B, gate, up, down, S.value_table("int", 5), x, ids, p, f"prefill {fmts} T={T}", parity_report)


def test_prefill_many_pairs_per_expert(B, parity_report):
    """One expert receives every token (> 128 pairs: several N tiles);
    ragged pair counts on the others; f16 table."""
    gate, up, down, x, ids, p = _case(300, ("iq2_ks",) * 3, E=6, H=768, F=512, T=333, topk=2, skew=3)
    _check(B, gate, up, down, S.value_table("f16", 6), x, ids, p, "prefill skewed", parity_report)


def test_prefill_matches_decode_math(B, parity_report):
    """Decode and prefill compute the same block: both within tolerance of
    the oracle on the same inputs (T=16, 64 experts)."""
    gate, up, down, x, ids, p = _case(301, ("iq2_k",) * 3, E=64, H=1024, F=512, T=16, topk=6)
    values = S.value_table("int", 7)
    _check(B, gate, up, down, values, x, ids, p, "prefill", parity_report)
    _check(B, gate, up, down, values, x, ids, p, "decode", parity_report, prefill=False)


def test_prefill_bad_ids(B, parity_report):
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
    valid = (bad >= 0) & (bad < 8)
    h = read_h(B, ws, 1, 5, 3, 8, 256, 256, valid_pairs=int(valid.sum()))
    out = check_block(from_dev_bf16(y), h, O.moe(gate, up, down, values, x, fixed, pv), down, values, fixed, pv,
                      "prefill bad ids", pairs=valid)
    parity_report("prefill bad ids", flat_stats(out))


@pytest.fixture(scope="module")
def full_prefill(B):
    """The prefill workload at full size: 2048 tokens, 256 experts, top-6,
    IQ2_KS (about 48 pairs per expert), int table."""
    rng = S.rng_for(4)
    gate, up, down = S.moe_weights(rng, "iq2_ks", S.EXPERTS, S.HIDDEN, S.INTER)
    x = S.random_bf16(rng, (2048, S.HIDDEN))
    ids, p = S.routing(rng, 2048, S.EXPERTS, S.TOPK)
    values = S.value_table("int", 4)
    y, h = run_block(B, gate, up, down, values, x, ids, p, prefill=True)
    return gate, up, down, values, x, ids, p, y, h


def test_prefill_full_every_expert_last_tile(B, full_prefill, parity_report):
    """Tokens chosen so that every expert's last (ragged) N tile of pairs is
    checked: for each expert, the token of its last pair in expert order."""
    gate, up, down, values, x, ids, p, y, h = full_prefill
    flat = ids.reshape(-1)
    order = np.argsort(flat, kind="stable")
    last = {}
    for i in order:
        last[int(flat[i])] = int(i) // ids.shape[1]
    toks = np.array(sorted(set(last.values())))
    ref = O.moe(gate, up, down, values, x, ids, p, tokens=toks)
    out = check_block(y[toks], h[toks], ref, down, values, ids[toks], p[toks],
                      f"prefill 2048 tokens, {len(toks)} tokens covering every expert's last tile")
    parity_report("prefill 2048, last tiles", flat_stats(out))


def test_prefill_full_all_tokens(B, full_prefill, parity_report):
    """Every output and every h of the full prefill workload."""
    gate, up, down, values, x, ids, p, y, h = full_prefill
    ref = O.moe(gate, up, down, values, x, ids, p)
    out = check_block(y, h, ref, down, values, ids, p, "prefill 2048 tokens, all")
    parity_report("prefill 2048, all tokens", flat_stats(out))


@pytest.mark.parametrize("fmt,rows,cols,table", [("iq2_k", 200, 512, "f16"), ("iq2_ks", 200, 512, "int"),
                                                 ("iq2_k", 160, 4096, "int"), ("iq2_ks", 272, 2048, "f16")])
def test_producer_tile_is_the_rounded_weight(B, fmt, rows, cols, table):
    """The prefill A operand (what the producer warps store into tensor
    memory) is the oracle's float32 weight rounded to bf16, bit for bit.
    IQ2_K: bf16_rn((d*idx)*value). IQ2_KS: bf16_rn(idx*value), the row
    scale d going to the epilogue; pinned with d = 1 (fp16 0x3C00), where the
    oracle's weight is exactly float(idx)*value. Rows from an offset to a
    ragged end; a row of zero scale (IQ2_K) for the signs of zero."""
    rng = S.rng_for(700 + rows)
    host = S.random_streams(rng, fmt, 3, rows, cols)
    if fmt == "iq2_ks":
        host.dv[...] = 0x3C00
    else:
        host.dv[1, 7, :] = 0  # every weight of row 7 of expert 1 is +-0
    values = S.value_table(table, 11)
    w = B.Weights.from_host(host)
    e, row0 = 1, 5
    nrows = rows - row0
    a = B.iqk_prefill_a_tile(w, e, row0, nrows, values)
    torch.cuda.synchronize()
    got = a.view(torch.int16).cpu().numpy().view(np.uint16)
    ref = O.bf16_round(O.dequant_expert(host, e, values)[row0:row0 + nrows])
    assert got.shape == ref.shape
    bad = np.argwhere(got != ref)
    assert bad.size == 0, f"{len(bad)} mismatches, first at {bad[:3].tolist()}"
