"""GPU parity: dequantization, GEMV, routed decode, grouping and the floor arm,
each through the C ABI against the CPU oracle on the same seeded inputs."""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.encode import encode, idx_range, sub_size
from tests.util import check_block, check_fp32, flat_stats, from_dev_bf16, read_h, run_block, to_dev_bf16

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def bits_equal(a, b):
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))


# ------------------------------------------------------------------ dequant

@pytest.mark.parametrize("case", S.MATRIX_CASES)
@pytest.mark.parametrize("table", ["int", "f16"])
def test_dequant_bitexact_matrix_cases(B, case, table):
    w, _, _ = S.matrix_case(case)
    values = S.value_table(table, S.seed_of(case))
    dw = B.Weights.from_host(w)
    got = B.iqk_dequant(dw, 0, values).cpu().numpy()
    assert bits_equal(got, O.dequant_expert(w, 0, values))


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
def test_dequant_edge_fields_multi_expert(B, fmt):
    """Zero/subnormal/negative scales, every index, ragged row count, expert > 0."""
    rng = np.random.default_rng(41)
    rows, cols = 37, 768
    experts = []
    for e in range(3):
        lo, hi = idx_range(fmt)
        nsub = cols // sub_size(fmt)
        codes = rng.integers(0, 4, size=(rows, cols))
        idx = rng.integers(lo, hi + 1, size=(rows, nsub))
        alpha = rng.integers(0, 2, size=(rows, nsub))
        dshape = (rows,) if fmt == "iq2_ks" else (rows, cols // 256)
        d = rng.uniform(1e-3, 1e-2, size=dshape).astype(np.float16)
        m = rng.random(dshape)
        d[m < 0.1] = (rng.integers(1, 1024, size=(m < 0.1).sum()) * 2.0 ** -24).astype(np.float16)
        d[(m >= 0.1) & (m < 0.15)] = 0
        d *= rng.choice([-1, 1], size=dshape).astype(np.float16)
        experts.append(encode(fmt, codes, idx, alpha, d.view(np.uint16)))
    st = S.Streams(fmt, 3, rows, cols, *[None if getattr(experts[0], k) is None else
                                         np.concatenate([getattr(x, k) for x in experts])
                                         for k in ("qs", "scl", "sch", "sex", "dv")])
    values = S.value_table("f16", 9)
    dw = B.Weights.from_host(st)
    for e in range(3):
        got = B.iqk_dequant(dw, e, values).cpu().numpy()
        assert bits_equal(got, O.dequant_expert(st, e, values)), e


@pytest.mark.parametrize("case", S.MATRIX_CASES)
def test_dequant_bf16_is_rounded_fp32(B, case):
    w, _, _ = S.matrix_case(case)
    values = S.value_table("f16", S.seed_of(case))
    dw = B.Weights.from_host(w)
    got = B.iqk_dequant_bf16(dw, 0, values).view(torch.int16).cpu().numpy().view(np.uint16)
    assert np.array_equal(got, O.bf16_round(O.dequant_expert(w, 0, values)))


# --------------------------------------------------------------------- gemv

@pytest.mark.parametrize("case", S.MATRIX_CASES)
@pytest.mark.parametrize("T", [1, 3, 8])
def test_gemv_matrix_cases(B, case, T):
    w, x, values = S.matrix_case(case)
    rng = S.rng_for(100 + T)
    x = np.concatenate([x, S.random_bf16(rng, (T - 1, w.cols))]) if T > 1 else x
    dw = B.Weights.from_host(w)
    y = B.iqk_gemv(dw, 0, values, to_dev_bf16(x)).cpu().numpy()
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 0, values), x)
    check_fp32(y, y_ref, Sabs, f"gemv {case} T={T}")


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
@pytest.mark.parametrize("rows,cols,T", [(2048, 4096, 1), (2048, 4096, 4), (1030, 5120, 1), (1030, 5120, 2)])
def test_gemv_tile_path(B, fmt, rows, cols, T):
    """Tall matrices with at most 4 tokens take the tile kernel with
    two-block items (scales from the planes): 2048 x 4096 gives one tile per
    CTA and one item per warp; 1030 x 5120 gives a ragged last tile and ten
    slices, so two warps take a second item. Expert 2 of 3, f16 table."""
    rng = S.rng_for(rows + cols + T)
    w = S.random_streams(rng, fmt, 3, rows, cols)
    x = S.random_bf16(rng, (T, cols))
    values = S.value_table("f16", 5)
    dw = B.Weights.from_host(w)
    y = B.iqk_gemv(dw, 2, values, to_dev_bf16(x)).cpu().numpy()
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 2, values), x)
    check_fp32(y, y_ref, Sabs, f"gemv tile path {fmt} {rows}x{cols} T={T}")


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
@pytest.mark.parametrize("T", [9, 16, 33, 64])
def test_gemv_ragged_and_many_tokens(B, fmt, T):
    rng = S.rng_for(7 + T)
    w = S.random_streams(rng, fmt, 2, 200, 1280)  # rows not a multiple of 16; 5 blocks
    x = S.random_bf16(rng, (T, 1280))
    values = S.value_table("f16", 4)
    dw = B.Weights.from_host(w)
    y = B.iqk_gemv(dw, 1, values, to_dev_bf16(x)).cpu().numpy()
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 1, values), x)
    check_fp32(y, y_ref, Sabs, f"gemv {fmt} T={T}")


# ------------------------------------------------------------- moe decode

def _moe_case(seed, fg, fu, fd, E, H, F, T, topk):
    rng = S.rng_for(seed)
    gate = S.random_streams(rng, fg, E, F, H)
    up = S.random_streams(rng, fu, E, F, H)
    down = S.random_streams(rng, fd, E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, topk)
    return gate, up, down, x, ids, p


def _check(B, gate, up, down, values, x, ids, p, what, report):
    y, h = run_block(B, gate, up, down, values, x, ids, p)
    ref = O.moe(gate, up, down, values, x, ids, p)
    out = check_block(y, h, ref, down, values, ids, p, what)
    report(what, flat_stats(out))
    return out


@pytest.mark.parametrize("fmts", [("iq2_ks",) * 3, ("iq2_k",) * 3, ("iq2_ks", "iq2_k", "iq2_ks"),
                                  ("iq2_k", "iq2_ks", "iq2_k")])
@pytest.mark.parametrize("T", [1, 4, 16])
def test_moe_decode_small(B, fmts, T, parity_report):
    gate, up, down, x, ids, p = _moe_case(50 + T, *fmts, E=12, H=512, F=768, T=T, topk=6)
    _check(B, gate, up, down, S.value_table("int", 1), x, ids, p, f"decode {fmts} T={T}", parity_report)


def test_moe_decode_topk_edge(B, parity_report):
    """topk = 1 and topk = 16, T = 64 (the decode limits)."""
    for T, k in [(3, 1), (64, 16)]:
        gate, up, down, x, ids, p = _moe_case(60 + k, "iq2_ks", "iq2_ks", "iq2_k", E=40, H=256, F=256, T=T, topk=k)
        _check(B, gate, up, down, S.value_table("f16", 2), x, ids, p, f"decode T={T} topk={k}", parity_report)


def test_moe_decode_bad_ids_skipped_and_flagged(B, parity_report):
    gate, up, down, x, ids, p = _moe_case(77, "iq2_ks", "iq2_ks", "iq2_ks", E=8, H=256, F=256, T=2, topk=3)
    values = S.value_table("int", 0)
    bad = ids.copy()
    bad[0, 1] = 8
    bad[1, 2] = -1
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, 2, 3, 8, 256, 256))
    y = B.iqk_moe_decode(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(bad).cuda(),
                         torch.from_numpy(p).cuda(), ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_EINVAL
    pv = p.copy()
    pv[0, 1] = 0.0
    pv[1, 2] = 0.0
    fixed = ids.copy()
    fixed[0, 1] = 0
    fixed[1, 2] = 0
    ref = O.moe(gate, up, down, values, x, fixed, pv)
    h = read_h(B, ws, 0, 2, 3, 8, 256, 256)
    valid = (bad >= 0) & (bad < 8)
    out = check_block(from_dev_bf16(y), h, ref, down, values, fixed, pv, "bad ids", pairs=valid)
    parity_report("bad ids", flat_stats(out))
    # a clean call resets the status word
    B.iqk_moe_decode(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(ids).cuda(),
                     torch.from_numpy(p).cuda(), ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_OK


# full-size geometry: 256 experts, gate/up [2048, 4096], down [4096, 2048]
@pytest.fixture(scope="module")
def full_ks(B):
    rng = S.rng_for(2)
    return S.moe_weights(rng, "iq2_ks", S.EXPERTS, S.HIDDEN, S.INTER)


@pytest.fixture(scope="module")
def full_k(B):
    rng = S.rng_for(3)
    return S.moe_weights(rng, "iq2_k", S.EXPERTS, S.HIDDEN, S.INTER)


@pytest.mark.parametrize("table", ["int", "f16"])
def test_moe_decode_full_iq2_ks_e256_top6(B, full_ks, table, parity_report):
    gate, up, down = full_ks
    rng = S.rng_for(20)
    x = S.random_bf16(rng, (1, S.HIDDEN))
    ids, p = S.routing(rng, 1, S.EXPERTS, S.TOPK)
    _check(B, gate, up, down, S.value_table(table, 2), x, ids, p,
           f"IQ2_KS decode, 256 experts, top-6, 1 token, {table} table", parity_report)


@pytest.mark.parametrize("T", [1, 4, 16])
@pytest.mark.parametrize("table", ["int", "f16"])
def test_moe_decode_full_iq2_k_e256_top6(B, full_k, T, table, parity_report):
    gate, up, down = full_k
    rng = S.rng_for(30 + T)
    x = S.random_bf16(rng, (T, S.HIDDEN))
    ids, p = S.routing(rng, T, S.EXPERTS, S.TOPK)
    _check(B, gate, up, down, S.value_table(table, 3), x, ids, p,
           f"IQ2_K decode, 256 experts, top-6, T={T}, {table} table", parity_report)


# ------------------------------------------------------------------- route

@pytest.mark.parametrize("T,E,k", [(1, 8, 6), (100, 16, 6), (2048, 256, 6), (3000, 1000, 4)])
def test_route_bitexact(B, T, E, k):
    rng = S.rng_for(T + E)
    ids, _ = S.routing(rng, T, E, k)
    counts, offsets, perm, _ = B.iqk_moe_route(torch.from_numpy(ids).cuda(), E)
    c_ref, o_ref, p_ref = O.route_prep(ids, E)
    assert np.array_equal(counts.cpu().numpy(), c_ref)
    assert np.array_equal(offsets.cpu().numpy(), o_ref)
    assert np.array_equal(perm.cpu().numpy(), p_ref)


def test_route_bad_ids(B):
    ids = np.array([[0, 5, 9], [2, 2, -3]], np.int32)
    counts, offsets, perm, ws = B.iqk_moe_route(torch.from_numpy(ids).cuda(), 8)
    assert B.iqk_moe_status(ws) == B.IQK_EINVAL
    assert offsets.cpu().numpy()[-1] == 4
    assert list(perm.cpu().numpy()[:4]) == [0, 3, 4, 1]


# ------------------------------------------------------------------- floor

@pytest.mark.parametrize("fmt,rows,cols", [("iq2_ks", 2048, 4096), ("iq2_k", 4096, 2048), ("iq2_ks", 37, 512)])
def test_floor_xor_bitexact(B, fmt, rows, cols):
    rng = S.rng_for(rows)
    w = S.random_streams(rng, fmt, 4, rows, cols)
    dw = B.Weights.from_host(w)
    elist = torch.tensor([3, 1], dtype=torch.int32, device="cuda")
    out = B.iqk_floor(dw, elist).cpu().numpy().view(np.uint32)
    assert np.array_equal(out[0], O.floor_xor(w, 3))
    assert np.array_equal(out[1], O.floor_xor(w, 1))


@pytest.mark.parametrize("fmt,rows,cols", [("iq2_ks", 2048, 4096), ("iq2_k", 4096, 2048), ("iq2_ks", 37, 512),
                                           ("iq2_k", 5, 256)])
@pytest.mark.parametrize("bf16", [False, True])
def test_dequant_floor_bitexact(B, fmt, rows, cols, bf16):
    rng = S.rng_for(rows + 1)
    w = S.random_streams(rng, fmt, 3, rows, cols)
    dw = B.Weights.from_host(w)
    for e in (2, 0):
        out = B.iqk_dequant_floor(dw, e, bf16=bf16).cpu().numpy().view(np.uint32)
        assert np.array_equal(out, O.dequant_floor(w, e, bf16=bf16)), (fmt, rows, cols, bf16, e)


def test_moe_decode_duplicate_ids(B, parity_report):
    """A token listing one expert twice: both slots are computed as separate
    pairs. One token listing one expert in all twelve slots: more pairs than
    one MMA column group, split into runs, each run a separate pass."""
    gate, up, down, x, ids, p = _moe_case(77, "iq2_ks", "iq2_ks", "iq2_ks", E=12, H=512, F=768, T=2, topk=4)
    ids = ids.copy()
    ids[0, 1] = ids[0, 0]
    ids[1, 3] = ids[1, 2]
    vals = S.value_table("int", 3)
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, 2, 4, 12, 512, 768))
    _check_ws(B, gate, up, down, vals, x, ids, p, ws, "duplicate ids", parity_report)
    assert B.iqk_moe_status(ws) == B.IQK_OK
    ids12 = np.full((1, 12), 5, np.int32)
    p12 = np.full((1, 12), 1.0 / 12, np.float32)
    ws12 = B.workspace(B.iqk_moe_workspace_bytes(0, 1, 12, 12, 512, 768))
    _check_ws(B, gate, up, down, vals, x[:1], ids12, p12, ws12, "twelve slots, one expert", parity_report)
    assert B.iqk_moe_status(ws12) == B.IQK_OK


@pytest.mark.parametrize("T,topk,E,dup", [(2, 10, 20, True), (33, 6, 12, False), (40, 4, 64, False)])
def test_moe_decode_runs_of_pairs(B, T, topk, E, dup, parity_report):
    """Experts with more pairs than the MMA columns: split into runs (one
    column group when experts average at most 8 pairs, two otherwise)."""
    gate, up, down, x, ids, p = _moe_case(300 + T, "iq2_k", "iq2_ks", "iq2_ks", E=E, H=512, F=256, T=T, topk=topk)
    if dup:  # token 0 puts one expert in every slot: 10 pairs, 2 runs of one column group
        ids = ids.copy()
        ids[0, :] = ids[1, 0]
    _check(B, gate, up, down, S.value_table("f16", 6), x, ids, p, f"decode runs T={T} topk={topk} E={E}",
           parity_report)


def _check_ws(B, gate, up, down, values, x, ids, p, ws, what, report):
    y, h = run_block(B, gate, up, down, values, x, ids, p, ws=ws)
    out = check_block(y, h, O.moe(gate, up, down, values, x, ids, p), down, values, ids, p, what)
    report(what, flat_stats(out))
