"""Switch linear (routed single projection) against the oracle, both kernels."""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.util import check_fp32, to_dev_bf16

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def _case(seed, fmt, E, rows, cols, T, topk, bad=False):
    rng = S.rng_for(seed)
    w = S.random_streams(rng, fmt, E, rows, cols)
    x = S.random_bf16(rng, (T, cols))
    ids, _ = S.routing(rng, T, E, topk)
    if bad:
        ids = ids.copy()
        ids[0, 0] = E + 3
    return w, x, ids


def _run(B, w, x, ids, values, mode):
    dw = B.Weights.from_host(w)
    ids_d = torch.from_numpy(ids).cuda()
    ws = B.workspace(B.iqk_switch_linear_workspace_bytes(mode, ids.shape[0], ids.shape[1], w.experts, w.rows, w.cols))
    y = B.iqk_switch_linear(dw, values, to_dev_bf16(x), ids_d, mode=mode, ws=ws).cpu().numpy()
    return y, B.iqk_moe_status(ws)


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
@pytest.mark.parametrize("T", [1, 5, 20])
def test_switch_decode_kernel(B, fmt, T):
    w, x, ids = _case(90 + T, fmt, 12, 200, 768, T, 6)  # ragged rows, 3 blocks per row
    vals = S.value_table("f16", 5)
    y, st = _run(B, w, x, ids, vals, mode=1)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st == 0
    check_fp32(y, y_ref, Sabs, f"switch decode {fmt} T={T}")


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
@pytest.mark.parametrize("T", [1, 37])
def test_switch_gemm_kernel(B, fmt, T):
    w, x, ids = _case(95 + T, fmt, 10, 512, 1024, T, 4)
    vals = S.value_table("int", 6)
    y, st = _run(B, w, x, ids, vals, mode=2)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st == 0
    check_fp32(y, y_ref, Sabs, f"switch gemm {fmt} T={T}")


@pytest.mark.parametrize("mode", [1, 2])
def test_switch_out_of_range_id(B, mode):
    w, x, ids = _case(99, "iq2_ks", 8, 256, 512, 3, 2, bad=True)
    vals = S.value_table("int", 7)
    y, st = _run(B, w, x, ids, vals, mode=mode)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st & 1
    assert not y[0, 0].any()
    check_fp32(y, y_ref, Sabs, f"switch bad id mode {mode}")


@pytest.mark.parametrize("T", [1, 64, 100])
def test_switch_auto_config_geometry(B, T):
    """Gate-projection geometry of the routed block (2048 x 4096, 32 experts
    resident); auto mode picks the decode kernel at 6 and 384 pairs and the
    grouped GEMM at 600. Sampled rows are checked against the oracle."""
    w, x, ids = _case(120 + T, "iq2_ks", 32, 2048, 4096, T, 6)
    vals = S.value_table("int", 8)
    y, st = _run(B, w, x, ids, vals, mode=0)
    assert st == 0
    rng = np.random.default_rng(T)
    toks = rng.choice(T, size=min(T, 4), replace=False)
    sub = ids[toks]
    y_ref, Sabs = O.switch_linear(w, vals, x[toks], sub)
    check_fp32(y[toks], y_ref, Sabs, f"switch auto T={T}")


@pytest.mark.parametrize("fmt,rows,cols,T", [
    ("iq2_ks", 37, 256, 1),    # one slice per row: 8 tiles per group, ragged last group
    ("iq2_k", 100, 1024, 3),   # two slices: 4 tiles per group
    ("iq2_ks", 48, 5120, 2),   # five slices: one tile per group
    ("iq2_k", 33, 9216, 1),    # nine slices: a warp takes two items of a group
    ("iq2_ks", 200, 768, 12),  # two column groups, activations through the read-only path
    ("iq2_k", 130, 2048, 16),  # sixteen columns per expert at most
])
def test_switch_decode_tile_geometries(B, fmt, rows, cols, T):
    """The decode kernel's group shapes (tiles per group from the slices per
    row) at ragged row counts, one and two MMA column groups."""
    w, x, ids = _case(200 + rows, fmt, 10, rows, cols, T, 6)
    vals = S.value_table("int", 9)
    y, st = _run(B, w, x, ids, vals, mode=1)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st == 0
    check_fp32(y, y_ref, Sabs, f"switch decode {fmt} {rows}x{cols} T={T}")


def test_switch_decode_duplicate_slot(B):
    """A token listing one expert in two slots gets the same row in both."""
    w, x, ids = _case(210, "iq2_ks", 6, 64, 512, 2, 3)
    ids = ids.copy()
    ids[0, 2] = ids[0, 0]
    vals = S.value_table("int", 10)
    y, st = _run(B, w, x, ids, vals, mode=1)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st == 0
    check_fp32(y, y_ref, Sabs, "switch decode duplicate slot")
    assert np.array_equal(y[0, 0], y[0, 2])


@pytest.mark.parametrize("T,topk,E", [(1, 12, 4), (40, 6, 10), (64, 6, 256)])
def test_switch_decode_runs_of_pairs(B, T, topk, E):
    """More pairs per expert than one MMA column group (split into runs), and
    the mid-size token counts the decode kernel now takes."""
    rng = S.rng_for(220 + T)
    w = S.random_streams(rng, "iq2_k", E, 96, 512)
    x = S.random_bf16(rng, (T, 512))
    ids = rng.integers(0, E, size=(T, topk)).astype(np.int32)  # repeats within a token allowed
    vals = S.value_table("int", 11)
    y, st = _run(B, w, x, ids, vals, mode=1)
    y_ref, Sabs = O.switch_linear(w, vals, x, ids)
    assert st == 0
    check_fp32(y, y_ref, Sabs, f"switch decode runs T={T} topk={topk} E={E}")
