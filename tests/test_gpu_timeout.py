"""Bounded device waits: a wait that runs out reports IQK_ETIMEOUT, the
kernel finishes (its copies in flight land first), and the next call on the
same workspace and stream is correct.

The wait is made to run out with the library's testing hook: warp 0 of every
CTA also waits on a barrier nothing arrives on, bounded at 100 us. No GPU
fault, trap or hang is involved; every other wait keeps its normal bound.
"""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.util import check_block, check_fp32, run_block, to_dev_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LIMIT_NS = 100_000


@pytest.fixture(scope="module")
def B():
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


class expire_waits:
    def __init__(self, B):
        self.B = B

    def __enter__(self):
        self.B.iqk_set_wait_limit_ns(LIMIT_NS, True)

    def __exit__(self, *a):
        self.B.iqk_set_wait_limit_ns(0, False)


def test_decode_wait_runs_out_then_recovers(B):
    rng = S.rng_for(610)
    E, H, F, T, k = 16, 1024, 512, 2, 6
    gate, up, down = S.moe_weights(rng, "iq2_ks", E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, k)
    values = S.value_table("int", 1)
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, T, k, E, H, F))
    with expire_waits(B):
        run_block(B, gate, up, down, values, x, ids, p, ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_ETIMEOUT
    y, h = run_block(B, gate, up, down, values, x, ids, p, ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_OK
    check_block(y, h, O.moe(gate, up, down, values, x, ids, p), down, values, ids, p, "decode after a timeout")


def test_gemv_and_switch_waits_run_out_then_recover(B):
    w, x, values = S.matrix_case(S.MATRIX_CASES[1])
    dw = B.Weights.from_host(w)
    xd = to_dev_bf16(x)
    ws = B.workspace(B.iqk_gemv_workspace_bytes(1, w.rows, w.cols))
    with expire_waits(B):
        B.iqk_gemv(dw, 0, values, xd, ws=ws)
    assert B.iqk_moe_status(ws) == B.IQK_ETIMEOUT
    y = B.iqk_gemv(dw, 0, values, xd, ws=ws).cpu().numpy()
    assert B.iqk_moe_status(ws) == B.IQK_OK
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 0, values), x)
    check_fp32(y, y_ref, Sabs, "gemv after a timeout")

    rng = S.rng_for(611)
    ws_e = S.random_streams(rng, "iq2_k", 8, 512, 1024)
    dws = B.Weights.from_host(ws_e)
    xs = S.random_bf16(rng, (3, 1024))
    ids, _ = S.routing(rng, 3, 8, 4)
    idd = torch.from_numpy(ids).cuda()
    wsw = B.workspace(B.iqk_switch_linear_workspace_bytes(1, 3, 4, 8, 512, 1024))
    with expire_waits(B):
        B.iqk_switch_linear(dws, values, to_dev_bf16(xs), idd, mode=1, ws=wsw)
    assert B.iqk_moe_status(wsw) == B.IQK_ETIMEOUT
    ys = B.iqk_switch_linear(dws, values, to_dev_bf16(xs), idd, mode=1, ws=wsw).cpu().numpy()
    assert B.iqk_moe_status(wsw) == B.IQK_OK
    ys_ref, ys_S = O.switch_linear(ws_e, values, xs, ids)
    assert np.all(np.abs(ys - ys_ref) <= 2e-3 * ys_S + 1e-30)


def test_floor_wait_runs_out_then_recovers(B):
    rng = S.rng_for(612)
    w = S.random_streams(rng, "iq2_ks", 4, 512, 2048)
    dw = B.Weights.from_host(w)
    elist = torch.tensor([2, 0], dtype=torch.int32, device="cuda")
    with expire_waits(B):
        B.iqk_floor(dw, elist)
    assert B.iqk_floor_status() == B.IQK_ETIMEOUT
    out = B.iqk_floor(dw, elist).cpu().numpy().view(np.uint32)
    assert B.iqk_floor_status() == B.IQK_OK
    assert np.array_equal(out[0], O.floor_xor(w, 2))
    assert np.array_equal(out[1], O.floor_xor(w, 0))
