"""Pricing against the deleted-decode floor (mlx-iqk 0.1.1 PKG-INFO, section
"Pricing"): the validation half. Every arm the benchmark times is checked
against the oracle here: the routed projection decode within the stated
tolerance, the dequantizer and both floors' integer signatures bit for bit
(every load reached the output).

Per member (IQ2_KS, IQ2_K) and projection (gate/up [2048 x 4096], down
[4096 x 2048]), 256 experts resident. The timed half -- the declared ratio
bar, the floor-rate band and no kernel faster than its own floor -- runs in
bench.py (details.pricing), so that a slow box cannot turn a parity run red.
"""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from util import check_fp32

torch = pytest.importorskip("torch")

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def B():
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def _validate(cell):
    w, c = cell.w, 0
    torch.cuda.synchronize()
    with torch.cuda.stream(cell.stream):
        cell.decode(c)
        cell.floor(c)
        cell.dequant(c)
        cell.dequant_floor(c)
    torch.cuda.synchronize()
    y_ref, S_ref = O.switch_linear(w, cell.values, cell.x_h[c], cell.ids_h[c])
    check_fp32(cell.y[c].cpu().numpy(), y_ref, S_ref, f"{w.fmt} {w.rows}x{w.cols} decode arm")
    fo = cell.fout[c].cpu().numpy().view(np.uint32)
    for i, e in enumerate(cell.elist[c].cpu().numpy()):
        assert np.array_equal(fo[i], O.floor_xor(w, int(e))), "floor arm signature"
    e = cell.deq_e[c]
    assert np.array_equal(cell.dq[c % 4].cpu().numpy().view(np.uint32),
                          O.dequant_expert(w, e, cell.values).view(np.uint32)), "dequant arm"
    assert np.array_equal(cell.dqf[c % 4].cpu().numpy().view(np.uint32), O.dequant_floor(w, e)), "dequant floor signature"


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
def test_pricing_arms_validate(B, fmt):
    import bench as BE
    rng = S.rng_for(77)
    values = S.value_table("int" if fmt == "iq2_ks" else "f16", 5)
    device, stream = torch.device("cuda:0"), torch.cuda.Stream()
    for seed, (rows, cols) in enumerate(((S.INTER, S.HIDDEN), (S.HIDDEN, S.INTER))):
        w = S.random_streams(rng, fmt, S.EXPERTS, rows, cols)
        cell = BE.PriceCell(torch, B, w, values, device, stream, seed=seed + 3, calls=84)
        _validate(cell)
        assert B.iqk_floor_status(stream) == B.IQK_OK
        del cell, w
        torch.cuda.empty_cache()
