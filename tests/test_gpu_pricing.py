"""Pricing against the deleted-decode floor (mlx-iqk 0.1.1 PKG-INFO, section
"Pricing"): validation first, then the timed arms and the declared gates.

Per member (IQ2_KS, IQ2_K) and projection (gate/up [2048 x 4096], down
[4096 x 2048]), 256 experts resident: the routed projection decode and the
dequantizer, each against its own floor. Before any timing, every arm's output
is checked against the oracle (the floors' integer signatures bit for bit,
which shows that every load reached the output). Then the gates: the declared
ratio bar, the floor-rate band and no kernel faster than its own floor.
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
    assert np.array_equal(cell.dq.cpu().numpy().view(np.uint32),
                          O.dequant_expert(w, e, cell.values).view(np.uint32)), "dequant arm"
    assert np.array_equal(cell.dqf.cpu().numpy().view(np.uint32), O.dequant_floor(w, e)), "dequant floor signature"


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
def test_pricing_cells_validate_then_meet_the_declared_gates(B, fmt):
    import bench as BE
    peaks = BE.measured_peaks()
    rng = S.rng_for(77)
    values = S.value_table("int" if fmt == "iq2_ks" else "f16", 5)
    device, stream = torch.device("cuda:0"), torch.cuda.Stream()
    cells = []
    for proj, (rows, cols) in (("gate/up", (S.INTER, S.HIDDEN)), ("down", (S.HIDDEN, S.INTER))):
        w = S.random_streams(rng, fmt, S.EXPERTS, rows, cols)
        cell = BE.PriceCell(torch, B, w, values, device, stream, seed=len(cells) + 3, calls=84)
        _validate(cell)
        t = cell.time(reps=3)
        cells.append({"member": fmt, "projection": proj,
                      "decode_over_floor": t["decode"] / t["floor"],
                      "dequant_over_floor": t["dequant"] / t["dequant_floor"],
                      "floor_gbs": cell.decode_bytes / (t["floor"] * 1e-6) / 1e9,
                      "dequant_floor_gbs": cell.dequant_bytes / (t["dequant_floor"] * 1e-6) / 1e9})
        del cell, w
        torch.cuda.empty_cache()
    fails = BE.price_gates(cells, peaks["hbm_gbs"])
    assert not fails, "\n".join(fails) + f"\n{cells}"
