"""Host logic of the pricing gates (no GPU): each declared gate fires on the
condition it names and on nothing else."""
import bench as BE


def _cell(**kw):
    c = {"member": "IQ2_KS", "projection": "gate/up", "decode_over_floor": 1.5, "dequant_over_floor": 1.05,
         "floor_gbs": 5000.0, "dequant_floor_gbs": 5000.0}
    c.update(kw)
    return c


def test_a_clean_table_passes():
    assert BE.price_gates([_cell(), _cell(projection="down")], 6500.0) == []


def test_each_gate_fires_on_its_own_condition():
    hbm = 6500.0
    cases = [
        (_cell(decode_over_floor=BE.PRICE_BAR["decode"] + 0.01), "above the declared bar"),
        (_cell(dequant_over_floor=BE.PRICE_BAR["dequant"] + 0.01), "above the declared bar"),
        (_cell(decode_over_floor=BE.PRICE_MIN_RATIO - 0.01), "deleted-load signature"),
        (_cell(dequant_over_floor=0.5), "deleted-load signature"),
        (_cell(floor_gbs=BE.FLOOR_BAND[1] * hbm * 1.01), "floor band"),
        (_cell(dequant_floor_gbs=BE.FLOOR_BAND[0] * hbm * 0.99), "floor band"),
    ]
    for cell, phrase in cases:
        fails = BE.price_gates([cell], hbm)
        assert len(fails) == 1 and phrase in fails[0], (cell, fails)
