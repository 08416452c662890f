"""The routed-block parity checks must be able to fail.

Each case builds a routed block at the page's per-expert geometry (gate/up
2048 x 4096, down 4096 x 2048, top-6; mlx-iqk 0.1.1 PKG-INFO, the benchmark
geometry paragraph) with only the routed experts resident, computes it with
the oracle, and confirms that (a) the oracle's own output passes
``tests.util.check_block`` and (b) every planted mistake, computed on the CPU
from the oracle's pieces, is rejected by it: the output zeroed, a routing
slot dropped, uniform routing weights, gate and up swapped, sigmoid in place
of silu, h left unrounded.
"""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.util import bf16_value, check_block

H, F = S.HIDDEN, S.INTER

CASES = {
    # the headline decode: IQ2_KS, one token, six distinct experts
    "decode_iq2_ks_T1": dict(fmt="iq2_ks", E=8, T=1, seed=2),
    # IQ2_K decode, four tokens (experts shared between tokens)
    "decode_iq2_k_T4": dict(fmt="iq2_k", E=12, T=4, seed=3),
    # prefill rows: IQ2_KS, several tokens per expert
    "prefill_iq2_ks_T8": dict(fmt="iq2_ks", E=6, T=8, seed=4),
}


def _block_from_h(down, values, ids, p, h_vals, cache):
    """y = sum_j p_j Wd_j h_j in float64 for given h values, rounded to bf16
    (the oracle's combine, with the down matrices dequantized by the oracle)."""
    ids = np.atleast_2d(ids)
    y = np.zeros((ids.shape[0], down.rows))
    for e in np.unique(ids):
        rows_n, slots = np.nonzero(ids == e)
        if int(e) not in cache:
            cache[int(e)] = O.dequant_expert(down, int(e), values).astype(np.float64)
        wd = cache[int(e)]
        np.add.at(y, rows_n, p[rows_n, slots].astype(np.float64)[:, None] * (h_vals[rows_n, slots] @ wd.T))
    return O.bf16_round(y.astype(np.float32))


@pytest.fixture(scope="module", params=list(CASES))
def case(request):
    c = CASES[request.param]
    rng = S.rng_for(c["seed"])
    gate, up, down = S.moe_weights(rng, c["fmt"], c["E"], H, F)
    x = S.random_bf16(rng, (c["T"], H))
    ids, p = S.routing(rng, c["T"], c["E"], S.TOPK)
    return request.param, gate, up, down, x, ids, p


@pytest.mark.parametrize("table", ["int", "f16"])
def test_checks_pass_the_oracle_and_reject_planted_mistakes(case, table):
    name, gate, up, down, x, ids, p = case
    values = S.value_table(table, 2)
    ref = O.moe(gate, up, down, values, x, ids, p)
    h_ok = bf16_value(ref["h_bits"])
    check_block(ref["y_bits"], h_ok, ref, down, values, ids, p, f"{name} oracle")

    g = ref["g"].astype(np.float64)
    u = ref["u"].astype(np.float64)
    with np.errstate(over="ignore"):
        sig = 1.0 / (1.0 + np.exp(-g))
    h_sigmoid = bf16_value(O.bf16_round((sig * u).astype(np.float32)))
    h_unrounded = (g * sig * u).astype(np.float32).astype(np.float64)
    p_drop0 = p.copy()
    p_drop0[:, 0] = 0
    p_droplast = p.copy()
    p_droplast[:, -1] = 0
    p_uniform = np.full_like(p, 1.0 / p.shape[1])
    swapped = O.moe(up, gate, down, values, x, ids, p)
    cache = {}
    # the combine is linear in p: mistakes in the routing weights reuse the oracle's h
    mutants = {
        "output zeroed": (np.zeros_like(ref["y_bits"]), h_ok),
        "slot 0 dropped": (_block_from_h(down, values, ids, p_drop0, h_ok, cache), h_ok),
        "last slot dropped": (_block_from_h(down, values, ids, p_droplast, h_ok, cache), h_ok),
        "uniform routing weights": (_block_from_h(down, values, ids, p_uniform, h_ok, cache), h_ok),
        "gate and up swapped": (swapped["y_bits"], bf16_value(swapped["h_bits"])),
        "sigmoid in place of silu": (_block_from_h(down, values, ids, p, h_sigmoid, cache), h_sigmoid),
        "h left unrounded": (_block_from_h(down, values, ids, p, h_unrounded, cache), h_unrounded),
    }
    for what, (y_m, h_m) in mutants.items():
        with pytest.raises(AssertionError):
            check_block(y_m, h_m, ref, down, values, ids, p, f"{name} {what}")
        if what in ("slot 0 dropped", "last slot dropped", "uniform routing weights", "output zeroed"):
            # the output check alone rejects the combine mistakes
            with pytest.raises(AssertionError):
                check_block(y_m, None, ref, down, values, ids, p, f"{name} {what} (y only)")
