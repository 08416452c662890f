"""Pins of the CPU oracle against what the page and the mathematics fix.

Every expected value here comes from something other than the oracle's own
formula: exact rational arithmetic with one IEEE rounding, library
conversions (numpy float16, torch bfloat16, scipy expit), hand-built one-hot
streams, the byte budgets printed on the page, brute force on tiny inputs.
"""
import ctypes
import json
import os
import subprocess
from fractions import Fraction

import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from tests.encode import encode, idx_range, sub_size

GOLD = os.path.join(os.path.dirname(__file__), "golden")


# ------------------------------------------------------------------ helpers

def exact_weight(d_bits, idx, v):
    """The page's chain for fp16 d, integer index and an fp16-exact table
    entry: d*idx is exact in float32 (<= 16 significant bits), so the chain
    equals the exact product d*idx*v rounded once to float32 (<= 27 bits, exact
    in float64 first). Zero keeps the IEEE product sign."""
    d = float(np.uint16(d_bits).view(np.float16))
    exact = Fraction(d) * idx * Fraction(float(v))
    if exact == 0:
        # IEEE: the sign of a product is the XOR of the signs; float(0) is +0
        neg = bool(np.signbit(d)) ^ (idx < 0) ^ bool(np.signbit(np.float32(v)))
        return np.float32(-0.0) if neg else np.float32(0.0)
    return np.float32(float(exact))


def expected_matrix(fmt, codes, idx, alpha, d_bits, values):
    rows, cols = codes.shape
    ss = sub_size(fmt)
    out = np.empty((rows, cols), np.float32)
    for r in range(rows):
        for k in range(cols):
            j = k // ss
            db = d_bits[r] if fmt == "iq2_ks" else d_bits[r, k // 256]
            out[r, k] = exact_weight(db, int(idx[r, j]), values[4 * int(alpha[r, j]) + int(codes[r, k])])
    return out


def oracle_dq(s, values):
    return O.dequant_expert(s, 0, values)


def random_fields(rng, fmt, rows, cols):
    lo, hi = idx_range(fmt)
    nsub = cols // sub_size(fmt)
    codes = rng.integers(0, 4, size=(rows, cols))
    idx = rng.integers(lo, hi + 1, size=(rows, nsub))
    alpha = rng.integers(0, 2, size=(rows, nsub))
    dshape = (rows,) if fmt == "iq2_ks" else (rows, cols // 256)
    # fp16 scales across normal, subnormal and zero, both signs
    d = rng.uniform(1e-3, 1e-2, size=dshape).astype(np.float16)
    sub = rng.random(dshape) < 0.1
    d[sub] = (rng.integers(1, 1024, size=sub.sum()) * 2.0 ** -24).astype(np.float16)
    d[rng.random(dshape) < 0.05] = 0
    d *= rng.choice([-1, 1], size=dshape).astype(np.float16)
    return codes, idx, alpha, d.view(np.uint16)


def same_bits(a, b):
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))


FMTS = ["iq2_ks", "iq2_k"]


# -------------------------------------------------------------- conversions

def test_half_to_float_matches_numpy_for_every_pattern():
    bits = np.arange(65536, dtype=np.uint16)
    got = O.half_to_float(bits)
    ref = bits.view(np.float16).astype(np.float32)
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def test_bf16_round_matches_torch():
    torch = pytest.importorskip("torch")
    rng = np.random.default_rng(5)
    f = np.concatenate([
        rng.standard_normal(200000).astype(np.float32) * np.float32(10.0) ** rng.integers(-30, 30, 200000).astype(np.float32),
        np.array([0.0, -0.0, np.inf, -np.inf, 1.0, 3.4e38, -3.4e38, 1e-40, -1e-45], np.float32),
        # exact ties: lower 16 bits 0x8000, both parities of bit 16
        (np.arange(1000, dtype=np.uint32) << 16 | 0x8000).view(np.float32),
        (np.arange(1000, dtype=np.uint32) << 16 | 0x18000).view(np.float32),
    ]).astype(np.float32)
    f = f[np.isfinite(f) | np.isinf(f)]
    got = O.bf16_round(f)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    assert np.array_equal(got, ref)
    nanb = O.bf16_round(np.array([np.nan], np.float32))
    assert (nanb[0] & 0x7F80) == 0x7F80 and (nanb[0] & 0x7F) != 0


# ------------------------------------------------ reconstruction, exact pins

@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("table", ["f16", "int"])
def test_round_trip_fields_match_exact_chain(fmt, table):
    rng = np.random.default_rng(11)
    values = S.value_table(table, 3)
    codes, idx, alpha, d = random_fields(rng, fmt, 6, 512)
    s = encode(fmt, codes, idx, alpha, d)
    assert same_bits(oracle_dq(s, values), expected_matrix(fmt, codes, idx, alpha, d, values))


@pytest.mark.parametrize("fmt", FMTS)
def test_exhaustive_index_alphabet_code(fmt):
    """Every (scale index, alphabet, code) combination of the signed range."""
    lo, hi = idx_range(fmt)
    values = S.value_table("f16", 7)
    combos = [(i, a, c) for i in range(lo, hi + 1) for a in (0, 1) for c in range(4)]
    ss = sub_size(fmt)
    nsub_needed = len(combos) // 4  # one sub-block per (i, a), 4 codes each
    cols = 256 * ((nsub_needed * ss + 255) // 256)
    nsub = cols // ss
    codes = np.zeros((1, cols), int)
    idx = np.full((1, nsub), lo)
    alpha = np.zeros((1, nsub), int)
    for n, (i, a) in enumerate([(i, a) for i in range(lo, hi + 1) for a in (0, 1)]):
        idx[0, n], alpha[0, n] = i, a
        for c in range(4):
            codes[0, n * ss + c] = c
    d = np.full((1,) if fmt == "iq2_ks" else (1, cols // 256), np.float16(0.0078125)).view(np.uint16)
    s = encode(fmt, codes, idx, alpha, d)
    got = oracle_dq(s, values)
    for n, (i, a) in enumerate([(i, a) for i in range(lo, hi + 1) for a in (0, 1)]):
        for c in range(4):
            assert got[0, n * ss + c] == np.float32(0.0078125 * i * float(values[4 * a + c])), (i, a, c)
    assert got.min() >= -np.abs(values).max() * 16 * 0.0078125
    # the full range is reachable: both ends of the index appear
    assert lo in idx and hi in idx


@pytest.mark.parametrize("fmt", FMTS)
def test_one_hot_code_positions(fmt):
    """A single code set to 3 in an all-zero-code row changes exactly that weight."""
    values = np.array([1, 2, 4, 8, 16, 32, 64, 128], np.float32)
    cols = 512
    s0 = S.empty_streams(fmt, 1, 1, cols)
    s0.dv[...] = np.float16(1.0).view(np.uint16)
    base = oracle_dq(s0, values)
    for k in range(cols):
        s = S.empty_streams(fmt, 1, 1, cols)
        s.dv[...] = np.float16(1.0).view(np.uint16)
        s.qs[0, 0, k // 16] = np.uint32(3) << np.uint32(2 * (k % 16))
        got = oracle_dq(s, values)
        diff = np.nonzero(got != base)[1]
        assert list(diff) == [k]
        lo = idx_range(fmt)[0]
        assert got[0, k] == np.float32(lo * 8.0)


@pytest.mark.parametrize("fmt", FMTS)
@pytest.mark.parametrize("field", ["scl", "sch", "sex"])
def test_one_hot_subblock_fields(fmt, field):
    if fmt == "iq2_k" and field == "sch":
        pytest.skip("IQ2_K has no sch stream")
    values = np.array([3, 5, 7, 11, 13, 17, 19, 23], np.float32)
    cols, ss = 512, sub_size(fmt)
    def fresh():
        s = S.empty_streams(fmt, 1, 1, cols)
        s.dv[...] = np.float16(1.0).view(np.uint16)
        s.qs[...] = 0x1B1B1B1B  # codes 3,2,1,0 repeating
        return s
    base = oracle_dq(fresh(), values)
    for j in range(cols // ss):
        s = fresh()
        if field == "scl":
            s.scl[0, 0, j >> 3] = np.uint32(5) << np.uint32(4 * (j & 7))
        elif field == "sch":
            s.sch[0, 0, j >> 3] = np.uint8(1 << (j & 7))
        elif fmt == "iq2_ks":
            s.sex[0, 0, j >> 3] = np.uint8(1 << (j & 7))
        else:
            s.sex[0, 0, j >> 4] = np.uint16(1 << (j & 15))
        got = oracle_dq(s, values)
        changed = np.nonzero(got[0] != base[0])[0]
        assert list(changed) == list(range(j * ss, (j + 1) * ss)), (field, j)


def test_one_hot_iq2_k_super_block_scale():
    values = np.arange(1, 9, dtype=np.float32)
    cols = 1024
    for b in range(cols // 256):
        s = S.empty_streams("iq2_k", 1, 1, cols)
        s.qs[...] = 0xFFFFFFFF
        s.dv[0, 0, b] = np.float16(2.0).view(np.uint16)
        got = oracle_dq(s, values)
        nz = np.nonzero(got[0])[0]
        assert list(nz) == list(range(256 * b, 256 * (b + 1)))
        assert np.all(got[0, nz] == np.float32(2.0 * -8 * 4.0))


@pytest.mark.parametrize("fmt", FMTS)
def test_zero_scale_signs(fmt):
    """dv = +-0 or index 0 gives zeros carrying the IEEE product sign."""
    values = np.array([-1, 2, -3, 4, 5, -6, 7, -8], np.float32)
    rng = np.random.default_rng(3)
    codes, idx, alpha, d = random_fields(rng, fmt, 4, 256)
    d[...] = np.where(rng.random(d.shape) < 0.5, np.float16(-0.0), np.float16(0.0)).view(np.uint16)
    idx[1] = 0
    s = encode(fmt, codes, idx, alpha, d)
    got = oracle_dq(s, values)
    assert np.all(got == 0)
    assert same_bits(got, expected_matrix(fmt, codes, idx, alpha, d, values))
    d2 = np.full(d.shape, np.float16(0.5)).view(np.uint16)
    idx[...] = 0
    got2 = oracle_dq(encode(fmt, codes, idx, alpha, d2), values)
    assert same_bits(got2, expected_matrix(fmt, codes, idx, alpha, d2, values))


def test_byte_budgets_match_page():
    gold = json.load(open(os.path.join(GOLD, "page_budgets.json")))
    rng = np.random.default_rng(0)
    for fmt in FMTS:
        for n in (256, 512, 2048, 4096):
            s = S.random_streams(rng, fmt, 1, 3, n)
            per_row = s.stream_bytes_per_row()
            expect = eval(gold[fmt]["row_bytes"], {"n": n})
            assert per_row == expect, (fmt, n)
            bpw = (8 * per_row - gold[fmt]["row_scale_bits"]) / n
            assert bpw == gold[fmt]["bits_per_weight"]


# --------------------------------------------------------------------- gemv

def test_gemv_brute_force_exact():
    """Dyadic table, power-of-two scales and short bf16 activations make every
    product exact; the float64 sum must equal the rational sum exactly."""
    rng = np.random.default_rng(21)
    values = S.value_table("dyadic", 1)
    for fmt in FMTS:
        rows, cols = 5, 256
        codes, idx, alpha, _ = random_fields(rng, fmt, rows, cols)
        dshape = (rows,) if fmt == "iq2_ks" else (rows, 1)
        d = (2.0 ** rng.integers(-6, 3, size=dshape)).astype(np.float16).view(np.uint16)
        s = encode(fmt, codes, idx, alpha, d)
        xs = (rng.integers(-64, 65, size=(2, cols)) / 16.0).astype(np.float32)
        xb = (xs.view(np.uint32) >> 16).astype(np.uint16)
        assert np.array_equal((xb.astype(np.uint32) << 16).view(np.float32), xs)
        y, Sabs = O.gemv(oracle_dq(s, values), xb)
        ss = sub_size(fmt)
        for t in range(2):
            for r in range(rows):
                acc = Fraction(0)
                aabs = Fraction(0)
                for k in range(cols):
                    j = k // ss
                    dd = Fraction(float(np.uint16(d.reshape(rows, -1)[r, 0]).view(np.float16)))
                    w = dd * int(idx[r, j]) * Fraction(float(values[4 * alpha[r, j] + codes[r, k]]))
                    acc += w * Fraction(float(xs[t, k]))
                    aabs += abs(w * Fraction(float(xs[t, k])))
                assert Fraction(y[t, r]) == acc
                assert Fraction(Sabs[t, r]) == aabs


def test_constant_scale_reduces_to_table_lookup_and_matvec():
    rng = np.random.default_rng(2)
    values = S.value_table("f16", 2)
    for fmt in FMTS:
        rows, cols = 7, 768
        codes = rng.integers(0, 4, size=(rows, cols))
        nsub = cols // sub_size(fmt)
        idx = np.ones((rows, nsub), int)
        alpha = np.zeros((rows, nsub), int)
        d = np.full((rows,) if fmt == "iq2_ks" else (rows, cols // 256), np.float16(1.0)).view(np.uint16)
        w = oracle_dq(encode(fmt, codes, idx, alpha, d), values)
        assert np.array_equal(w, values[codes])
        x = S.random_bf16(rng, (3, cols))
        y, _ = O.gemv(w, x)
        xf = (x.astype(np.uint32) << 16).view(np.float32).astype(np.float64)
        ref = np.einsum("ok,tk->to", values[codes].astype(np.float64), xf)
        assert np.allclose(y, ref, rtol=1e-13, atol=1e-13)


# ---------------------------------------------------------------------- moe

def test_silu_grad_matches_central_difference():
    g = np.linspace(-30, 30, 2001)
    h = 1e-6
    num = (O.silu(g + h) - O.silu(g - h)) / (2 * h)
    assert np.allclose(O.silu_grad(g), num, rtol=1e-7, atol=1e-9)


def test_bf16_spacing_is_the_gap_to_the_next_bfloat16():
    torch = pytest.importorskip("torch")
    v = np.array([1.0, 1.5, 3.0, 1e-3, 7e4, -2.5], np.float64)
    t = torch.tensor(v, dtype=torch.bfloat16)
    nxt = torch.nextafter(t.abs(), torch.tensor(float("inf"), dtype=torch.bfloat16))
    assert np.allclose(O.bf16_spacing(v), (nxt - t.abs()).double().numpy(), rtol=0, atol=0)


def test_silu_matches_scipy():
    special = pytest.importorskip("scipy.special")
    g = np.linspace(-40, 40, 10001)
    assert np.allclose(O.silu(g), g * special.expit(g), rtol=1e-14, atol=1e-300)
    assert O.silu(np.array([0.0]))[0] == 0.0


def _small_moe(seed, fmt="iq2_ks", E=5, H=256, F=512, T=3, topk=2):
    rng = S.rng_for(seed)
    gate, up, down = S.moe_weights(rng, fmt, E, H, F)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, topk)
    return gate, up, down, x, ids, p


def test_moe_linear_in_routing_weights_and_slot_order():
    gate, up, down, x, ids, p = _small_moe(1)
    v = S.value_table("int", 0)
    a = O.moe(gate, up, down, v, x, ids, p)
    b = O.moe(gate, up, down, v, x, ids, 4.0 * p)
    assert np.array_equal(b["y"], 4.0 * a["y"])
    c = O.moe(gate, up, down, v, x, ids[:, ::-1].copy(), p[:, ::-1].copy())
    assert np.allclose(c["y"], a["y"], rtol=1e-12, atol=1e-12 * np.abs(a["y"]).max())
    assert np.array_equal(c["h_bits"][:, ::-1], a["h_bits"])


def test_moe_single_expert_is_composition_of_gemvs():
    gate, up, down, x, ids, _ = _small_moe(2, fmt="iq2_k", topk=1)
    v = S.value_table("f16", 0)
    p = np.ones_like(ids, dtype=np.float32)
    out = O.moe(gate, up, down, v, x, ids, p)
    for t in range(x.shape[0]):
        e = int(ids[t, 0])
        g, _ = O.gemv(O.dequant_expert(gate, e, v), x[t])
        u, _ = O.gemv(O.dequant_expert(up, e, v), x[t])
        h = O.bf16_round((g / (1 + np.exp(-g)) * u).astype(np.float32))[0]
        y, _ = O.gemv(O.dequant_expert(down, e, v), h)
        assert np.array_equal(out["h_bits"][t, 0], h)
        assert np.allclose(out["y"][t], y[0], rtol=0, atol=1e-12 * np.abs(y).max())


# --------------------------------------------------------------- route prep

def test_route_prep_against_sorted():
    rng = np.random.default_rng(4)
    for T, E, k in [(1, 8, 3), (37, 16, 6), (200, 256, 6)]:
        ids, _ = S.routing(rng, T, E, k)
        counts, offsets, perm = O.route_prep(ids, E)
        flat = ids.reshape(-1)
        ref = sorted(range(flat.size), key=lambda i: (flat[i], i))
        assert list(perm) == ref
        assert counts.sum() == T * k and offsets[-1] == T * k
        for e in range(E):
            assert counts[e] == int(np.sum(flat == e))
            assert offsets[e] == int(np.sum(flat < e))
    with pytest.raises(ValueError):
        O.route_prep(np.array([[0, 9]]), 8)


# -------------------------------------------------------------------- floor

def test_floor_xor_brute_force():
    rng = S.rng_for(9)
    for fmt in FMTS:
        w = S.random_streams(rng, fmt, 2, 3, 512)
        got = O.floor_xor(w, 1)
        for r in range(3):
            h = 0
            for a in (w.qs, w.scl, w.sch, w.sex, w.dv):
                if a is None:
                    continue
                raw = np.ascontiguousarray(a[1]).reshape(3, -1).view(np.uint8)[r]
                for i, byte in enumerate(raw.tolist()):
                    h ^= byte << (8 * (i % 4))
            assert got[r] == h


# ------------------------------------------------------ planted mistakes

MUTANTS = [
    ("offset 15 instead of 16", "(int32_t)(lo | (hi << 4)) - 16", "(int32_t)(lo | (hi << 4)) - 15"),
    ("IQ2_K nibble from the wrong word", "(scl[j >> 3] >> (4 * (j & 7))) & 15u;\n  uint32_t a = ((uint32_t)sex[j >> 4]",
     "(scl[j >> 4] >> (4 * (j & 7))) & 15u;\n  uint32_t a = ((uint32_t)sex[j >> 4]"),
    ("alphabet bit shifted", "((uint32_t)sex[j >> 3] >> (j & 7)) & 1u", "((uint32_t)sex[j >> 3] >> ((j + 1) & 7)) & 1u"),
    ("alphabet stride 2", "values[4 * alpha + code]", "values[2 * alpha + code]"),
    ("scale held in half precision", "float w = t * values[4 * alpha + code];",
     "float w = (float)(_Float16)t * values[4 * alpha + code];"),
]


@pytest.mark.parametrize("name,old,new", MUTANTS)
def test_pins_catch_planted_mistakes(name, old, new, tmp_path):
    src = open(O._SRC).read()
    assert old in src, name
    path = tmp_path / "mut.c"
    path.write_text(src.replace(old, new))
    so = tmp_path / "mut.so"
    subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fPIC", "-shared", "-o", str(so), str(path), "-lm"])
    L = ctypes.CDLL(str(so))
    caught = False
    rng = np.random.default_rng(17)
    for fmt in FMTS:
        values = S.value_table("f16", 5)
        codes, idx, alpha, d = random_fields(rng, fmt, 4, 512)
        s = encode(fmt, codes, idx, alpha, d)
        out = np.empty((4, 512), np.float32)
        v = np.ascontiguousarray(values, np.float32)
        P = lambda a: np.ascontiguousarray(a).ctypes.data_as(ctypes.c_void_p)
        q, sc, sx, dv = (np.ascontiguousarray(s.qs[0]), np.ascontiguousarray(s.scl[0]),
                         np.ascontiguousarray(s.sex[0]), np.ascontiguousarray(s.dv[0]))
        if fmt == "iq2_ks":
            sh = np.ascontiguousarray(s.sch[0])
            L.oracle_dequant_iq2_ks(ctypes.c_int64(4), ctypes.c_int64(512), P(q), P(sc), P(sh), P(sx), P(dv), P(v), P(out))
        else:
            L.oracle_dequant_iq2_k(ctypes.c_int64(4), ctypes.c_int64(512), P(q), P(sc), P(sx), P(dv), P(v), P(out))
        if not same_bits(out, expected_matrix(fmt, codes, idx, alpha, d, values)):
            caught = True
    assert caught, f"planted mistake not caught: {name}"


# ------------------------------------------------------------- switch linear

def test_switch_linear_brute_force_and_out_of_range():
    """Every (token, slot) output equals the brute-force sum over k of the
    pinned dequantized weight times x; out-of-range ids give zero rows."""
    rng = S.rng_for(77)
    w = S.random_streams(rng, "iq2_k", 3, 5, 256)
    x = S.random_bf16(rng, (2, 256))
    vals = S.value_table("dyadic", 1)
    ids = np.array([[2, 0, 7], [1, 2, -1]], np.int32)
    y, Sabs = O.switch_linear(w, vals, x, ids)
    xf = O.bf16_to_float(x).astype(np.float64)
    for t in range(2):
        for j in range(3):
            e = ids[t, j]
            if e < 0 or e >= 3:
                assert not y[t, j].any() and not Sabs[t, j].any()
                continue
            wd = O.dequant_expert(w, int(e), vals).astype(np.float64)
            for o in range(5):
                acc = sum(wd[o, k] * xf[t, k] for k in range(256))
                assert abs(y[t, j, o] - acc) <= 1e-9 * max(1.0, abs(acc))
                assert abs(Sabs[t, j, o] - sum(abs(wd[o, k] * xf[t, k]) for k in range(256))) <= 1e-9 * max(1.0, Sabs[t, j, o])


# ------------------------------------------------------- dequantizer floor

def _nonzero_index_streams(rng, fmt, rows, cols):
    """Random streams in which no sub-block has scale index 0, so every field
    of a 16-weight group moves at least one of its dequantized values."""
    w = S.random_streams(rng, fmt, 2, rows, cols)
    if fmt == "iq2_ks":
        w.sch[:] = 0  # index = low nibble - 16, never 0
    else:
        for n in range(8):  # nibble 8 (index 0) -> 9
            nib = (w.scl >> np.uint32(4 * n)) & np.uint32(15)
            w.scl ^= np.where(nib == 8, np.uint32(1 << (4 * n)), np.uint32(0)).astype(np.uint32)
    return w


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
def test_dequant_floor_reads_what_the_dequantizer_reads(fmt):
    """Flipping every bit of one element of any stream changes the floor's
    output in exactly the 16-weight groups whose dequantized values change
    (the pinned dequantizer decides which), for the float32 and the bfloat16
    layouts alike: no loaded field is dropped, none is read at the wrong
    place, and nothing else reaches the output."""
    rng = S.rng_for(31)
    rows, cols = 3, 512
    vals = np.array([3, -5, 7, -11, 13, -17, 19, -23], np.float32)  # distinct, non-zero
    w = _nonzero_index_streams(rng, fmt, rows, cols)
    d0 = O.dequant_expert(w, 1, vals).view(np.uint32).reshape(rows, cols // 16, 16)
    f0 = O.dequant_floor(w, 1).reshape(rows, cols // 16, 16)
    b0 = O.dequant_floor(w, 1, bf16=True).reshape(rows, cols // 16, 8)
    assert np.array_equal(f0 ^ f0[..., :1], np.broadcast_to(np.arange(16, dtype=np.uint32), f0.shape))
    assert np.array_equal(b0 ^ b0[..., :1], np.broadcast_to(np.arange(8, dtype=np.uint32), b0.shape))
    for name in ("qs", "scl", "sch", "sex", "dv"):
        arr = getattr(w, name)
        if arr is None:
            continue
        flat = arr[1].reshape(-1)
        for pos in rng.choice(flat.size, size=min(6, flat.size), replace=False):
            saved = flat[pos]
            flat[pos] = saved ^ np.iinfo(arr.dtype).max
            arr[1] = flat.reshape(arr[1].shape)
            d1 = O.dequant_expert(w, 1, vals).view(np.uint32).reshape(rows, cols // 16, 16)
            f1 = O.dequant_floor(w, 1).reshape(rows, cols // 16, 16)
            b1 = O.dequant_floor(w, 1, bf16=True).reshape(rows, cols // 16, 8)
            flat[pos] = saved
            arr[1] = flat.reshape(arr[1].shape)
            moved = np.any(d1 != d0, axis=2)
            assert moved.any(), (name, pos)
            assert np.array_equal(np.any(f1 != f0, axis=2), moved), (name, pos)
            assert np.array_equal(np.any(b1 != b0, axis=2), moved), (name, pos)


@pytest.mark.parametrize("fmt", ["iq2_ks", "iq2_k"])
def test_dequant_floor_of_empty_streams_is_the_word_index(fmt):
    """All-zero streams fold to 0, so output word k of every group is k."""
    w = S.empty_streams(fmt, 1, 2, 256)
    assert np.array_equal(O.dequant_floor(w, 0), np.tile(np.arange(16, dtype=np.uint32), (2, 16)))
    assert np.array_equal(O.dequant_floor(w, 0, bf16=True), np.tile(np.arange(8, dtype=np.uint32), (2, 16)))
