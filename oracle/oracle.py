"""CPU oracle for the IQ2_KS / IQ2_K routed-expert path.

TEST INFRASTRUCTURE ONLY. Only the tests, the package smoke check and the
benchmark's CPU-baseline leg may import this module; the product path never
does, and this module imports nothing from the CUDA library. It shares no
code, header, table or constant generator with it.

What it computes, and where each step is defined:

* ``dequant``: the page's reconstruction ``d * float(scale_index) *
  values[4*alphabet + code]`` in float32, each product rounded once, in that
  order (mlx-iqk 0.1.1 PKG-INFO, section "Format", the paragraph after the
  stream tables). Implemented in plain C (``iqk_oracle.c``), built with
  ``-ffp-contract=off``.
* ``gemv``: the plain definition ``y[t,o] = sum_k w[o,k] * x[t,k]`` in float64
  (a library matmul as the one step), plus ``S[t,o] = sum_k |w[o,k] * x[t,k]|``,
  the scale of the stated tolerance ``|y - y_ref| <= 2e-3 * S``.
* ``moe``: the routed-expert block the page's geometry describes (gate/up,
  SwiGLU, down, weighted combine; section "Surface" and the benchmark geometry
  paragraph). The page does not write the block out; the plain reading used
  here: ``g = Wg x``, ``u = Wu x``, ``h = bf16_rn(float32(silu(g) * u))`` with
  ``silu(g) = g / (1 + exp(-g))`` in float64, ``y = sum_j p_j * (Wd_j h_j)`` in
  float64, output ``bf16_rn(float32(y))``. Prefill is the same per token.
* ``route_prep``: expert histogram, exclusive prefix sum and the stable
  permutation of (token, slot) pairs sorted by expert -- what "grouped by
  expert ... each expert's weights read once" requires (section "Surface").
* ``floor_xor``: the deleted-decode address floor's checksum (section
  "Pricing": identical loads, decode removed, an integer accumulator).
* ``moe_shard``: one expert-parallel rank's part of ``moe`` (the slots
  routed to its experts), so that the parts of a partition sum to ``moe``.
* ``dequant_floor``: the dequantizer's own floor signature (same section):
  per qs word, the XOR of the stream fields its 16 weights are decoded from,
  written where the dequantizer writes those weights.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "iqk_oracle.c")
_SO = os.path.join(_HERE, "_build", "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile the C part of the oracle (plain gcc, strict float semantics)."""
    os.makedirs(os.path.dirname(_SO), exist_ok=True)
    if force or not os.path.exists(_SO) or os.path.getmtime(_SO) < os.path.getmtime(_SRC):
        tmp = _SO + f".{os.getpid()}.tmp"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _SO)
    return _SO


def lib():
    global _lib
    with _lock:
        if _lib is None:
            L = ctypes.CDLL(build())
            i64, u32p, f32p = ctypes.c_int64, ctypes.c_void_p, ctypes.c_void_p
            L.oracle_half_to_float.restype = ctypes.c_float
            L.oracle_half_to_float.argtypes = [ctypes.c_uint16]
            L.oracle_float_to_bf16.restype = ctypes.c_uint16
            L.oracle_float_to_bf16.argtypes = [ctypes.c_float]
            L.oracle_dequant_iq2_ks.restype = ctypes.c_int
            L.oracle_dequant_iq2_ks.argtypes = [i64, i64] + [ctypes.c_void_p] * 7
            L.oracle_dequant_iq2_k.restype = ctypes.c_int
            L.oracle_dequant_iq2_k.argtypes = [i64, i64] + [ctypes.c_void_p] * 6
            L.oracle_f32_to_bf16_array.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i64]
            L.oracle_half_to_float_array.argtypes = [ctypes.c_void_p, ctypes.c_void_p, i64]
            L.oracle_fields_iq2_ks.argtypes = [ctypes.c_void_p] * 4 + [i64] + [ctypes.c_void_p] * 3
            L.oracle_fields_iq2_k.argtypes = [ctypes.c_void_p] * 3 + [i64] + [ctypes.c_void_p] * 3
            L.oracle_floor_xor.argtypes = [i64, i64, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
            _lib = L
    return _lib


def _p(a: np.ndarray):
    assert a.flags["C_CONTIGUOUS"], "oracle inputs must be C-contiguous"
    return a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dt):
    return np.ascontiguousarray(a, dtype=dt)


# ---------------------------------------------------------------- conversions

def half_to_float(bits) -> np.ndarray:
    b = _c(bits, np.uint16)
    out = np.empty(b.shape, np.float32)
    lib().oracle_half_to_float_array(_p(b), _p(out), b.size)
    return out


def bf16_round(x) -> np.ndarray:
    """float32 -> bfloat16 bit patterns, round to nearest even."""
    f = _c(x, np.float32)
    out = np.empty(f.shape, np.uint16)
    lib().oracle_f32_to_bf16_array(_p(f), _p(out), f.size)
    return out


def bf16_to_float(bits) -> np.ndarray:
    """bfloat16 bit patterns -> float32 (exact: the pattern is the upper half)."""
    return (_c(bits, np.uint16).astype(np.uint32) << 16).view(np.float32)


# --------------------------------------------------------------------- fields

def fields(fmt: str, qs_row, scl_row, sch_row, sex_row, k: int):
    """(code, scale_index, alphabet) of weight ``k`` of one row."""
    c, i, a = ctypes.c_int32(), ctypes.c_int32(), ctypes.c_int32()
    L = lib()
    if fmt == "iq2_ks":
        q, s, h, x = (_c(qs_row, np.uint32), _c(scl_row, np.uint32), _c(sch_row, np.uint8),
                      _c(sex_row, np.uint8))
        L.oracle_fields_iq2_ks(_p(q), _p(s), _p(h), _p(x), k, ctypes.byref(c), ctypes.byref(i),
                               ctypes.byref(a))
    elif fmt == "iq2_k":
        q, s, x = _c(qs_row, np.uint32), _c(scl_row, np.uint32), _c(sex_row, np.uint16)
        L.oracle_fields_iq2_k(_p(q), _p(s), _p(x), k, ctypes.byref(c), ctypes.byref(i), ctypes.byref(a))
    else:
        raise ValueError(fmt)
    return c.value, i.value, a.value


# -------------------------------------------------------------------- dequant

def dequant(fmt: str, rows: int, cols: int, qs, scl, sch, sex, dv, values) -> np.ndarray:
    """float32 [rows, cols] reconstruction of one matrix (bit-exact reference)."""
    v = _c(values, np.float32)
    if v.shape != (8,):
        raise ValueError("values must hold 8 entries")
    out = np.empty((rows, cols), np.float32)
    L = lib()
    if fmt == "iq2_ks":
        rc = L.oracle_dequant_iq2_ks(rows, cols, _p(_c(qs, np.uint32)), _p(_c(scl, np.uint32)),
                                     _p(_c(sch, np.uint8)), _p(_c(sex, np.uint8)),
                                     _p(_c(dv, np.uint16)), _p(v), _p(out))
    elif fmt == "iq2_k":
        rc = L.oracle_dequant_iq2_k(rows, cols, _p(_c(qs, np.uint32)), _p(_c(scl, np.uint32)),
                                    _p(_c(sex, np.uint16)), _p(_c(dv, np.uint16)), _p(v), _p(out))
    else:
        raise ValueError(fmt)
    if rc != 0:
        raise ValueError(f"bad shape rows={rows} cols={cols}")
    return out


def dequant_expert(w, e: int, values) -> np.ndarray:
    """Dequantize expert ``e`` of a stacked-stream object (attributes fmt, rows,
    cols, qs, scl, sch, sex, dv with a leading expert axis)."""
    return dequant(w.fmt, w.rows, w.cols, w.qs[e], w.scl[e], None if w.sch is None else w.sch[e],
                   w.sex[e], w.dv[e], values)


# ----------------------------------------------------------------------- gemv

def gemv(w: np.ndarray, x_bits) -> tuple[np.ndarray, np.ndarray]:
    """y[t, o] = sum_k w[o, k] x[t, k] in float64, and S = sum_k |w x|."""
    x = bf16_to_float(np.atleast_2d(x_bits)).astype(np.float64)
    wd = w.astype(np.float64)
    return x @ wd.T, np.abs(x) @ np.abs(wd).T


# ------------------------------------------------------------------------ moe

def silu(g: np.ndarray) -> np.ndarray:
    """g / (1 + exp(-g)); exp(-g) may overflow to inf for very negative g,
    where the quotient's limit -0/0 is the right value."""
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def silu_grad(g: np.ndarray) -> np.ndarray:
    with np.errstate(over="ignore"):
        s = 1.0 / (1.0 + np.exp(-g))
    return s * (1.0 + g * (1.0 - s))


def bf16_spacing(v: np.ndarray) -> np.ndarray:
    """Distance between consecutive bfloat16 numbers at |v| (normal range)."""
    a = np.maximum(np.abs(v), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def moe(gate, up, down, values, x_bits, ids, p, tokens=None):
    """Routed-expert block for the listed tokens (all by default).

    For every (token t, slot j) pair with expert e = ids[t, j]:
      g = Wg_e x_t, u = Wu_e x_t (float64), h = bf16_rn(float32(silu(g) * u)),
    and y_t = sum_j p_tj * (Wd_e h) in float64, output bf16_rn(float32(y_t)).
    The pairs are visited expert by expert (each expert's three matrices are
    dequantized once per call); the sum over a token's slots is a plain sum,
    so its order does not enter the definition.

    Returns a dict with
      y_bits   bf16 [n, hidden], the rounded output;
      y        float64 [n, hidden] before the final rounding;
      S        sum_j |p_j| sum_f |Wd_jf h_jf|: the scale of the down GEMV's
               stated tolerance;
      h_bits   bf16 [n, topk, inter];
      g, u     the gate and up GEMV results [n, topk, inter] (computed in
               float64, stored as float32);
      S_g, S_u their scales sum_k |w x| (same storage).
    Expert ids must lie in [0, experts).
    """
    x_bits = np.atleast_2d(x_bits)
    ids = np.atleast_2d(np.asarray(ids))
    p = np.atleast_2d(np.asarray(p))
    toks = np.arange(x_bits.shape[0]) if tokens is None else np.asarray(list(tokens), np.int64)
    idn = ids[toks].astype(np.int64)
    if idn.size and (idn.min() < 0 or idn.max() >= gate.experts):
        raise ValueError("expert id out of range")
    pn = p[toks].astype(np.float64)
    xs = bf16_to_float(x_bits[toks]).astype(np.float64)
    n, topk = idn.shape
    H, F = down.rows, down.cols
    y = np.zeros((n, H))
    S = np.zeros((n, H))
    hb = np.zeros((n, topk, F), np.uint16)
    g_out = np.zeros((n, topk, F), np.float32)
    u_out = np.zeros((n, topk, F), np.float32)
    sg_out = np.zeros((n, topk, F), np.float32)
    su_out = np.zeros((n, topk, F), np.float32)
    for e in np.unique(idn):
        rows_n, slots = np.nonzero(idn == e)
        X = xs[rows_n]
        aX = np.abs(X)
        wg = dequant_expert(gate, int(e), values).astype(np.float64)
        wu = dequant_expert(up, int(e), values).astype(np.float64)
        G = X @ wg.T
        U = X @ wu.T
        h = bf16_round((silu(G) * U).astype(np.float32))
        hf = bf16_to_float(h).astype(np.float64)
        wd = dequant_expert(down, int(e), values).astype(np.float64)
        pw = pn[rows_n, slots][:, None]
        np.add.at(y, rows_n, pw * (hf @ wd.T))
        np.add.at(S, rows_n, np.abs(pw) * (np.abs(hf) @ np.abs(wd).T))
        hb[rows_n, slots] = h
        g_out[rows_n, slots] = G
        u_out[rows_n, slots] = U
        sg_out[rows_n, slots] = aX @ np.abs(wg).T
        su_out[rows_n, slots] = aX @ np.abs(wu).T
    return dict(y_bits=bf16_round(y.astype(np.float32)), y=y, S=S, h_bits=hb, g=g_out, u=u_out,
                S_g=sg_out, S_u=su_out)


# -------------------------------------------------------------- switch linear

def switch_linear(w, values, x_bits, ids):
    """Routed single projection (mlx-iqk 0.1.1 page, section "Surface": the
    switch linear's y = proj(x, indices)): y[t, j] = W_{ids[t, j]} x[t] in
    float64 for every (token, slot) pair, with S[t, j] = sum_k |w x| for the
    tolerance. Out-of-range ids give zero rows (and S = 0)."""
    ids = np.asarray(ids, np.int64)
    T, topk = ids.shape
    x_bits = np.atleast_2d(x_bits)
    y = np.zeros((T, topk, w.rows))
    S = np.zeros((T, topk, w.rows))
    for e in np.unique(ids):
        if e < 0 or e >= w.experts:
            continue
        t_idx, j_idx = np.nonzero(ids == e)
        ye, Se = gemv(dequant_expert(w, int(e), values), x_bits[t_idx])
        y[t_idx, j_idx] = ye
        S[t_idx, j_idx] = Se
    return y, S


# ----------------------------------------------------------------- route prep

def route_prep(ids, experts: int):
    """counts[e], offsets[e] (exclusive prefix sum, offsets[E] = total) and the
    pair permutation: pair indices t*topk + j sorted by expert, ties in pair
    order."""
    flat = np.asarray(ids, np.int64).reshape(-1)
    if flat.size and (flat.min() < 0 or flat.max() >= experts):
        raise ValueError("expert id out of range")
    counts = np.bincount(flat, minlength=experts).astype(np.int32)
    offsets = np.zeros(experts + 1, np.int32)
    offsets[1:] = np.cumsum(counts)
    perm = np.argsort(flat, kind="stable").astype(np.int32)
    return counts, offsets, perm


# ---------------------------------------------------------------------- floor

def floor_xor(w, e: int) -> np.ndarray:
    """Per-row XOR fold of every stream byte of expert ``e`` (uint32 [rows])."""
    streams = [a[e] for a in (w.qs, w.scl, w.sch, w.sex, w.dv) if a is not None]
    rows = w.rows
    arrs = [np.ascontiguousarray(a).reshape(rows, -1).view(np.uint8) for a in streams]
    ptrs = (ctypes.c_void_p * len(arrs))(*[a.ctypes.data for a in arrs])
    rb = np.array([a.shape[1] for a in arrs], np.int64)
    out = np.empty(rows, np.uint32)
    lib().oracle_floor_xor(rows, len(arrs), ptrs, _p(rb), _p(out))
    return out


def dequant_floor(w, e: int, bf16: bool = False) -> np.ndarray:
    """Signature the dequantizer's deleted-decode floor writes for expert ``e``.

    Qs word wk of row r carries weights 16*wk .. 16*wk+15; the fields those
    weights are decoded from (section "Format": IQ2_KS one scl word, one sch
    and one sex byte per 256 weights and one dv per row; IQ2_K one scl word
    per 128 weights, one sex halfword and one dv per 256) fold into
    ``m = qs ^ scl ^ sch ^ (sex << 8) ^ (dv << 16)``. The floor stores m ^ k
    in the k-th 32-bit word of the weights' output bytes: 16 words per qs word
    for the float32 output, 8 for bfloat16. uint32 [rows][cols] or
    [rows][cols / 2].
    """
    rows, cols = w.rows, w.cols
    wpr = cols // 16
    wk = np.arange(wpr)
    q = np.asarray(w.qs[e]).reshape(rows, wpr).astype(np.uint32)
    blk = wk // 16  # 256-weight block of each qs word
    if w.fmt == "iq2_ks":
        s = np.asarray(w.scl[e]).reshape(rows, -1)[:, blk].astype(np.uint32)
        h = np.asarray(w.sch[e]).reshape(rows, -1)[:, blk].astype(np.uint32)
        x = np.asarray(w.sex[e]).reshape(rows, -1)[:, blk].astype(np.uint32)
        dv = np.repeat(np.asarray(w.dv[e]).reshape(rows, 1).astype(np.uint32), wpr, axis=1)
    elif w.fmt == "iq2_k":
        s = np.asarray(w.scl[e]).reshape(rows, -1)[:, wk // 8].astype(np.uint32)
        h = np.zeros((rows, wpr), np.uint32)
        x = np.asarray(w.sex[e]).reshape(rows, -1)[:, blk].astype(np.uint32)
        dv = np.asarray(w.dv[e]).reshape(rows, -1)[:, blk].astype(np.uint32)
    else:
        raise ValueError(f"unknown format {w.fmt!r}")
    m = q ^ s ^ h ^ (x << np.uint32(8)) ^ (dv << np.uint32(16))
    n = 8 if bf16 else 16
    return (m[:, :, None] ^ np.arange(n, dtype=np.uint32)[None, None, :]).reshape(rows, wpr * n)


def moe_shard(gate, up, down, values, x_bits, ids, p, lo: int, hi: int):
    """One rank's part of the routed block when its experts are partitioned
    over ranks (expert parallelism): the block's weighted sum over slots,
    restricted to the slots routed to experts [lo, hi); every other slot
    weighs 0. The parts of a partition of the experts add up to ``moe``'s
    float64 y (the sum over slots regrouped by owner). Same dict as ``moe``."""
    ids = np.atleast_2d(ids)
    p = np.where((ids >= lo) & (ids < hi), np.atleast_2d(p), 0.0)
    return moe(gate, up, down, values, x_bits, ids, p)
