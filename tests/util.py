"""Shared helpers for the parity tests (comparison rules and device upload).

The stated tolerance is per GEMV output: |y - y_ref| <= 2e-3 * sum |w x|,
bf16 outputs compared after rounding (plus one bf16 spacing). The routed
block chains three GEMVs, so it is checked stage by stage:

* ``check_h``: the SwiGLU output h = bf16(silu(g) u) read back from the
  kernel. With g and u each within 2e-3 of their own GEMV scale, silu(g) u
  lies in an interval that follows from the monotone pieces of silu; the
  kernel's h must be a bfloat16 number between the bfloat16 roundings of
  that interval's ends. An h that is not a bfloat16 number fails.
* ``check_y``: the combined output. The down GEMV reads the kernel's own h,
  which may differ from the oracle's; with dh = |h_kernel - h_oracle| and
  R = sum_j |p_j| |Wd_j| dh_j (computed by ``h_reach``),
      |y - y_ref| <= 2e-3 (S + R) + R + spacing_bf16(y).
  With the kernel's h equal to the oracle's, R = 0 and this is the stated
  per-output rule for the down GEMV.
"""
import numpy as np

TOL = 2e-3  # stated tolerance: |y - y_ref| <= 2e-3 * sum |w x| per output
SILU_ARGMIN = -1.2784645427610738  # silu is decreasing below this point and increasing above it


def bf16_ulp(v):
    """Spacing of bfloat16 numbers at |v| (normal range; 2^-133 below)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def bf16_value(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def check_fp32(y, y_ref, S, what=""):
    """float32 outputs: |y - y_ref| <= 2e-3 * S. Returns the worst err / (2e-3 S)."""
    y = np.asarray(y, np.float64)
    err = np.abs(y - y_ref)
    bound = TOL * S + 1e-30
    ratio = float(np.max(err / np.maximum(TOL * S, 1e-30))) if err.size else 0.0
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} outputs out of tolerance; worst err/(2e-3 S) = {ratio:.3f}"
    return ratio


def check_bf16(y_bits, y_ref, S, what=""):
    """bf16 outputs compared after rounding: |y - y_ref| <= 2e-3 * S + 1 bf16 spacing."""
    y = bf16_value(y_bits)
    err = np.abs(y - y_ref)
    ulp = bf16_ulp(np.maximum(np.abs(y), np.abs(y_ref)))
    bound = TOL * S + ulp
    bad = err > bound
    ratio = float(np.max(err / bound)) if err.size else 0.0
    assert not bad.any(), f"{what}: {bad.sum()} outputs out of tolerance; worst err/bound = {ratio:.3f}"
    return ratio


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bf16(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def _silu(g):
    with np.errstate(over="ignore"):
        return g / (1.0 + np.exp(-g))


def h_interval(ref):
    """[lo, hi] of silu(g') u' over |g' - g| <= 2e-3 S_g and |u' - u| <= 2e-3 S_u,
    from the oracle's g, u, S_g, S_u (exact interval arithmetic: silu is
    monotone on either side of its minimum; a product of intervals takes its
    extremes at the corners)."""
    g = ref["g"].astype(np.float64)
    u = ref["u"].astype(np.float64)
    dg = TOL * ref["S_g"].astype(np.float64)
    du = TOL * ref["S_u"].astype(np.float64)
    s1, s2 = _silu(g - dg), _silu(g + dg)
    s_lo = np.minimum(s1, s2)
    inside = (g - dg < SILU_ARGMIN) & (g + dg > SILU_ARGMIN)
    s_lo = np.where(inside, _silu(np.float64(SILU_ARGMIN)), s_lo)
    s_hi = np.maximum(s1, s2)
    c = np.stack([s_lo * (u - du), s_lo * (u + du), s_hi * (u - du), s_hi * (u + du)])
    lo, hi = c.min(axis=0), c.max(axis=0)
    # the kernel evaluates silu and the product in float32 with its own exp:
    # a relative 2^-20 on top (float32 keeps 24 bits), and an absolute floor
    # for e^g below float32's normal range (2^-126), where silu(g) = g e^g /
    # (1 + e^g) can lose up to |g| 2^-126 before the product with u
    slack = (2.0 ** -20 * np.maximum(np.abs(lo), np.abs(hi))
             + 2.0 ** -126 * np.maximum(1.0, np.abs(g) + dg) * (np.abs(u) + du) + 2.0 ** -149)
    return lo - slack, hi + slack


def _bf16_rn_f64(v):
    """bfloat16 round-to-nearest-even of float64 values (via float32, rounded
    outward first so the float32 step never moves a value across the interval)."""
    from oracle import oracle as O
    return bf16_value(O.bf16_round(v.astype(np.float32)))


def check_h(h_vals, ref, what=""):
    """The kernel's SwiGLU output against the interval the stated tolerance
    allows (see the module docstring). h_vals: float values [n, topk, inter]
    (bfloat16 numbers for a correct kernel). Returns statistics."""
    h = np.asarray(h_vals, np.float64)
    lo, hi = h_interval(ref)
    lo32 = np.nextafter(lo.astype(np.float32), np.float32(-np.inf))
    hi32 = np.nextafter(hi.astype(np.float32), np.float32(np.inf))
    lo_b, hi_b = _bf16_rn_f64(lo32.astype(np.float64)), _bf16_rn_f64(hi32.astype(np.float64))
    is_bf16 = (h.astype(np.float32).view(np.uint32) & 0xFFFF) == 0
    is_bf16 &= h.astype(np.float32).astype(np.float64) == h
    inside = (h >= lo_b) & (h <= hi_b)
    bad = ~(is_bf16 & inside)
    ho = bf16_value(ref["h_bits"])
    diff = np.abs(h - ho)
    spac = bf16_ulp(ho)
    stats = {"exact": float(np.mean(diff == 0)) if h.size else 1.0,
             "max_spacings": float(np.max(diff / spac)) if h.size else 0.0,
             "within_one_spacing": float(np.mean(diff <= spac)) if h.size else 1.0}
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {h.size} h values outside the tolerance interval "
                           f"({int((~is_bf16).sum())} not bfloat16 numbers); stats {stats}")
    return stats


def h_reach(down, values, ids, p, dh):
    """R[n, o] = sum_j |p_nj| sum_f |Wd_{ids[n,j]}[o, f]| dh[n, j, f]: how far the
    down GEMV's result can move between the oracle's h and h + dh."""
    from oracle import oracle as O
    ids = np.atleast_2d(ids)
    p = np.atleast_2d(p)
    n = ids.shape[0]
    R = np.zeros((n, down.rows))
    nz = np.any(dh != 0, axis=2)
    for e in np.unique(ids[nz]):
        rows_n, slots = np.nonzero((ids == e) & nz)
        awd = np.abs(O.dequant_expert(down, int(e), values).astype(np.float64))
        contrib = (np.abs(p[rows_n, slots])[:, None]) * (dh[rows_n, slots] @ awd.T)
        np.add.at(R, rows_n, contrib)
    return R


def check_y(y_bits, ref, R=None, what=""):
    """The block's bf16 output: |y - y_ref| <= 2e-3 (S + R) + R + spacing_bf16(y).
    Returns the worst err / bound and the worst err / (2e-3 S)."""
    y = bf16_value(y_bits)
    R = 0.0 if R is None else R
    err = np.abs(y - ref["y"])
    ulp = bf16_ulp(np.maximum(np.abs(y), np.abs(ref["y"])))
    bound = TOL * (ref["S"] + R) + R + ulp
    bad = err > bound
    frac = float(np.max(err / bound)) if err.size else 0.0
    rel = float(np.max(np.maximum(err - ulp, 0) / np.maximum(TOL * ref["S"], 1e-300))) if err.size else 0.0
    assert not bad.any(), (f"{what}: {int(bad.sum())} of {err.size} outputs out of tolerance; "
                           f"worst err/bound = {frac:.3f}")
    return {"err_over_bound": frac, "err_minus_ulp_over_2e-3S": rel}


def check_block(y_bits, h_vals, ref, down, values, ids, p, what="", pairs=None, y_f32=False):
    """Both stages of the routed block: h (interval rule), then y with the
    reach of the kernel's h differences. h_vals may be None where the kernel's
    h is not available (then y must meet the rule with R = 0). ``pairs``
    (bool [n, topk]) limits the h check to the pairs the kernel computed;
    the others must carry zero routing weight in ``p``. ``y_f32``: y is a
    float32 array (an expert-parallel partial: no output rounding)."""
    out = {}
    R = None
    if h_vals is not None:
        h = np.asarray(h_vals, np.float64)
        ho = bf16_value(ref["h_bits"])
        if pairs is not None:
            h = np.where(pairs[:, :, None], h, ho)
        out["h"] = check_h(h, ref, what + " h")
        R = h_reach(down, values, ids, p, np.abs(h - ho))
    if y_f32:
        y = np.asarray(y_bits, np.float64)
        Rv = 0.0 if R is None else R
        err = np.abs(y - ref["y"])
        bound = TOL * (ref["S"] + Rv) + Rv + 1e-300
        frac = float(np.max(err / bound)) if err.size else 0.0
        assert (err <= bound).all(), f"{what} y: {int((err > bound).sum())} outputs out of tolerance; worst {frac:.3f}"
        out["y"] = {"err_over_bound": frac}
    else:
        out["y"] = check_y(y_bits, ref, R, what + " y")
    return out


def read_h(B, ws, mode, T, topk, experts, hidden, inter, valid_pairs=None):
    """The kernel's SwiGLU output of the last call on ``ws``, as float64
    values [T, topk, inter] (pairs it did not compute: NaN), from the layout
    iqk_moe_workspace_layout reports. ``valid_pairs``: the number of pairs
    with an in-range id (prefill rows past it are unused)."""
    L = B.iqk_moe_workspace_layout(mode, T, topk, experts, hidden, inter)
    n = L.h_rows
    raw = ws[L.h:L.h + n * inter * 2].cpu().numpy().view(np.uint16).reshape(n, inter)
    f = np.arange(inter)
    raw = raw[:, (f & ~15) | ((f & 3) << 2) | ((f >> 2) & 3)]  # undo the slot transpose
    h = np.full((n, inter), np.nan)
    if mode == 0:
        h[:] = bf16_value(raw)
    else:
        order = ws[L.h_order:L.h_order + n * 4].cpu().numpy().view(np.int32)
        ok = (order >= 0) & (order < n) & (np.arange(n) < (n if valid_pairs is None else valid_pairs))
        h[order[ok]] = bf16_value(raw[ok])
    return h.reshape(T, topk, inter)


def run_block(B, gate, up, down, values, x, ids, p, prefill=False, valid_pairs=None, ws=None):
    """One routed-block call through the C ABI on device copies of the host
    inputs; returns (y bf16 bits [T, hidden], the kernel's h [T, topk, inter])."""
    import torch
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    mode = 1 if prefill else 0
    T, k = ids.shape
    if ws is None:
        ws = B.workspace(B.iqk_moe_workspace_bytes(mode, T, k, gate.experts, gate.cols, gate.rows))
    fn = B.iqk_moe_prefill if prefill else B.iqk_moe_decode
    y = fn(dg, du, dd, values, to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda(), ws=ws)
    torch.cuda.synchronize()
    h = read_h(B, ws, mode, T, k, gate.experts, gate.cols, gate.rows, valid_pairs)
    return from_dev_bf16(y), h


def flat_stats(out):
    """check_block's nested statistics as one flat dict (for the parity report)."""
    r = {}
    for stage, d in out.items():
        for k, v in d.items():
            r[f"{stage}_{k}"] = v
    return r
