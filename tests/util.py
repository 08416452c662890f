"""Shared helpers for the parity tests (comparison rules and device upload)."""
import numpy as np

TOL = 2e-3  # stated tolerance: |y - y_ref| <= 2e-3 * sum |w x| per output


def bf16_ulp(v):
    """Spacing of bfloat16 numbers at |v| (normal range; 2^-133 below)."""
    a = np.maximum(np.abs(np.asarray(v, np.float64)), 2.0 ** -126)
    return 2.0 ** (np.floor(np.log2(a)) - 7)


def check_fp32(y, y_ref, S, what=""):
    """float32 outputs: |y - y_ref| <= 2e-3 * S. Returns the worst ratio."""
    y = np.asarray(y, np.float64)
    err = np.abs(y - y_ref)
    bound = TOL * S + 1e-30
    ratio = float(np.max(err / np.maximum(S, 1e-30)))
    bad = err > bound
    assert not bad.any(), f"{what}: {bad.sum()} outputs out of tolerance; worst err/S = {ratio:.3e}"
    return ratio


def check_bf16(y_bits, y_ref, S, what=""):
    """bf16 outputs compared after rounding: |y - y_ref| <= 2e-3 * S + 1 bf16 ulp."""
    y = (np.asarray(y_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(y - y_ref)
    bound = TOL * S + bf16_ulp(np.maximum(np.abs(y), np.abs(y_ref)))
    bad = err > bound
    ratio = float(np.max(np.maximum(err - bf16_ulp(np.maximum(np.abs(y), np.abs(y_ref))), 0) / np.maximum(S, 1e-30)))
    assert not bad.any(), f"{what}: {bad.sum()} outputs out of tolerance; worst (err-ulp)/S = {ratio:.3e}"
    return ratio


def to_dev_bf16(bits):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


def from_dev_bf16(t):
    import torch
    return t.view(torch.int16).cpu().numpy().view(np.uint16)


def check_moe(y_bits, ref, what=""):
    """Routed-block outputs. Each GEMV stage is held to the stated 2e-3 of its
    own sum |w x|; that error propagates to y through h = silu(g) u (first
    order, ref["S_prop"]), h may round to the neighbouring bfloat16
    (ref["S_round"]), and y is compared after rounding (one ulp):
        |y - y_ref| <= 2e-3 (S + S_prop) + S_round + ulp(y).
    Returns the worst error as a fraction of that bound."""
    y = (np.asarray(y_bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)
    err = np.abs(y - ref["y"])
    bound = TOL * (ref["S"] + ref["S_prop"]) + ref["S_round"] + bf16_ulp(np.maximum(np.abs(y), np.abs(ref["y"])))
    frac = float(np.max(err / bound))
    assert frac <= 1.0, f"{what}: {(err > bound).sum()} outputs out of tolerance; worst err/bound = {frac:.3f}"
    return frac
