"""The C-ABI library loads, exports every declared entry point and rejects bad
arguments on the host before touching a GPU (no compute calls here)."""
import ctypes
import os
import re

import numpy as np
import pytest

from gemm_iq2_ks_b200 import binding as B

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    src = open(os.path.join(ROOT, "include", "iqk.h")).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(iqk_[a-z0-9_]+)\s*\(", src)))


def test_header_declares_the_binding_exports():
    assert set(declared_symbols()) == set(B.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = B.lib()
    for name in declared_symbols():
        assert hasattr(L, name), name


def test_row_bytes_and_version():
    L = B.lib()
    assert L.iqk_version() == 2
    assert L.iqk_row_bytes(0, 4096) == 2 + 70 * 4096 // 256
    assert L.iqk_row_bytes(1, 2048) == 76 * 2048 // 256
    assert L.iqk_row_bytes(0, 100) == -1
    assert L.iqk_row_bytes(7, 256) == -1


def _w(fmt=0, experts=1, rows=16, cols=256, sch=True, slots=None):
    return B.IqkWeights(fmt, experts, rows, cols, 4096, 4096, 4096 if sch else None, 4096, 4096, slots)


def test_slot_image_sizes_and_checks():
    """One image per (expert, 16-row tile, slice) of the decode kernels'
    slice width: IQ2_KS 64*bpi + 160 bytes, IQ2_K 192*bpi bytes, with bpi
    4 blocks at 4096 columns and 2 at 2048 (4 slices per row either way)."""
    L = B.lib()
    w = _w(fmt=0, experts=2, rows=2048, cols=4096)
    assert L.iqk_slots_bytes(ctypes.byref(w)) == 2 * 128 * 4 * (64 * 4 + 160)
    w = _w(fmt=1, experts=1, rows=4096, cols=2048, sch=False)
    assert L.iqk_slots_bytes(ctypes.byref(w)) == 256 * 4 * (192 * 2)
    w = _w(fmt=0, experts=3, rows=20, cols=512)  # ragged last tile; 2 blocks per row, bpi 2, one slice
    assert L.iqk_slots_bytes(ctypes.byref(w)) == 3 * 2 * 1 * (64 * 2 + 160)
    assert L.iqk_slots_bytes(ctypes.byref(_w(cols=100))) == 0
    w = _w(fmt=0, experts=1, rows=16, cols=256)
    n = L.iqk_slots_bytes(ctypes.byref(w))
    assert L.iqk_pack_slots(ctypes.byref(w), 4096 + 8, n, None) == B.IQK_EWORKSPACE  # misaligned
    assert L.iqk_pack_slots(ctypes.byref(w), 4096, n - 16, None) == B.IQK_EWORKSPACE  # too small
    assert L.iqk_pack_slots(ctypes.byref(w), None, n, None) == B.IQK_EWORKSPACE
    v = np.zeros(8, np.float32)
    w = _w(slots=4096 + 4)  # images must be 16-byte aligned
    assert L.iqk_dequant(ctypes.byref(w), 0, v.ctypes.data, 4096, None) == B.IQK_EINVAL


def test_host_validation_rejects_before_any_launch():
    L = B.lib()
    v = np.zeros(8, np.float32)
    P = v.ctypes.data
    bad = [
        (_w(cols=100), B.IQK_ESHAPE),
        (_w(cols=0), B.IQK_ESHAPE),
        (_w(rows=0), B.IQK_ESHAPE),
        (_w(fmt=5), B.IQK_EINVAL),
        (_w(fmt=1, sch=True), B.IQK_EINVAL),   # IQ2_K takes no sch plane
        (_w(fmt=0, sch=False), B.IQK_EINVAL),  # IQ2_KS needs it
    ]
    for w, rc in bad:
        assert L.iqk_dequant(ctypes.byref(w), 0, P, 4096, None) == rc
    w = _w()
    assert L.iqk_dequant(ctypes.byref(w), 1, P, 4096, None) == B.IQK_EINVAL  # expert out of range
    assert L.iqk_dequant(ctypes.byref(w), 0, None, 4096, None) == B.IQK_EINVAL  # no table
    assert L.iqk_dequant(None, 0, P, 4096, None) == B.IQK_EINVAL
    # dequantizer floor: same checks, no table
    assert L.iqk_dequant_floor(ctypes.byref(_w(cols=100)), 0, 0, 4096, None) == B.IQK_ESHAPE
    assert L.iqk_dequant_floor(ctypes.byref(w), 1, 0, 4096, None) == B.IQK_EINVAL  # expert out of range
    assert L.iqk_dequant_floor(ctypes.byref(w), 0, 1, None, None) == B.IQK_EINVAL  # no output
    assert L.iqk_dequant_floor(ctypes.byref(w), 0, 0, 4100, None) == B.IQK_EINVAL  # output misaligned
    # gemv: token count and workspace
    assert L.iqk_gemv(ctypes.byref(w), 0, P, 4096, 65, 4096, 4096, 1 << 20, None) == B.IQK_EUNSUPPORTED
    assert L.iqk_gemv(ctypes.byref(w), 0, P, 4096, 1, 4096, None, 0, None) == B.IQK_EWORKSPACE
    assert L.iqk_gemv(ctypes.byref(w), 0, P, 4096, 1, 4096, 4097, 1 << 20, None) == B.IQK_EWORKSPACE
    assert L.iqk_gemv(ctypes.byref(w), 0, P, 4098, 1, 4096, 4096, 1 << 20, None) == B.IQK_EINVAL  # x misaligned


def test_moe_shape_checks():
    L = B.lib()
    v = np.zeros(8, np.float32).ctypes.data
    g = _w(experts=4, rows=512, cols=256)
    u = _w(experts=4, rows=512, cols=256)
    d = _w(experts=4, rows=256, cols=512)
    d_bad = _w(experts=4, rows=256, cols=768)
    e_bad = _w(experts=3, rows=256, cols=512)
    args = lambda dd, T=1, k=6: (ctypes.byref(g), ctypes.byref(u), ctypes.byref(dd), v, 4096, T, 4096, 4096, k,
                                 4096, None, 0, None)
    assert L.iqk_moe_decode(*args(d_bad)) == B.IQK_EINVAL
    assert L.iqk_moe_decode(*args(e_bad)) == B.IQK_EINVAL
    assert L.iqk_moe_decode(*args(d, k=17)) == B.IQK_EINVAL
    assert L.iqk_moe_decode(*args(d, T=65)) == B.IQK_EUNSUPPORTED
    assert L.iqk_moe_decode(*args(d, T=0)) == B.IQK_OK  # empty call is a no-op
    assert L.iqk_moe_decode(*args(d)) == B.IQK_EWORKSPACE
    assert L.iqk_moe_prefill(*args(d, T=70000)) == B.IQK_EUNSUPPORTED
    assert L.iqk_moe_workspace_bytes(0, 65, 6, 4, 256, 512) == 0
    assert L.iqk_moe_workspace_bytes(0, 1, 6, 4, 256, 512) > 0
    # the expert-parallel shard: same checks, plus a non-negative expert base
    sargs = lambda dd, T=1, k=6, base=0, ws=None: (ctypes.byref(g), ctypes.byref(u), ctypes.byref(dd), v, 4096, T,
                                                   4096, 4096, k, base, 4096, ws, 0, None)
    assert L.iqk_moe_decode_shard(*sargs(d_bad)) == B.IQK_EINVAL
    assert L.iqk_moe_decode_shard(*sargs(d, base=-1)) == B.IQK_EINVAL
    assert L.iqk_moe_decode_shard(*sargs(d, T=65)) == B.IQK_EUNSUPPORTED
    assert L.iqk_moe_decode_shard(*sargs(d, T=0)) == B.IQK_OK
    assert L.iqk_moe_decode_shard(*sargs(d)) == B.IQK_EWORKSPACE
    assert L.iqk_f32_to_bf16(None, None, 0, None) == B.IQK_OK
    assert L.iqk_f32_to_bf16(None, 4096, 8, None) == B.IQK_EINVAL
    assert L.iqk_f32_to_bf16(4096, 4096, -1, None) == B.IQK_EINVAL


def test_switch_linear_mode_checks():
    L = B.lib()
    v = np.zeros(8, np.float32).ctypes.data
    w = _w(experts=4, rows=200, cols=512)   # rows not a multiple of 256: no grouped GEMM
    assert L.iqk_switch_linear_workspace_bytes(2, 4, 2, 4, 200, 512) == 0
    assert L.iqk_switch_linear_workspace_bytes(1, 4, 2, 4, 200, 512) > 0
    assert L.iqk_switch_linear_workspace_bytes(1, 65, 2, 4, 200, 512) == 0
    assert L.iqk_switch_linear(ctypes.byref(w), v, 4096, 4, 4096, 2, 4096, 2, 4096, 1 << 20, None) == B.IQK_EUNSUPPORTED
    assert L.iqk_switch_linear(ctypes.byref(w), v, 4096, 4, 4096, 2, 4096, 7, 4096, 1 << 20, None) == B.IQK_EINVAL
    assert L.iqk_switch_linear(ctypes.byref(w), v, 4096, 4, 4096, 17, 4096, 1, 4096, 1 << 20, None) == B.IQK_EINVAL
    assert L.iqk_switch_linear(ctypes.byref(w), v, 4096, 4, 4096, 2, 4096, 1, None, 0, None) == B.IQK_EWORKSPACE
    assert L.iqk_switch_linear(ctypes.byref(w), v, 4096, 0, 4096, 2, 4096, 1, None, 0, None) == B.IQK_OK


def test_strerror_covers_every_status():
    L = B.lib()
    for rc in range(0, -7, -1):
        assert L.iqk_strerror(rc) not in (b"", b"unknown status")
    assert L.iqk_strerror(-99) == b"unknown status"


def test_workspace_layout_inside_the_workspace():
    """The intermediates' offsets lie inside the workspace the same call
    needs, aligned, and the layout refuses shapes the mode cannot take."""
    for mode, T, k, E, H, F in [(0, 1, 6, 256, 4096, 2048), (0, 64, 16, 40, 256, 512), (1, 2048, 6, 256, 4096, 2048),
                                (1, 5, 3, 8, 256, 256)]:
        need = B.iqk_moe_workspace_bytes(mode, T, k, E, H, F)
        L = B.iqk_moe_workspace_layout(mode, T, k, E, H, F)
        assert L.h_rows == T * k
        assert L.status == 0
        assert L.h % 256 == 0 and L.h + L.h_rows * F * 2 <= need
        if mode == 0:
            assert L.h_order == -1
        else:
            assert L.h_order % 256 == 0 and L.h_order + T * k * 4 <= need
            assert not (L.h_order < L.h + L.h_rows * F * 2 and L.h < L.h_order + T * k * 4)
    lib = B.lib()
    out = B.IqkWsLayout()
    assert lib.iqk_moe_workspace_layout(0, 65, 6, 4, 256, 512, ctypes.byref(out)) == B.IQK_EINVAL
    assert lib.iqk_moe_workspace_layout(2, 1, 6, 4, 256, 512, ctypes.byref(out)) == B.IQK_EINVAL
    assert lib.iqk_moe_workspace_layout(0, 1, 6, 4, 256, 512, None) == B.IQK_EINVAL
