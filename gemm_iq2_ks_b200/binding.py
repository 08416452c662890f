"""Thin Python binding of the C ABI in include/iqk.h (argument marshalling only).

Every function here has the C entry point's name and forwards device
pointers, sizes and the current CUDA stream to ``libiqk.so``; all
computation happens in the library's CUDA kernels. PyTorch provides device
memory and streams. There is no fallback: if the library cannot be loaded,
the call raises.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional, Sequence

import numpy as np

from . import build as _build

IQK_OK, IQK_EINVAL, IQK_ESHAPE, IQK_EUNSUPPORTED, IQK_ECUDA, IQK_ETIMEOUT, IQK_EWORKSPACE = 0, -1, -2, -3, -4, -5, -6
FMT = {"iq2_ks": 0, "iq2_k": 1}

EXPORTS = (
    "iqk_strerror", "iqk_last_cuda_error", "iqk_version", "iqk_row_bytes",
    "iqk_dequant", "iqk_dequant_bf16", "iqk_dequant_floor", "iqk_gemv_workspace_bytes", "iqk_gemv", "iqk_gemv_static",
    "iqk_moe_workspace_bytes", "iqk_moe_workspace_layout", "iqk_moe_decode", "iqk_moe_decode_host",
    "iqk_moe_decode_shard", "iqk_f32_to_bf16",
    "iqk_moe_prefill", "iqk_moe_prefill_shard", "iqk_moe_combine", "iqk_moe_status",
    "iqk_route_workspace_bytes", "iqk_moe_route", "iqk_floor", "iqk_floor_status", "iqk_set_wait_limit_ns",
    "iqk_switch_linear_workspace_bytes", "iqk_switch_linear", "iqk_slots_bytes", "iqk_pack_slots",
    "iqk_prefill_a_tile",
)


class IqkWsLayout(ctypes.Structure):
    _fields_ = [("status", ctypes.c_int64), ("h", ctypes.c_int64), ("h_order", ctypes.c_int64),
                ("h_rows", ctypes.c_int32), ("reserved", ctypes.c_int32)]


class IqkWeights(ctypes.Structure):
    _fields_ = [("fmt", ctypes.c_int32), ("experts", ctypes.c_int32), ("rows", ctypes.c_int32),
                ("cols", ctypes.c_int32), ("qs", ctypes.c_void_p), ("scl", ctypes.c_void_p),
                ("sch", ctypes.c_void_p), ("sex", ctypes.c_void_p), ("dv", ctypes.c_void_p),
                ("slots", ctypes.c_void_p)]


_lib = None


def library_path() -> str:
    return _build.LIB


def lib(build_if_missing: bool = True) -> ctypes.CDLL:
    """Load libiqk.so (building it in-tree first if it is missing or stale)."""
    global _lib
    if _lib is None:
        path = _build.LIB
        if build_if_missing and not _build.up_to_date():
            _build.build()
        if not os.path.exists(path):
            raise RuntimeError(f"CUDA library not built: {path}")
        L = ctypes.CDLL(path)
        vp, i32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_size_t
        W = ctypes.POINTER(IqkWeights)
        sig = {
            "iqk_strerror": (ctypes.c_char_p, [ctypes.c_int]),
            "iqk_last_cuda_error": (ctypes.c_char_p, []),
            "iqk_version": (ctypes.c_int, []),
            "iqk_row_bytes": (ctypes.c_int64, [i32, i32]),
            "iqk_dequant": (ctypes.c_int, [W, i32, vp, vp, vp]),
            "iqk_dequant_bf16": (ctypes.c_int, [W, i32, vp, vp, vp]),
            "iqk_dequant_floor": (ctypes.c_int, [W, i32, i32, vp, vp]),
            "iqk_gemv_workspace_bytes": (sz, [i32, i32, i32]),
            "iqk_gemv": (ctypes.c_int, [W, i32, vp, vp, i32, vp, vp, sz, vp]),
            "iqk_gemv_static": (ctypes.c_int, [W, i32, vp, vp, i32, vp, vp]),
            "iqk_moe_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
            "iqk_moe_workspace_layout": (ctypes.c_int, [i32, i32, i32, i32, i32, i32,
                                                        ctypes.POINTER(IqkWsLayout)]),
            "iqk_moe_decode": (ctypes.c_int, [W, W, W, vp, vp, i32, vp, vp, i32, vp, vp, sz, vp]),
            "iqk_moe_decode_host": (ctypes.c_int, [W, W, W, vp, vp, i32, vp, vp, i32, vp, vp, sz, vp]),
            "iqk_moe_decode_shard": (ctypes.c_int, [W, W, W, vp, vp, i32, vp, vp, i32, i32, vp, vp, sz, vp]),
            "iqk_f32_to_bf16": (ctypes.c_int, [vp, vp, ctypes.c_int64, vp]),
            "iqk_moe_prefill": (ctypes.c_int, [W, W, W, vp, vp, i32, vp, vp, i32, vp, vp, sz, vp]),
            "iqk_moe_prefill_shard": (ctypes.c_int, [W, W, W, vp, vp, i32, vp, vp, i32, i32, vp, vp, sz, vp]),
            "iqk_moe_combine": (ctypes.c_int, [vp, vp, i32, i32, i32, vp, vp]),
            "iqk_moe_status": (ctypes.c_int, [vp, vp]),
            "iqk_route_workspace_bytes": (sz, [i32, i32, i32]),
            "iqk_moe_route": (ctypes.c_int, [vp, i32, i32, i32, vp, vp, vp, vp, sz, vp]),
            "iqk_floor": (ctypes.c_int, [W, vp, i32, vp, vp]),
            "iqk_floor_status": (ctypes.c_int, [vp]),
            "iqk_set_wait_limit_ns": (ctypes.c_int, [ctypes.c_uint64, i32]),
            "iqk_switch_linear_workspace_bytes": (sz, [i32, i32, i32, i32, i32, i32]),
            "iqk_switch_linear": (ctypes.c_int, [W, vp, vp, i32, vp, i32, vp, i32, vp, sz, vp]),
            "iqk_slots_bytes": (sz, [W]),
            "iqk_pack_slots": (ctypes.c_int, [W, vp, sz, vp]),
            "iqk_prefill_a_tile": (ctypes.c_int, [W, i32, i32, i32, vp, vp, vp]),
        }
        for name, (res, args) in sig.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def _check(rc: int, what: str) -> None:
    if rc == IQK_OK:
        return
    L = lib()
    msg = f"{what}: {L.iqk_strerror(rc).decode()} ({rc})"
    if rc == IQK_ECUDA:
        msg += f": {L.iqk_last_cuda_error().decode()}"
    if rc in (IQK_EINVAL, IQK_ESHAPE):
        raise ValueError(msg)
    raise RuntimeError(msg)


def _torch():
    import torch
    return torch


def _stream(stream) -> ctypes.c_void_p:
    torch = _torch()
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _values(values) -> np.ndarray:
    v = np.ascontiguousarray(values, dtype=np.float32)
    if v.shape != (8,):
        raise ValueError("values must hold 8 floats")
    return v


def _ptr(t) -> Optional[int]:
    return None if t is None else t.data_ptr()


class Weights:
    """Device-resident stacked streams of one weight tensor (torch CUDA tensors)."""

    def __init__(self, fmt: str, experts: int, rows: int, cols: int, qs, scl, sch, sex, dv, slots=None):
        self.fmt, self.experts, self.rows, self.cols = fmt, experts, rows, cols
        self.qs, self.scl, self.sch, self.sex, self.dv = qs, scl, sch, sex, dv
        self.slots = slots
        self._c = IqkWeights(FMT[fmt], experts, rows, cols, _ptr(qs), _ptr(scl), _ptr(sch), _ptr(sex), _ptr(dv),
                             _ptr(slots))

    @classmethod
    def from_host(cls, s, device="cuda", pack: bool = True) -> "Weights":
        """Upload host streams (attributes fmt, experts, rows, cols, qs, scl, sch,
        sex, dv); with `pack` and a CUDA device, also their scale-slot images
        (iqk_pack_slots)."""
        torch = _torch()

        def up(a, dt):
            if a is None:
                return None
            return torch.from_numpy(np.ascontiguousarray(a).view(dt)).to(device)

        w = cls(s.fmt, s.experts, s.rows, s.cols, up(s.qs, np.int32), up(s.scl, np.int32),
                up(s.sch, np.uint8), up(s.sex, np.uint8 if s.fmt == "iq2_ks" else np.int16),
                up(s.dv, np.int16))
        return w.packed() if pack and torch.device(device).type == "cuda" else w

    def packed(self, stream=None) -> "Weights":
        """These planes with their scale-slot images (iqk_pack_slots), packed on
        `stream` and complete when this returns."""
        torch = _torch()
        plain = self.unpacked()
        n = lib().iqk_slots_bytes(ctypes.byref(plain.c))
        if n == 0:
            raise ValueError("invalid weights")
        slots = torch.empty((n,), dtype=torch.uint8, device=self.qs.device)
        st = _stream(stream)
        _check(lib().iqk_pack_slots(ctypes.byref(plain.c), slots.data_ptr(), n, st), "iqk_pack_slots")
        torch.cuda.synchronize(self.qs.device)
        return Weights(self.fmt, self.experts, self.rows, self.cols, self.qs, self.scl, self.sch, self.sex, self.dv,
                       slots)

    def unpacked(self) -> "Weights":
        """The same planes without scale-slot images (per-lane scale copies)."""
        return Weights(self.fmt, self.experts, self.rows, self.cols, self.qs, self.scl, self.sch, self.sex, self.dv)

    @property
    def c(self) -> IqkWeights:
        return self._c

    def nbytes(self) -> int:
        return sum(t.numel() * t.element_size() for t in (self.qs, self.scl, self.sch, self.sex, self.dv)
                   if t is not None)


def _empty(shape, dtype, device):
    return _torch().empty(shape, dtype=dtype, device=device)


# ------------------------------------------------------------------ entry points

def iqk_row_bytes(fmt: str, cols: int) -> int:
    return lib().iqk_row_bytes(FMT[fmt], cols)


def iqk_prefill_a_tile(w: Weights, expert: int, row0: int, nrows: int, values, out=None, stream=None):
    """The prefill producer's bf16 A operand of rows [row0, row0 + nrows) of
    one expert, in k order ([nrows, cols] bf16)."""
    torch = _torch()
    out = _empty((nrows, w.cols), torch.bfloat16, w.qs.device) if out is None else out
    v = _values(values)
    _check(lib().iqk_prefill_a_tile(ctypes.byref(w.c), expert, row0, nrows, v.ctypes.data, out.data_ptr(),
                                    _stream(stream)), "iqk_prefill_a_tile")
    return out


def iqk_dequant(w: Weights, expert: int, values, out=None, stream=None):
    torch = _torch()
    out = _empty((w.rows, w.cols), torch.float32, w.qs.device) if out is None else out
    v = _values(values)
    _check(lib().iqk_dequant(ctypes.byref(w.c), expert, v.ctypes.data, out.data_ptr(), _stream(stream)),
           "iqk_dequant")
    return out


def iqk_dequant_bf16(w: Weights, expert: int, values, out=None, stream=None):
    torch = _torch()
    out = _empty((w.rows, w.cols), torch.bfloat16, w.qs.device) if out is None else out
    v = _values(values)
    _check(lib().iqk_dequant_bf16(ctypes.byref(w.c), expert, v.ctypes.data, out.data_ptr(), _stream(stream)),
           "iqk_dequant_bf16")
    return out


def iqk_dequant_floor(w: Weights, expert: int, bf16: bool = False, out=None, stream=None):
    """The dequantizer's deleted-decode floor: int32 [rows][cols] (or
    [rows][cols/2] with bf16), the integer signature of every loaded word."""
    torch = _torch()
    out = _empty((w.rows, w.cols // 2 if bf16 else w.cols), torch.int32, w.qs.device) if out is None else out
    _check(lib().iqk_dequant_floor(ctypes.byref(w.c), expert, int(bool(bf16)), out.data_ptr(), _stream(stream)),
           "iqk_dequant_floor")
    return out


def iqk_gemv_workspace_bytes(T: int, rows: int, cols: int) -> int:
    return lib().iqk_gemv_workspace_bytes(T, rows, cols)


def workspace(nbytes: int, device="cuda"):
    """A 256-byte aligned device workspace (torch allocations are)."""
    return _empty((max(nbytes, 256),), _torch().uint8, device)


def iqk_gemv(w: Weights, expert: int, values, x, y=None, ws=None, stream=None):
    torch = _torch()
    T = x.shape[0]
    y = _empty((T, w.rows), torch.float32, x.device) if y is None else y
    need = iqk_gemv_workspace_bytes(T, w.rows, w.cols)
    ws = workspace(need, x.device) if ws is None else ws
    v = _values(values)
    _check(lib().iqk_gemv(ctypes.byref(w.c), expert, v.ctypes.data, x.data_ptr(), T, y.data_ptr(), ws.data_ptr(),
                          ws.numel(), _stream(stream)), "iqk_gemv")
    return y


def iqk_gemv_static(w: Weights, expert: int, values, x, y=None, stream=None):
    """iqk_gemv with the library's static scratch (no workspace argument)."""
    torch = _torch()
    T = x.shape[0]
    y = _empty((T, w.rows), torch.float32, x.device) if y is None else y
    v = _values(values)
    _check(lib().iqk_gemv_static(ctypes.byref(w.c), expert, v.ctypes.data, x.data_ptr(), T, y.data_ptr(),
                                 _stream(stream)), "iqk_gemv_static")
    return y


def iqk_switch_linear_workspace_bytes(mode: int, T: int, topk: int, experts: int, rows: int, cols: int) -> int:
    return lib().iqk_switch_linear_workspace_bytes(mode, T, topk, experts, rows, cols)


def iqk_switch_linear(w: Weights, values, x, ids, mode: int = 0, y=None, ws=None, stream=None):
    """y[t, j] = W_{ids[t, j]} x[t] (float32 [T, topk, rows])."""
    torch = _torch()
    T, topk = ids.shape
    y = _empty((T, topk, w.rows), torch.float32, x.device) if y is None else y
    if ws is None:
        need = iqk_switch_linear_workspace_bytes(mode, T, topk, w.experts, w.rows, w.cols)
        if need == 0:
            raise RuntimeError("iqk_switch_linear: the mode cannot take this shape")
        ws = workspace(need, x.device)
    v = _values(values)
    _check(lib().iqk_switch_linear(ctypes.byref(w.c), v.ctypes.data, x.data_ptr(), T, ids.data_ptr(), topk,
                                   y.data_ptr(), mode, ws.data_ptr(), ws.numel(), _stream(stream)),
           "iqk_switch_linear")
    return y


def iqk_moe_workspace_bytes(mode: int, T: int, topk: int, experts: int, hidden: int, inter: int) -> int:
    return lib().iqk_moe_workspace_bytes(mode, T, topk, experts, hidden, inter)


def iqk_moe_workspace_layout(mode: int, T: int, topk: int, experts: int, hidden: int, inter: int) -> IqkWsLayout:
    out = IqkWsLayout()
    _check(lib().iqk_moe_workspace_layout(mode, T, topk, experts, hidden, inter, ctypes.byref(out)),
           "iqk_moe_workspace_layout")
    return out


def _moe(fn, mode, gate, up, down, values, x, ids, p, y, ws, stream):
    torch = _torch()
    T, topk = ids.shape
    y = _empty((T, down.rows), torch.bfloat16, x.device) if y is None else y
    need = iqk_moe_workspace_bytes(mode, T, topk, gate.experts, gate.cols, gate.rows)
    if need == 0:
        raise ValueError("unsupported token count / topk for this call")
    ws = workspace(need, x.device) if ws is None else ws
    v = _values(values)
    _check(fn(ctypes.byref(gate.c), ctypes.byref(up.c), ctypes.byref(down.c), v.ctypes.data, x.data_ptr(), T,
              ids.data_ptr(), p.data_ptr(), topk, y.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           fn.__name__)
    return y


def iqk_moe_decode(gate: Weights, up: Weights, down: Weights, values, x, ids, p, y=None, ws=None, stream=None):
    return _moe(lib().iqk_moe_decode, 0, gate, up, down, values, x, ids, p, y, ws, stream)


def iqk_moe_decode_host(gate: Weights, up: Weights, down: Weights, values, x, ids, p, y=None, ws=None, stream=None):
    """iqk_moe_decode on page-locked host tensors (x, ids, p and y pinned CPU
    tensors); the call's kernels read the inputs and write y over the host
    link. y is complete once the stream has passed the call. The workspace is
    device memory on the current device."""
    torch = _torch()
    T, topk = ids.shape
    if y is None:
        y = torch.empty((T, down.rows), dtype=torch.bfloat16, pin_memory=True)
    if ws is None:
        ws = workspace(iqk_moe_workspace_bytes(0, T, topk, gate.experts, gate.cols, gate.rows),
                       torch.device("cuda", torch.cuda.current_device()))
    v = _values(values)
    _check(lib().iqk_moe_decode_host(ctypes.byref(gate.c), ctypes.byref(up.c), ctypes.byref(down.c), v.ctypes.data,
                                     x.data_ptr(), T, ids.data_ptr(), p.data_ptr(), topk, y.data_ptr(),
                                     ws.data_ptr(), ws.numel(), _stream(stream)),
           "iqk_moe_decode_host")
    return y


def iqk_moe_prefill(gate: Weights, up: Weights, down: Weights, values, x, ids, p, y=None, ws=None, stream=None):
    return _moe(lib().iqk_moe_prefill, 1, gate, up, down, values, x, ids, p, y, ws, stream)


def iqk_moe_decode_shard(gate: Weights, up: Weights, down: Weights, values, x, ids, p, expert_base: int,
                         y=None, ws=None, stream=None):
    """One expert-parallel rank's float32 partial [T, hidden] (its experts
    [expert_base, expert_base + gate.experts); other ids skipped)."""
    torch = _torch()
    T, topk = ids.shape
    y = _empty((T, down.rows), torch.float32, x.device) if y is None else y
    if ws is None:
        ws = workspace(iqk_moe_workspace_bytes(0, T, topk, gate.experts, gate.cols, gate.rows), x.device)
    v = _values(values)
    _check(lib().iqk_moe_decode_shard(ctypes.byref(gate.c), ctypes.byref(up.c), ctypes.byref(down.c), v.ctypes.data,
                                      x.data_ptr(), T, ids.data_ptr(), p.data_ptr(), topk, expert_base,
                                      y.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           "iqk_moe_decode_shard")
    return y


def iqk_moe_prefill_shard(gate: Weights, up: Weights, down: Weights, values, x, ids, p, expert_base: int,
                          y=None, ws=None, stream=None):
    """One expert-parallel rank's float32 prefill partial [T, hidden]."""
    torch = _torch()
    T, topk = ids.shape
    y = _empty((T, down.rows), torch.float32, x.device) if y is None else y
    if ws is None:
        ws = workspace(iqk_moe_workspace_bytes(1, T, topk, gate.experts, gate.cols, gate.rows), x.device)
    v = _values(values)
    _check(lib().iqk_moe_prefill_shard(ctypes.byref(gate.c), ctypes.byref(up.c), ctypes.byref(down.c),
                                       v.ctypes.data, x.data_ptr(), T, ids.data_ptr(), p.data_ptr(), topk,
                                       expert_base, y.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)),
           "iqk_moe_prefill_shard")
    return y


def iqk_moe_combine(rows, p, y=None, stream=None):
    """y[t] = bf16(sum_j p[t, j] rows[t * topk + j]) in slot order."""
    torch = _torch()
    T, topk = p.shape
    H = rows.shape[-1]
    y = _empty((T, H), torch.bfloat16, rows.device) if y is None else y
    _check(lib().iqk_moe_combine(rows.data_ptr(), p.data_ptr(), T, topk, H, y.data_ptr(), _stream(stream)),
           "iqk_moe_combine")
    return y


def iqk_f32_to_bf16(x, out=None, stream=None):
    torch = _torch()
    out = _empty(tuple(x.shape), torch.bfloat16, x.device) if out is None else out
    _check(lib().iqk_f32_to_bf16(x.data_ptr(), out.data_ptr(), x.numel(), _stream(stream)), "iqk_f32_to_bf16")
    return out


def iqk_moe_status(ws, stream=None) -> int:
    return lib().iqk_moe_status(ws.data_ptr(), _stream(stream))


def iqk_route_workspace_bytes(T: int, topk: int, experts: int) -> int:
    return lib().iqk_route_workspace_bytes(T, topk, experts)


def iqk_moe_route(ids, experts: int, ws=None, stream=None):
    torch = _torch()
    T, topk = ids.shape
    dev = ids.device
    counts = _empty((experts,), torch.int32, dev)
    offsets = _empty((experts + 1,), torch.int32, dev)
    perm = torch.full((T * topk,), -1, dtype=torch.int32, device=dev)
    ws = workspace(iqk_route_workspace_bytes(T, topk, experts), dev) if ws is None else ws
    _check(lib().iqk_moe_route(ids.data_ptr(), T, topk, experts, counts.data_ptr(), offsets.data_ptr(),
                               perm.data_ptr(), ws.data_ptr(), ws.numel(), _stream(stream)), "iqk_moe_route")
    return counts, offsets, perm, ws


def iqk_floor(w: Weights, expert_list, out=None, stream=None):
    torch = _torch()
    n = expert_list.numel()
    out = _empty((n, w.rows), torch.int32, expert_list.device) if out is None else out
    _check(lib().iqk_floor(ctypes.byref(w.c), expert_list.data_ptr(), n, out.data_ptr(), _stream(stream)),
           "iqk_floor")
    return out


def iqk_floor_status(stream=None) -> int:
    return lib().iqk_floor_status(_stream(stream))


def iqk_set_wait_limit_ns(limit_ns: int, expire: bool = False) -> int:
    return lib().iqk_set_wait_limit_ns(int(limit_ns), int(bool(expire)))


# --------------------------------------------------------------- module form

class IqkSwitchLinear:
    """The switch-linear projection of the mlx-iqk 0.1.1 page (section
    "Surface"): ``proj = IqkSwitchLinear(member, num_experts, out_features,
    in_features, values)``, ``proj.load_streams(streams)``, ``y = proj(x,
    indices)`` with ``y[..., j, :] = W_{indices[..., j]} x[...]``.

    The member (``"iq2_ks"`` or ``"iq2_k"``) is fixed per instance, so the
    projections of one layer can carry different members. ``values`` is the
    8-entry value table (entries 0-3 alphabet 0, 4-7 alphabet 1); the page
    does not print it, so it is an argument. Every call goes through
    ``iqk_switch_linear``: its auto mode runs the decode kernel for few
    (token, slot) pairs and the grouped GEMM for many. Both group the pairs by
    expert on the device, so each expert's weights are read once per call
    whatever ``sorted_indices`` says; the flag is accepted for interface
    parity and changes nothing.

    Errors: widths that are not a positive multiple of 256 and mismatched
    streams raise ValueError before any launch; a shape the kernels do not
    take raises RuntimeError. Ids outside [0, num_experts) give zero rows and
    make ``status()`` report IQK_EINVAL.

    Each (mode, shape, stream) gets its own workspace, so calls on different
    streams never share scratch; ``status()`` reports the last call made
    through this instance.
    """

    def __init__(self, member: str, num_experts: int, out_features: int, in_features: int, values,
                 device="cuda"):
        if member not in FMT:
            raise ValueError(f"unknown member {member!r} (expected one of {sorted(FMT)})")
        if in_features <= 0 or in_features % 256:
            raise ValueError(f"in_features {in_features} is not a positive multiple of 256")
        if out_features <= 0 or num_experts <= 0:
            raise ValueError("out_features and num_experts must be positive")
        self.member, self.num_experts = member, num_experts
        self.out_features, self.in_features = out_features, in_features
        self.values = _values(values)
        self.device = device
        self.weights: Optional[Weights] = None
        self._ws = {}
        self._last_ws = None

    def load_streams(self, streams) -> "IqkSwitchLinear":
        """Take host streams (fmt, experts, rows, cols and the five planes) or
        device ``Weights``; their member and shape must match the instance."""
        got = (streams.fmt, streams.experts, streams.rows, streams.cols)
        want = (self.member, self.num_experts, self.out_features, self.in_features)
        if got != want:
            raise ValueError(f"streams are {got}, the projection is {want}")
        self.weights = streams if isinstance(streams, Weights) else Weights.from_host(streams, self.device)
        return self

    def __call__(self, x, indices, sorted_indices: bool = False, mode: int = 0, stream=None):
        if self.weights is None:
            raise RuntimeError("IqkSwitchLinear: load_streams() first")
        torch = _torch()
        if x.dtype != torch.bfloat16 or x.shape[-1] != self.in_features:
            raise ValueError(f"x must be bfloat16 [..., {self.in_features}]")
        if indices.shape[:-1] != x.shape[:-1]:
            raise ValueError("indices must be [..., k] over the same leading shape as x")
        lead, k = tuple(x.shape[:-1]), indices.shape[-1]
        xt = x.reshape(-1, self.in_features).contiguous()
        ids = indices.reshape(-1, k).to(torch.int32).contiguous()
        T = xt.shape[0]
        st = torch.cuda.current_stream(x.device) if stream is None else stream
        key = (mode, T, k, st.cuda_stream)
        ws = self._ws.get(key)
        if ws is None:
            need = iqk_switch_linear_workspace_bytes(mode, T, k, self.num_experts, self.out_features,
                                                     self.in_features)
            if need == 0:
                raise RuntimeError(f"IqkSwitchLinear: mode {mode} cannot take {T} tokens x {k} slots")
            ws = self._ws[key] = workspace(need, x.device)
        self._last_ws = (ws, st)
        y = iqk_switch_linear(self.weights, self.values, xt, ids, mode=mode, ws=ws, stream=st)
        return y.reshape(*lead, k, self.out_features)

    def status(self, stream=None) -> int:
        """Status of the last call as iqk_moe_status reports it: IQK_OK,
        IQK_EINVAL (an id was out of range), IQK_EUNSUPPORTED or IQK_ETIMEOUT."""
        if self._last_ws is None:
            return 0
        ws, st = self._last_ws
        return iqk_moe_status(ws, st if stream is None else stream)
