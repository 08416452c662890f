"""Seeded synthetic inputs for the IQ2_KS / IQ2_K routed-expert path.

This module only draws random numbers and lays them out in the stream format;
it performs none of the method's arithmetic (no field decode, no
reconstruction, no products). Both the CPU oracle (through the tests) and the
CUDA path consume what it produces.

Stream format (one logical weight tensor ``[rows, cols]`` per expert, experts
stacked on a leading axis; every stream a separate row-major, k-contiguous
plane).  Format tables: mlx-iqk 0.1.1 PKG-INFO, section "Format".

IQ2_KS (2.1875 bits per weight plus a 16-bit row scale):
  qs  uint32 [E, rows, cols/16]   weight k: word k>>4, bits 2*(k&15)..+1
  scl uint32 [E, rows, cols/256]  32-weight sub-block j=k>>5: word j>>3, nibble j&7
                                  (low 4 bits of the signed scale index)
  sch uint8  [E, rows, cols/256]  bit j&7 of byte j>>3 (high bit of the index)
  sex uint8  [E, rows, cols/256]  bit j&7 of byte j>>3 (alphabet select)
  dv  uint16 [E, rows]            fp16 row scale (bit pattern)

IQ2_K (2.375 bits per weight):
  qs  uint32 [E, rows, cols/16]   as above
  scl uint32 [E, rows, cols/128]  16-weight sub-block j=k>>4: word j>>3, nibble j&7
                                  (4-bit offset-8 signed scale index)
  sex uint16 [E, rows, cols/256]  bit j&15 of halfword j>>4 (alphabet select)
  dv  uint16 [E, rows, cols/256]  fp16 super-block scale per 256 weights
"""
from __future__ import annotations

from dataclasses import dataclass, field
from typing import Optional

import numpy as np

FORMATS = ("iq2_ks", "iq2_k")


@dataclass
class Streams:
    """Host-side streams of ``experts`` stacked ``[rows, cols]`` matrices."""

    fmt: str
    experts: int
    rows: int
    cols: int
    qs: np.ndarray
    scl: np.ndarray
    sch: Optional[np.ndarray]
    sex: np.ndarray
    dv: np.ndarray
    meta: dict = field(default_factory=dict)

    def stream_bytes_per_row(self) -> int:
        """Bytes one row occupies across all streams."""
        per_row = 0
        for a in (self.qs, self.scl, self.sch, self.sex, self.dv):
            if a is None:
                continue
            per_row += a.nbytes // (self.experts * self.rows)
        return per_row

    def expert(self, e: int) -> "Streams":
        """A one-expert view of expert ``e``."""
        sl = slice(e, e + 1)
        return Streams(self.fmt, 1, self.rows, self.cols, self.qs[sl], self.scl[sl],
                       None if self.sch is None else self.sch[sl], self.sex[sl], self.dv[sl])

    def nbytes(self) -> int:
        return sum(a.nbytes for a in (self.qs, self.scl, self.sch, self.sex, self.dv) if a is not None)


def _check(fmt: str, cols: int) -> None:
    if fmt not in FORMATS:
        raise ValueError(f"unknown format {fmt!r}")
    if cols <= 0 or cols % 256:
        raise ValueError(f"cols must be a positive multiple of 256, got {cols}")


def empty_streams(fmt: str, experts: int, rows: int, cols: int) -> Streams:
    """All-zero streams of the right shapes (for hand-built one-hot cases)."""
    _check(fmt, cols)
    E, R = experts, rows
    qs = np.zeros((E, R, cols // 16), np.uint32)
    if fmt == "iq2_ks":
        return Streams(fmt, E, R, cols, qs,
                       np.zeros((E, R, cols // 256), np.uint32),
                       np.zeros((E, R, cols // 256), np.uint8),
                       np.zeros((E, R, cols // 256), np.uint8),
                       np.zeros((E, R), np.uint16))
    return Streams(fmt, E, R, cols, qs,
                   np.zeros((E, R, cols // 128), np.uint32), None,
                   np.zeros((E, R, cols // 256), np.uint16),
                   np.zeros((E, R, cols // 256), np.uint16))


def _fp16_bits_uniform(rng: np.random.Generator, shape, lo: float, hi: float) -> np.ndarray:
    return rng.uniform(lo, hi, size=shape).astype(np.float16).view(np.uint16)


def random_streams(rng: np.random.Generator, fmt: str, experts: int, rows: int, cols: int,
                   dv_range=(1e-3, 1e-2)) -> Streams:
    """Uniform codes 0..3, uniform signed scale index over its full range,
    Bernoulli(0.5) alphabet bit and fp16 scales uniform in ``dv_range``:
    every bit of qs/scl/sch/sex is an independent fair coin."""
    _check(fmt, cols)
    E, R = experts, rows

    def words(n, dt):
        size = E * R * n * np.dtype(dt).itemsize
        return np.frombuffer(rng.bytes(size), dtype=dt).reshape(E, R, n).copy()

    qs = words(cols // 16, np.uint32)
    if fmt == "iq2_ks":
        scl = words(cols // 256, np.uint32)
        sch = words(cols // 256, np.uint8)
        sex = words(cols // 256, np.uint8)
        dv = _fp16_bits_uniform(rng, (E, R), *dv_range)
        return Streams(fmt, E, R, cols, qs, scl, sch, sex, dv)
    scl = words(cols // 128, np.uint32)
    sex = words(cols // 256, np.uint16)
    dv = _fp16_bits_uniform(rng, (E, R, cols // 256), *dv_range)
    return Streams(fmt, E, R, cols, qs, scl, None, sex, dv)


def random_bf16(rng: np.random.Generator, shape, scale: float = 1.0) -> np.ndarray:
    """bf16 bit patterns of N(0, scale^2) samples (upper half of the float32 pattern)."""
    f = (rng.standard_normal(size=shape) * scale).astype(np.float32)
    return (f.view(np.uint32) >> 16).astype(np.uint16)


def value_table(kind: str, seed: int = 0) -> np.ndarray:
    """A builder-chosen 8-entry table (entries 0-3 alphabet 0, 4-7 alphabet 1).

    ``int``: 8 distinct signed integers in [-127, 127] (fp16-exact).
    ``f16``: 8 random finite fp16 values with magnitudes in [2^-6, 2^6].
    ``dyadic``: 8 small dyadic rationals k/4, |k| <= 64 (exact in every format used).
    """
    rng = np.random.default_rng(np.random.PCG64(1000 + seed))
    if kind == "int":
        v = rng.choice(np.arange(-127, 128), size=8, replace=False)
        return v.astype(np.float32)
    if kind == "f16":
        mag = np.exp2(rng.uniform(-6, 6, size=8))
        sgn = rng.choice([-1.0, 1.0], size=8)
        return (sgn * mag).astype(np.float16).astype(np.float32)
    if kind == "dyadic":
        v = rng.choice(np.arange(-64, 65), size=8, replace=False)
        return (v / 4.0).astype(np.float32)
    raise ValueError(kind)


def routing(rng: np.random.Generator, tokens: int, experts: int, topk: int):
    """Top-k routing uniform over experts, without replacement per token;
    weights are the softmax of the selected experts' N(0,1) logits.
    Returns (ids int32 [T, topk], p float32 [T, topk])."""
    ids = np.empty((tokens, topk), np.int32)
    for t in range(tokens):
        ids[t] = rng.choice(experts, size=topk, replace=False)
    logits = rng.standard_normal(size=(tokens, topk))
    ex = np.exp(logits - logits.max(axis=1, keepdims=True))
    p = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    return ids, p


def routing_ring(rng: np.random.Generator, calls: int, experts: int, topk: int):
    """Single-token routings for ``calls`` consecutive decode calls.

    Each call's experts are ``topk`` consecutive entries of a random
    permutation of all experts (a uniformly random distinct set), so no expert
    repeats within ``experts // topk`` consecutive calls and a call never finds
    the previous calls' weights in L2. Returns (ids [calls, 1, topk], p [calls, 1, topk])."""
    per = experts // topk
    ids = np.empty((calls, 1, topk), np.int32)
    for c0 in range(0, calls, per):
        perm = rng.permutation(experts)
        for c in range(c0, min(calls, c0 + per)):
            ids[c, 0] = perm[(c - c0) * topk:(c - c0 + 1) * topk]
    logits = rng.standard_normal(size=(calls, 1, topk))
    ex = np.exp(logits - logits.max(axis=2, keepdims=True))
    p = (ex / ex.sum(axis=2, keepdims=True)).astype(np.float32)
    return ids, p


# The five workloads (routed geometry: 256 experts, top-6, gate/up
# [2048,4096], down [4096,2048]), by name; `seed` seeds each one's inputs.
HIDDEN, INTER, EXPERTS, TOPK = 4096, 2048, 256, 6

WORKLOADS = {
    "gemv_iq2_ks_256x512": dict(kind="matrix", fmt="iq2_ks", rows=256, cols=512, tokens=1, seed=0),
    "gemv_iq2_k_2048x4096": dict(kind="matrix", fmt="iq2_k", rows=2048, cols=4096, tokens=1, seed=1),
    "decode_iq2_ks_e256_top6": dict(kind="decode", fmt="iq2_ks", experts=EXPERTS, hidden=HIDDEN, inter=INTER,
                                    topk=TOPK, tokens=(1,), seed=2),
    "decode_iq2_k_e256_top6": dict(kind="decode", fmt="iq2_k", experts=EXPERTS, hidden=HIDDEN, inter=INTER,
                                   topk=TOPK, tokens=(1, 4, 16), seed=3),
    "prefill_iq2_ks_e256_top6_2048": dict(kind="prefill", fmt="iq2_ks", experts=EXPERTS, hidden=HIDDEN,
                                          inter=INTER, topk=TOPK, tokens=(2048,), seed=4),
}
MATRIX_CASES = ("gemv_iq2_ks_256x512", "gemv_iq2_k_2048x4096")


def seed_of(name: str) -> int:
    return WORKLOADS[name]["seed"]


def rng_for(seed: int) -> np.random.Generator:
    return np.random.Generator(np.random.PCG64(seed))


def matrix_case(name: str, value_kind: str = "int"):
    """A single-matrix workload (MATRIX_CASES): one matrix, one activation
    row and a value table."""
    c = WORKLOADS[name]
    rng = rng_for(c["seed"])
    w = random_streams(rng, c["fmt"], 1, c["rows"], c["cols"])
    x = random_bf16(rng, (c["tokens"], c["cols"]))
    return w, x, value_table(value_kind, c["seed"])


def moe_weights(rng: np.random.Generator, fmt: str, experts: int, hidden: int, inter: int):
    """Stacked gate [E, inter, hidden], up [E, inter, hidden], down [E, hidden, inter]."""
    gate = random_streams(rng, fmt, experts, inter, hidden)
    up = random_streams(rng, fmt, experts, inter, hidden)
    down = random_streams(rng, fmt, experts, hidden, inter)
    return gate, up, down
