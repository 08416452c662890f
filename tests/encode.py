"""Test-side encoder: per-weight fields -> stream planes (the inverse of decoding).

Used to pin the oracle's bit addressing by round trip: a decoder that reads a
field from the wrong bits cannot reproduce fields this encoder wrote, unless
the encoder makes the mirror-image mistake (which the one-hot position tests
rule out separately).
"""
import numpy as np

from iqk_synth import Streams


def encode(fmt, codes, idx, alpha, d_bits):
    """codes int [rows, cols] in 0..3; idx int [rows, nsub]; alpha int [rows, nsub];
    d_bits uint16 [rows] (IQ2_KS) or [rows, cols/256] (IQ2_K). Single expert."""
    rows, cols = codes.shape
    qs = np.zeros((rows, cols // 16), np.uint64)
    for k in range(cols):
        qs[:, k >> 4] |= codes[:, k].astype(np.uint64) << np.uint64(2 * (k & 15))
    qs = qs.astype(np.uint32)
    if fmt == "iq2_ks":
        nsub = cols // 32
        assert idx.shape == (rows, nsub)
        biased = idx + 16
        assert biased.min() >= 0 and biased.max() < 32
        scl = np.zeros((rows, cols // 256), np.uint64)
        sch = np.zeros((rows, cols // 256), np.uint64)
        sex = np.zeros((rows, cols // 256), np.uint64)
        for j in range(nsub):
            scl[:, j >> 3] |= (biased[:, j] & 15).astype(np.uint64) << np.uint64(4 * (j & 7))
            sch[:, j >> 3] |= (biased[:, j] >> 4).astype(np.uint64) << np.uint64(j & 7)
            sex[:, j >> 3] |= alpha[:, j].astype(np.uint64) << np.uint64(j & 7)
        return Streams(fmt, 1, rows, cols, qs[None], scl.astype(np.uint32)[None],
                       sch.astype(np.uint8)[None], sex.astype(np.uint8)[None],
                       np.asarray(d_bits, np.uint16).reshape(rows)[None])
    nsub = cols // 16
    assert idx.shape == (rows, nsub)
    biased = idx + 8
    assert biased.min() >= 0 and biased.max() < 16
    scl = np.zeros((rows, cols // 128), np.uint64)
    sex = np.zeros((rows, cols // 256), np.uint64)
    for j in range(nsub):
        scl[:, j >> 3] |= biased[:, j].astype(np.uint64) << np.uint64(4 * (j & 7))
        sex[:, j >> 4] |= alpha[:, j].astype(np.uint64) << np.uint64(j & 15)
    return Streams(fmt, 1, rows, cols, qs[None], scl.astype(np.uint32)[None], None,
                   sex.astype(np.uint16)[None],
                   np.asarray(d_bits, np.uint16).reshape(rows, cols // 256)[None])


def sub_size(fmt):
    return 32 if fmt == "iq2_ks" else 16


def idx_range(fmt):
    return (-16, 15) if fmt == "iq2_ks" else (-8, 7)
