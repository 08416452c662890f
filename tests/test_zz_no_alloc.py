"""iqk_gemv_static: the GEMV with the library's static scratch array.

Collected last (file name), so the GPU test also runs after every other test
has used the library in the same process.
"""
import ctypes

import numpy as np
import pytest

import iqk_synth as S
from gemm_iq2_ks_b200 import binding as B
from oracle import oracle as O
from util import check_fp32, to_dev_bf16


def test_static_scratch_limit_is_refused_on_the_host():
    """A shape whose scratch exceeds the static array returns IQK_EWORKSPACE
    before touching the device (fake device pointers are never read)."""
    L = B.lib()
    v = np.zeros(8, np.float32)
    w = B.IqkWeights(0, 1, 16384, 16384, 4096, 4096, 4096, 4096, 4096)
    assert B.iqk_gemv_workspace_bytes(64, 16384, 16384) > (4 << 20)
    assert L.iqk_gemv_static(ctypes.byref(w), 0, v.ctypes.data, 4096, 64, 4096, None) == B.IQK_EWORKSPACE
    assert L.iqk_gemv_static(ctypes.byref(w), 0, v.ctypes.data, 4098, 1, 4096, None) == B.IQK_EINVAL  # x misaligned
    assert L.iqk_gemv_static(ctypes.byref(w), 0, v.ctypes.data, 4096, 65, 4096, None) == B.IQK_EUNSUPPORTED


@pytest.mark.gpu
@pytest.mark.parametrize("case,T", [(S.MATRIX_CASES[0], 1), (S.MATRIX_CASES[1], 1), (S.MATRIX_CASES[1], 3)])
def test_static_matches_workspace_gemv_twice(case, T):
    w, x, values = S.matrix_case(case)
    if T > 1:
        x = np.concatenate([x, S.random_bf16(S.rng_for(300 + T), (T - 1, w.cols))])
    dw = B.Weights.from_host(w)
    xd = to_dev_bf16(x)
    y_ws = B.iqk_gemv(dw, 0, values, xd).cpu().numpy().astype(np.float64)
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 0, values), x)
    for k in range(2):  # two calls in a row reuse the same scratch
        y_st = B.iqk_gemv_static(dw, 0, values, xd).cpu().numpy()
        # against the workspace entry point, within the stated tolerance ...
        check_fp32(y_st, y_ws, Sabs, f"static gemv vs iqk_gemv, {case} T={T} call {k}")
        # ... and against the oracle
        check_fp32(y_st, y_ref, Sabs, f"static gemv vs oracle, {case} T={T} call {k}")
