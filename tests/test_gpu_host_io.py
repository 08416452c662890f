"""iqk_moe_decode_host: x, ids, p and y in page-locked host memory.

The call's own kernels move the data: the prep kernel reads each input byte
once over the host link into the workspace, the tile kernels read those
copies, and the down kernel writes y to host memory. The kernels and their
arithmetic are those of iqk_moe_decode, so the results must equal, bit for
bit, the same call on device tensors (itself checked against the oracle in
test_gpu_decode.py): y, and the status word. T = 1 stages x rows in shared
memory with per-run readiness; T = 4 stages x rows in shared memory without
it; T = 8 reads x through the prep kernel's transposed copy.
"""
import numpy as np
import pytest

import iqk_synth as S
from util import to_dev_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

E, H, F, K = 32, 4096, 2048, 6


@pytest.fixture(scope="module")
def B():
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


@pytest.fixture(scope="module")
def weights(B):
    rng = S.rng_for(950)
    g, u, d = (S.random_streams(rng, "iq2_ks", E, r, c) for r, c in ((F, H), (F, H), (H, F)))
    return [B.Weights.from_host(w) for w in (g, u, d)]


def _pinned(a, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.view(dtype)
    return t.pin_memory()


def _inputs(seed, T):
    rng = S.rng_for(seed)
    x = S.random_bf16(rng, (T, H))
    ids, p = S.routing(rng, T, E, K)
    return x, ids, p


def _device_call(B, weights, values, x, ids, p):
    g, u, d = weights
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, x.shape[0], K, E, H, F))
    y = B.iqk_moe_decode(g, u, d, values, to_dev_bf16(x), torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda(),
                         ws=ws)
    torch.cuda.synchronize()
    return y.cpu().view(torch.int16).numpy(), B.iqk_moe_status(ws)


@pytest.mark.parametrize("T", [1, 4, 8])
def test_host_io_equals_device_call(B, weights, T):
    values = S.value_table("int", 9)
    x, ids, p = _inputs(960 + T, T)
    if T == 8:
        ids[3, 2] = E + 5  # an id outside [0, E): flagged, its slot skipped
    want, want_status = _device_call(B, weights, values, x, ids, p)
    g, u, d = weights
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, T, K, E, H, F))
    hx, hids, hp = _pinned(x.view(np.int16), torch.bfloat16), _pinned(ids), _pinned(p)
    hy = torch.full((T, H), -1, dtype=torch.int16).pin_memory()
    B.iqk_moe_decode_host(g, u, d, values, hx, hids, hp, y=hy.view(torch.bfloat16), ws=ws)
    torch.cuda.synchronize()
    assert np.array_equal(hy.numpy(), want), f"T={T}"
    assert B.iqk_moe_status(ws) == want_status
    assert want_status == (B.IQK_EINVAL if T == 8 else B.IQK_OK)


def test_host_io_chained_calls_on_one_workspace(B, weights):
    """Three calls back to back on one stream and one workspace, no
    synchronisation between them: each call's prep kernel rewrites the
    staged inputs only after the previous call's kernels are done."""
    values = S.value_table("f16", 9)
    g, u, d = weights
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, 1, K, E, H, F))
    cases, outs, keep = [], [], []  # the pinned inputs stay alive until the stream has passed the calls
    for c in range(3):
        x, ids, p = _inputs(970 + c, 1)
        cases.append((x, ids, p))
        hin = (_pinned(x.view(np.int16), torch.bfloat16), _pinned(ids), _pinned(p))
        keep.append(hin)
        hy = torch.zeros((1, H), dtype=torch.int16).pin_memory()
        B.iqk_moe_decode_host(g, u, d, values, *hin, y=hy.view(torch.bfloat16), ws=ws)
        outs.append(hy)
    torch.cuda.synchronize()
    for (x, ids, p), hy in zip(cases, outs):
        want, _ = _device_call(B, weights, values, x, ids, p)
        assert np.array_equal(hy.numpy(), want)


def test_host_io_output_feeds_the_next_call(B):
    """Four layers chained through host memory, no synchronisation: call
    N+1's x is call N's y. Each call's prep kernel reads x only after the
    previous call's kernels have completed, so the chain must equal, bit for
    bit, the same chain through device tensors."""
    rng = S.rng_for(990)
    # small row scales keep four chained layers (quadratic through SwiGLU) finite and non-zero
    g, u, d = (B.Weights.from_host(S.random_streams(rng, "iq2_ks", E, r, c, dv_range=(3e-4, 5e-4)))
               for r, c in ((F, H), (F, H), (H, F)))
    values = S.value_table("dyadic", 8)
    layers = 4
    x0 = S.random_bf16(rng, (1, H))
    routes = [S.routing(rng, 1, E, K) for _ in range(layers)]
    ws_d = B.workspace(B.iqk_moe_workspace_bytes(0, 1, K, E, H, F))
    xd = to_dev_bf16(x0)
    want = []
    for ids, p in routes:
        xd = B.iqk_moe_decode(g, u, d, values, xd, torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda(), ws=ws_d)
        want.append(xd.cpu().view(torch.int16).numpy())
    torch.cuda.synchronize()
    ws_h = B.workspace(B.iqk_moe_workspace_bytes(0, 1, K, E, H, F))
    hx = _pinned(x0.view(np.int16), torch.bfloat16)
    keep, outs = [hx], []
    for ids, p in routes:
        hids, hp = _pinned(ids), _pinned(p)
        hy = torch.zeros((1, H), dtype=torch.int16).pin_memory()
        B.iqk_moe_decode_host(g, u, d, values, hx, hids, hp, y=hy.view(torch.bfloat16), ws=ws_h)
        keep += [hids, hp, hy]
        outs.append(hy)
        hx = hy.view(torch.bfloat16)
    torch.cuda.synchronize()
    for n, (hy, w) in enumerate(zip(outs, want)):
        assert np.array_equal(hy.numpy(), w), f"layer {n}"
    assert np.any(want[-1] != 0)


def test_host_io_rejects_other_memory(B, weights):
    values = S.value_table("int", 9)
    g, u, d = weights
    x, ids, p = _inputs(980, 1)
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, 1, K, E, H, F))
    hy = torch.zeros((1, H), dtype=torch.bfloat16).pin_memory()
    pageable_x = torch.from_numpy(x.view(np.int16)).view(torch.bfloat16)  # not page-locked
    with pytest.raises(ValueError):
        B.iqk_moe_decode_host(g, u, d, values, pageable_x, _pinned(ids), _pinned(p), y=hy, ws=ws)
    with pytest.raises(ValueError):  # device tensors belong to iqk_moe_decode
        B.iqk_moe_decode_host(g, u, d, values, to_dev_bf16(x), _pinned(ids), _pinned(p), y=hy, ws=ws)
