"""Consecutive calls on one stream, each reading the previous call's output.

Calls launch as programmatic dependents of whatever precedes them, so call
N+1's kernels may start while call N's last kernel runs. Each kernel waits
for its predecessor before it reads anything but its parameters; here call
N+1's x is call N's y, so a kernel reading x too early would see a partial y.
The kernels are deterministic, so the chained results must equal, bit for
bit, the same calls with the stream synchronised between them (eagerly and
replayed from a CUDA graph). The first call is checked against the oracle.
"""
import numpy as np
import pytest

import iqk_synth as S
from oracle import oracle as O
from util import check_block, from_dev_bf16, read_h, run_block, to_dev_bf16

torch = pytest.importorskip("torch")
pytestmark = pytest.mark.gpu

LAYERS = 4


@pytest.fixture(scope="module")
def B():
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


@pytest.mark.parametrize("T", [1, 4, 24])
def test_chained_decode_calls_read_the_previous_output(B, T):
    """T = 24 stages x and h through the workspace (transposed by the prep
    kernel, read through L1) instead of shared memory."""
    rng = S.rng_for(800 + T)
    E, H, F, k = 32, 1024, 512, 6
    # small row scales keep four chained layers (quadratic through SwiGLU) finite and non-zero
    gate, up, down = (S.random_streams(rng, "iq2_ks", E, r, c, dv_range=(3e-4, 5e-4))
                      for r, c in ((F, H), (F, H), (H, F)))
    values = S.value_table("dyadic", 8)
    x0 = S.random_bf16(rng, (T, H))
    routes = [S.routing(rng, T, E, k) for _ in range(LAYERS)]
    dg, du, dd = (B.Weights.from_host(w) for w in (gate, up, down))
    ids = [torch.from_numpy(i).cuda() for i, _ in routes]
    ps = [torch.from_numpy(p).cuda() for _, p in routes]
    ws = B.workspace(B.iqk_moe_workspace_bytes(0, T, k, E, H, F))
    stream = torch.cuda.Stream()
    xs = [to_dev_bf16(x0)] + [torch.empty((T, H), dtype=torch.bfloat16, device="cuda") for _ in range(LAYERS)]

    def chain(sync):
        for l in range(LAYERS):
            B.iqk_moe_decode(dg, du, dd, values, xs[l], ids[l], ps[l], y=xs[l + 1], ws=ws, stream=stream)
            if sync:
                stream.synchronize()

    with torch.cuda.stream(stream):
        chain(sync=True)
    torch.cuda.synchronize()
    ref = [t.clone() for t in xs[1:]]
    # the first call against the oracle (its h from a fresh workspace)
    y0, h0 = run_block(B, gate, up, down, values, x0, routes[0][0], routes[0][1])
    assert np.array_equal(y0, from_dev_bf16(ref[0]))
    check_block(y0, h0, O.moe(gate, up, down, values, x0, routes[0][0], routes[0][1]), down, values, routes[0][0],
                routes[0][1], "layer 0")
    for l in range(LAYERS):  # every layer's output is a real signal (the comparisons below are bitwise)
        assert (ref[l].float() != 0).any(), f"layer {l} output is all zero"

    for t in xs[1:]:
        t.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        chain(sync=False)
    torch.cuda.synchronize()
    for l in range(LAYERS):
        assert torch.equal(xs[l + 1].view(torch.int16), ref[l].view(torch.int16)), f"eager chain, layer {l}"

    for t in xs[1:]:
        t.zero_()
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            chain(sync=False)
    for t in xs[1:]:
        t.zero_()
    torch.cuda.synchronize()
    for _ in range(3):
        with torch.cuda.stream(stream):
            g.replay()
    torch.cuda.synchronize()
    for l in range(LAYERS):
        assert torch.equal(xs[l + 1].view(torch.int16), ref[l].view(torch.int16)), f"graph chain, layer {l}"
    del g


def _chain_vs_sync(stream, calls, outs):
    """Run `calls` (list of zero-argument launches on `stream`) once with the
    stream synchronised after each, then back to back eagerly and from a CUDA
    graph; every output must be identical bit for bit."""
    with torch.cuda.stream(stream):
        for c in calls:
            c()
            stream.synchronize()
    torch.cuda.synchronize()
    ref = [o.clone() for o in outs]
    for o in outs:
        o.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        for c in calls:
            c()
    torch.cuda.synchronize()
    for i, (o, r) in enumerate(zip(outs, ref)):
        assert torch.equal(o, r), f"eager chain, call {i}"
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for c in calls:
                c()
    for o in outs:
        o.zero_()
    torch.cuda.synchronize()
    with torch.cuda.stream(stream):
        g.replay()
        g.replay()
    torch.cuda.synchronize()
    for i, (o, r) in enumerate(zip(outs, ref)):
        assert torch.equal(o, r), f"graph chain, call {i}"
    del g
    return ref


@pytest.mark.parametrize("T", [1, 9])
def test_chained_gemv_calls_share_one_workspace(B, T):
    """Back-to-back GEMVs of different experts on one workspace (tile
    counters and partial sums reused by every call); T = 9 reads x through
    the workspace."""
    rng = S.rng_for(900 + T)
    w = S.random_streams(rng, "iq2_k", 6, 2048, 4096)
    values = S.value_table("f16", 1)
    dw = B.Weights.from_host(w)
    xs = [to_dev_bf16(S.random_bf16(rng, (T, 4096))) for _ in range(6)]
    ys = [torch.empty((T, 2048), dtype=torch.float32, device="cuda") for _ in range(6)]
    ws = B.workspace(B.iqk_gemv_workspace_bytes(T, 2048, 4096))
    stream = torch.cuda.Stream()
    calls = [lambda e=e: B.iqk_gemv(dw, e, values, xs[e], y=ys[e], ws=ws, stream=stream) for e in range(6)]
    ref = _chain_vs_sync(stream, calls, ys)
    from tests.util import check_fp32
    y_ref, Sabs = O.gemv(O.dequant_expert(w, 2, values), from_dev_bf16(xs[2]))
    check_fp32(ref[2].cpu().numpy(), y_ref, Sabs, "chained gemv, expert 2")


@pytest.mark.parametrize("T", [1, 16])
def test_chained_switch_calls_share_one_workspace(B, T):
    """Back-to-back routed single projections on one workspace."""
    rng = S.rng_for(950 + T)
    w = S.random_streams(rng, "iq2_ks", 24, 1024, 2048)
    values = S.value_table("int", 2)
    dw = B.Weights.from_host(w)
    n = 5
    xs = [to_dev_bf16(S.random_bf16(rng, (T, 2048))) for _ in range(n)]
    ids = [torch.from_numpy(S.routing(rng, T, 24, 6)[0]).cuda() for _ in range(n)]
    ys = [torch.empty((T, 6, 1024), dtype=torch.float32, device="cuda") for _ in range(n)]
    ws = B.workspace(B.iqk_switch_linear_workspace_bytes(1, T, 6, 24, 1024, 2048))
    stream = torch.cuda.Stream()
    calls = [lambda c=c: B.iqk_switch_linear(dw, values, xs[c], ids[c], mode=1, y=ys[c], ws=ws, stream=stream)
             for c in range(n)]
    ref = _chain_vs_sync(stream, calls, ys)
    y_ref, Sabs = O.switch_linear(w, values, from_dev_bf16(xs[1]), ids[1].cpu().numpy())
    assert np.all(np.abs(ref[1].cpu().numpy() - y_ref) <= 2e-3 * Sabs + 1e-30)
