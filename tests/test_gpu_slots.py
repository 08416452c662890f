"""The decode paths read an item's scales either from the planes (per-lane
copies) or from the scale-slot images (one bulk copy). The images hold the
planes' bytes, so both paths compute the same arithmetic on the same values:
their outputs must agree bit for bit. (Each path is also checked against the
oracle by the parity tests; the binding packs images by default.)"""
import numpy as np
import pytest

import iqk_synth as S

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")


@pytest.fixture(scope="module")
def B():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from gemm_iq2_ks_b200 import binding
    binding.lib()
    return binding


def _both(B, host):
    w = B.Weights.from_host(host, pack=False)
    return w, w.packed()


def _x(rng, T, cols):
    return torch.from_numpy(S.random_bf16(rng, (T, cols)).view(np.int16)).cuda().view(torch.bfloat16)


# (format, experts, rows, cols): slice widths 4 (cols 4096), 2 (2048, 512) and
# 1 (768) blocks; ragged last tiles (rows 40, 72)
SHAPES = [("iq2_ks", 5, 40, 512), ("iq2_k", 4, 72, 768), ("iq2_ks", 3, 256, 4096), ("iq2_k", 3, 512, 2048)]


@pytest.mark.parametrize("fmt,E,rows,cols", SHAPES)
def test_gemv_switch_and_floor_match_with_images(B, fmt, E, rows, cols):
    rng = S.rng_for(900 + rows)
    host = S.random_streams(rng, fmt, E, rows, cols)
    plain, packed = _both(B, host)
    values = S.value_table("f16" if fmt == "iq2_k" else "int", 3)
    for T in (1, 3):
        x = _x(rng, T, cols)
        a = B.iqk_gemv(plain, E - 1, values, x)
        b = B.iqk_gemv(packed, E - 1, values, x)
        torch.cuda.synchronize()
        assert torch.equal(a.view(torch.int32), b.view(torch.int32)), f"gemv T={T}"
    x = _x(rng, 2, cols)
    ids = torch.from_numpy(np.array([[0, E - 1], [E - 1, 1]], np.int32)).cuda()
    a = B.iqk_switch_linear(plain, values, x, ids, mode=1)
    b = B.iqk_switch_linear(packed, values, x, ids, mode=1)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int32), b.view(torch.int32)), "switch (decode kernel)"
    lst = torch.from_numpy(np.arange(E, dtype=np.int32)).cuda()
    a = B.iqk_floor(plain, lst)
    b = B.iqk_floor(packed, lst)
    torch.cuda.synchronize()
    assert torch.equal(a, b), "floor signatures"


@pytest.mark.parametrize("T", [1, 4])
def test_routed_decode_matches_with_images(B, T):
    rng = S.rng_for(950 + T)
    E, H, F = 8, 1024, 512
    hosts = (S.random_streams(rng, "iq2_ks", E, F, H), S.random_streams(rng, "iq2_k", E, F, H),
             S.random_streams(rng, "iq2_ks", E, H, F))
    plain, packed = zip(*(_both(B, h) for h in hosts))
    values = S.value_table("int", 6)
    x = _x(rng, T, H)
    ids, p = S.routing(rng, T, E, 6)
    idsd, pd = torch.from_numpy(ids).cuda(), torch.from_numpy(p).cuda()
    a = B.iqk_moe_decode(*plain, values, x, idsd, pd)
    b = B.iqk_moe_decode(*packed, values, x, idsd, pd)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
