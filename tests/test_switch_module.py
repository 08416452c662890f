"""IqkSwitchLinear, the page's module surface (mlx-iqk 0.1.1 PKG-INFO, section
"Surface"): host-side refusals on CPU, results against the oracle on GPU."""
import numpy as np
import pytest

import iqk_synth as S
from gemm_iq2_ks_b200 import binding as B

VALS = np.array([3, -5, 7, -11, 13, -17, 19, -23], np.float32)


def test_unsized_widths_and_unknown_members_are_refused():
    with pytest.raises(ValueError):
        B.IqkSwitchLinear("iq2_ks", 8, 256, 1000, VALS)
    with pytest.raises(ValueError):
        B.IqkSwitchLinear("iq2_ks", 8, 256, 0, VALS)
    with pytest.raises(ValueError):
        B.IqkSwitchLinear("iq1_s", 8, 256, 512, VALS)
    with pytest.raises(ValueError):
        B.IqkSwitchLinear("iq2_k", 8, 256, 512, VALS[:4])


def test_streams_must_match_member_and_shape():
    proj = B.IqkSwitchLinear("iq2_ks", 4, 64, 512, VALS)
    with pytest.raises(ValueError):
        proj.load_streams(S.empty_streams("iq2_k", 4, 64, 512))
    with pytest.raises(ValueError):
        proj.load_streams(S.empty_streams("iq2_ks", 4, 64, 768))
    with pytest.raises(RuntimeError):
        proj(None, None)  # nothing loaded


@pytest.mark.gpu
@pytest.mark.parametrize("lead", [(1,), (2, 3), (48,)])
def test_layer_of_two_members_matches_the_oracle(lead):
    """One layer's projections with different members; leading dims are kept;
    1 token takes the decode kernel, 48 the grouped GEMM (auto mode)."""
    torch = pytest.importorskip("torch")
    from oracle import oracle as O
    from util import check_fp32
    rng = S.rng_for(400 + int(np.prod(lead)))
    E, k, H, F = 12, 4, 512, 256
    wg = S.random_streams(rng, "iq2_ks", E, F, H)
    wd = S.random_streams(rng, "iq2_k", E, H, F)
    gate = B.IqkSwitchLinear("iq2_ks", E, F, H, VALS).load_streams(wg)
    down = B.IqkSwitchLinear("iq2_k", E, H, F, VALS).load_streams(wd)
    T = int(np.prod(lead))
    x = S.random_bf16(rng, (T, H))
    ids, _ = S.routing(rng, T, E, k)
    xd = torch.from_numpy(x.view(np.int16)).cuda().view(torch.bfloat16).reshape(*lead, H)
    idd = torch.from_numpy(ids).cuda().reshape(*lead, k)
    g = gate(xd, idd, sorted_indices=True)
    assert tuple(g.shape) == (*lead, k, F) and gate.status() == B.IQK_OK
    y_ref, S_ref = O.switch_linear(wg, VALS, x, ids)
    check_fp32(g.reshape(T, k, F).cpu().numpy(), y_ref, S_ref, f"gate {lead}")
    # the layer's other projection on its own seeded input, routed the same way
    hb = S.random_bf16(rng, (T, F))
    h = torch.from_numpy(hb.view(np.int16)).cuda().view(torch.bfloat16).reshape(*lead, F)
    d = down(h, idd, sorted_indices=False)
    y2, S2 = O.switch_linear(wd, VALS, hb, ids)
    check_fp32(d.reshape(T, k, H).cpu().numpy(), y2, S2, f"down {lead}")


@pytest.mark.gpu
def test_out_of_range_id_reports_through_status():
    torch = pytest.importorskip("torch")
    rng = S.rng_for(410)
    w = S.random_streams(rng, "iq2_ks", 6, 64, 512)
    proj = B.IqkSwitchLinear("iq2_ks", 6, 64, 512, VALS).load_streams(w)
    x = torch.from_numpy(S.random_bf16(rng, (2, 512)).view(np.int16)).cuda().view(torch.bfloat16)
    ids = torch.tensor([[0, 9], [1, 2]], dtype=torch.int32, device="cuda")
    y = proj(x, ids)
    assert proj.status() == B.IQK_EINVAL
    assert not y[0, 1].any()


def test_call_checks_shapes_before_any_launch():
    """Host-side refusals of a loaded projection (streams kept on the CPU:
    nothing reaches the library)."""
    torch = pytest.importorskip("torch")
    w = S.random_streams(S.rng_for(3), "iq2_k", 4, 32, 512)
    proj = B.IqkSwitchLinear("iq2_k", 4, 32, 512, VALS, device="cpu").load_streams(w)
    ids = torch.zeros((2, 3), dtype=torch.int32)
    with pytest.raises(ValueError):
        proj(torch.zeros((2, 512), dtype=torch.float32), ids)      # not bf16
    with pytest.raises(ValueError):
        proj(torch.zeros((2, 256), dtype=torch.bfloat16), ids)     # wrong width
    with pytest.raises(ValueError):
        proj(torch.zeros((3, 512), dtype=torch.bfloat16), ids)     # leading shapes differ
