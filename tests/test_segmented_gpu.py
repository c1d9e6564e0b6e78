"""The two-level chunk scan on the GPU (gdn2_chunk_fwd_segmented, gdn2_state_map).

Checked through the C ABI against the fp64 oracles:
  * the segmented forward equals the token recurrence (rel-L2 <= 2e-2 in bf16
    I/O, the bar of the other bf16 paths) and stays close to gdn2_chunk_fwd,
    for segments of 1 chunk, several chunks, more chunks than a sequence has,
    the library's own choice, dense and packed rows (empty and one-token
    sequences), dv = 64 and 128, with and without h0;
  * gdn2_state_map equals the oracle's affine map (Phi, Psi) of each
    sequence, and Phi h0 + Psi equals the final state of gdn2_chunk_fwd;
  * state passing between ranges of one sequence (what ranks holding parts of
    a long sequence do): the maps of the first ranges give the start state of
    the next, and the outputs of the ranges run from there equal the whole
    sequence's.
"""
import numpy as np
import pytest

from oracle import state_map as osm
from tests.helpers import TOL, compare, rel_l2, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


CASES = [
    dict(B=1, T=1000, H=3, dv=128, lengths=None, L=3, h0=0.05),
    dict(B=1, T=777, H=2, dv=64, lengths=None, L=1, h0=0.05),
    dict(B=2, T=300, H=2, dv=128, lengths=None, L=100, h0=None),
    dict(B=1, T=None, H=3, dv=128, lengths=[130, 0, 64, 1, 500], L=2, h0=0.05),
    dict(B=1, T=2000, H=2, dv=128, lengths=None, L=0, h0=0.05),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}T{c['T']}H{c['H']}dv{c['dv']}L{c['L']}")
def test_segmented_matches_oracle_and_fwd(gdn2, case):
    lengths = case["lengths"]
    T = sum(lengths) if lengths else case["T"]
    x = make_inputs(case["B"], T, case["H"], 128, case["dv"], io="bf16", seed=71, decay="strong",
                    h0_std=case["h0"], lengths=lengths)
    d = to_device(x)
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale)
    o, h = gdn2.chunk_fwd_segmented(*args, h0=d["h0"], cu_seqlens=d["cu_seqlens"], segment_chunks=case["L"])
    o_ref, h_ref = gdn2.chunk_fwd(*args, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    o, h = o.float().cpu().numpy(), h.cpu().numpy()
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(h))
    ro, rh = compare(x, o, h)
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)
    assert rel_l2(o, o_ref.float().cpu().numpy()) <= 1e-2
    assert rel_l2(h, h_ref.cpu().numpy()) <= 1e-2


@pytest.mark.parametrize("dv,lengths", [(128, None), (64, [150, 0, 65, 9])])
def test_state_map_matches_oracle(gdn2, dv, lengths):
    # mild decay and short sequences: over long ranges Phi decays below the
    # fp32 range (the oracle's fp64 values there are ~1e-60)
    T = sum(lengths) if lengths else 160
    x = make_inputs(1, T, 2, 128, dv, io="bf16", seed=72, decay="mild", h0_std=0.05, lengths=lengths)
    x.log_alpha = (0.1 * x.log_alpha).astype(np.float32)   # Phi of order one
    d = to_device(x)
    phi, psi = gdn2.state_map(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu_seqlens=d["cu_seqlens"])
    P, Q = osm.state_map(x.k, x.v, x.log_alpha, x.b, x.w, cu_seqlens=x.cu_seqlens)
    assert rel_l2(phi.cpu().numpy(), P) <= TOL["bf16"] and rel_l2(psi.cpu().numpy(), Q) <= TOL["bf16"]
    _, hT = gdn2.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, h0=d["h0"],
                           cu_seqlens=d["cu_seqlens"])
    via_map = (phi @ d["h0"] + psi).cpu().numpy()
    assert rel_l2(via_map, hT.cpu().numpy()) <= 1e-2


def test_state_passing_between_ranges(gdn2):
    """Three ranges of one 1100-token sequence (not chunk-aligned), as three
    ranks would hold them: each range's map, composed in order from h0, gives
    the next range's start state; running each range from its start state
    reproduces the whole sequence."""
    import torch
    x = make_inputs(1, 1100, 2, 128, 128, io="bf16", seed=73, decay="strong", h0_std=0.05)
    d = to_device(x)
    cuts = [0, 350, 801, 1100]
    S = d["h0"]
    outs = []
    for r in range(3):
        s = slice(cuts[r], cuts[r + 1])
        part = [t[:, s].contiguous() for t in (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"])]
        o, _ = gdn2.chunk_fwd(*part, x.scale, h0=S.contiguous())
        outs.append(o.float().cpu().numpy())
        phi, psi = gdn2.state_map(*part)
        S = phi @ S + psi
    o = np.concatenate(outs, axis=1)
    ro, rh = compare(x, o, S.cpu().numpy())
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)
    torch.cuda.synchronize()
