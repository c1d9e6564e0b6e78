"""The fused prep + walk launch (bf16 I/O, dk = 128, few walk CTAs).

gdn2_chunk_fwd takes the fused path whenever the walk fits beside enough prep
CTAs; the per-chunk arithmetic is the same code as the two stage kernels run
back to back, so the two orders must agree bit for bit.  Checked here through
the C ABI:
  * chunk_fwd (fused) == chunk_prep + chunk_walk, bitwise, dense and packed,
    dv = 128 and 64, with and without h0;
  * chunk_plan + chunk_fused alone == chunk_fwd when no chunk is handed back;
  * a chunk with decay too steep for the tensor-core prep ends the fused walk
    early (redo flag), and the exact redo that follows still gives the
    sequential result and stays within the oracle tolerance;
  * the ready flags and the redo flag the launch leaves in the workspace.
"""
import numpy as np
import pytest

from tests.helpers import TOL, compare, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


def _sequential(gdn2, x, d, shape):
    import torch
    lay = gdn2.workspace_layout(*shape, gdn2.GDN2_IO_BF16, 0 if x.cu_seqlens is None else len(x.cu_seqlens) - 1)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    gdn2.chunk_prep(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], cu_seqlens=d["cu_seqlens"], workspace=ws)
    o, h = gdn2.chunk_walk(ws, shape, torch.bfloat16, x.scale, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    torch.cuda.synchronize()
    return o, h


def _fused(gdn2, x, d, shape):
    import torch
    ns = 0 if x.cu_seqlens is None else len(x.cu_seqlens) - 1
    lay = gdn2.workspace_layout(*shape, gdn2.GDN2_IO_BF16, ns)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    o, h = gdn2.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, h0=d["h0"],
                          cu_seqlens=d["cu_seqlens"], workspace=ws)
    torch.cuda.synchronize()
    return o, h, ws, lay


CASES = [
    dict(B=1, T=1000, H=4, dv=128, lengths=None, h0=0.0),
    dict(B=1, T=777, H=3, dv=64, lengths=None, h0=0.05),
    dict(B=2, T=300, H=2, dv=128, lengths=None, h0=0.05),
    dict(B=1, T=None, H=3, dv=128, lengths=[130, 0, 64, 1, 500], h0=0.05),
    # 20 heads: the walk CTAs take prep tasks first (switch point above 0)
    dict(B=1, T=300, H=20, dv=128, lengths=None, h0=0.05),
    # long sequences (79 and 71 chunks), and a packed row of long ones
    dict(B=1, T=5000, H=3, dv=128, lengths=None, h0=0.05),
    dict(B=1, T=4500, H=2, dv=64, lengths=None, h0=0.05),
    dict(B=1, T=None, H=2, dv=128, lengths=[2100, 0, 70, 2500], h0=0.05),
]


@pytest.mark.parametrize("case", CASES, ids=lambda c: f"B{c['B']}-H{c['H']}-dv{c['dv']}-{'var' if c['lengths'] else 'dense'}")
def test_fused_equals_sequential_bitwise(gdn2, case):
    lengths = case["lengths"]
    T = sum(lengths) if lengths else case["T"]
    x = make_inputs(case["B"], T, case["H"], 128, case["dv"], io="bf16", seed=71 + case["H"],
                    h0_std=case["h0"], lengths=lengths)
    d = to_device(x)
    shape = (case["B"], T, case["H"], 128, case["dv"])
    o_s, h_s = _sequential(gdn2, x, d, shape)
    o_f, h_f, ws, lay = _fused(gdn2, x, d, shape)
    import torch
    assert torch.equal(o_f, o_s) and torch.equal(h_f, h_s)
    # every (chunk, head) the walk took was published by both storing threads
    sync = ws[lay["off_sync"]:].view(torch.int32)
    nch = lay["max_chunks"] * case["H"]
    ready = sync[2:2 + nch].cpu().numpy()
    chunk_off = ws[lay["off_chunk_offsets"]:].view(torch.int32)
    n_seq = len(lengths) if lengths else case["B"]
    used = int(chunk_off[n_seq].item()) * case["H"]
    assert np.all(ready[:used] == 2) and np.all(ready[used:] == 0)
    assert int(sync[1].item()) == 0          # no redo
    assert int(sync[0].item()) >= used       # every task was taken


def test_fused_stage_alone_equals_chunk_fwd(gdn2):
    import torch
    x = make_inputs(1, 2000, 4, 128, 128, io="bf16", seed=75, h0_std=0.05)
    d = to_device(x)
    shape = (1, 2000, 4, 128, 128)
    o_f, h_f, _, lay = _fused(gdn2, x, d, shape)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    out = torch.empty_like(d["v"])
    hT = torch.empty((1, 4, 128, 128), dtype=torch.float32, device="cuda")
    gdn2.chunk_plan(shape, torch.bfloat16, ws)
    gdn2.chunk_fused(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, ws, h0=d["h0"],
                     out=out, hT=hT)
    torch.cuda.synchronize()
    assert torch.equal(out, o_f) and torch.equal(hT, h_f)


def test_fused_stage_rejects_shapes_it_does_not_take(gdn2):
    import torch
    x = make_inputs(1, 100, 2, 64, 64, io="bf16", seed=76)
    d = to_device(x)
    shape = (1, 100, 2, 64, 64)
    lay = gdn2.workspace_layout(*shape, gdn2.GDN2_IO_BF16)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    gdn2.chunk_plan(shape, torch.bfloat16, ws)
    with pytest.raises(gdn2.GDN2Error):
        gdn2.chunk_fused(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, ws,
                         out=torch.empty_like(d["v"]))


def test_fused_steep_chunk_in_a_long_sequence_redoes_the_walk(gdn2):
    """A steep chunk early in an 80-chunk sequence: the fused walk stops
    there, and the redo (exact chunks, walk again) still gives the sequential
    result."""
    import torch
    x = make_inputs(1, 80 * 64, 2, 128, 128, io="bf16", seed=44, h0_std=0.05)
    x.log_alpha[0, 5 * 64 + 2:5 * 64 + 30, :, :8] = -6.0     # chunk 5: ~170 nats in 28 tokens
    d = to_device(x)
    shape = (1, 80 * 64, 2, 128, 128)
    o_s, h_s = _sequential(gdn2, x, d, shape)
    o_f, h_f, ws, lay = _fused(gdn2, x, d, shape)
    sync = ws[lay["off_sync"]:].view(torch.int32)
    assert int(sync[1].item()) == 1
    assert torch.equal(o_f, o_s) and torch.equal(h_f, h_s)
    ro, rh = compare(x, o_f.float().cpu().numpy(), h_f.cpu().numpy())
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)


def test_fused_steep_chunk_redoes_the_walk(gdn2):
    import torch
    x = make_inputs(1, 300, 2, 128, 128, io="bf16", seed=43, h0_std=0.05)
    x.log_alpha[0, 70:100, :, :16] = -6.0      # ~180 nats over 30 tokens in 16 channels
    d = to_device(x)
    shape = (1, 300, 2, 128, 128)
    o_s, h_s = _sequential(gdn2, x, d, shape)
    o_f, h_f, ws, lay = _fused(gdn2, x, d, shape)
    sync = ws[lay["off_sync"]:].view(torch.int32)
    assert int(sync[1].item()) == 1            # the fused walk met a handed-back chunk
    ready = sync[2:2 + lay["max_chunks"] * 2].cpu().numpy()
    assert np.sum(ready == 3) >= 2             # chunk 1 of both heads
    assert torch.equal(o_f, o_s) and torch.equal(h_f, h_s)
    ro, rh = compare(x, o_f.float().cpu().numpy(), h_f.cpu().numpy())
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)
