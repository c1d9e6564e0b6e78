"""Bounded device waits, made to run out on purpose (no fault, no hang).

The walk of the fused path takes each chunk only once the prep has raised
that chunk's ready flag in the workspace.  gdn2_chunk_walk_flagged runs that
walk on its own with a short wait limit.  Checked here through the C ABI:
  * with every flag left at 0 (nobody raises them) each bounded wait gives up
    after the limit: the launch completes, the workspace status word reads
    GDN2_ERR_DEVICE_TIMEOUT, and the context stays usable (a normal call
    right after it gives the usual result);
  * with every flag raised by hand after the prep, the flagged walk gives
    bitwise the same O and hT as the plain walk.
"""
import time

import numpy as np
import pytest

from tests.helpers import TOL, compare, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu

GDN2_ERR_DEVICE_TIMEOUT = 8


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


def _status(ws, lay):
    import torch
    off = lay["off_status"]
    return int(ws[off:off + 4].view(torch.int32).item())


@pytest.mark.parametrize("dv", [128, 64])
def test_walk_wait_runs_out_when_no_flag_is_raised(gdn2, dv):
    import torch
    x = make_inputs(1, 300, 2, 128, dv, io="bf16", seed=61, h0_std=0.05)
    d = to_device(x)
    shape = (1, 300, 2, 128, dv)
    lay = gdn2.workspace_layout(*shape, gdn2.GDN2_IO_BF16)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    # the prep's plan clears the status word and every ready flag
    gdn2.chunk_prep(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], workspace=ws)
    torch.cuda.synchronize()
    assert _status(ws, lay) == 0
    t0 = time.perf_counter()
    gdn2.chunk_walk_flagged(ws, shape, torch.bfloat16, x.scale, h0=d["h0"], wait_budget_ns=1_000_000)
    torch.cuda.synchronize()
    assert time.perf_counter() - t0 < 5.0
    assert _status(ws, lay) == GDN2_ERR_DEVICE_TIMEOUT
    # the context is still usable and the next call is right
    o, h = gdn2.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, h0=d["h0"])
    ro, rh = compare(x, o.float().cpu().numpy(), h.cpu().numpy())
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"]


def test_flagged_walk_with_raised_flags_equals_walk(gdn2):
    import torch
    x = make_inputs(1, 700, 3, 128, 128, io="bf16", seed=62, h0_std=0.05, decay="strong")
    d = to_device(x)
    shape = (1, 700, 3, 128, 128)
    lay = gdn2.workspace_layout(*shape, gdn2.GDN2_IO_BF16)
    ws = torch.zeros(lay["total_bytes"], dtype=torch.uint8, device="cuda")
    gdn2.chunk_prep(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], workspace=ws)
    ref_o, ref_h = gdn2.chunk_walk(ws, shape, torch.bfloat16, x.scale, h0=d["h0"])
    n_flags = lay["max_chunks"] * 3
    off = lay["off_sync"]
    ws[off:off + 4 * (2 + n_flags)].view(torch.int32)[2:] = 2
    o, h = gdn2.chunk_walk_flagged(ws, shape, torch.bfloat16, x.scale, h0=d["h0"], wait_budget_ns=1_000_000_000)
    torch.cuda.synchronize()
    assert _status(ws, lay) == 0
    assert np.array_equal(o.float().cpu().numpy(), ref_o.float().cpu().numpy())
    assert np.array_equal(h.cpu().numpy(), ref_h.cpu().numpy())
