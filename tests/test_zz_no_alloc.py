"""gdn2_chunk_fwd_noalloc: the forward pass for callers that cannot allocate
device memory where they run it (a plugin whose host framework owns all device
memory, code running under CUDA graph capture, a path that must not risk the
synchronisation an allocation can cause).  It uses a fixed scratch array
inside the library instead of a caller-provided workspace.

Checked here through the C ABI: two calls in a row (different inputs, so the
second call also shows that what the first left in the shared scratch does
not leak into its result) give bitwise the same O and hT as gdn2_chunk_fwd
(the same kernels on the same inputs), the status word of a call can be read
back (gdn2_noalloc_status, here on a malformed cu_seqlens), and a problem
larger than the scratch is rejected before anything is launched.  Every call
gets real device buffers of the right size.  This file is collected last on
purpose."""
import ctypes

import numpy as np
import pytest

from tests.helpers import to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu

GDN2_ERR_SEQLENS = 5
GDN2_ERR_WORKSPACE = 6


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


def _both(gdn2, x):
    d = to_device(x)
    args = (d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale)
    ref_o, ref_h = gdn2.chunk_fwd(*args, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    o, h = gdn2.chunk_fwd_noalloc(*args, h0=d["h0"], cu_seqlens=d["cu_seqlens"])
    st = gdn2.noalloc_status(d["q"], d["v"], d["cu_seqlens"])
    return (o.float().cpu().numpy(), h.cpu().numpy()), (ref_o.float().cpu().numpy(), ref_h.cpu().numpy()), int(st.item())


@pytest.mark.parametrize("io,dk,dv,lengths", [("bf16", 128, 128, None), ("bf16", 128, 64, [70, 0, 131, 5]),
                                              ("f32", 64, 128, None)])
def test_noalloc_matches_workspace_entry_point_twice(gdn2, io, dk, dv, lengths):
    for call, seed in enumerate((51, 52)):
        if lengths is None:
            x = make_inputs(2, 200, 3, dk, dv, io=io, seed=seed + dk, h0_std=0.05)
        else:
            x = make_inputs(1, sum(lengths), 3, dk, dv, io=io, seed=seed + dk, h0_std=0.05, lengths=lengths)
        (o, h), (ro, rh), st = _both(gdn2, x)
        assert st == 0, call
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(h)), call
        assert np.array_equal(o, ro) and np.array_equal(h, rh), call


def test_noalloc_status_reports_malformed_seqlens(gdn2):
    import torch
    x = make_inputs(1, 300, 2, 128, 128, io="bf16", seed=53, lengths=[100, 200])
    d = to_device(x)
    bad = torch.tensor([0, 250, 200], dtype=torch.int32, device="cuda")   # decreasing pair
    gdn2.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale, cu_seqlens=bad)
    assert int(gdn2.noalloc_status(d["q"], d["v"], bad).item()) == GDN2_ERR_SEQLENS
    # a good call afterwards clears it
    gdn2.chunk_fwd_noalloc(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale,
                           cu_seqlens=d["cu_seqlens"])
    assert int(gdn2.noalloc_status(d["q"], d["v"], d["cu_seqlens"]).item()) == 0


def test_noalloc_rejects_problems_beyond_its_scratch(gdn2):
    """Real, correctly sized device buffers: if the size check ever stopped
    returning first, the call would compute on valid memory (and this test
    would fail on the status), never touch memory it does not own."""
    import torch
    lib = gdn2.load_library()
    B, T, H, dk, dv = 1, 2048, 16, 128, 128
    assert gdn2.workspace_size(B, T, H, dk, dv, gdn2.GDN2_IO_BF16) > gdn2.NOALLOC_SCRATCH_BYTES
    bf = dict(dtype=torch.bfloat16, device="cuda")
    f32 = dict(dtype=torch.float32, device="cuda")
    q, k, v = (torch.zeros((B, T, H, d), **bf) for d in (dk, dk, dv))
    la, b, w = (torch.zeros((B, T, H, d), **f32) for d in (dk, dk, dv))
    out = torch.empty((B, T, H, dv), **bf)
    hT = torch.empty((B, H, dk, dv), **f32)
    d = gdn2.make_desc(B, T, H, dk, dv, gdn2.GDN2_IO_BF16)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    st = lib.gdn2_chunk_fwd_noalloc(ctypes.byref(d), P(q), P(k), P(v), P(la), P(b), P(w), 0.1, None, None,
                                    P(out), P(hT), None)
    assert st == GDN2_ERR_WORKSPACE
    flag = torch.zeros(4, dtype=torch.int32, device="cuda")
    assert lib.gdn2_noalloc_status(ctypes.byref(d), P(flag), None) == GDN2_ERR_WORKSPACE
    torch.cuda.synchronize()
