"""gdn2_chunk_fwd_noalloc: the forward pass for callers that cannot allocate
device memory where they run it (a plugin whose host framework owns all device
memory, code running under CUDA graph capture, a path that must not risk the
synchronisation an allocation can cause).  It uses a fixed scratch array
inside the library instead of a caller-provided workspace.

Checked here through the C ABI: two calls in a row (different inputs, so the
second call also shows that what the first left in the shared scratch does
not leak into its result) agree with gdn2_chunk_fwd within the tolerance the
parity tests use, and a problem larger than the scratch is rejected before
anything is launched.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from tests.helpers import TOL, rel_l2, to_device
from workloads import make_inputs

pytestmark = pytest.mark.gpu

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
    return (o.float().cpu().numpy(), h.cpu().numpy()), (ref_o.float().cpu().numpy(), ref_h.cpu().numpy())


@pytest.mark.parametrize("io,dk,dv,lengths", [("bf16", 128, 128, None), ("bf16", 128, 64, [70, 0, 131, 5]),
                                              ("f32", 64, 128, None)])
def test_noalloc_matches_workspace_entry_point_twice(gdn2, io, dk, dv, lengths):
    for call, seed in enumerate((51, 52)):
        if lengths is None:
            x = make_inputs(2, 200, 3, dk, dv, io=io, seed=seed + dk, h0_std=0.05)
        else:
            x = make_inputs(1, sum(lengths), 3, dk, dv, io=io, seed=seed + dk, h0_std=0.05, lengths=lengths)
        (o, h), (ro, rh) = _both(gdn2, x)
        assert np.all(np.isfinite(o)) and np.all(np.isfinite(h)), call
        assert rel_l2(o, ro) <= TOL[io] and rel_l2(h, rh) <= TOL[io], call


def test_noalloc_rejects_problems_beyond_its_scratch(gdn2):
    lib = gdn2.load_library()
    B, T, H, dk, dv = 1, 16384, 16, 128, 128
    assert gdn2.workspace_size(B, T, H, dk, dv, gdn2.GDN2_IO_BF16) > gdn2.NOALLOC_SCRATCH_BYTES
    d = gdn2.make_desc(B, T, H, dk, dv, gdn2.GDN2_IO_BF16)
    fake = [ctypes.c_void_p(0x10000 + 0x100 * i) for i in range(6)]
    st = lib.gdn2_chunk_fwd_noalloc(ctypes.byref(d), *fake, 0.1, None, None, ctypes.c_void_p(0x20000),
                                    None, None)
    assert st == GDN2_ERR_WORKSPACE
