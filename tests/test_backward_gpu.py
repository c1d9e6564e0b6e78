"""GPU parity of gdn2_chunk_bwd (through the C ABI) against the fp64 backward
oracle (``oracle/backward.py``, pinned by finite differences of the forward).

The kernel computes in fp32 from the same (bf16-representable) inputs the
oracle sees and writes fp32 gradients, so the tolerance is the fp32 one in
both I/O modes: rel-L2 <= 1e-4 over each gradient tensor (fp64 comparison),
on shapes that span several chunks, a ragged tail, packed sequences with empty
and one-token ones, dk / dv 64 and 128, with and without h0 and dhT,
chunks whose decay is too steep for the scaled-product form (the pair-by-pair
path), and two heads of the full 16K x 1 workload.
"""
import numpy as np
import pytest

from tests.helpers import rel_l2
from workloads import make_inputs, round_bf16

pytestmark = pytest.mark.gpu

NAMES = ("q", "k", "v", "log_alpha", "b", "w")


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


CASES = [
    dict(io="f32", dk=64, dv=64, B=2, T=150, H=2, lengths=None, decay="mild", h0=True, dhT=True),
    dict(io="bf16", dk=128, dv=128, B=1, T=200, H=2, lengths=None, decay="strong", h0=True, dhT=True),
    dict(io="f32", dk=128, dv=64, B=1, T=None, H=2, lengths=[70, 0, 1, 130], decay="mild", h0=True, dhT=True),
    dict(io="bf16", dk=64, dv=128, B=2, T=65, H=1, lengths=None, decay="mild", h0=False, dhT=False),
    # a chunk whose decay spans ~96 nats on each side of its middle token: the
    # pair-by-pair path instead of the scaled products
    dict(io="bf16", dk=128, dv=128, B=1, T=192, H=2, lengths=None, decay="mild", h0=True, dhT=True, steep=True),
    dict(io="f32", dk=64, dv=64, B=1, T=None, H=2, lengths=[100, 3, 90], decay="mild", h0=True, dhT=True,
         steep=True),
]


def _ids(c):
    return (f"{c['io']}-dk{c['dk']}-dv{c['dv']}-{'var' if c['lengths'] else 'B%d' % c['B']}"
            + ("-steep" if c.get("steep") else ""))


@pytest.mark.parametrize("case", CASES, ids=_ids)
def test_backward_matches_oracle(gdn2, case):
    import torch

    import oracle.backward as ob
    lengths = case["lengths"]
    T = sum(lengths) if lengths else case["T"]
    x = make_inputs(case["B"], T, case["H"], case["dk"], case["dv"], io=case["io"], seed=91 + case["dk"],
                    decay=case["decay"], h0_std=0.05 if case["h0"] else None, lengths=lengths)
    if case.get("steep"):
        x.log_alpha[:, 64:128] = -3.0
    rng = np.random.default_rng(92)
    dO = rng.standard_normal(x.v.shape).astype(np.float32)
    if case["io"] == "bf16":
        dO = round_bf16(dO)
    N = x.num_seqs
    dhT = rng.standard_normal((N, case["H"], case["dk"], case["dv"])).astype(np.float32) if case["dhT"] else None
    ref = ob.backward(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, dO, dhT=dhT, h0=x.h0, cu_seqlens=x.cu_seqlens)

    io = torch.bfloat16 if case["io"] == "bf16" else torch.float32
    t = lambda a, dt: None if a is None else torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)  # noqa: E731
    got = gdn2.chunk_bwd(t(x.q, io), t(x.k, io), t(x.v, io), t(x.log_alpha, torch.float32), t(x.b, torch.float32),
                         t(x.w, torch.float32), x.scale, t(dO, io), h0=t(x.h0, torch.float32),
                         dhT=t(dhT, torch.float32), cu_seqlens=t(x.cu_seqlens, torch.int32))
    torch.cuda.synchronize()
    for name in NAMES + ("h0",):
        g = got[name].cpu().numpy()
        assert np.all(np.isfinite(g)), name
        r = rel_l2(g, ref[name])
        assert r <= 1e-4, (name, r)


def test_backward_malformed_seqlens_sets_status(gdn2):
    import torch
    x = make_inputs(1, 100, 1, 64, 64, io="f32", seed=93, lengths=[50, 10, 40])
    cu = torch.tensor([0, 50, 40, 100], dtype=torch.int32, device="cuda")   # sequence 1 ends before it starts
    nbytes = gdn2.backward_workspace_size(1, 100, 1, 64, 64, gdn2.GDN2_IO_F32, 3)
    ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", torch.float32)  # noqa: E731
    dO = torch.ones((1, 100, 1, 64), dtype=torch.float32, device="cuda")
    gdn2.chunk_bwd(t(x.q), t(x.k), t(x.v), t(x.log_alpha), t(x.b), t(x.w), x.scale, dO, cu_seqlens=cu, workspace=ws)
    torch.cuda.synchronize()
    assert gdn2.STATUS[int(ws[:4].view(torch.int32).item())] == "GDN2_ERR_SEQLENS"


@pytest.mark.parametrize("heads", [(0, 11)])
def test_backward_full_size_sampled_heads(gdn2, heads):
    """The 16K x 1 workload (H = 16, bf16 inputs) in the launch configuration
    bench.py times; heads are independent, so two of them are checked against
    the chunkwise fp64 oracle run on that head alone."""
    import torch

    import oracle.chunk_backward as ocb
    from workloads import config
    x = config(2)
    rng = np.random.default_rng(96)
    dO = round_bf16(rng.standard_normal(x.v.shape).astype(np.float32))
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)  # noqa: E731
    bf, f32 = torch.bfloat16, torch.float32
    got = gdn2.chunk_bwd(t(x.q, bf), t(x.k, bf), t(x.v, bf), t(x.log_alpha, f32), t(x.b, f32), t(x.w, f32),
                         x.scale, t(dO, bf))
    torch.cuda.synchronize()
    for h in heads:
        one = lambda a: np.ascontiguousarray(a[:, :, h:h + 1])  # noqa: E731
        ref = ocb.backward(one(x.q), one(x.k), one(x.v), one(x.log_alpha), one(x.b), one(x.w), x.scale, one(dO))
        for name in NAMES:
            g = got[name][:, :, h:h + 1].cpu().numpy()
            assert np.all(np.isfinite(g)), (h, name)
            r = rel_l2(g, ref[name])
            assert r <= 1e-4, (h, name, r)
        r = rel_l2(got["h0"][:, h:h + 1].cpu().numpy(), ref["h0"])
        assert r <= 1e-4, (h, "h0", r)
