"""The token path around the operator on the GPU (gdn2_token_prologue,
gdn2_token_epilogue), through the C ABI, against the fp64 oracle
(oracle/token_path.py):
  * the prologue's q, k, v for dense and packed rows (sequence starts reset
    the convolution; empty and one-token sequences), dk / dv 64 and 128,
    every width 1..8 (each its own kernel), tiles with sequence starts
    inside a warp's run of tokens, fp32 I/O (rel-L2 <= 1e-5) and bf16 I/O (<= 1e-2: one
    bf16 rounding of the result);
  * the epilogue likewise (row counts that leave a block part-filled), and
    in place (out = o);
  * the whole path (prologue, operator, epilogue) against the oracles chained,
    at the operator's bf16 bar.
"""
import numpy as np
import pytest

import oracle
from oracle import token_path as otp
from tests.helpers import TOL, rel_l2
from workloads import round_bf16

pytestmark = pytest.mark.gpu

BAR = {"f32": 1e-5, "bf16": 1e-2}


@pytest.fixture(scope="module")
def gdn2(cuda_device):
    import gated_delta_rule_129_b200 as mod
    mod.load_library()
    return mod


def _raw(B, T, H, dk, dv, io, seed, W):
    rng = np.random.default_rng(seed)
    r = lambda *s: rng.standard_normal(s).astype(np.float32)  # noqa: E731
    x = dict(q=r(B, T, H, dk), k=r(B, T, H, dk), v=r(B, T, H, dv))
    if io == "bf16":
        x = {n: round_bf16(a) for n, a in x.items()}
    x["wq"], x["wk"], x["wv"] = r(H * dk, W) * 0.5, r(H * dk, W) * 0.5, r(H * dv, W) * 0.5
    return x


def _dev(a, dt):
    import torch
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dt)


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dk,dv,W,lengths", [(128, 128, 4, None), (64, 128, 1, None), (128, 64, 4, [9, 0, 1, 70]),
                                             (128, 128, 3, [200, 17, 0, 90]), (64, 64, 8, [5, 1, 300, 0]),
                                             (128, 128, 6, None), (64, 128, 2, [130, 7]), (128, 64, 5, None),
                                             (128, 128, 7, [3, 140])])
def test_prologue_matches_oracle(gdn2, io, dk, dv, W, lengths):
    import torch
    T = sum(lengths) if lengths else 50
    B = 1 if lengths else 2
    x = _raw(B, T, 3, dk, dv, io, 81, W)
    cu = None if lengths is None else np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    dt = torch.float32 if io == "f32" else torch.bfloat16
    q, k, v = gdn2.token_prologue(_dev(x["q"], dt), _dev(x["k"], dt), _dev(x["v"], dt), _dev(x["wq"], torch.float32),
                                  _dev(x["wk"], torch.float32), _dev(x["wv"], torch.float32),
                                  None if cu is None else _dev(cu, torch.int32))
    rq, rk, rv = otp.prologue(x["q"], x["k"], x["v"], x["wq"], x["wk"], x["wv"], cu)
    for got, ref in ((q, rq), (k, rk), (v, rv)):
        assert rel_l2(got.float().cpu().numpy(), ref) <= BAR[io]
    # L2-normalised rows
    n = np.linalg.norm(q.float().cpu().numpy().astype(np.float64), axis=-1)
    assert np.all(np.abs(n - 1) < (1e-5 if io == "f32" else 1e-2))


@pytest.mark.parametrize("io", ["f32", "bf16"])
@pytest.mark.parametrize("dv", [64, 128])
@pytest.mark.parametrize("shape", [(2, 40, 3), (1, 37, 3)])
def test_epilogue_matches_oracle(gdn2, io, dv, shape):
    import torch
    rng = np.random.default_rng(82)
    o = rng.standard_normal((*shape, dv)).astype(np.float32)
    g = rng.standard_normal((*shape, dv)).astype(np.float32)
    if io == "bf16":
        o, g = round_bf16(o), round_bf16(g)
    wt = rng.uniform(0.5, 1.5, dv).astype(np.float32)
    dt = torch.float32 if io == "f32" else torch.bfloat16
    od = _dev(o, dt)
    out = gdn2.token_epilogue(od, _dev(g, dt), _dev(wt, torch.float32))
    ref = otp.epilogue(o, g, wt)
    assert rel_l2(out.float().cpu().numpy(), ref) <= BAR[io]
    gdn2.token_epilogue(od, _dev(g, dt), _dev(wt, torch.float32), out=od)   # in place
    assert np.array_equal(od.float().cpu().numpy(), out.float().cpu().numpy())


def test_whole_token_path_matches_chained_oracles(gdn2):
    import torch
    from workloads import make_inputs
    lengths = [130, 0, 64, 1, 300]
    T = sum(lengths)
    gates = make_inputs(1, T, 2, 128, 128, io="bf16", seed=83, decay="strong", h0_std=0.05, lengths=lengths)
    x = _raw(1, T, 2, 128, 128, "bf16", 84, 4)
    rng = np.random.default_rng(85)
    g = round_bf16(rng.standard_normal((1, T, 2, 128)).astype(np.float32))
    wt = rng.uniform(0.5, 1.5, 128).astype(np.float32)
    cu = gates.cu_seqlens
    bf, f32 = torch.bfloat16, torch.float32
    out, hT = gdn2.token_path_fwd(_dev(x["q"], bf), _dev(x["k"], bf), _dev(x["v"], bf),
                                  _dev(gates.log_alpha, f32), _dev(gates.b, f32), _dev(gates.w, f32), _dev(g, bf),
                                  _dev(x["wq"], f32), _dev(x["wk"], f32), _dev(x["wv"], f32), _dev(wt, f32),
                                  gates.scale, h0=_dev(gates.h0, f32), cu_seqlens=_dev(cu, torch.int32))
    q, k, v = otp.prologue(x["q"], x["k"], x["v"], x["wq"], x["wk"], x["wv"], cu)
    q, k, v = (round_bf16(a.astype(np.float32)) for a in (q, k, v))   # what the operator is handed
    o, h = oracle.recurrent(q, k, v, gates.log_alpha, gates.b, gates.w, gates.scale, h0=gates.h0, cu_seqlens=cu)
    ref = otp.epilogue(round_bf16(o.astype(np.float32)), g, wt)
    assert rel_l2(out.float().cpu().numpy(), ref) <= TOL["bf16"]
    assert rel_l2(hT.cpu().numpy(), h) <= TOL["bf16"]
