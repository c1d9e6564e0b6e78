"""Parity at the full workload sizes, in the launch configuration bench.py times.

  2Kx8      B=8, T=2048, H=16, dk=dv=128, bf16 -- every sequence against the oracle
  16Kx1     B=1, T=16384, strong decay variety (256 chunks of state walk)
  reduce-a  B=4, T=4096, b = w = beta: also against the separate KDA oracle
  reduce-b  as (a) with a scalar decay: also against the Gated DeltaNet oracle
  varlen    32 packed sequences: every sequence against the oracle, and
            bitwise identity of every sequence run on its own
"""
import numpy as np
import pytest

from tests.helpers import TOL, compare, rel_l2, run_gpu, to_device
from workloads import config

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _gpu(cuda_device):
    import gated_delta_rule_129_b200 as gdn2
    gdn2.load_library()


@pytest.mark.parametrize("i", [1, 2])
def test_training_and_long_context_workloads(i):
    x = config(i)
    o, hT = run_gpu(x)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(hT))
    ro, rh = compare(x, o, hT)
    assert hT.size == x.num_seqs * 262_144
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)


@pytest.mark.parametrize("variant", ["a", "b"])
def test_reduction_workloads(variant):
    import oracle
    x = config(3, variant)
    o, hT = run_gpu(x)
    ro, rh = compare(x, o, hT)
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)
    if variant == "a":
        o2, h2 = oracle.kda(x.q, x.k, x.v, x.log_alpha, x.beta, x.scale)
    else:
        o2, h2 = oracle.gdn(x.q, x.k, x.v, x.log_alpha_scalar, x.beta, x.scale)
    assert rel_l2(o, o2) <= TOL["bf16"] and rel_l2(hT, h2) <= TOL["bf16"]


def test_varlen_workload():
    """Every one of the 32 packed sequences: against the oracle, and bitwise
    against the same sequence run on its own (with its own h0)."""
    import gated_delta_rule_129_b200 as gdn2
    x = config(4)
    o, hT = run_gpu(x)
    assert np.all(np.isfinite(o)) and np.all(np.isfinite(hT))
    ro, rh = compare(x, o, hT)
    assert ro <= TOL["bf16"] and rh <= TOL["bf16"], (ro, rh)
    d = to_device(x)
    cu = x.cu_seqlens
    for n in range(len(cu) - 1):
        s = slice(int(cu[n]), int(cu[n + 1]))
        sub = lambda t: t[:, s].contiguous()  # noqa: E731
        on, hn = gdn2.chunk_fwd(sub(d["q"]), sub(d["k"]), sub(d["v"]), sub(d["log_alpha"]),
                                sub(d["b"]), sub(d["w"]), x.scale, h0=d["h0"][n:n + 1].contiguous())
        assert np.array_equal(on.float().cpu().numpy(), o[:, s]), n
        assert np.array_equal(hn[0].cpu().numpy(), hT[n]), n
