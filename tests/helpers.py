"""Shared helpers for the GPU tests: move seeded inputs to the device, call the
CUDA path through the binding, and measure relative L2 error in fp64."""
import numpy as np

TOL = {"f32": 1e-4, "bf16": 2e-2}   # rel-L2 of O and hT against the fp64 oracle


def rel_l2(x, ref):
    x = np.asarray(x, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    den = np.linalg.norm(ref.ravel())
    return float(np.linalg.norm((x - ref).ravel()) / (den if den > 0 else 1.0))


def to_device(x, device="cuda"):
    import torch
    io = torch.bfloat16 if x.io == "bf16" else torch.float32
    t = lambda a, dt: torch.from_numpy(np.ascontiguousarray(a)).to(device=device, dtype=dt)  # noqa: E731
    d = dict(q=t(x.q, io), k=t(x.k, io), v=t(x.v, io), log_alpha=t(x.log_alpha, torch.float32),
             b=t(x.b, torch.float32), w=t(x.w, torch.float32))
    d["h0"] = None if x.h0 is None else t(x.h0, torch.float32)
    d["cu_seqlens"] = None if x.cu_seqlens is None else t(x.cu_seqlens, torch.int32)
    return d


def run_gpu(x, **kw):
    import gated_delta_rule_129_b200 as gdn2
    d = to_device(x)
    o, hT = gdn2.chunk_fwd(d["q"], d["k"], d["v"], d["log_alpha"], d["b"], d["w"], x.scale,
                           h0=d["h0"], cu_seqlens=d["cu_seqlens"], **kw)
    return o.float().cpu().numpy(), hT.cpu().numpy()


def run_oracle(x, seqs=None):
    """The fp64 oracle on all sequences, or only on ``seqs`` (list of indices);
    returns per-sequence outputs [(o_n [len, H, dv], hT_n [H, dk, dv]), ...]."""
    import oracle
    if x.cu_seqlens is None:
        B, T = x.q.shape[:2]
        if seqs is None:
            o, hT = oracle.recurrent(x.q, x.k, x.v, x.log_alpha, x.b, x.w, x.scale, h0=x.h0)
            return [(o[n], hT[n]) for n in range(B)]
        res = []
        for n in seqs:
            h0 = None if x.h0 is None else x.h0[n:n + 1]
            o, hT = oracle.recurrent(*(a[n:n + 1] for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)),
                                     x.scale, h0=h0)
            res.append((o[0], hT[0]))
        return res
    cu = x.cu_seqlens
    seqs = range(len(cu) - 1) if seqs is None else seqs
    res = []
    for n in seqs:
        s = slice(int(cu[n]), int(cu[n + 1]))
        h0 = None if x.h0 is None else x.h0[n:n + 1]
        o, hT = oracle.recurrent(*(a[:, s] for a in (x.q, x.k, x.v, x.log_alpha, x.b, x.w)),
                                 x.scale, h0=h0)
        res.append((o[0], hT[0]))
    return res


def gpu_per_seq(x, o, hT, seqs=None):
    """Split GPU outputs the same way as :func:`run_oracle`."""
    if x.cu_seqlens is None:
        B = x.q.shape[0]
        seqs = range(B) if seqs is None else seqs
        return [(o[n], hT[n]) for n in seqs]
    cu = x.cu_seqlens
    seqs = range(len(cu) - 1) if seqs is None else seqs
    return [(o[0, int(cu[n]):int(cu[n + 1])], hT[n]) for n in seqs]


def compare(x, o, hT, seqs=None):
    """rel-L2 of O and of hT over the chosen sequences (concatenated)."""
    ref = run_oracle(x, seqs)
    got = gpu_per_seq(x, o, hT, seqs)
    ro = rel_l2(np.concatenate([g[0].ravel() for g in got]), np.concatenate([r[0].ravel() for r in ref]))
    rh = rel_l2(np.concatenate([g[1].ravel() for g in got]), np.concatenate([r[1].ravel() for r in ref]))
    return ro, rh
