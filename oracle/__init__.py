"""fp64 CPU oracle for the Gated DeltaNet-2 forward operator.

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
``cpu_baseline`` / ``--impl reference`` legs of ``bench.py`` may import this
package.  It shares no code with the CUDA path (``gated_delta_rule_129_b200``)
and the CUDA path never calls it.

Contents
--------
* :func:`recurrent` -- the token-by-token Gated Delta Rule-2 recurrence in fp64
  (C, ``gdn2_oracle.c``).  Page "Gated DeltaNet-2：将擦除与写入分开"
  (iplexlaw blog), section "在两个维度上独立控制": e = b*k, z = w*v,
  Sbar = diag(alpha) S, r = Sbar^T e, S = Sbar + k (z - r)^T, and the query
  reads the updated state.
* :func:`kda`, :func:`gdn`, :func:`deltanet` -- the scalar-gate recurrences the
  method reduces to (page "Gated DeltaNet-2: Decoupling Erase and Write in
  Linear Attention", cere-bro blog, section "TL;DR").
* :func:`recurrent_step` -- one decode step on a batch of states: the same
  recurrence with every sequence one token long.
* :mod:`oracle.chunk_wy` -- the 64-token chunkwise WY restatement in fp64
  (numpy), used to check the chunk algebra and to give per-chunk intermediates.
* :mod:`oracle.backward` -- the gradients of O and hT with respect to every
  input, reverse mode through the token recurrence in fp64 (numpy; small cases),
  pinned by finite differences of :func:`recurrent`.
* :mod:`oracle.chunk_backward` -- the same gradients through the 64-token chunk
  form (the algebra a backward over chunks evaluates), checked against
  :mod:`oracle.backward`.
* :mod:`oracle.token_path` -- the token path around the operator (short causal
  convolution, SiLU, L2 normalisation of q and k; RMS normalisation and the
  output gate of the operator's output), fp64 numpy.
* :mod:`oracle.state_map` -- the affine state map (Phi, Psi) of a token range
  and the composition of consecutive maps (the two-level chunk scan and the
  state passing between ranges of one sequence), fp64 numpy.

Arrays use the token-major layout ``[B, T, H, D]`` (or ``[1, T_total, H, D]``
with ``cu_seqlens``).  Inputs of any float dtype are upcast to fp64 exactly.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn2_oracle.c")
_LIB_PATH = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile ``gdn2_oracle.c`` into ``liboracle.so`` with gcc (IEEE fp64, no fast-math)."""
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread",
           "-fno-fast-math", "-ffp-contract=off", _SRC, "-o", tmp, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            build()
            lib = ctypes.CDLL(_LIB_PATH)
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            i = ctypes.c_int
            d = ctypes.c_double
            lib.oracle_gdn2_recurrent_f64.argtypes = [i, i, i, i, ip, dp, dp, dp, dp, dp, dp, d, dp, dp, dp, i]
            lib.oracle_kda_f64.argtypes = [i, i, i, i, ip, dp, dp, dp, dp, dp, d, dp, dp, dp, i]
            lib.oracle_gdn_f64.argtypes = [i, i, i, i, ip, dp, dp, dp, dp, dp, d, dp, dp, dp, i]
            lib.oracle_deltanet_f64.argtypes = [i, i, i, i, ip, dp, dp, dp, d, dp, dp, dp, i]
            for f in (lib.oracle_gdn2_recurrent_f64, lib.oracle_kda_f64,
                      lib.oracle_gdn_f64, lib.oracle_deltanet_f64):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _pack(x):
    """[B, T, H, D] -> ([B*T, H, D] fp64 contiguous)."""
    x = _f64(x)
    return x.reshape(-1, x.shape[-2], x.shape[-1])


def _seqlens(B, T, cu_seqlens):
    if cu_seqlens is None:
        return (np.arange(B + 1, dtype=np.int64) * T).astype(np.int32)
    cu = np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int32))
    if B != 1:
        raise ValueError("cu_seqlens requires B == 1 (packed layout)")
    if cu[0] != 0 or cu[-1] != T or np.any(np.diff(cu) < 0):
        raise ValueError("cu_seqlens must start at 0, be non-decreasing and end at T")
    return cu


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


def recurrent(q, k, v, log_alpha, b, w, scale, h0=None, cu_seqlens=None, nthreads=None):
    """Gated Delta Rule-2 recurrence in fp64.

    Returns ``(o, hT)``: ``o`` with the shape of ``v`` and ``hT`` of shape
    ``[N, H, dk, dv]`` (N = number of sequences).
    """
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    cu = _seqlens(B, T, cu_seqlens)
    N = len(cu) - 1
    qq, kk, vv, la, bb, ww = (_pack(x) for x in (q, k, v, log_alpha, b, w))
    h0a = None if h0 is None else _f64(h0).reshape(N, H, dk, dv)
    o = np.zeros((B * T, H, dv), dtype=np.float64)
    hT = np.zeros((N, H, dk, dv), dtype=np.float64)
    rc = _load().oracle_gdn2_recurrent_f64(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(qq), _ptr(kk), _ptr(vv), _ptr(la), _ptr(bb), _ptr(ww), float(scale),
        _ptr(h0a), _ptr(o), _ptr(hT), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle_gdn2_recurrent_f64 failed")
    return o.reshape(B, T, H, dv), hT


def kda(q, k, v, log_alpha, beta, scale, h0=None, cu_seqlens=None, nthreads=None):
    """KDA: scalar beta ``[B, T, H]``, channel-wise log-decay ``[B, T, H, dk]``."""
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    cu = _seqlens(B, T, cu_seqlens)
    N = len(cu) - 1
    qq, kk, vv, la = (_pack(x) for x in (q, k, v, log_alpha))
    be = _f64(beta).reshape(-1)
    h0a = None if h0 is None else _f64(h0).reshape(N, H, dk, dv)
    o = np.zeros((B * T, H, dv))
    hT = np.zeros((N, H, dk, dv))
    rc = _load().oracle_kda_f64(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(qq), _ptr(kk), _ptr(vv), _ptr(la), _ptr(be), float(scale),
        _ptr(h0a), _ptr(o), _ptr(hT), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle_kda_f64 failed")
    return o.reshape(B, T, H, dv), hT


def gdn(q, k, v, log_alpha_scalar, beta, scale, h0=None, cu_seqlens=None, nthreads=None):
    """Gated DeltaNet: scalar beta and scalar log-decay, both ``[B, T, H]``."""
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    cu = _seqlens(B, T, cu_seqlens)
    N = len(cu) - 1
    qq, kk, vv = (_pack(x) for x in (q, k, v))
    las = _f64(log_alpha_scalar).reshape(-1)
    be = _f64(beta).reshape(-1)
    h0a = None if h0 is None else _f64(h0).reshape(N, H, dk, dv)
    o = np.zeros((B * T, H, dv))
    hT = np.zeros((N, H, dk, dv))
    rc = _load().oracle_gdn_f64(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(qq), _ptr(kk), _ptr(vv), _ptr(las), _ptr(be), float(scale),
        _ptr(h0a), _ptr(o), _ptr(hT), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle_gdn_f64 failed")
    return o.reshape(B, T, H, dv), hT


def deltanet(q, k, v, scale, h0=None, cu_seqlens=None, nthreads=None):
    """Plain DeltaNet (beta = 1, no decay)."""
    B, T, H, dk = np.shape(q)
    dv = np.shape(v)[-1]
    cu = _seqlens(B, T, cu_seqlens)
    N = len(cu) - 1
    qq, kk, vv = (_pack(x) for x in (q, k, v))
    h0a = None if h0 is None else _f64(h0).reshape(N, H, dk, dv)
    o = np.zeros((B * T, H, dv))
    hT = np.zeros((N, H, dk, dv))
    rc = _load().oracle_deltanet_f64(
        N, H, dk, dv, cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int32)),
        _ptr(qq), _ptr(kk), _ptr(vv), float(scale),
        _ptr(h0a), _ptr(o), _ptr(hT), int(nthreads or default_threads()))
    if rc != 0:
        raise RuntimeError("oracle_deltanet_f64 failed")
    return o.reshape(B, T, H, dv), hT


def recurrent_step(q, k, v, log_alpha, b, w, scale, state, nthreads=None):
    """One decode step for a batch of states.

    ``q, k, log_alpha, b`` are ``[B, H, dk]``; ``v, w`` are ``[B, H, dv]``;
    ``state`` is ``[B, H, dk, dv]``.  Returns ``(o [B, H, dv], new_state)``:
    the recurrence of :func:`recurrent` run for one token per batch element.
    """
    Bn = np.shape(q)[0]
    add_t = lambda x: _f64(x)[None]  # noqa: E731  -> [1, B, H, D]
    cu = np.arange(Bn + 1, dtype=np.int32)
    o, hT = recurrent(add_t(q), add_t(k), add_t(v), add_t(log_alpha), add_t(b), add_t(w),
                      scale, h0=state, cu_seqlens=cu, nthreads=nthreads)
    return o[0], hT
