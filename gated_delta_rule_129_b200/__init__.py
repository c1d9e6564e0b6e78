"""B200 (sm_100a) Gated DeltaNet-2 forward operator -- Python binding.

A thin ctypes layer over ``libgdn2.so`` (declared in ``include/gdn2.h``).  It
only marshals arguments: every step of the computation runs in the library's
CUDA kernels.  PyTorch supplies device memory and the current stream.  There
is no CPU fallback: if the library is missing, every call raises.

Public functions mirror the C entry points:

* :func:`chunk_fwd`        -- ``gdn2_chunk_fwd``
* :func:`chunk_prep`       -- ``gdn2_chunk_prep`` (gate prep + intra-chunk WY)
* :func:`chunk_walk`       -- ``gdn2_chunk_walk`` (state walk + output)
* :func:`chunk_plan`, :func:`chunk_fused` -- ``gdn2_chunk_plan``, ``gdn2_chunk_fused``
  (the fused prep + walk launch on its own, for timing and tests)
* :func:`recurrent_step`   -- ``gdn2_recurrent_step`` (one decode token)
* :func:`workspace_size`, :func:`workspace_layout`, :func:`status_string`
"""
from __future__ import annotations

import ctypes
import os
import threading

__all__ = ["chunk_fwd", "chunk_fwd_noalloc", "noalloc_status", "chunk_walk_flagged", "chunk_fwd_segmented",
           "segmented_workspace_size", "state_map", "token_prologue", "token_epilogue", "token_path_fwd", "chunk_prep", "chunk_walk", "chunk_plan", "chunk_fused",
           "recurrent_step", "workspace_size",
           "workspace_layout", "status_string", "GDN2Error", "lib_path", "load_library"]

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB_PATH = os.path.join(_HERE, "libgdn2.so")
_lock = threading.Lock()
_lib = None

GDN2_IO_F32 = 0
GDN2_IO_BF16 = 1

STATUS = {0: "GDN2_OK", 1: "GDN2_ERR_NULL", 2: "GDN2_ERR_SHAPE", 3: "GDN2_ERR_DTYPE",
          4: "GDN2_ERR_ALIGN", 5: "GDN2_ERR_SEQLENS", 6: "GDN2_ERR_WORKSPACE",
          7: "GDN2_ERR_CUDA", 8: "GDN2_ERR_DEVICE_TIMEOUT", 9: "GDN2_ERR_UNSUPPORTED"}

EXPORTED = ("gdn2_workspace_size", "gdn2_workspace_layout", "gdn2_chunk_fwd", "gdn2_chunk_fwd_noalloc",
            "gdn2_chunk_prep", "gdn2_chunk_walk", "gdn2_chunk_plan", "gdn2_chunk_fused",
            "gdn2_recurrent_step", "gdn2_status_string", "gdn2_version", "gdn2_backward_workspace_size",
            "gdn2_chunk_bwd", "gdn2_noalloc_status", "gdn2_chunk_walk_flagged",
            "gdn2_segmented_workspace_size", "gdn2_chunk_fwd_segmented", "gdn2_state_map",
            "gdn2_token_prologue", "gdn2_token_epilogue")


class GDN2Error(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)} ({status_string(status)})")


class Desc(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("H", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("num_seqs", ctypes.c_int),
                ("io", ctypes.c_int), ("workspace", ctypes.c_void_p),
                ("workspace_bytes", ctypes.c_size_t)]


class WsLayout(ctypes.Structure):
    _fields_ = [("total_bytes", ctypes.c_size_t), ("max_chunks", ctypes.c_int),
                ("factor_elem_bytes", ctypes.c_int), ("factor_set", ctypes.c_int),
                ("reserved", ctypes.c_int), ("off_W", ctypes.c_size_t),
                ("off_Ut", ctypes.c_size_t), ("off_Kbar", ctypes.c_size_t),
                ("off_Qeff", ctypes.c_size_t), ("off_Opart", ctypes.c_size_t),
                ("off_gamma_last", ctypes.c_size_t), ("off_Mp", ctypes.c_size_t),
                ("off_Nc", ctypes.c_size_t), ("off_chunk_offsets", ctypes.c_size_t),
                ("off_status", ctypes.c_size_t), ("off_fix", ctypes.c_size_t),
                ("off_sync", ctypes.c_size_t), ("off_colscale", ctypes.c_size_t)]

    def as_dict(self):
        return {name: getattr(self, name) for name, _ in self._fields_}


def lib_path() -> str:
    return _LIB_PATH


def load_library():
    """Load ``libgdn2.so``; raises if it has not been built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        if not os.path.exists(_LIB_PATH):
            raise RuntimeError(f"{_LIB_PATH} is missing: build it with "
                               "`python -m gated_delta_rule_129_b200.build` (nvcc, sm_100a)")
        lib = ctypes.CDLL(_LIB_PATH)
        vp, i, f, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
        dp = ctypes.POINTER(Desc)
        lib.gdn2_workspace_size.argtypes = [dp]
        lib.gdn2_workspace_size.restype = sz
        lib.gdn2_workspace_layout.argtypes = [dp, ctypes.POINTER(WsLayout)]
        lib.gdn2_workspace_layout.restype = i
        lib.gdn2_chunk_fwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_fwd.restype = i
        lib.gdn2_chunk_fwd_noalloc.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_fwd_noalloc.restype = i
        lib.gdn2_noalloc_status.argtypes = [dp, vp, vp]
        lib.gdn2_noalloc_status.restype = i
        lib.gdn2_chunk_walk_flagged.argtypes = [dp, f, vp, vp, vp, vp, ctypes.c_ulonglong, vp]
        lib.gdn2_chunk_walk_flagged.restype = i
        lib.gdn2_segmented_workspace_size.argtypes = [dp, i]
        lib.gdn2_segmented_workspace_size.restype = sz
        lib.gdn2_chunk_fwd_segmented.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, i, vp]
        lib.gdn2_chunk_fwd_segmented.restype = i
        lib.gdn2_state_map.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.gdn2_state_map.restype = i
        lib.gdn2_token_prologue.argtypes = [dp, vp, vp, vp, vp, vp, vp, i, vp, vp, vp, vp, vp]
        lib.gdn2_token_prologue.restype = i
        lib.gdn2_token_epilogue.argtypes = [dp, vp, vp, vp, vp, vp]
        lib.gdn2_token_epilogue.restype = i
        lib.gdn2_chunk_prep.argtypes = [dp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_prep.restype = i
        lib.gdn2_chunk_walk.argtypes = [dp, f, vp, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_walk.restype = i
        lib.gdn2_chunk_plan.argtypes = [dp, vp, vp]
        lib.gdn2_chunk_plan.restype = i
        lib.gdn2_chunk_fused.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_fused.restype = i
        lib.gdn2_recurrent_step.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp]
        lib.gdn2_backward_workspace_size.argtypes = [dp]
        lib.gdn2_backward_workspace_size.restype = sz
        lib.gdn2_chunk_bwd.argtypes = [dp, vp, vp, vp, vp, vp, vp, f, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp, vp]
        lib.gdn2_chunk_bwd.restype = i
        lib.gdn2_recurrent_step.restype = i
        lib.gdn2_status_string.argtypes = [i]
        lib.gdn2_status_string.restype = ctypes.c_char_p
        lib.gdn2_version.argtypes = []
        lib.gdn2_version.restype = i
        _lib = lib
        return lib


def status_string(status: int) -> str:
    return load_library().gdn2_status_string(int(status)).decode()


def _check(status: int, where: str):
    if status != 0:
        raise GDN2Error(status, where)


# ------------------------------------------------------------------ helpers --

def _torch():
    import torch
    return torch


def _io_of(dtype) -> int:
    torch = _torch()
    if dtype == torch.float32:
        return GDN2_IO_F32
    if dtype == torch.bfloat16:
        return GDN2_IO_BF16
    raise TypeError(f"q/k/v must be float32 or bfloat16, got {dtype}")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    torch = _torch()
    s = stream if stream is not None else torch.cuda.current_stream()
    return ctypes.c_void_p(s.cuda_stream)


def make_desc(B, T, H, dk, dv, io, num_seqs=0, workspace=None, workspace_bytes=0) -> Desc:
    return Desc(int(B), int(T), int(H), int(dk), int(dv), int(num_seqs), int(io),
                None if workspace is None else ctypes.c_void_p(workspace),
                int(workspace_bytes))


def workspace_size(B, T, H, dk, dv, io=GDN2_IO_BF16, num_seqs=0) -> int:
    d = make_desc(B, T, H, dk, dv, io, num_seqs)
    return int(load_library().gdn2_workspace_size(ctypes.byref(d)))


def workspace_layout(B, T, H, dk, dv, io=GDN2_IO_BF16, num_seqs=0) -> dict:
    d = make_desc(B, T, H, dk, dv, io, num_seqs)
    lay = WsLayout()
    _check(load_library().gdn2_workspace_layout(ctypes.byref(d), ctypes.byref(lay)),
           "gdn2_workspace_layout")
    return lay.as_dict()


def _shapes(q, v, cu_seqlens):
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    num_seqs = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
    return B, T, H, dk, dv, num_seqs


def _alloc_workspace(desc_args, device):
    torch = _torch()
    nbytes = workspace_size(*desc_args)
    if nbytes == 0:
        raise GDN2Error(2, "gdn2_workspace_size")
    return torch.empty(nbytes, dtype=torch.uint8, device=device)


def _need_contig(*ts):
    for t in ts:
        if t is not None and not t.is_contiguous():
            raise ValueError("all tensors must be contiguous")


# -------------------------------------------------------------- entry points --

def chunk_fwd(q, k, v, log_alpha, b, w, scale=None, h0=None, cu_seqlens=None, *,
              out=None, hT=None, workspace=None, output_final_state=True, stream=None):
    """Gated DeltaNet-2 chunkwise forward.  Returns ``(out, hT)``.

    ``q, k, v`` are float32 or bfloat16 ``[B, T, H, d]`` CUDA tensors;
    ``log_alpha, b, w`` float32 of the same leading shape; ``h0`` float32
    ``[N, H, dk, dv]`` or None; ``cu_seqlens`` int32 ``[N + 1]`` CUDA tensor
    or None.  ``scale`` defaults to ``dk ** -0.5``.
    """
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    N = ns if cu_seqlens is not None else B
    if scale is None:
        scale = dk ** -0.5
    _need_contig(q, k, v, log_alpha, b, w, h0, cu_seqlens)
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _alloc_workspace((B, T, H, dk, dv, io, ns), q.device)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_fwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                       _ptr(b), _ptr(w), float(scale), _ptr(h0), _ptr(cu_seqlens),
                                       _ptr(out), _ptr(hT), _stream(stream))
    _check(st, "gdn2_chunk_fwd")
    return out, hT


def chunk_plan(shape, dtype, workspace, cu_seqlens=None, *, stream=None):
    """``gdn2_chunk_plan`` for ``shape = (B, T, H, dk, dv)`` into ``workspace``."""
    B, T, H, dk, dv = shape
    ns = 0 if cu_seqlens is None else cu_seqlens.numel() - 1
    d = make_desc(B, T, H, dk, dv, _io_of(dtype), ns, workspace.data_ptr(),
                  workspace.numel() * workspace.element_size())
    _check(load_library().gdn2_chunk_plan(ctypes.byref(d), _ptr(cu_seqlens), _stream(stream)), "gdn2_chunk_plan")


def chunk_fused(q, k, v, log_alpha, b, w, scale, workspace, h0=None, cu_seqlens=None, *, out, hT=None,
                stream=None):
    """``gdn2_chunk_fused``: the fused prep + walk launch alone (run
    :func:`chunk_plan` on the same workspace first).  Raises ``GDN2Error``
    (``GDN2_ERR_UNSUPPORTED``) when the problem does not take the fused path."""
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    _need_contig(q, k, v, log_alpha, b, w, h0, cu_seqlens)
    d = make_desc(B, T, H, dk, dv, _io_of(q.dtype), ns, workspace.data_ptr(),
                  workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_fused(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b),
                                         _ptr(w), float(scale), _ptr(h0), _ptr(cu_seqlens), _ptr(out), _ptr(hT),
                                         _stream(stream))
    _check(st, "gdn2_chunk_fused")
    return out, hT


NOALLOC_SCRATCH_BYTES = 32 << 20


def chunk_fwd_noalloc(q, k, v, log_alpha, b, w, scale=None, h0=None, cu_seqlens=None, *,
                      out=None, hT=None, output_final_state=True, stream=None):
    """``gdn2_chunk_fwd_noalloc``: like :func:`chunk_fwd`, but the library uses
    its own fixed device scratch (``NOALLOC_SCRATCH_BYTES``) instead of a
    workspace, for callers that cannot allocate device memory where they run
    the operator.  Problems whose workspace would exceed the scratch raise
    ``GDN2Error`` (``GDN2_ERR_WORKSPACE``).  Calls share the scratch, so calls
    that overlap on the GPU race; keep them on one stream.  ``out``/``hT``
    are allocated here only if not given."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    N = ns if cu_seqlens is not None else B
    if scale is None:
        scale = dk ** -0.5
    _need_contig(q, k, v, log_alpha, b, w, h0, cu_seqlens)
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    d = make_desc(B, T, H, dk, dv, io, ns)
    st = load_library().gdn2_chunk_fwd_noalloc(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                               _ptr(b), _ptr(w), float(scale), _ptr(h0), _ptr(cu_seqlens),
                                               _ptr(out), _ptr(hT), _stream(stream))
    _check(st, "gdn2_chunk_fwd_noalloc")
    return out, hT


def noalloc_status(q, v, cu_seqlens=None, *, stream=None):
    """``gdn2_noalloc_status``: the device status word of the last
    :func:`chunk_fwd_noalloc` call on inputs shaped like ``q``, ``v``
    (``cu_seqlens`` for a packed call), as an int32 CUDA tensor of one element
    filled on ``stream`` (0 = ok, 5 = malformed cu_seqlens, 8 = a bounded
    device wait gave up)."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    out = torch.empty(4, dtype=torch.int32, device=q.device)
    d = make_desc(B, T, H, dk, dv, _io_of(q.dtype), ns)
    _check(load_library().gdn2_noalloc_status(ctypes.byref(d), _ptr(out), _stream(stream)), "gdn2_noalloc_status")
    return out[:1]


def chunk_prep(q, k, v, log_alpha, b, w, cu_seqlens=None, *, workspace=None, stream=None):
    """Stage 1 only.  Returns the workspace tensor holding the chunk factors."""
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    _need_contig(q, k, v, log_alpha, b, w, cu_seqlens)
    if workspace is None:
        workspace = _alloc_workspace((B, T, H, dk, dv, io, ns), q.device)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_prep(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                        _ptr(b), _ptr(w), _ptr(cu_seqlens), _stream(stream))
    _check(st, "gdn2_chunk_prep")
    return workspace


def chunk_walk(workspace, shape, io_dtype, scale, h0=None, cu_seqlens=None, *, out=None, hT=None,
               chunk_states=None, stream=None):
    """Stage 2 only, from a workspace filled by :func:`chunk_prep`.

    ``shape`` is ``(B, T, H, dk, dv)``; ``io_dtype`` the torch dtype of q/k/v.
    Returns ``(out, hT)``.
    """
    torch = _torch()
    B, T, H, dk, dv = shape
    ns = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
    N = ns if cu_seqlens is not None else B
    io = _io_of(io_dtype)
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io_dtype, device=workspace.device)
    if hT is None:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=workspace.device)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_walk(ctypes.byref(d), float(scale), _ptr(h0), _ptr(cu_seqlens),
                                        _ptr(out), _ptr(hT), _ptr(chunk_states), _stream(stream))
    _check(st, "gdn2_chunk_walk")
    return out, hT


def chunk_walk_flagged(workspace, shape, io_dtype, scale, h0=None, cu_seqlens=None, *, out=None, hT=None,
                       wait_budget_ns=0, stream=None):
    """``gdn2_chunk_walk_flagged``: :func:`chunk_walk` that takes each chunk
    only once its ready flag in the workspace is raised, with every bounded
    device wait limited to ``wait_budget_ns`` (0 = 2 s).  Returns ``(out, hT)``;
    a wait that gave up shows in the workspace status word."""
    torch = _torch()
    B, T, H, dk, dv = shape
    ns = 0 if cu_seqlens is None else int(cu_seqlens.numel()) - 1
    N = ns if cu_seqlens is not None else B
    if out is None:
        out = torch.empty((B, T, H, dv), dtype=io_dtype, device=workspace.device)
    if hT is None:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=workspace.device)
    d = make_desc(B, T, H, dk, dv, _io_of(io_dtype), ns, workspace.data_ptr(),
                  workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_walk_flagged(ctypes.byref(d), float(scale), _ptr(h0), _ptr(cu_seqlens),
                                                _ptr(out), _ptr(hT), ctypes.c_ulonglong(int(wait_budget_ns)),
                                                _stream(stream))
    _check(st, "gdn2_chunk_walk_flagged")
    return out, hT


def segmented_workspace_size(B, T, H, dk, dv, io=GDN2_IO_BF16, num_seqs=0, segment_chunks=0) -> int:
    d = make_desc(B, T, H, dk, dv, io, num_seqs)
    return int(load_library().gdn2_segmented_workspace_size(ctypes.byref(d), int(segment_chunks)))


def chunk_fwd_segmented(q, k, v, log_alpha, b, w, scale=None, h0=None, cu_seqlens=None, *, segment_chunks=0,
                        out=None, hT=None, workspace=None, output_final_state=True, stream=None):
    """``gdn2_chunk_fwd_segmented``: :func:`chunk_fwd` through the two-level
    chunk scan, each sequence split into segments of ``segment_chunks``
    64-token chunks (0 = the library's choice).  Returns ``(out, hT)``."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    N = ns if cu_seqlens is not None else B
    if scale is None:
        scale = dk ** -0.5
    _need_contig(q, k, v, log_alpha, b, w, h0, cu_seqlens)
    if out is None:
        out = torch.empty(v.shape, dtype=q.dtype, device=q.device)
    if hT is None and output_final_state:
        hT = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        nbytes = segmented_workspace_size(B, T, H, dk, dv, io, ns, segment_chunks)
        if nbytes == 0:
            raise GDN2Error(9, "gdn2_segmented_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_fwd_segmented(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                                 _ptr(b), _ptr(w), float(scale), _ptr(h0), _ptr(cu_seqlens),
                                                 _ptr(out), _ptr(hT), int(segment_chunks), _stream(stream))
    _check(st, "gdn2_chunk_fwd_segmented")
    return out, hT


def state_map(q, k, v, log_alpha, b, w, cu_seqlens=None, *, phi=None, psi=None, workspace=None, stream=None):
    """``gdn2_state_map``: the affine map of every sequence, ``(phi [N, H, dk,
    dk], psi [N, H, dk, dv])`` fp32, with final state = phi @ S_start + psi."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    N = ns if cu_seqlens is not None else B
    _need_contig(q, k, v, log_alpha, b, w, cu_seqlens)
    if phi is None:
        phi = torch.empty((N, H, dk, dk), dtype=torch.float32, device=q.device)
    if psi is None:
        psi = torch.empty((N, H, dk, dv), dtype=torch.float32, device=q.device)
    if workspace is None:
        workspace = _alloc_workspace((B, T, H, dk, dv, io, ns), q.device)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_state_map(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b),
                                       _ptr(w), _ptr(cu_seqlens), _ptr(phi), _ptr(psi), _stream(stream))
    _check(st, "gdn2_state_map")
    return phi, psi


def token_prologue(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, cu_seqlens=None, *, q=None, k=None, v=None,
                   stream=None):
    """``gdn2_token_prologue``: ``(q, k, v)`` for the operator from the
    projections' outputs (short causal convolution with weights ``conv_*``
    ``[H * d, W]`` fp32, SiLU, and L2 normalisation of q and k)."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q_raw, v_raw, cu_seqlens)
    io = _io_of(q_raw.dtype)
    _need_contig(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, cu_seqlens)
    W = int(conv_q.shape[-1])
    q = torch.empty_like(q_raw) if q is None else q
    k = torch.empty_like(k_raw) if k is None else k
    v = torch.empty_like(v_raw) if v is None else v
    d = make_desc(B, T, H, dk, dv, io, ns)
    st = load_library().gdn2_token_prologue(ctypes.byref(d), _ptr(q_raw), _ptr(k_raw), _ptr(v_raw), _ptr(conv_q),
                                            _ptr(conv_k), _ptr(conv_v), W, _ptr(cu_seqlens), _ptr(q), _ptr(k), _ptr(v),
                                            _stream(stream))
    _check(st, "gdn2_token_prologue")
    return q, k, v


def token_epilogue(o, gate, norm_weight, *, out=None, stream=None):
    """``gdn2_token_epilogue``: ``rmsnorm(o) * norm_weight * sigmoid(gate)``."""
    torch = _torch()
    B, T, H, dv = o.shape
    _need_contig(o, gate, norm_weight)
    out = torch.empty_like(o) if out is None else out
    d = make_desc(B, T, H, 128, dv, _io_of(o.dtype))
    st = load_library().gdn2_token_epilogue(ctypes.byref(d), _ptr(o), _ptr(gate), _ptr(norm_weight), _ptr(out),
                                            _stream(stream))
    _check(st, "gdn2_token_epilogue")
    return out


def token_path_fwd(q_raw, k_raw, v_raw, log_alpha, b, w, gate, conv_q, conv_k, conv_v, norm_weight, scale=None,
                   h0=None, cu_seqlens=None, *, workspace=None, stream=None):
    """The operator with its token path: :func:`token_prologue`, then
    :func:`chunk_fwd`, then :func:`token_epilogue`.  Returns ``(out, hT)``
    (``out`` before the caller's output projection)."""
    q, k, v = token_prologue(q_raw, k_raw, v_raw, conv_q, conv_k, conv_v, cu_seqlens, stream=stream)
    o, hT = chunk_fwd(q, k, v, log_alpha, b, w, scale, h0, cu_seqlens, workspace=workspace, stream=stream)
    return token_epilogue(o, gate, norm_weight, out=o, stream=stream), hT


def backward_workspace_size(B, T, H, dk, dv, io=GDN2_IO_BF16, num_seqs=0) -> int:
    d = make_desc(B, T, H, dk, dv, io, num_seqs)
    return int(load_library().gdn2_backward_workspace_size(ctypes.byref(d)))


def chunk_bwd(q, k, v, log_alpha, b, w, scale, dO, h0=None, dhT=None, cu_seqlens=None, *, workspace=None,
              stream=None):
    """``gdn2_chunk_bwd``: gradients of :func:`chunk_fwd`'s ``(out, hT)``
    contracted with ``dO`` (``[B, T, H, dv]``, the dtype of ``q``) and ``dhT``
    (``[N, H, dk, dv]`` fp32 or None).  Returns a dict of fp32 tensors
    ``q, k, v, log_alpha, b, w`` (input shapes) and ``h0`` ``[N, H, dk, dv]``."""
    torch = _torch()
    B, T, H, dk, dv, ns = _shapes(q, v, cu_seqlens)
    io = _io_of(q.dtype)
    N = ns if cu_seqlens is not None else B
    _need_contig(q, k, v, log_alpha, b, w, h0, cu_seqlens, dO, dhT)
    if workspace is None:
        nbytes = backward_workspace_size(B, T, H, dk, dv, io, ns)
        if nbytes == 0:
            raise GDN2Error(2, "gdn2_backward_workspace_size")
        workspace = torch.empty(nbytes, dtype=torch.uint8, device=q.device)
    f32 = dict(dtype=torch.float32, device=q.device)
    g = {n: torch.empty(t.shape, **f32) for n, t in (("q", q), ("k", k), ("v", v), ("log_alpha", log_alpha),
                                                       ("b", b), ("w", w))}
    g["h0"] = torch.empty((N, H, dk, dv), **f32)
    d = make_desc(B, T, H, dk, dv, io, ns, workspace.data_ptr(), workspace.numel() * workspace.element_size())
    st = load_library().gdn2_chunk_bwd(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha), _ptr(b),
                                       _ptr(w), float(scale), _ptr(h0), _ptr(cu_seqlens), _ptr(dO), _ptr(dhT),
                                       _ptr(g["q"]), _ptr(g["k"]), _ptr(g["v"]), _ptr(g["log_alpha"]), _ptr(g["b"]),
                                       _ptr(g["w"]), _ptr(g["h0"]), _stream(stream))
    _check(st, "gdn2_chunk_bwd")
    return g


def recurrent_step(q, k, v, log_alpha, b, w, scale, state, *, out=None, stream=None):
    """One decode token; ``state`` ``[B, H, dk, dv]`` fp32 is updated in place.

    ``q, k, log_alpha, b`` are ``[B, H, dk]``; ``v, w`` ``[B, H, dv]``.
    Returns ``out`` ``[B, H, dv]``.
    """
    torch = _torch()
    Bn, H, dk = q.shape
    dv = v.shape[-1]
    io = _io_of(q.dtype)
    _need_contig(q, k, v, log_alpha, b, w, state)
    if out is None:
        out = torch.empty((Bn, H, dv), dtype=q.dtype, device=q.device)
    d = make_desc(Bn, 1, H, dk, dv, io)
    st = load_library().gdn2_recurrent_step(ctypes.byref(d), _ptr(q), _ptr(k), _ptr(v), _ptr(log_alpha),
                                            _ptr(b), _ptr(w), float(scale), _ptr(state), _ptr(out),
                                            _stream(stream))
    _check(st, "gdn2_recurrent_step")
    return out
