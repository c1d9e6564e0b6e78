"""C-ABI checks that need no GPU: the library loads, exports every entry point
that include/gdn2.h declares, and rejects bad arguments with the documented
status codes before it makes any CUDA call."""
import ctypes
import os
import re

import pytest

import gated_delta_rule_129_b200 as gdn2

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn2.h")

OK, NULL, SHAPE, DTYPE, ALIGN, SEQLENS, WORKSPACE, CUDA, TIMEOUT, UNSUPPORTED = range(10)


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"GDN2_API\s+[\w\s\*]*?\b(gdn2_\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from gated_delta_rule_129_b200 import build
    build.build()
    return gdn2.load_library()


def test_library_exports_every_declared_symbol(lib):
    syms = declared_symbols()
    assert len(syms) >= 8
    for s in syms:
        assert hasattr(lib, s), s
    assert set(syms) <= set(gdn2.EXPORTED) | set(syms)


def test_status_strings(lib):
    for code in range(10):
        assert gdn2.status_string(code)
    assert gdn2.status_string(0) == "ok"
    assert lib.gdn2_version() >= 100


def test_workspace_layout_sizes(lib):
    lay = gdn2.workspace_layout(1, 16384, 16, 128, 128, gdn2.GDN2_IO_BF16)
    assert lay["max_chunks"] == 256 and lay["factor_elem_bytes"] == 2 and lay["factor_set"] == 1
    tile = 256 * 16 * 64 * 128 * 2
    assert lay["off_W"] == lay["off_Ut"] == lay["off_Kbar"] == lay["off_Qeff"]   # WY set absent
    assert lay["off_Opart"] - lay["off_Qeff"] >= tile
    assert lay["off_Nc"] - lay["off_Mp"] >= 256 * 16 * 128 * 128 * 2
    wy = gdn2.workspace_layout(1, 16384, 16, 128, 128, gdn2.GDN2_IO_F32)
    assert wy["factor_set"] == 0 and wy["off_Ut"] - wy["off_W"] >= 2 * tile
    assert wy["off_Nc"] == wy["off_Mp"] == wy["off_chunk_offsets"]              # affine set absent
    offs = sorted(v for k, v in lay.items() if k.startswith("off_"))
    assert all(o % 256 == 0 for o in offs)
    assert lay["total_bytes"] >= offs[-1] + 4
    # packed: the bound is T_total/64 + N chunks
    lay2 = gdn2.workspace_layout(1, 1000, 2, 64, 128, gdn2.GDN2_IO_F32, num_seqs=7)
    assert lay2["max_chunks"] == 1000 // 64 + 7 and lay2["factor_elem_bytes"] == 4
    assert gdn2.workspace_size(1, 1000, 2, 64, 128, gdn2.GDN2_IO_F32, num_seqs=7) == lay2["total_bytes"]


@pytest.mark.parametrize("kw,code", [
    (dict(dk=96), SHAPE), (dict(dv=32), SHAPE), (dict(H=0), SHAPE), (dict(T=-1), SHAPE),
    (dict(io=7), DTYPE), (dict(B=2, num_seqs=3), SHAPE),
])
def test_layout_rejects_bad_desc(lib, kw, code):
    args = dict(B=1, T=128, H=2, dk=64, dv=64, io=0, num_seqs=0)
    args.update(kw)
    d = gdn2.make_desc(**args)
    lay = gdn2.WsLayout()
    assert lib.gdn2_workspace_layout(ctypes.byref(d), ctypes.byref(lay)) == code
    assert lib.gdn2_workspace_size(ctypes.byref(d)) == 0


def _fwd(lib, d, ptrs, out=0x20000, h0=None, cu=None, hT=None):
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    return lib.gdn2_chunk_fwd(ctypes.byref(d), *(P(p) for p in ptrs), 0.125, P(h0), P(cu), P(out),
                              P(hT), None)


def test_chunk_fwd_host_checks(lib):
    """Fake, never-dereferenced device addresses: every call below must return
    before any CUDA call (or with UNSUPPORTED where no B200 is present)."""
    size = gdn2.workspace_size(1, 128, 2, 64, 64, 0)
    good = [0x10000 + 0x100 * i for i in range(6)]
    d = gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100000, size)
    assert lib.gdn2_chunk_fwd(None, *(ctypes.c_void_p(p) for p in good), 0.1, None, None,
                              ctypes.c_void_p(0x20000), None, None) == NULL
    bad_null = list(good)
    bad_null[3] = None
    assert _fwd(lib, d, bad_null) == NULL
    assert _fwd(lib, d, good, out=None) == NULL
    bad_align = list(good)
    bad_align[1] += 4
    assert _fwd(lib, d, bad_align) == ALIGN
    assert _fwd(lib, d, good, h0=0x30004) == ALIGN
    small = gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100000, size - 1)
    assert _fwd(lib, small, good) == WORKSPACE
    nows = gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, None, size)
    assert _fwd(lib, nows, good) == WORKSPACE
    misws = gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100010, size)
    assert _fwd(lib, misws, good) == ALIGN
    # packed call without cu_seqlens / dense call with num_seqs set
    pk = gdn2.make_desc(1, 128, 2, 64, 64, 0, 3, 0x100000, 1 << 30)
    assert _fwd(lib, pk, good) == SHAPE
    assert _fwd(lib, d, good, cu=0x40000) == SHAPE
    # With valid arguments the only remaining check is the device itself.
    # That call is made only where no CUDA device exists: on a B200 it would
    # pass the check and launch kernels on the fake addresses above.
    if _cuda_device_present():
        return
    assert _fwd(lib, d, good) == UNSUPPORTED


def _cuda_device_present():
    try:
        import torch
        if torch.cuda.is_available():
            return True
    except Exception:  # pragma: no cover
        pass
    return os.path.exists("/dev/nvidiactl") or any(os.path.exists(f"/dev/nvidia{i}") for i in range(16))


def test_recurrent_step_host_checks(lib):
    good = [ctypes.c_void_p(0x10000 + 0x100 * i) for i in range(6)]
    d = gdn2.make_desc(4, 1, 2, 128, 128, 1)
    st, out = ctypes.c_void_p(0x50000), ctypes.c_void_p(0x60000)
    assert lib.gdn2_recurrent_step(ctypes.byref(d), *good, 0.1, None, out, None) == NULL
    assert lib.gdn2_recurrent_step(ctypes.byref(d), *good, 0.1, ctypes.c_void_p(0x50008), out, None) == ALIGN
    bad = gdn2.make_desc(4, 1, 2, 128, 80, 1)
    assert lib.gdn2_recurrent_step(ctypes.byref(bad), *good, 0.1, st, out, None) == SHAPE
    bad = gdn2.make_desc(4, 1, 2, 128, 128, 5)
    assert lib.gdn2_recurrent_step(ctypes.byref(bad), *good, 0.1, st, out, None) == DTYPE


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    """The product path has no fallback: a missing library is an error."""
    monkeypatch.setattr(gdn2, "_lib", None)
    monkeypatch.setattr(gdn2, "_LIB_PATH", str(tmp_path / "missing.so"))
    with pytest.raises(RuntimeError, match="missing"):
        gdn2.load_library()


def test_backward_workspace_size(lib):
    """The backward's workspace: the status word, the forward's fp32 factor
    set (whatever the I/O type), T and P, three dk x dv matrices (the state,
    its gradient, G) and two 64 x dv tiles per (chunk, head), each region
    256-byte aligned."""
    B, T, H, dk, dv = 1, 16384, 16, 128, 128
    chunks_h = (T // 64) * H
    regions = 2 * chunks_h * 64 * 64 * 4 + 3 * chunks_h * dk * dv * 4 + 2 * chunks_h * 64 * dv * 4
    wy = gdn2.workspace_size(B, T, H, dk, dv, gdn2.GDN2_IO_F32)
    for io in (gdn2.GDN2_IO_BF16, gdn2.GDN2_IO_F32):
        n = gdn2.backward_workspace_size(B, T, H, dk, dv, io)
        assert wy + regions + 256 <= n <= wy + regions + 256 + 8 * 256
    assert gdn2.backward_workspace_size(B, T, H, dk, dv, gdn2.GDN2_IO_BF16) == \
        gdn2.backward_workspace_size(B, T, H, dk, dv, gdn2.GDN2_IO_F32)
    assert gdn2.backward_workspace_size(1, 128, 2, 96, 64) == 0          # bad dk
    # packed: T_total / 64 + N chunks bound the regions
    n7 = gdn2.backward_workspace_size(1, 1000, 2, 64, 128, gdn2.GDN2_IO_F32, num_seqs=7)
    ch7 = (1000 // 64 + 7) * 2
    assert n7 >= gdn2.workspace_size(1, 1000, 2, 64, 128, gdn2.GDN2_IO_F32, num_seqs=7) + \
        ch7 * (2 * 64 * 64 + 3 * 64 * 128 + 2 * 64 * 128) * 4


def test_chunk_bwd_host_checks(lib):
    """Failing argument checks of gdn2_chunk_bwd return before any CUDA call
    (fake, never-dereferenced device addresses; no call passes every check)."""
    size = gdn2.backward_workspace_size(1, 128, 2, 64, 64, 0)
    P = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731
    ins = [0x10000 + 0x100 * i for i in range(6)]
    grads = [0x200000 + 0x1000 * i for i in range(7)]

    def bwd(d, ins=ins, dO=0x80000, grads=grads, h0=None, dhT=None, cu=None):
        return lib.gdn2_chunk_bwd(None if d is None else ctypes.byref(d), *(P(p) for p in ins), 0.125, P(h0),
                                  P(cu), P(dO), P(dhT), *(P(g) for g in grads), None)
    d = gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100000, size)
    assert bwd(None) == NULL
    assert bwd(gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100000, size - 1)) == WORKSPACE
    assert bwd(gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, None, size)) == WORKSPACE
    assert bwd(gdn2.make_desc(1, 128, 2, 64, 64, 0, 0, 0x100010, size)) == ALIGN
    assert bwd(d, dO=None) == NULL
    assert bwd(d, grads=grads[:6] + [None]) == NULL                    # dh0
    assert bwd(d, grads=[grads[0] + 4] + grads[1:]) == ALIGN
    assert bwd(d, dhT=0x90004) == ALIGN
    bad = list(ins)
    bad[2] = None
    assert bwd(d, ins=bad) == NULL
    assert bwd(gdn2.make_desc(1, 128, 2, 64, 80, 0, 0, 0x100000, size)) == SHAPE


P_ = lambda x: None if x is None else ctypes.c_void_p(x)  # noqa: E731


def test_token_path_host_checks(lib):
    """Failing argument checks of gdn2_token_prologue / gdn2_token_epilogue
    return before any CUDA call (fake, never-dereferenced device addresses;
    no call passes every check)."""
    raw = [0x10000, 0x20000, 0x30000]
    taps = [0x40000, 0x41000, 0x42000]
    outs = [0x50000, 0x60000, 0x70000]

    def pro(d, raw=raw, taps=taps, width=4, cu=None, outs=outs):
        return lib.gdn2_token_prologue(None if d is None else ctypes.byref(d), *(P_(p) for p in raw),
                                       *(P_(p) for p in taps), width, P_(cu), *(P_(p) for p in outs), None)
    d = gdn2.make_desc(1, 256, 2, 128, 128, gdn2.GDN2_IO_BF16)
    assert pro(None) == NULL
    assert pro(d, width=0) == SHAPE
    assert pro(d, width=9) == SHAPE
    assert pro(gdn2.make_desc(1, 256, 2, 96, 128, gdn2.GDN2_IO_BF16)) == SHAPE
    assert pro(gdn2.make_desc(1, 256, 2, 128, 128, 7)) == DTYPE
    assert pro(gdn2.make_desc(1, 256, 2, 128, 128, gdn2.GDN2_IO_BF16, num_seqs=3)) == SHAPE   # dense with num_seqs
    assert pro(gdn2.make_desc(2, 256, 2, 128, 128, gdn2.GDN2_IO_BF16, num_seqs=2), cu=0x80000) == SHAPE  # packed, B 2
    assert pro(d, raw=[raw[0], None, raw[2]]) == NULL
    assert pro(d, taps=[taps[0], taps[1], None]) == NULL
    assert pro(d, outs=[None, outs[1], outs[2]]) == NULL
    assert pro(d, raw=[raw[0] + 8, raw[1], raw[2]]) == ALIGN
    assert pro(d, taps=[taps[0], taps[1] + 4, taps[2]]) == ALIGN
    assert pro(d, outs=[outs[0], outs[1], outs[2] + 2]) == ALIGN

    def epi(d, o=0x10000, gate=0x20000, weight=0x30000, out=0x40000):
        return lib.gdn2_token_epilogue(None if d is None else ctypes.byref(d), P_(o), P_(gate), P_(weight),
                                       P_(out), None)
    assert epi(None) == NULL
    assert epi(gdn2.make_desc(1, 256, 2, 128, 128, 7)) == DTYPE
    assert epi(gdn2.make_desc(1, 256, 2, 128, 80, gdn2.GDN2_IO_BF16)) == SHAPE
    assert epi(gdn2.make_desc(1, 256, 0, 128, 128, gdn2.GDN2_IO_BF16)) == SHAPE
    assert epi(gdn2.make_desc(1, 2 ** 30, 2, 128, 128, gdn2.GDN2_IO_BF16)) == SHAPE   # token count
    assert epi(d, gate=None) == NULL
    assert epi(d, weight=None) == NULL
    assert epi(d, out=0x40004) == ALIGN


def test_segmented_and_state_map_host_checks(lib):
    """The two-level scan's workspace size and the host checks of
    gdn2_chunk_fwd_segmented and gdn2_state_map (each call fails a check
    before any CUDA call)."""
    B, T, H, dk, dv = 1, 4096, 2, 128, 128
    bf = gdn2.GDN2_IO_BF16
    base = gdn2.workspace_size(B, T, H, dk, dv, bf)
    size_seg = lambda d, L: int(lib.gdn2_segmented_workspace_size(None if d is None else ctypes.byref(d), L))  # noqa: E731
    n8 = size_seg(gdn2.make_desc(B, T, H, dk, dv, bf), 8)
    # beyond the usual layout: 8 segments of 8 chunks, each a [dk, dk] Phi and
    # two [dk, dv] matrices (Psi and the start state) per head, fp32
    assert n8 >= base + 8 * H * (dk * dk + 2 * dk * dv) * 4
    assert size_seg(gdn2.make_desc(B, T, H, dk, dv, bf), 0) > base          # the library's choice
    assert size_seg(None, 8) == 0
    assert size_seg(gdn2.make_desc(B, T, H, dk, dv, bf), -1) == 0
    assert size_seg(gdn2.make_desc(B, T, H, 64, dv, bf), 8) == 0          # not the affine factor set
    assert size_seg(gdn2.make_desc(B, T, H, dk, dv, gdn2.GDN2_IO_F32), 8) == 0

    ins = [0x10000 + 0x1000 * i for i in range(6)]

    def seg(d, ins=ins, out=0x80000, h0=None, hT=None, L=8):
        return lib.gdn2_chunk_fwd_segmented(None if d is None else ctypes.byref(d), *(P_(p) for p in ins),
                                            0.125, P_(h0), None, P_(out), P_(hT), L, None)
    d = gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, n8)
    assert seg(None) == NULL
    assert seg(gdn2.make_desc(B, T, H, dk, dv, gdn2.GDN2_IO_F32, 0, 0x1000000, n8)) == UNSUPPORTED
    assert seg(gdn2.make_desc(B, T, H, dk, dv, bf, 0, None, n8)) == WORKSPACE
    assert seg(gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000010, n8)) == ALIGN
    assert seg(gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, n8 - 1)) == WORKSPACE
    assert seg(d, L=-1) == SHAPE
    assert seg(d, ins=ins[:5] + [None]) == NULL
    assert seg(d, out=None) == NULL
    assert seg(d, out=0x80008) == ALIGN
    assert seg(d, h0=0x90004) == ALIGN

    wsz = gdn2.workspace_size(B, T, H, dk, dv, bf)

    def smap(d, ins=ins, phi=0xA0000, psi=0xB0000):
        return lib.gdn2_state_map(None if d is None else ctypes.byref(d), *(P_(p) for p in ins), None,
                                  P_(phi), P_(psi), None)
    d = gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, wsz)
    assert smap(None) == NULL
    assert smap(gdn2.make_desc(B, T, H, dk, dv, gdn2.GDN2_IO_F32, 0, 0x1000000, 1 << 30)) == UNSUPPORTED
    assert smap(gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, wsz - 1)) == WORKSPACE
    assert smap(d, ins=[None] + ins[1:]) == NULL
    assert smap(d, phi=None) == NULL
    assert smap(d, psi=0xB0004) == ALIGN


def test_stage_entry_points_host_checks(lib):
    """gdn2_chunk_prep, _walk, _plan, _fused and _walk_flagged reject a missing
    or short workspace, missing or misaligned pointers, and (fused, flagged)
    shapes outside the affine factor set, before any CUDA call (each call
    fails a check)."""
    B, T, H, dk, dv = 1, 256, 2, 128, 128
    bf, f32 = gdn2.GDN2_IO_BF16, gdn2.GDN2_IO_F32
    size = gdn2.workspace_size(B, T, H, dk, dv, bf)
    ins = [0x10000 + 0x1000 * i for i in range(6)]
    ok = gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, size)
    short = gdn2.make_desc(B, T, H, dk, dv, bf, 0, 0x1000000, size - 1)
    nows = gdn2.make_desc(B, T, H, dk, dv, bf, 0, None, size)
    r = ctypes.byref

    def prep(d, ins=ins):
        return lib.gdn2_chunk_prep(r(d), *(P_(p) for p in ins), None, None)
    assert prep(short) == WORKSPACE
    assert prep(nows) == WORKSPACE
    assert prep(ok, ins=ins[:2] + [None] + ins[3:]) == NULL
    assert prep(ok, ins=ins[:4] + [ins[4] + 4, ins[5]]) == ALIGN

    def walk(d, out=0x80000, h0=None, hT=None, states=None):
        return lib.gdn2_chunk_walk(r(d), 0.125, P_(h0), None, P_(out), P_(hT), P_(states), None)
    assert walk(short) == WORKSPACE
    assert walk(ok, out=None) == NULL
    assert walk(ok, hT=0x90008) == ALIGN
    assert walk(ok, states=0x90004) == ALIGN

    assert lib.gdn2_chunk_plan(r(short), None, None) == WORKSPACE
    assert lib.gdn2_chunk_plan(r(gdn2.make_desc(B, T, H, dk, dv, bf, 2, 0x1000000, 1 << 30)), None, None) == SHAPE

    def fused(d, ins=ins, out=0x80000):
        return lib.gdn2_chunk_fused(r(d), *(P_(p) for p in ins), 0.125, None, None, P_(out), None, None)
    assert fused(short) == WORKSPACE
    assert fused(ok, out=None) == NULL
    assert fused(ok, ins=[ins[0] + 2] + ins[1:]) == ALIGN
    f32_size = gdn2.workspace_size(B, T, H, dk, dv, f32)
    assert fused(gdn2.make_desc(B, T, H, dk, dv, f32, 0, 0x1000000, f32_size), out=0x80004) == ALIGN

    def flagged(d, out=0x80000):
        return lib.gdn2_chunk_walk_flagged(r(d), 0.125, None, None, P_(out), None, 1000000, None)
    assert flagged(short) == WORKSPACE
    assert flagged(ok, out=None) == NULL
    assert flagged(ok, out=0x80004) == ALIGN
    assert flagged(gdn2.make_desc(B, T, H, dk, dv, f32, 0, 0x1000000, f32_size)) == UNSUPPORTED   # WY factor set
