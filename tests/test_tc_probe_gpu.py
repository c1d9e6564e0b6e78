"""Building blocks of the tensor-core kernels, checked one at a time.

Each UMMA case places a random bf16 A (M x K) and B (K x N) in shared memory
in one of the operand layouts the kernels use (K-major SW128, MN-major
SW128, MN-major interleaved), runs the tcgen05.mma K-loop, reads the fp32
accumulator back from tensor memory and compares it with A @ B.  The TMA case
checks the byte image of a SWIZZLE_128B load against the software swizzle
the kernels use to write operands.  The probe library is built here from
tests/csrc/tc_probe.cu (it includes the product's tc.cuh)."""
import ctypes
import os
import subprocess

import numpy as np
import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "csrc", "tc_probe.cu")
LIB = os.path.join(ROOT, "tests", "csrc", "libtcprobe.so")
CSRC = os.path.join(ROOT, "gated_delta_rule_129_b200", "csrc")


def build_probe():
    deps = [SRC] + [os.path.join(CSRC, f) for f in ("tc.cuh", "tmap.cuh")]
    if os.path.exists(LIB) and all(os.path.getmtime(d) <= os.path.getmtime(LIB) for d in deps):
        return LIB
    tmp = LIB + f".tmp{os.getpid()}"
    subprocess.run(["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O2", "-std=c++17", "-shared",
                    "-Xcompiler", "-fPIC", "-I", CSRC, SRC, "-o", tmp], check=True)
    os.replace(tmp, LIB)
    return LIB


def test_probe_library_compiles():
    """Cross-compiles for sm_100a without a GPU."""
    assert os.path.exists(build_probe())


def sw128_off(row, e):
    b = e * 2
    return row * 128 + ((((b >> 4) ^ (row & 7)) << 4) | (b & 15))


@pytest.fixture(scope="module")
def probe(cuda_device):
    lib = ctypes.CDLL(build_probe())
    vp = ctypes.c_void_p
    lib.probe_umma.argtypes = [ctypes.c_int, vp, vp, vp, vp]
    lib.probe_tma.argtypes = [vp, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int, vp, vp]
    lib.probe_mode_shape.argtypes = [ctypes.c_int] + [ctypes.POINTER(ctypes.c_int)] * 3
    return lib


@pytest.mark.gpu
@pytest.mark.parametrize("mode", range(8))
def test_umma_layouts(probe, mode):
    import torch
    M, N, K = ctypes.c_int(), ctypes.c_int(), ctypes.c_int()
    assert probe.probe_mode_shape(mode, ctypes.byref(M), ctypes.byref(N), ctypes.byref(K)) == 0
    M, N, K = M.value, N.value, K.value
    g = torch.Generator(device="cpu").manual_seed(mode)
    A = torch.randn(M, K, generator=g).to(torch.bfloat16).cuda()
    B = torch.randn(K, N, generator=g).to(torch.bfloat16).cuda()
    D = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert probe.probe_umma(mode, A.data_ptr(), B.data_ptr(), D.data_ptr(), st.data_ptr()) == 0
    torch.cuda.synchronize()
    assert st.item() == 0, "bounded wait gave up"
    ref = A.float().cpu().double() @ B.float().cpu().double()
    got = D.cpu().double()
    err = (got - ref).abs().max().item()
    assert err < 1e-3 * max(1.0, ref.abs().max().item()), (mode, err)


@pytest.mark.gpu
@pytest.mark.parametrize("c0,c1,rows", [(0, 0, 64), (64, 3, 16), (64, 40, 128)])
def test_tma_swizzle_128b_image(probe, c0, c1, rows):
    import torch
    width, height = 128, 200
    vals = torch.arange(width * height, dtype=torch.int32).remainder(30000).to(torch.int16)
    src = vals.view(height, width).cuda()
    out = torch.zeros(rows * 128, dtype=torch.uint8, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert probe.probe_tma(src.data_ptr(), width, height, c0, c1, rows, out.data_ptr(), st.data_ptr()) == 0
    torch.cuda.synchronize()
    assert st.item() == 0
    img = out.cpu().numpy().view(np.int16)
    host = vals.view(height, width).numpy()
    for r in range(rows):
        for e in range(64):
            gr, gc = c1 + r, c0 + e
            want = host[gr, gc] if gr < height else 0
            assert img[sw128_off(r, e) // 2] == want, (r, e)
