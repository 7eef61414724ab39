"""Single-CTA GPU probes of the sm_100a building blocks of the chunk kernel:
tensor-memory store/load, TMA 4-D tile loads with the 128-byte swizzle and
zero fill, and tcgen05.mma with K-major / MN-major operands at M = 64 and
M = 128 (accumulator lane layouts included), each checked against torch."""
import ctypes
import os
import subprocess

import pytest
import torch

pytestmark = pytest.mark.gpu

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
SRC = os.path.join(HERE, "csrc", "tc_probe.cu")
OUT = os.path.join(HERE, "_build", "libtcprobe.so")


def _lib():
    os.makedirs(os.path.dirname(OUT), exist_ok=True)
    deps = [SRC, os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "csrc", "tc_ptx.cuh"),
            os.path.join(ROOT, "gated_deltanet_sequence_gdn_b200", "csrc", "common.cuh")]
    if not os.path.exists(OUT) or os.path.getmtime(OUT) < max(os.path.getmtime(d) for d in deps):
        subprocess.run(["/usr/local/cuda/bin/nvcc", "-gencode", "arch=compute_100a,code=sm_100a",
                        "-O2", "-std=c++17", "-lineinfo", "-Xcompiler", "-fPIC", "-shared",
                        "-I", os.path.join(ROOT, "include"), "-o", OUT, SRC], check=True)
    lib = ctypes.CDLL(OUT)
    vp, i = ctypes.c_void_p, ctypes.c_int
    lib.probe_tmem_roundtrip.argtypes = [vp, vp]
    lib.probe_tma_load.argtypes = [vp, i, i, i, i, i, i, i, vp, vp]
    lib.probe_mma.argtypes = [vp, vp, vp, i, i, i, i, i, i, i, vp]
    return lib


@pytest.fixture(scope="module")
def lib():
    return _lib()


def _p(t):
    return ctypes.c_void_p(t.data_ptr())


def test_tmem_roundtrip(lib):
    out = torch.full((128 * 4 * 16,), -1.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.probe_tmem_roundtrip(_p(out), _p(st)) == 0
    torch.cuda.synchronize()
    tid = torch.arange(128).view(128, 1, 1)
    blk = torch.arange(4).view(1, 4, 1)
    c = torch.arange(16).view(1, 1, 16)
    ref = (tid * 1000 + blk * 100 + c).float().reshape(-1)
    assert torch.equal(out.cpu(), ref)
    assert st.item() == 0


@pytest.mark.parametrize("T,H,c0,h,t0", [(64, 1, 0, 0, 0), (100, 3, 64, 2, 64), (1, 1, 64, 0, 0)])
def test_tma_tile_load(lib, T, H, c0, h, t0):
    src = torch.randn(1, T, H, 128, device="cuda").to(torch.bfloat16)
    out = torch.full((64, 64), -7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.probe_tma_load(_p(src), T, H, c0, h, t0, 1, 0, _p(out), _p(st))
    assert rc == 0, rc
    torch.cuda.synchronize()
    ref = torch.zeros(64, 64)
    n = max(0, min(64, T - t0))
    ref[:n] = src[0, t0:t0 + n, h, c0:c0 + 64].float().cpu()
    assert st.item() == 0
    assert torch.equal(out.cpu(), ref)


@pytest.mark.parametrize("prefetch", [0, 1])
def test_tma_five_boxes_one_barrier(lib, prefetch):
    """Five boxes (both channel halves of q and k, and v, as the chunk kernel
    issues them) complete on one barrier; the tensor map may be prefetched."""
    T, H = 1, 1
    src = torch.randn(1, T, H, 128, device="cuda").to(torch.bfloat16)
    out = torch.full((5, 64, 64), -7.0, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.probe_tma_load(_p(src), T, H, 0, 0, 0, 5, prefetch, _p(out), _p(st))
    assert rc == 0, rc
    torch.cuda.synchronize()
    assert st.item() == 0
    for b in range(5):
        ref = torch.zeros(64, 64)
        ref[:1] = src[0, :1, 0, 64 * (b % 2):64 * (b % 2) + 64].float().cpu()
        assert torch.equal(out[b].cpu(), ref), b


@pytest.mark.parametrize("M,N,a_mn,b_mn,dcol,base_off,atom", [
    # operands high in a large dynamic shared-memory window, 16 KB atom stride
    (64, 128, 0, 1, 128, 65536, 16384), (128, 64, 1, 1, 0, 81920, 16384),
    (64, 64, 0, 1, 320, 98304, 8192), (128, 64, 0, 0, 64, 114688, 8192),
])
def test_mma_high_smem_and_wide_atoms(lib, M, N, a_mn, b_mn, dcol, base_off, atom):
    g = torch.Generator(device="cuda").manual_seed(base_off + atom)
    A = torch.randn(M, 64, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(64, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.probe_mma(_p(A), _p(B), _p(D), M, N, a_mn, b_mn, dcol, base_off, atom,
                         _p(st)) == 0
    torch.cuda.synchronize()
    assert st.item() == 0
    torch.testing.assert_close(D, A.float() @ B.float(), rtol=1e-5, atol=1e-4)


@pytest.mark.parametrize("M,N,a_mn,b_mn,dcol", [
    (128, 64, 0, 0, 0),   # [K;Q] K^T
    (64, 64, 0, 1, 0),    # U = A2 V ; P = W S ; Aqk U~
    (64, 128, 0, 1, 0),   # W = A1 K (two MN atoms in B)
    (128, 64, 1, 1, 0),   # S += K^T U~s (two MN atoms in A)
    (64, 64, 0, 0, 0), (128, 128, 0, 0, 0), (128, 128, 1, 0, 0),
    # accumulators away from column 0, as the chunk kernel places them
    (128, 64, 0, 0, 64), (64, 128, 0, 1, 128), (64, 64, 0, 1, 256), (64, 64, 0, 1, 320),
    (64, 64, 0, 1, 384), (64, 64, 0, 1, 448), (128, 64, 1, 1, 448),
])
def test_mma_layouts(lib, M, N, a_mn, b_mn, dcol):
    g = torch.Generator(device="cuda").manual_seed(M * 7 + N + 3 * a_mn + b_mn)
    A = torch.randn(M, 64, device="cuda", generator=g).to(torch.bfloat16)
    B = torch.randn(64, N, device="cuda", generator=g).to(torch.bfloat16)
    D = torch.full((M, N), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    assert lib.probe_mma(_p(A), _p(B), _p(D), M, N, a_mn, b_mn, dcol, 1024, 8192, _p(st)) == 0
    torch.cuda.synchronize()
    assert st.item() == 0
    ref = A.float() @ B.float()
    torch.testing.assert_close(D, ref, rtol=1e-5, atol=1e-4)
