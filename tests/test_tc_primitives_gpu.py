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
    lib.probe_skeleton.argtypes = [vp, vp, vp, vp, vp, vp, i, i, vp]
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


def _swz(tile):
    """bf16 [R][64] -> the 128-byte-swizzled byte image the kernels use
    (16-byte chunk c of row r stored at chunk position c ^ (r % 8))."""
    t = tile.contiguous().view(torch.int16).cpu().numpy().reshape(-1, 8, 8)
    R = t.shape[0]
    out = t.copy()
    for r in range(R):
        for p in range(8):
            out[r, p] = t[r, p ^ (r % 8)]
    return torch.from_numpy(out.reshape(-1)).view(torch.uint8)


@pytest.mark.parametrize("tma_T,mode", [(0, 0), (1, 0), (64, 0), (1, 1), (1, 8), (1, 4), (1, 2),
                                        (1, 15), (0, 16), (1, 31), (0, 32), (1, 32), (1, 63)])
def test_mma_tmem_choreography(lib, tma_T, mode):
    """Four commit/wait rounds on one barrier with interleaved MMAs of different
    shapes, tile stores while the tensor cores run, at the chunk kernel's
    shared-memory offsets (grid of two CTAs, 150 KB of shared memory).  With
    tma_T > 0 the K, Q and V tiles are TMA loads of real [1, T, 1, 128] tensors
    (rows past T zero-filled), as the chunk kernel issues them."""
    g = torch.Generator().manual_seed(5)
    bf = lambda *s: torch.randn(*s, generator=g).to(torch.bfloat16)
    K, Q, V = bf(64, 128), bf(64, 128), bf(64, 64)
    qd = kd = vd = None
    if tma_T:
        qd = bf(1, tma_T, 1, 128).cuda()
        kd = bf(1, tma_T, 1, 128).cuda()
        vd = bf(1, tma_T, 1, 128).cuda()
        Q = torch.zeros(64, 128, dtype=torch.bfloat16); Q[:tma_T] = qd[0, :, 0].cpu()
        K = torch.zeros(64, 128, dtype=torch.bfloat16); K[:tma_T] = kd[0, :, 0].cpu()
        Vfull = torch.zeros(64, 128, dtype=torch.bfloat16); Vfull[:tma_T] = vd[0, :, 0].cpu()
    Aqk, A1, A2, Wt, S = bf(64, 64), bf(64, 64), bf(64, 64), bf(64, 128), bf(128, 64)
    Ut, Us = bf(64, 64), bf(64, 64)
    img = torch.zeros(149056, dtype=torch.uint8)

    def put(off, tile):
        b = _swz(tile)
        img[off:off + b.numel()] = b

    put(0, K[:, :64]); put(8192, Q[:, :64]); put(16384, K[:, 64:]); put(24576, Q[:, 64:])
    put(32768, V); put(40960, Aqk); put(49152, A1); put(57344, A2)
    put(65536, Wt[:, :64]); put(73728, Wt[:, 64:]); put(81920, S)
    put(98304, Ut); put(106496, Us)
    tiles = img.cuda()
    out = torch.full((2, 40960), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    ptr = lambda t: None if t is None else _p(t)
    sink = torch.zeros(1, device="cuda")
    assert lib.probe_skeleton(_p(tiles), _p(out), _p(st), ptr(qd), ptr(kd), ptr(vd), tma_T, mode,
                              _p(sink)) == 0
    torch.cuda.synchronize()
    assert st.item() == 0
    f = lambda t: t.float()
    for cta in range(2):
        Vc = Vfull[:, 64 * cta:64 * cta + 64] if tma_T else V
        refs = [(0, (torch.cat([K, Q]).float() @ f(K).T)), (8192, f(A1) @ f(K)),
                (16384, f(A2) @ f(Vc)), (20480, f(Wt) @ f(S)), (24576, f(Q) @ f(S)),
                (28672, f(Aqk) @ f(Ut)), (32768, f(K).T @ f(Us))]
        for off, ref in refs:
            got = out[cta, off:off + ref.numel()].view(ref.shape).cpu()
            torch.testing.assert_close(got, ref, rtol=1e-5, atol=1e-3, msg=f"cta {cta} @ {off}")


@pytest.mark.parametrize("T,stages", [(1, 0), (64, 0), (1, 1), (64, 1), (1, 2), (64, 2), (1, 3),
                                      (64, 3)])
def test_chunk_prologue_on_skeleton(lib, T, stages):
    """The chunk kernel's own prologue code (gates from gate tensors, q norms,
    KK / QK epilogue, forward substitution, A1 / A2) on the validated skeleton,
    launched like the chunk kernel; then the W / U round on the computed tiles."""
    lib.probe_prologue.argtypes = [ctypes.c_void_p] * 8 + [ctypes.c_int, ctypes.c_float,
                                                           ctypes.c_void_p, ctypes.c_void_p,
                                                           ctypes.c_void_p, ctypes.c_int]
    g = torch.Generator(device="cuda").manual_seed(T)
    r = lambda *s, dt=torch.bfloat16: torch.randn(*s, device="cuda", generator=g).to(dt)
    q, k, v = r(1, T, 1, 128), r(1, T, 1, 128), r(1, T, 1, 128)
    a, b = r(1, T, 1), r(1, T, 1)
    A_log = torch.rand(1, device="cuda", generator=g) * 2.7
    dt_bias = -1 - 3 * torch.rand(1, device="cuda", generator=g)
    h0 = r(1, 1, 128, 128, dt=torch.float32) * 0.02
    o = torch.zeros(1, T, 1, 128, device="cuda", dtype=torch.bfloat16)
    out = torch.full((2, 69632), float("nan"), device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    rc = lib.probe_prologue(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(dt_bias), _p(h0), T,
                            128 ** -0.5, _p(o), _p(out), _p(st), stages)
    assert rc == 0, rc
    torch.cuda.synchronize()
    assert st.item() == 0
    K = torch.zeros(64, 128); K[:T] = k[0, :, 0].float().cpu()
    V = torch.zeros(64, 128); V[:T] = v[0, :, 0].float().cpu()
    for cta in range(2):
        A1 = out[cta, :4096].view(64, 64).cpu()
        A2 = out[cta, 4096:8192].view(64, 64).cpu()
        assert torch.isfinite(A1).all() and torch.isfinite(A2).all()
        torch.testing.assert_close(out[cta, 8192:16384].view(64, 128).cpu(), A1 @ K,
                                   rtol=1e-4, atol=1e-3)
        torch.testing.assert_close(out[cta, 16384:20480].view(64, 64).cpu(),
                                   A2 @ V[:, 64 * cta:64 * cta + 64], rtol=1e-4, atol=1e-3)
        Sb = h0[0, 0, :, 64 * cta:64 * cta + 64].to(torch.bfloat16).float().cpu()
        assert torch.equal(out[cta, 20480:28672].view(128, 64).cpu(), Sb)
        if stages >= 1:
            Wb = out[cta, 8192:16384].view(64, 128).cpu().to(torch.bfloat16).float()
            Q = torch.zeros(64, 128); Q[:T] = q[0, :, 0].float().cpu()
            torch.testing.assert_close(out[cta, 28672:32768].view(64, 64).cpu(), Wb @ Sb,
                                       rtol=1e-3, atol=1e-3)
            torch.testing.assert_close(out[cta, 32768:36864].view(64, 64).cpu(), Q @ Sb,
                                       rtol=1e-3, atol=1e-3)
        if stages >= 2:
            Aqk = out[cta, 36864:40960].view(64, 64).cpu()
            Ut = out[cta, 40960:45056].view(64, 64).cpu()
            Us = out[cta, 45056:49152].view(64, 64).cpu()
            torch.testing.assert_close(out[cta, 49152:53248].view(64, 64).cpu(), Aqk @ Ut,
                                       rtol=1e-3, atol=1e-3)
            Kb = K.to(torch.bfloat16).float()
            torch.testing.assert_close(out[cta, 53248:61440].view(128, 64).cpu(), Kb.T @ Us,
                                       rtol=1e-3, atol=1e-3)
        if stages >= 3:
            S_new = out[cta, 61440:69632].view(128, 64).cpu()
            assert torch.isfinite(S_new).all()
    if stages >= 3:
        assert torch.isfinite(o.float()).all()
