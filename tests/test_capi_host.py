"""The C-ABI library loads, exports every entry point include/gdn.h declares,
and rejects bad arguments on the host before touching a GPU (no CUDA call is
made on these paths, so they run without a device)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "gdn.h")

import gated_deltanet_sequence_gdn_b200 as G  # noqa: E402

FAKE = 0x10000  # 16-byte aligned, never dereferenced on the host paths tested


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:int|size_t|const char\*)\s+(gdn2?_\w+)\s*\(", src,
                                 flags=re.M)))


def test_header_declares_the_entry_points():
    names = declared_functions()
    for n in ("gdn_gate_prep", "gdn_chunk_fwd", "gdn_recurrent_step", "gdn2_chunk_fwd",
              "gdn_check_status", "gdn_status_string"):
        assert n in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(G.LIB_PATH)
    for n in declared_functions():
        assert hasattr(lib, n), f"{n} declared in gdn.h but not exported"


def test_only_declared_symbols_are_exported():
    import subprocess
    out = subprocess.run(["nm", "-D", "--defined-only", G.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = sorted(l.split()[-1] for l in out.splitlines() if l.strip())
    assert exported == declared_functions()


def test_status_strings_and_version():
    assert G.lib.gdn_status_string(0) == b"GDN_OK"
    assert G.lib.gdn_status_string(-1) == b"GDN_ERR_INVALID_ARG"
    assert G.lib.gdn_status_string(-4) == b"GDN_ERR_TIMEOUT"
    assert G.lib.gdn_status_string(-6) == b"GDN_ERR_RANGE"
    assert G.lib.gdn_status_string(12345) == b"GDN_ERR_UNKNOWN"
    assert G.lib.gdn_version() >= 100


def test_workspace_sizes():
    """Tensor-core path (bf16, d = 128): per padded token and value head an fp16
    W row (256 B), a float32 U row (512 B) and an fp16 A_qk row (128 B); per
    padded token and key head fp16 q and k rows (512 B); 1040 B of factors per
    chunk and value head."""
    ws = G.lib.gdn_chunk_workspace_bytes
    assert ws(1, 8192, 16, 64, 128, 128, 1) == 64 * (8192 * 896 + 128 * 1040) + 16 * 8192 * 512
    assert ws(2, 100, 2, 4, 128, 128, 1) == 2 * 4 * (128 * 896 + 2 * 1040) + 2 * 2 * 128 * 512
    assert ws(1, 64, 1, 1, 128, 128, 1) == 64 * 896 + 1040 + 64 * 512
    # no workspace: float32, other head sizes, empty inputs, Gated DeltaNet-2
    assert ws(1, 8192, 16, 64, 128, 128, 0) == 0
    assert ws(1, 256, 2, 2, 64, 64, 1) == 0
    assert ws(0, 256, 2, 2, 128, 128, 1) == 0
    assert ws(1, 0, 2, 2, 128, 128, 1) == 0
    # Gated DeltaNet-2 (bf16, d = 128): the same layout with one key head per head
    assert G.lib.gdn2_chunk_workspace_bytes(4, 4096, 16, 128, 128, 1) == \
        4 * 16 * (4096 * 896 + 64 * 1040) + 4 * 16 * 4096 * 512
    assert G.lib.gdn2_chunk_workspace_bytes(4, 4096, 16, 128, 128, 0) == 0


def test_missing_workspace_rejected():
    """A bf16 d = 128 call without (enough) workspace is refused before any launch."""
    assert _chunk() == -5
    need = 4 * (896 * 64 + 1040) + 2 * 64 * 512  # B=1, T=64, Hk=2, Hv=4
    assert _chunk(ws=FAKE, ws_bytes=need - 1) == -5
    assert _chunk(ws=FAKE + 8, ws_bytes=1 << 20) == -5  # misaligned
    assert _chunk(ws=FAKE, ws_bytes=need, flags=9) == -1  # a bad flag is reported first


def _chunk(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, h0=None,
                B=1, T=64, Hk=2, Hv=4, dk=128, dv=128, dtype=1, scale=0.1, flags=1, o=FAKE,
                ht=None, ws=None, ws_bytes=0)
    args.update(kw)
    return G.lib.gdn_chunk_fwd(args["q"], args["k"], args["v"], args["a"], args["b"],
                               args["A_log"], args["dt_bias"], args["h0"], args["B"],
                               args["T"], args["Hk"], args["Hv"], args["dk"], args["dv"],
                               args["dtype"], args["scale"], args["flags"], args["o"],
                               args["ht"], args["ws"], args["ws_bytes"], None)


@pytest.mark.parametrize("kw,expect", [
    (dict(q=None), -1), (dict(o=None), -1), (dict(a=None), -1),
    (dict(q=FAKE + 2), -1), (dict(h0=FAKE + 8), -1), (dict(ht=FAKE + 4), -1),
    (dict(dtype=7), -1), (dict(B=-1), -1), (dict(T=-5), -1), (dict(flags=8), -1),
    (dict(flags=16), -1),
    (dict(A_log=None), -1), (dict(Hk=0), -1),
    (dict(dk=96), -2), (dict(dv=32), -2), (dict(Hk=3, Hv=4), -2),
])
def test_chunk_rejects_bad_arguments(kw, expect):
    assert _chunk(**kw) == expect


def test_gdn2_and_decode_reject_bad_arguments():
    L = G.lib
    assert L.gdn2_chunk_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, 1, 64, 2,
                            128, 128, 1, 0.1, 1, FAKE, None, None, 0, None) == -1
    assert L.gdn2_chunk_fwd(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, 1, 64, 2,
                            100, 128, 1, 0.1, 1, FAKE, None, None, 0, None) == -2
    # bf16, d = 128 (the tensor-core path) copies the gate tiles in 16-byte pieces:
    # element-aligned but not 16-byte-aligned gates are refused there, not on the
    # float32 path
    for bad in ((FAKE + 2, FAKE, FAKE), (FAKE, FAKE + 2, FAKE), (FAKE, FAKE, FAKE + 2)):
        assert L.gdn2_chunk_fwd(FAKE, FAKE, FAKE, *bad, FAKE, FAKE, None, 1, 64, 2, 128, 128, 1,
                                0.1, 1, FAKE, None, FAKE, 1 << 30, None) == -1
    # decode: conv weights given but no conv state
    assert L.gdn_recurrent_step(FAKE, FAKE, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 4,
                                128, 128, 1, 0.1, 0, None) == -1
    assert L.gdn_recurrent_step(FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 4, 6,
                                128, 128, 1, 0.1, 0, None) == -2
    assert L.gdn_recurrent_step(FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 4, 2, 4,
                                128, 128, 1, 0.1, 1, None) == -1
    assert L.gdn_gate_prep(FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, 4, 80, 0.1, FAKE,
                           FAKE, FAKE, FAKE, None) == -2
    assert L.gdn_gate_prep(FAKE, None, 1, FAKE, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 0.1, FAKE,
                           FAKE, FAKE, FAKE, None) == -1


def test_conv_prefill_rejects_bad_arguments():
    cp = G.lib.gdn_conv_prefill
    # (x, conv_w, conv_state, q, k, v, B, T, Hk, Hv, dk, dv, dtype, stream)
    assert cp(None, FAKE, None, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE, None, None, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE, FAKE, None, FAKE, None, FAKE, 1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE + 8, FAKE, None, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE, FAKE, FAKE + 1, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE, FAKE, None, FAKE, FAKE, FAKE, -1, 8, 2, 4, 128, 128, 1, None) == -1
    assert cp(FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 8, 2, 4, 128, 128, 7, None) == -1
    assert cp(FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 8, 2, 4, 96, 128, 1, None) == -2
    assert cp(FAKE, FAKE, None, FAKE, FAKE, FAKE, 1, 16 * 65535 + 1, 2, 4, 128, 128, 1,
              None) == -2
    # no tokens or no sequences: nothing enqueued, the window untouched
    assert cp(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 1, 0, 2, 4, 128, 128, 1, None) == 0
    assert cp(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 8, 2, 4, 128, 128, 1, None) == 0


def test_rmsnorm_gated_rejects_bad_arguments():
    rn = G.lib.gdn_rmsnorm_gated
    # (o, z, weight, y, rows, dv, dtype, eps, stream)
    assert rn(None, FAKE, FAKE, FAKE, 8, 128, 1, 1e-6, None) == -1
    assert rn(FAKE, FAKE, None, FAKE, 8, 128, 1, 1e-6, None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE + 8, 8, 128, 1, 1e-6, None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE, -1, 128, 1, 1e-6, None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE, 8, 128, 5, 1e-6, None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE, 8, 128, 1, -1.0, None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE, 8, 128, 1, float("nan"), None) == -1
    assert rn(FAKE, FAKE, FAKE, FAKE, 8, 96, 1, 1e-6, None) == -2
    assert rn(FAKE, FAKE, FAKE, FAKE, 0, 128, 1, 1e-6, None) == 0


def test_kda_workspace_and_arguments():
    """KDA's workspace: gdn2_chunk_fwd's, then the tiled erase and write gates
    (B*T*H rows of dk and dv gate elements), each rounded up to 256 bytes."""
    L = G.lib
    up = lambda x: (x + 255) // 256 * 256
    B, T, H, d = 2, 100, 3, 128
    for dtype, flags, ges in ((1, 0, 2), (1, 2, 4), (0, 0, 4)):
        want = (up(L.gdn2_chunk_workspace_bytes(B, T, H, d, d, dtype)) + 2 * up(B * T * H * d * ges))
        assert L.gdn_kda_chunk_workspace_bytes(B, T, H, d, d, dtype, flags) == want
    assert L.gdn_kda_chunk_workspace_bytes(-1, T, H, d, d, 1, 0) == 0
    n = L.gdn_kda_chunk_workspace_bytes(B, T, H, d, d, 1, 0)
    kda = L.gdn_kda_chunk_fwd
    # (q, k, v, a, beta, A_log, dt_bias, h0, B, T, H, dk, dv, dtype, scale, flags, o, ht,
    #  ws, ws_bytes, stream)
    assert kda(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, B, T, H, d, d, 1, 0.1, 1, FAKE,
               None, FAKE, n, None) == -1
    assert kda(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, B, T, H, d, d, 1, 0.1, 1, FAKE,
               None, None, 0, None) == -5
    assert kda(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, B, T, H, d, d, 1, 0.1, 1, FAKE,
               None, FAKE, n - 1, None) == -5
    assert kda(FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, B, T, H, 96, d, 1, 0.1, 1, FAKE,
               None, FAKE, 1 << 40, None) == -2
    # no tokens: nothing to tile, no state to copy
    assert kda(FAKE, FAKE, FAKE, FAKE, None, FAKE, FAKE, None, B, 0, H, d, d, 1, 0.1, 1, FAKE,
               None, None, 0, None) == 0


def test_varlen_checks_cu_seqlens_before_anything():
    import ctypes as C
    vl = G.lib.gdn_chunk_fwd_varlen
    arr = lambda *xs: (C.c_longlong * len(xs))(*xs)
    # (q, k, v, a, b, A_log, dt_bias, h0, cu, N, Hk, Hv, dk, dv, dtype, scale, flags, o, ht,
    #  ws, ws_bytes, stream)
    args = lambda cu, N, **kw: [kw.get("q", FAKE), FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, None, cu,
                                N, 2, 4, 128, 128, 1, 0.1, 1, FAKE, None,
                                kw.get("ws", FAKE), kw.get("ws_bytes", 1 << 40), None]
    assert vl(*args(arr(0, 5), 0)) == 0                    # N = 0
    assert vl(*args(None, 2)) == -1                        # no offsets
    assert vl(*args(arr(1, 5, 9), 2)) == -1                # does not start at 0
    assert vl(*args(arr(0, 9, 5), 2)) == -1                # decreasing
    assert vl(*args(arr(0, 0, 0), 2)) == 0                 # empty sequences, no ht: nothing
    assert vl(*args(arr(0, 64, 100), 2, ws=None, ws_bytes=0)) == -5
    assert vl(*args(arr(0, 64, 100), 2, q=None)) == -1
    # the workspace holds every chunk of the packed batch and its sequence table
    wsb = G.lib.gdn_chunk_varlen_workspace_bytes
    need = wsb(arr(0, 64, 364), 2, 2, 4, 128, 128, 1)
    assert need >= G.lib.gdn_chunk_workspace_bytes(1, 6 * 64, 2, 4, 128, 128, 1)
    assert vl(*args(arr(0, 64, 364), 2, ws_bytes=need - 1)) == -5
    assert wsb(arr(0, 64, 364), 2, 2, 4, 64, 64, 1) == 0      # the CUDA-core path: none
    assert wsb(arr(0, 64, 364), 2, 2, 4, 128, 128, 0) == 0    # float32: none
    assert wsb(arr(0, 9, 5), 2, 2, 4, 128, 128, 1) == 0       # decreasing offsets
    # empty sequences take no chunk: only the table's space
    assert wsb(arr(0, 0, 0), 2, 2, 4, 128, 128, 1) == wsb(arr(0, 0), 1, 2, 4, 128, 128, 1) > 0


def test_empty_calls_are_no_ops():
    # zero tokens / zero sequences return before any launch (no state pointers)
    assert _chunk(T=0) == 0
    assert _chunk(B=0) == 0
    assert G.lib.gdn_recurrent_step(FAKE, None, None, FAKE, FAKE, FAKE, FAKE, FAKE, FAKE, 0, 2,
                                    4, 128, 128, 1, 0.1, 0, None) == 0
    assert G.lib.gdn_gate_prep(FAKE, FAKE, 1, FAKE, FAKE, FAKE, FAKE, 1, 0, 2, 4, 128, 0.1,
                               FAKE, FAKE, FAKE, FAKE, None) == 0


def test_host_pipeline_workspace_bytes():
    """gdn_chunk_fwd_host's device scratch: two sets of piece buffers (q, k, v, a, b),
    two output pieces, the state, A_log and dt_bias, and the piece's chunk workspace,
    each rounded up to 256 bytes."""
    up = lambda x: (x + 255) // 256 * 256
    B, T, Hk, Hv, d, Tc = 1, 8192, 16, 64, 128, 1024
    rows = [Hk * d * 2, Hk * d * 2, Hv * d * 2, Hv * 2, Hv * 2]
    want = 2 * sum(up(B * Tc * r) for r in rows) + 2 * up(B * Tc * Hv * d * 2)
    want += up(B * Hv * d * d * 4) + 2 * up(Hv * 4)
    want += up(G.lib.gdn_chunk_workspace_bytes(B, Tc, Hk, Hv, d, d, 1))
    fn = G.lib.gdn_chunk_fwd_host_workspace_bytes
    assert fn(B, T, Hk, Hv, d, d, 1, 1, 0) == want          # default: about T / 8 per piece
    assert fn(B, T, Hk, Hv, d, d, 1, 1, 1000) == want       # rounded up to whole chunks
    # float32 outputs and precomputed (float32) gates widen the rows
    assert fn(B, T, Hk, Hv, d, d, 1, 1 | 4, 1024) > want
    assert fn(B, T, Hk, Hv, d, d, 1, 1 | 2, 1024) > want
    assert fn(0, T, Hk, Hv, d, d, 1, 1, 0) == 0 and fn(B, 0, Hk, Hv, d, d, 1, 1, 0) == 0
    assert fn(B, T, Hk, Hv, d, d, 9, 1, 0) == 0


def test_host_pipeline_rejects_bad_arguments():
    """Refusals before any CUDA call: null inputs or outputs, negative sizes, a
    missing or too small device scratch; B = 0 does nothing."""
    f = G.lib.gdn_chunk_fwd_host
    args = [FAKE] * 7 + [None, 1, 64, 2, 4, 128, 128, 1, 0.1, 1, FAKE, None, 64, None, 0, None]
    assert f(*args) == -5                                    # no device scratch
    bad = list(args); bad[0] = None
    assert f(*bad) == -1                                     # q missing
    bad = list(args); bad[17] = None
    assert f(*bad) == -1                                     # o missing
    bad = list(args); bad[9] = -1
    assert f(*bad) == -1                                     # negative T
    bad = list(args); bad[8] = 0
    assert f(*bad) == 0                                      # B = 0: nothing to do
    bad = list(args); bad[20] = FAKE; bad[21] = 1024
    assert f(*bad) == -5                                     # scratch too small


def _bwd(**kw):
    args = dict(q=FAKE, k=FAKE, v=FAKE, a=FAKE, b=FAKE, A_log=FAKE, dt_bias=FAKE, h0=None,
                do=FAKE, dht=None, B=1, T=64, Hk=2, Hv=4, dk=128, dv=128, dtype=1, scale=0.1,
                flags=1, dq=FAKE, dk_out=FAKE, dv_out=FAKE, da=FAKE, db=FAKE, dA_log=FAKE,
                ddt_bias=FAKE, dh0=None, ws=None, ws_bytes=0)
    args.update(kw)
    names = ("q", "k", "v", "a", "b", "A_log", "dt_bias", "h0", "do", "dht", "B", "T", "Hk",
             "Hv", "dk", "dv", "dtype", "scale", "flags", "dq", "dk_out", "dv_out", "da",
             "db", "dA_log", "ddt_bias", "dh0", "ws", "ws_bytes")
    return G.lib.gdn_chunk_bwd(*[args[n] for n in names], None)


def test_backward_arguments_checked_before_any_launch():
    """gdn_chunk_bwd refuses bad arguments and a short workspace on the host."""
    assert _bwd(dk=128, dv=64) == -2          # GDN_ERR_UNSUPPORTED: dk != dv
    assert _bwd(dk=96, dv=96) == -2           # head size outside {64, 128}
    assert _bwd(Hk=3, Hv=4) == -2             # Hv % Hk != 0
    assert _bwd(flags=4) == -1                # GDN_OUT_F32 has no meaning here
    assert _bwd(dtype=7) == -1
    assert _bwd(A_log=None) == -1             # gates from logits need A_log ...
    assert _bwd(dA_log=None) == -1            # ... and somewhere for its gradient
    assert _bwd(dq=FAKE + 4) == -1            # misaligned output
    assert _bwd() == -5                       # no workspace
    need = G.lib.gdn_chunk_bwd_workspace_bytes(1, 64, 2, 4, 128, 128)
    assert need > 0
    assert _bwd(ws=FAKE, ws_bytes=need - 1) == -5
    assert G.lib.gdn_chunk_bwd_workspace_bytes(1, 0, 2, 4, 128, 128) == 0
    assert G.lib.gdn_chunk_bwd_workspace_bytes(1, 64, 2, 4, 128, 64) == 0
