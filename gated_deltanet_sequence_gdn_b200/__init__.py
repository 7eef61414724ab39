"""Python binding of libgdn.so, the B200 (sm_100a) Gated DeltaNet hot path.

Argument marshalling only: every step of the computation runs in the CUDA
kernels of libgdn.so, called through its C ABI (include/gdn.h) with ctypes.
PyTorch provides device memory and the current stream.  There is no CPU or
Python fallback: importing this module fails if the library is not built, and
every call raises if the library reports an error.

Entry points (same names as the C ABI):
    gdn_gate_prep, gdn_chunk_fwd, gdn_chunk_workspace_bytes, gdn_chunk_fwd_noalloc,
    gdn_recurrent_step, gdn2_chunk_fwd, gdn_check_status
"""
from __future__ import annotations

import ctypes
import os

import torch

__all__ = ["gdn_gate_prep", "gdn_chunk_fwd", "gdn_chunk_workspace_bytes", "gdn_recurrent_step",
           "gdn_conv_prefill", "gdn_rmsnorm_gated", "gdn_kda_chunk_fwd",
           "gdn_kda_chunk_workspace_bytes", "gdn_chunk_fwd_varlen",
           "gdn_chunk_varlen_workspace_bytes",
           "gdn2_chunk_fwd", "gdn2_chunk_workspace_bytes", "gdn_chunk_fwd_noalloc",
           "gdn_chunk_fwd_gated_norm", "gdn_recurrent_step_gated_norm",
           "gdn_chunk_bwd", "gdn_chunk_bwd_workspace_bytes",
           "gdn_check_status", "gdn_status", "gdn_test_set_wait_fault", "GDNError",
           "LIB_PATH", "lib", "F32", "BF16",
           "QK_L2NORM", "GATES_PRECOMPUTED", "OUT_F32"]

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libgdn.so")

if not os.path.exists(LIB_PATH):
    raise ImportError(
        f"{LIB_PATH} is missing: build it with `python gated_deltanet_sequence_gdn_b200/build.py`"
        " (nvcc, sm_100a). There is no fallback implementation.")

lib = ctypes.CDLL(LIB_PATH)

F32, BF16 = 0, 1
QK_L2NORM, GATES_PRECOMPUTED, OUT_F32 = 1, 2, 4
_STATUS = {0: "GDN_OK", -1: "GDN_ERR_INVALID_ARG", -2: "GDN_ERR_UNSUPPORTED",
           -3: "GDN_ERR_CUDA", -4: "GDN_ERR_TIMEOUT", -5: "GDN_ERR_WORKSPACE",
           -6: "GDN_ERR_RANGE"}

_vp, _i, _f, _sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_size_t
lib.gdn_gate_prep.argtypes = [_vp, _vp, _i, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _f,
                              _vp, _vp, _vp, _vp, _vp]
lib.gdn_chunk_fwd.argtypes = [_vp] * 8 + [_i] * 7 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
lib.gdn2_chunk_fwd.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
lib.gdn_chunk_fwd_noalloc.argtypes = [_vp] * 8 + [_i] * 7 + [_f, _i, _vp, _vp, _vp]
lib.gdn_chunk_fwd_host.argtypes = [_vp] * 8 + [_i] * 7 + [_f, _i, _vp, _vp, _i, _vp, _sz, _vp]
lib.gdn_chunk_fwd_host_workspace_bytes.argtypes = [_i] * 9
lib.gdn_chunk_fwd_host_workspace_bytes.restype = _sz
lib.gdn_recurrent_step.argtypes = [_vp] * 9 + [_i] * 6 + [_f, _i, _vp]
lib.gdn_conv_prefill.argtypes = [_vp] * 6 + [_i] * 7 + [_vp]
lib.gdn_rmsnorm_gated.argtypes = [_vp] * 4 + [ctypes.c_long, _i, _i, _f, _vp]
lib.gdn_chunk_fwd_varlen.argtypes = ([_vp] * 8 + [ctypes.POINTER(ctypes.c_longlong)] + [_i] * 6
                                     + [_f, _i, _vp, _vp, _vp, _sz, _vp])
lib.gdn_chunk_varlen_workspace_bytes.argtypes = [ctypes.POINTER(ctypes.c_longlong)] + [_i] * 6
lib.gdn_chunk_varlen_workspace_bytes.restype = _sz
lib.gdn_kda_chunk_fwd.argtypes = [_vp] * 8 + [_i] * 6 + [_f, _i, _vp, _vp, _vp, _sz, _vp]
lib.gdn_kda_chunk_workspace_bytes.argtypes = [_i] * 7
lib.gdn_kda_chunk_workspace_bytes.restype = _sz
lib.gdn_chunk_workspace_bytes.argtypes = [_i] * 7
lib.gdn2_chunk_workspace_bytes.argtypes = [_i] * 6
lib.gdn_chunk_workspace_bytes.restype = _sz
lib.gdn2_chunk_workspace_bytes.restype = _sz
lib.gdn_chunk_fwd_gated_norm.argtypes = [_vp] * 10 + [_f] + [_i] * 7 + [_f, _i, _vp, _vp, _vp,
                                                                       _sz, _vp]
lib.gdn_recurrent_step_gated_norm.argtypes = [_vp] * 10 + [_f, _vp] + [_i] * 6 + [_f, _i, _vp]
lib.gdn_chunk_bwd.argtypes = [_vp] * 10 + [_i] * 7 + [_f, _i] + [_vp] * 9 + [_sz, _vp]
lib.gdn_chunk_bwd_workspace_bytes.argtypes = [_i] * 6
lib.gdn_chunk_bwd_workspace_bytes.restype = _sz
lib.gdn_check_status.argtypes = [_vp]
lib.gdn_test_set_wait_fault.argtypes = [_i, ctypes.c_uint]
lib.gdn_test_set_wait_fault.restype = _i
lib.gdn_status_string.argtypes = [_i]
lib.gdn_status_string.restype = ctypes.c_char_p
lib.gdn_version.argtypes = []
for _fn in (lib.gdn_gate_prep, lib.gdn_chunk_fwd, lib.gdn_chunk_fwd_noalloc, lib.gdn_chunk_fwd_host,
            lib.gdn_chunk_fwd_gated_norm, lib.gdn_recurrent_step_gated_norm,
            lib.gdn2_chunk_fwd,
            lib.gdn_recurrent_step, lib.gdn_conv_prefill, lib.gdn_rmsnorm_gated,
            lib.gdn_kda_chunk_fwd, lib.gdn_chunk_fwd_varlen,
            lib.gdn_check_status, lib.gdn_version):
    _fn.restype = _i


class GDNError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


def _check(status: int, where: str):
    if status != 0:
        raise GDNError(status, where)


def _dtype_code(t: torch.dtype) -> int:
    if t == torch.bfloat16:
        return BF16
    if t == torch.float32:
        return F32
    raise TypeError(f"unsupported dtype {t}; expected bfloat16 or float32")


def _p(t):
    """Device pointer of a contiguous CUDA tensor (None -> NULL)."""
    if t is None:
        return None
    if not t.is_cuda:
        raise ValueError("tensor must live on a CUDA device")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _ph(t):
    """Host pointer of a contiguous CPU tensor (None -> NULL); page-locked memory
    (tensor.pin_memory()) gives asynchronous copies."""
    if t is None:
        return None
    if t.is_cuda:
        raise ValueError("tensor must live in host memory")
    if not t.is_contiguous():
        raise ValueError("tensor must be contiguous")
    return ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream)


def _need(t, dtype, shape, name):
    if t.dtype != dtype:
        raise TypeError(f"{name}: expected {dtype}, got {t.dtype}")
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")


def gdn_gate_prep(q, k, a, b, A_log, dt_bias, *, scale=None, q_out=None, k_out=None,
                  g_out=None, beta_out=None, stream=None):
    """Gate + L2-norm prologue. Returns (q_hat, k_hat, g, beta)."""
    B, T, Hk, d = q.shape
    Hv = a.shape[2]
    dt = q.dtype
    scale = d ** -0.5 if scale is None else scale
    q_out = torch.empty_like(q) if q_out is None else q_out
    k_out = torch.empty_like(k) if k_out is None else k_out
    g_out = torch.empty((B, T, Hv), device=q.device, dtype=torch.float32) if g_out is None else g_out
    beta_out = torch.empty_like(g_out) if beta_out is None else beta_out
    _need(k, dt, q.shape, "k")
    _need(a, dt, (B, T, Hv), "a")
    _need(b, dt, (B, T, Hv), "b")
    _check(lib.gdn_gate_prep(_p(q), _p(k), _dtype_code(dt), _p(a), _p(b), _p(A_log),
                             _p(dt_bias), B, T, Hk, Hv, d, float(scale), _p(q_out), _p(k_out),
                             _p(g_out), _p(beta_out), _stream(stream)), "gdn_gate_prep")
    return q_out, k_out, g_out, beta_out


def gdn_chunk_workspace_bytes(B, T, Hk, Hv, dk, dv, dtype) -> int:
    """Bytes of device workspace gdn_chunk_fwd needs for these sizes (0 = none)."""
    return int(lib.gdn_chunk_workspace_bytes(B, T, Hk, Hv, dk, dv, _dtype_code(dtype)))


def gdn_chunk_fwd(q, k, v, a, b, A_log=None, dt_bias=None, h0=None, *, scale=None,
                  l2norm=True, gates_precomputed=False, out_f32=False, o=None, ht=None,
                  want_ht=True, workspace=None, stream=None):
    """Chunkwise GDN prefill. q, k [B,T,Hk,dk]; v [B,T,Hv,dv]; a, b [B,T,Hv]
    (float32 g, beta with gates_precomputed); A_log, dt_bias [Hv] float32;
    h0 [B,Hv,dk,dv] float32 or None.  Returns (o [B,T,Hv,dv], ht or None);
    o has the input dtype, or float32 with out_f32.  workspace: a uint8 CUDA
    tensor of at least gdn_chunk_workspace_bytes(...) bytes, allocated here
    when None."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    gdt = torch.float32 if gates_precomputed else dt
    _need(a, gdt, (B, T, Hv), "a")
    _need(b, gdt, (B, T, Hv), "b")
    if h0 is not None:
        _need(h0, torch.float32, (B, Hv, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, Hv, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (B, T, Hv, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    ws_need = gdn_chunk_workspace_bytes(B, T, Hk, Hv, dk, dv, dt)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn_chunk_fwd(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(dt_bias), _p(h0),
                             B, T, Hk, Hv, dk, dv, _dtype_code(dt), float(scale), flags, _p(o),
                             _p(ht), _p(workspace), ws_bytes, _stream(stream)), "gdn_chunk_fwd")
    return o, ht


def gdn_chunk_fwd_gated_norm(q, k, v, a, b, A_log, dt_bias, h0, z, norm_weight, *, eps=1e-6,
                             scale=None, l2norm=True, gates_precomputed=False, out_f32=False,
                             o=None, ht=None, want_ht=True, workspace=None, stream=None):
    """gdn_chunk_fwd with the gated RMSNorm of the output stage applied to o:
    o = core / sqrt(mean(core^2) + eps) * norm_weight * SiLU(z) per (token, value
    head); z [B,T,Hv,dv] in the input dtype, norm_weight [dv] float32.  Fused into
    the scan's output store on the bf16 d = 128 path.  Returns (o, ht)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    gdt = torch.float32 if gates_precomputed else dt
    _need(a, gdt, (B, T, Hv), "a")
    _need(b, gdt, (B, T, Hv), "b")
    _need(z, dt, (B, T, Hv, dv), "z")
    _need(norm_weight, torch.float32, (dv,), "norm_weight")
    if h0 is not None:
        _need(h0, torch.float32, (B, Hv, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, Hv, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (B, T, Hv, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    ws_need = gdn_chunk_workspace_bytes(B, T, Hk, Hv, dk, dv, dt)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn_chunk_fwd_gated_norm(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log),
                                        _p(dt_bias), _p(h0), _p(z), _p(norm_weight),
                                        float(eps), B, T, Hk, Hv, dk, dv, _dtype_code(dt),
                                        float(scale), flags, _p(o), _p(ht), _p(workspace),
                                        ws_bytes, _stream(stream)), "gdn_chunk_fwd_gated_norm")
    return o, ht


def gdn_chunk_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv):
    return lib.gdn_chunk_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv)


def gdn_chunk_bwd(q, k, v, a, b, A_log, dt_bias, h0, do, dht=None, *, scale=None, l2norm=True,
                  gates_precomputed=False, want_dh0=True, workspace=None, stream=None):
    """Gradients of sum(o * do) + sum(ht * dht) for gdn_chunk_fwd's (o, ht) on the same
    inputs (see include/gdn.h).  Returns a dict of float32 tensors dq, dk [B,T,Hk,dk],
    dv [B,T,Hv,dv], da, db [B,T,Hv] (with gates_precomputed: with respect to g and
    beta), dA_log, ddt_bias [Hv] (None with gates_precomputed) and dh0 [B,Hv,dk,dv]
    (None unless want_dh0)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    _need(do, dt, (B, T, Hv, dv), "do")
    gdt = torch.float32 if gates_precomputed else dt
    _need(a, gdt, (B, T, Hv), "a")
    _need(b, gdt, (B, T, Hv), "b")
    if h0 is not None:
        _need(h0, torch.float32, (B, Hv, dk, dv), "h0")
    if dht is not None:
        _need(dht, torch.float32, (B, Hv, dk, dv), "dht")
    f32 = dict(device=q.device, dtype=torch.float32)
    out = {"dq": torch.empty((B, T, Hk, dk), **f32), "dk": torch.empty((B, T, Hk, dk), **f32),
           "dv": torch.empty((B, T, Hv, dv), **f32), "da": torch.empty((B, T, Hv), **f32),
           "db": torch.empty((B, T, Hv), **f32),
           "dA_log": None if gates_precomputed else torch.empty((Hv,), **f32),
           "ddt_bias": None if gates_precomputed else torch.empty((Hv,), **f32),
           "dh0": torch.empty((B, Hv, dk, dv), **f32) if want_dh0 else None}
    flags = (QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
    ws_need = gdn_chunk_bwd_workspace_bytes(B, T, Hk, Hv, dk, dv)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn_chunk_bwd(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(dt_bias), _p(h0),
                             _p(do), _p(dht), B, T, Hk, Hv, dk, dv, _dtype_code(dt),
                             float(scale), flags, _p(out["dq"]), _p(out["dk"]), _p(out["dv"]),
                             _p(out["da"]), _p(out["db"]), _p(out["dA_log"]),
                             _p(out["ddt_bias"]), _p(out["dh0"]), _p(workspace), ws_bytes,
                             _stream(stream)), "gdn_chunk_bwd")
    return out


def gdn_chunk_fwd_noalloc(q, k, v, a, b, A_log=None, dt_bias=None, h0=None, *, scale=None,
                          l2norm=True, gates_precomputed=False, out_f32=False, o=None, ht=None,
                          want_ht=True, stream=None):
    """gdn_chunk_fwd with the library's fixed 64 MiB device scratch instead of a
    workspace (raises GDNError(GDN_ERR_WORKSPACE) when the sizes need more)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    gdt = torch.float32 if gates_precomputed else dt
    _need(a, gdt, (B, T, Hv), "a")
    _need(b, gdt, (B, T, Hv), "b")
    if h0 is not None:
        _need(h0, torch.float32, (B, Hv, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, Hv, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (B, T, Hv, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    _check(lib.gdn_chunk_fwd_noalloc(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(dt_bias),
                                     _p(h0), B, T, Hk, Hv, dk, dv, _dtype_code(dt), float(scale),
                                     flags, _p(o), _p(ht), _stream(stream)),
           "gdn_chunk_fwd_noalloc")
    return o, ht


def gdn_chunk_fwd_host_workspace_bytes(B, T, Hk, Hv, dk, dv, dtype, *, l2norm=True,
                                       gates_precomputed=False, out_f32=False,
                                       piece_tokens=0) -> int:
    """Bytes of device scratch gdn_chunk_fwd_host needs for these sizes."""
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    return int(lib.gdn_chunk_fwd_host_workspace_bytes(B, T, Hk, Hv, dk, dv, _dtype_code(dtype),
                                                      flags, piece_tokens))


def gdn_chunk_fwd_host(q, k, v, a, b, A_log=None, dt_bias=None, h0=None, *, scale=None,
                       l2norm=True, gates_precomputed=False, out_f32=False, o=None, ht=None,
                       want_ht=True, piece_tokens=0, dev_workspace=None, device=None,
                       stream=None, sync=True):
    """gdn_chunk_fwd for host (CPU) tensors: the library copies the sequence to the
    device piece by piece, overlapping the copies in, the compute and the copies
    out.  Arguments as gdn_chunk_fwd, all CPU tensors (pin_memory() for
    asynchronous copies); o / ht are CPU tensors (page-locked when allocated
    here).  dev_workspace: a uint8 CUDA tensor of at least
    gdn_chunk_fwd_host_workspace_bytes(...) bytes, allocated here when None.
    Returns (o, ht); with sync=True (the default) once the stream has completed, so
    that they hold the results; with sync=False as soon as the work is enqueued (the
    host buffers are written asynchronously until the stream completes, and a
    dev_workspace allocated here must not be reused before then)."""
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    gdt = torch.float32 if gates_precomputed else dt
    _need(a, gdt, (B, T, Hv), "a")
    _need(b, gdt, (B, T, Hv), "b")
    if h0 is not None:
        _need(h0, torch.float32, (B, Hv, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, Hv, dv), dtype=odt).pin_memory() if o is None else o
    _need(o, odt, (B, T, Hv, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, Hv, dk, dv), dtype=torch.float32).pin_memory()
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    need = lib.gdn_chunk_fwd_host_workspace_bytes(B, T, Hk, Hv, dk, dv, _dtype_code(dt), flags,
                                                  piece_tokens)
    if dev_workspace is None and need > 0:
        dev = device if device is not None else torch.device("cuda", torch.cuda.current_device())
        dev_workspace = torch.empty(need, device=dev, dtype=torch.uint8)
    ws_bytes = 0 if dev_workspace is None else dev_workspace.numel() * dev_workspace.element_size()
    st = _stream(stream)
    _check(lib.gdn_chunk_fwd_host(_ph(q), _ph(k), _ph(v), _ph(a), _ph(b), _ph(A_log),
                                  _ph(dt_bias), _ph(h0), B, T, Hk, Hv, dk, dv, _dtype_code(dt),
                                  float(scale), flags, _ph(o), _ph(ht), int(piece_tokens),
                                  _p(dev_workspace), ws_bytes, st), "gdn_chunk_fwd_host")
    if sync:
        (stream if stream is not None else torch.cuda.current_stream()).synchronize()
    return o, ht


def gdn2_chunk_workspace_bytes(B, T, H, dk, dv, dtype) -> int:
    """Bytes of device workspace gdn2_chunk_fwd needs for these sizes (0 = none)."""
    return int(lib.gdn2_chunk_workspace_bytes(B, T, H, dk, dv, _dtype_code(dtype)))


def gdn2_chunk_fwd(q, k, v, a, b_logit, w_logit, A_log=None, dt_bias=None, h0=None, *,
                   scale=None, l2norm=True, gates_precomputed=False, out_f32=False, o=None,
                   ht=None, want_ht=True, workspace=None, stream=None):
    """Chunkwise Gated DeltaNet-2 forward. q, k, a, b_logit [B,T,H,dk]; v, w_logit
    [B,T,H,dv]; A_log, dt_bias [H,dk] float32; h0 [B,H,dk,dv] or None.  With
    gates_precomputed, a is the per-channel log-decay and b_logit / w_logit are
    the gate values (float32).  workspace as for gdn_chunk_fwd."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    gdt = torch.float32 if gates_precomputed else dt
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, H, dv), "v")
    _need(a, gdt, (B, T, H, dk), "a")
    _need(b_logit, gdt, (B, T, H, dk), "b_logit")
    _need(w_logit, gdt, (B, T, H, dv), "w_logit")
    if h0 is not None:
        _need(h0, torch.float32, (B, H, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, H, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (B, T, H, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    ws_need = gdn2_chunk_workspace_bytes(B, T, H, dk, dv, dt)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn2_chunk_fwd(_p(q), _p(k), _p(v), _p(a), _p(b_logit), _p(w_logit), _p(A_log),
                              _p(dt_bias), _p(h0), B, T, H, dk, dv, _dtype_code(dt),
                              float(scale), flags, _p(o), _p(ht), _p(workspace), ws_bytes,
                              _stream(stream)),
           "gdn2_chunk_fwd")
    return o, ht


def gdn_chunk_varlen_workspace_bytes(cu_seqlens, Hk, Hv, dk, dv, dtype) -> int:
    """Device workspace bytes gdn_chunk_fwd_varlen needs for these N + 1 token
    offsets (0 when the call needs none)."""
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    if len(cu) < 2:
        return 0
    arr = (ctypes.c_longlong * len(cu))(*cu)
    return int(lib.gdn_chunk_varlen_workspace_bytes(arr, len(cu) - 1, Hk, Hv, dk, dv,
                                                    _dtype_code(dtype)))


def gdn_chunk_fwd_varlen(q, k, v, a, b, A_log, dt_bias, h0, cu_seqlens, *, scale=None,
                         l2norm=True, gates_precomputed=False, out_f32=False, o=None, ht=None,
                         want_ht=True, workspace=None, stream=None):
    """Chunkwise GDN prefill over a packed batch: q, k [T_total, Hk, dk]; v
    [T_total, Hv, dv]; a, b [T_total, Hv]; cu_seqlens: N + 1 token offsets (a list
    or a CPU int64 tensor, first 0); h0 [N, Hv, dk, dv] or None.  Returns
    (o [T_total, Hv, dv], ht [N, Hv, dk, dv] or None)."""
    cu = [int(x) for x in (cu_seqlens.tolist() if hasattr(cu_seqlens, "tolist") else cu_seqlens)]
    N = len(cu) - 1
    Tt, Hk, dk = q.shape
    Hv, dv = v.shape[1], v.shape[2]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    gdt = torch.float32 if gates_precomputed else dt
    _need(k, dt, q.shape, "k")
    _need(v, dt, (Tt, Hv, dv), "v")
    _need(a, gdt, (Tt, Hv), "a")
    _need(b, gdt, (Tt, Hv), "b")
    if N < 0 or cu[0] != 0 or cu[-1] != Tt:
        raise ValueError("cu_seqlens must start at 0 and end at the packed token count")
    if h0 is not None:
        _need(h0, torch.float32, (N, Hv, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((Tt, Hv, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (Tt, Hv, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((N, Hv, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    cu_arr = (ctypes.c_longlong * len(cu))(*cu)
    ws_need = gdn_chunk_varlen_workspace_bytes(cu, Hk, Hv, dk, dv, dt)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn_chunk_fwd_varlen(_p(q), _p(k), _p(v), _p(a), _p(b), _p(A_log), _p(dt_bias),
                                    _p(h0), cu_arr, N, Hk, Hv, dk, dv, _dtype_code(dt),
                                    float(scale), flags, _p(o), _p(ht), _p(workspace), ws_bytes,
                                    _stream(stream)),
           "gdn_chunk_fwd_varlen")
    return o, ht


def gdn_kda_chunk_workspace_bytes(B, T, H, dk, dv, dtype, gates_precomputed=False) -> int:
    """Bytes of device workspace gdn_kda_chunk_fwd needs (the tiled gates included)."""
    return int(lib.gdn_kda_chunk_workspace_bytes(B, T, H, dk, dv, _dtype_code(dtype),
                                                 GATES_PRECOMPUTED if gates_precomputed else 0))


def gdn_kda_chunk_fwd(q, k, v, a, beta, A_log=None, dt_bias=None, h0=None, *, scale=None,
                      l2norm=True, gates_precomputed=False, out_f32=False, o=None, ht=None,
                      want_ht=True, workspace=None, stream=None):
    """Chunkwise KDA forward: Gated DeltaNet-2 with one beta per (token, head) for
    the erase and the write.  q, k, a [B,T,H,dk]; v [B,T,H,dv]; beta [B,T,H] (the
    logit, or beta in float32 with gates_precomputed, a then the per-channel
    log-decay); A_log, dt_bias [H,dk] float32; h0 [B,H,dk,dv] or None."""
    B, T, H, dk = q.shape
    dv = v.shape[3]
    dt = q.dtype
    scale = dk ** -0.5 if scale is None else scale
    gdt = torch.float32 if gates_precomputed else dt
    _need(k, dt, q.shape, "k")
    _need(v, dt, (B, T, H, dv), "v")
    _need(a, gdt, (B, T, H, dk), "a")
    _need(beta, gdt, (B, T, H), "beta")
    if h0 is not None:
        _need(h0, torch.float32, (B, H, dk, dv), "h0")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((B, T, H, dv), device=q.device, dtype=odt) if o is None else o
    _need(o, odt, (B, T, H, dv), "o")
    if ht is None and want_ht:
        ht = torch.empty((B, H, dk, dv), device=q.device, dtype=torch.float32)
    flags = ((QK_L2NORM if l2norm else 0) | (GATES_PRECOMPUTED if gates_precomputed else 0)
             | (OUT_F32 if out_f32 else 0))
    ws_need = gdn_kda_chunk_workspace_bytes(B, T, H, dk, dv, dt, gates_precomputed)
    if workspace is None and ws_need > 0:
        workspace = torch.empty(ws_need, device=q.device, dtype=torch.uint8)
    ws_bytes = 0 if workspace is None else workspace.numel() * workspace.element_size()
    _check(lib.gdn_kda_chunk_fwd(_p(q), _p(k), _p(v), _p(a), _p(beta), _p(A_log), _p(dt_bias),
                                 _p(h0), B, T, H, dk, dv, _dtype_code(dt), float(scale), flags,
                                 _p(o), _p(ht), _p(workspace), ws_bytes, _stream(stream)),
           "gdn_kda_chunk_fwd")
    return o, ht


def gdn_recurrent_step(x, conv_w, conv_state, a, b, A_log, dt_bias, state, *, Hk, Hv, dk,
                       dv, scale=None, out_f32=False, o=None, stream=None):
    """One fused conv1d + GDN decode step for N sequences; conv_state and state
    are updated in place.  x [N, 2*Hk*dk + Hv*dv]; returns o [N, Hv, dv]."""
    N = x.shape[0]
    dt = x.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(x, dt, (N, 2 * Hk * dk + Hv * dv), "x")
    _need(a, dt, (N, Hv), "a")
    _need(b, dt, (N, Hv), "b")
    _need(state, torch.float32, (N, Hv, dk, dv), "state")
    if conv_w is not None:
        _need(conv_w, torch.float32, (x.shape[1], 4), "conv_w")
        _need(conv_state, dt, (N, x.shape[1], 3), "conv_state")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((N, Hv, dv), device=x.device, dtype=odt) if o is None else o
    _need(o, odt, (N, Hv, dv), "o")
    _check(lib.gdn_recurrent_step(_p(x), _p(conv_w), _p(conv_state), _p(a), _p(b), _p(A_log),
                                  _p(dt_bias), _p(state), _p(o), N, Hk, Hv, dk, dv,
                                  _dtype_code(dt), float(scale), OUT_F32 if out_f32 else 0,
                                  _stream(stream)),
           "gdn_recurrent_step")
    return o


def gdn_recurrent_step_gated_norm(x, conv_w, conv_state, a, b, A_log, dt_bias, state, z,
                                  norm_weight, *, Hk, Hv, dk, dv, eps=1e-6, scale=None,
                                  out_f32=False, o=None, stream=None):
    """gdn_recurrent_step with the gated RMSNorm of the output stage fused into the
    store of o; z [N, Hv, dv] in the input dtype, norm_weight [dv] float32."""
    N = x.shape[0]
    dt = x.dtype
    scale = dk ** -0.5 if scale is None else scale
    _need(x, dt, (N, 2 * Hk * dk + Hv * dv), "x")
    _need(a, dt, (N, Hv), "a")
    _need(b, dt, (N, Hv), "b")
    _need(state, torch.float32, (N, Hv, dk, dv), "state")
    _need(z, dt, (N, Hv, dv), "z")
    _need(norm_weight, torch.float32, (dv,), "norm_weight")
    if conv_w is not None:
        _need(conv_w, torch.float32, (x.shape[1], 4), "conv_w")
        _need(conv_state, dt, (N, x.shape[1], 3), "conv_state")
    odt = torch.float32 if out_f32 else dt
    o = torch.empty((N, Hv, dv), device=x.device, dtype=odt) if o is None else o
    _need(o, odt, (N, Hv, dv), "o")
    _check(lib.gdn_recurrent_step_gated_norm(_p(x), _p(conv_w), _p(conv_state), _p(a), _p(b),
                                             _p(A_log), _p(dt_bias), _p(state), _p(z),
                                             _p(norm_weight), float(eps), _p(o), N, Hk, Hv, dk,
                                             dv, _dtype_code(dt), float(scale),
                                             OUT_F32 if out_f32 else 0, _stream(stream)),
           "gdn_recurrent_step_gated_norm")
    return o


def gdn_conv_prefill(x, conv_w, conv_state, *, Hk, Hv, dk, dv, q=None, k=None, v=None,
                     stream=None):
    """Causal conv1d (kernel 4) + SiLU over a prefill of the mixed stream
    x [B, T, 2*Hk*dk + Hv*dv]; conv_state [B, Cc, 3] (or None: a zero window) is
    read and then overwritten in place with the last three inputs.  Returns
    (q [B,T,Hk,dk], k [B,T,Hk,dk], v [B,T,Hv,dv]), not normalised."""
    B, T = x.shape[0], x.shape[1]
    dt = x.dtype
    Cc = 2 * Hk * dk + Hv * dv
    _need(x, dt, (B, T, Cc), "x")
    _need(conv_w, torch.float32, (Cc, 4), "conv_w")
    if conv_state is not None:
        _need(conv_state, dt, (B, Cc, 3), "conv_state")
    q = torch.empty((B, T, Hk, dk), device=x.device, dtype=dt) if q is None else q
    k = torch.empty((B, T, Hk, dk), device=x.device, dtype=dt) if k is None else k
    v = torch.empty((B, T, Hv, dv), device=x.device, dtype=dt) if v is None else v
    _need(q, dt, (B, T, Hk, dk), "q")
    _need(k, dt, (B, T, Hk, dk), "k")
    _need(v, dt, (B, T, Hv, dv), "v")
    _check(lib.gdn_conv_prefill(_p(x), _p(conv_w), _p(conv_state), _p(q), _p(k), _p(v), B, T,
                                Hk, Hv, dk, dv, _dtype_code(dt), _stream(stream)),
           "gdn_conv_prefill")
    return q, k, v


def gdn_rmsnorm_gated(o, z, weight, *, eps=1e-6, y=None, stream=None):
    """Gated RMSNorm of the core output over its last axis (d_v):
    y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z).  o, z [..., dv] (same shape
    and dtype); weight [dv] float32.  y may be o or z (in place)."""
    dt = o.dtype
    dv = o.shape[-1]
    _need(z, dt, tuple(o.shape), "z")
    _need(weight, torch.float32, (dv,), "weight")
    y = torch.empty_like(o) if y is None else y
    _need(y, dt, tuple(o.shape), "y")
    rows = o.numel() // dv if dv else 0
    _check(lib.gdn_rmsnorm_gated(_p(o), _p(z), _p(weight), _p(y), rows, dv, _dtype_code(dt),
                                 float(eps), _stream(stream)),
           "gdn_rmsnorm_gated")
    return y


def gdn_check_status(stream=None):
    """Synchronise the stream and raise if a bounded device wait expired or an
    fp16 operand left its range since the last check."""
    _check(lib.gdn_check_status(_stream(stream)), "gdn_check_status")


def gdn_status(stream=None) -> int:
    """Synchronise the stream, read and clear the device status word: the raw
    gdn_check_status code (0 = GDN_OK, -4 = GDN_ERR_TIMEOUT, -6 = GDN_ERR_RANGE)."""
    return int(lib.gdn_check_status(_stream(stream)))


def gdn_test_set_wait_fault(site: int, spin_limit: int = 0):
    """Test hook: make the tensor-core chunk kernels leave one bounded wait to
    expire (site 1: the scan's first state hand-off, site 2: the prep's K / Q
    tiles; 0: none), with spin_limit polls per wait (0 = the default)."""
    _check(lib.gdn_test_set_wait_fault(int(site), int(spin_limit)), "gdn_test_set_wait_fault")
