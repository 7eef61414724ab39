"""fp64 CPU oracle for the Gated DeltaNet hot path -- TEST INFRASTRUCTURE ONLY.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  The product library never does, and the
two share no code: the arithmetic lives in ``gdn_oracle.c`` (plain C, double
precision, token by token), compiled here with gcc and called through ctypes.

Each function cites the passage it follows (page title and section):

* ``gdn_fwd``      -- "Qwen3.5" (rainlin-net), section GDN详解: the five-step
  recurrence and the gate lines of the module skeleton.
* ``gate_prep``    -- same gate lines; "从 Full Attention 到 Gated DeltaNet"
  section 9 (alpha = e^g, softplus).
* ``decode_step``  -- "gated-deltanet-qwen3.5" architecture diagram (decode
  updates conv_states / recurrent_states) and section 10 of the dingfen page
  (Linear -> CausalConv1D -> SiLU -> q, k, v).
* ``conv_step`` / ``conv_prefill`` -- that conv alone, for one token or a whole
  prefill ("gated-deltanet-qwen3.5" section 因果卷积: kernel 4, depthwise, causal).
* ``gdn_bwd`` / ``gdn2_bwd`` -- the backward of ``gdn_fwd`` / ``gdn2_fwd`` (the
  training direction of the method; "Gated DeltaNet-2", Gate-aware 反向传播 for the
  second): reverse-mode through the same steps, pinned by finite differences.
* ``kda_fwd``      -- "Gated DeltaNet-2" (zhichai), section 标量绑定的数学表达 (the
  KDA update with its erase projection written out) and 退化兼容性.
* ``rmsnorm_gated`` -- "gated-deltanet-qwen3.5" section 输出门控与 RMSNorm
  (RMSNormGated(core_attn_out, z): the norm, then the SwiGLU-like z gate).
* ``gdn2_fwd``     -- "Gated DeltaNet-2" (zhichai), section 新更新公式.

Parity: pinned by tests/test_oracle_pins.py (closed forms, special cases,
brute force; see the header of gdn_oracle.c for the list).
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_BUILD = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into oracle/_build/libgdn_oracle.so (gcc, OpenMP)."""
    os.makedirs(_BUILD, exist_ok=True)
    if (not force and os.path.exists(_LIB_PATH)
            and os.path.getmtime(_LIB_PATH) >= os.path.getmtime(_SRC)):
        return _LIB_PATH
    tmp = _LIB_PATH + f".tmp{os.getpid()}"
    cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
           "-Wall", "-Wextra", "-o", tmp, _SRC, "-lm"]
    subprocess.run(cmd, check=True)
    os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            vp, ip, dp = ctypes.c_void_p, ctypes.c_int, ctypes.c_double
            lib.oracle_gdn_fwd.argtypes = [vp] * 8 + [ip] * 7 + [dp, ip, ip, ip, vp, vp, vp, ip]
            lib.oracle_gate_prep.argtypes = [vp] * 6 + [ip] * 6 + [dp] + [vp] * 4
            lib.oracle_gdn_decode_step.argtypes = [vp] * 6 + [ip] * 6 + [dp, ip, vp, vp, vp, vp, ip]
            lib.oracle_gdn2_fwd.argtypes = [vp] * 9 + [ip] * 6 + [dp, ip, ip, ip, vp, vp, vp, ip]
            lib.oracle_conv_step.argtypes = [vp, vp, ip, ip, ip, vp, vp]
            lib.oracle_conv_prefill.argtypes = [vp, vp, ip, ip, ip, ip, vp, vp]
            lib.oracle_rmsnorm_gated.argtypes = [vp, vp, vp, ip, ip, ip, dp, vp]
            lib.oracle_kda_fwd.argtypes = [vp] * 8 + [ip] * 6 + [dp, ip, vp, vp, ip]
            lib.oracle_gdn_bwd.argtypes = [vp] * 10 + [ip] * 6 + [dp, ip, ip] + [vp] * 8
            lib.oracle_gdn2_bwd.argtypes = [vp] * 11 + [ip] * 5 + [dp, ip, ip] + [vp] * 9
            for f in (lib.oracle_gdn_fwd, lib.oracle_gate_prep, lib.oracle_conv_step,
                      lib.oracle_conv_prefill, lib.oracle_rmsnorm_gated, lib.oracle_kda_fwd,
                      lib.oracle_gdn_bwd, lib.oracle_gdn2_bwd,
                      lib.oracle_gdn_decode_step, lib.oracle_gdn2_fwd):
                f.restype = ctypes.c_int
            lib.oracle_max_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def _arr(x, f64: bool):
    """numpy array (C-contiguous, float64 or float32) from numpy / torch CPU input."""
    if x is None:
        return None
    if hasattr(x, "detach"):
        x = x.detach().cpu()
        x = x.double().numpy() if f64 else x.float().numpy()
    return np.ascontiguousarray(x, dtype=np.float64 if f64 else np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _sel(sel):
    if sel is None:
        return 0, None, None
    s = np.ascontiguousarray(np.asarray(sel, dtype=np.int32))
    return int(s.size), s, s.ctypes.data_as(ctypes.c_void_p)


def _check(rc: int, name: str):
    if rc != 0:
        raise RuntimeError(f"{name} failed with status {rc}")


def _is_f64(*xs) -> bool:
    for x in xs:
        if x is None:
            continue
        dt = getattr(x, "dtype", None)
        if dt is not None and str(dt) in ("float64", "torch.float64"):
            return True
    return False


def gdn_fwd(q, k, v, a, b, A_log=None, dt_bias=None, h0=None, *, scale=None,
            l2norm=True, gates_given=False, heads=None, want_o=True,
            want_ht=True, threads=None):
    """Token-by-token GDN forward.

    q, k: [B,T,Hk,dk]; v: [B,T,Hv,dv]; a, b: [B,T,Hv] (or g, beta when
    ``gates_given``); A_log, dt_bias: [Hv]; h0: [B,Hv,dk,dv] or None.
    ``heads``: list of flat indices b*Hv+hv to compute (None = all).
    Returns (o, ht): with heads=None, o is [B,T,Hv,dv] and ht [B,Hv,dk,dv];
    with a selection, o is [n_sel,T,dv] and ht [n_sel,dk,dv].  float64.
    """
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    f64 = _is_f64(q, k, v, a, b, A_log, dt_bias, h0)
    arrs = [_arr(x, f64) for x in (q, k, v, a, b, A_log, dt_bias, h0)]
    if gates_given:
        arrs[5] = arrs[6] = None
    if scale is None:
        scale = dk ** -0.5
    n_sel, sel_arr, sel_p = _sel(heads)
    nh = n_sel if n_sel else B * Hv
    o = np.zeros((nh, T, dv), np.float64) if want_o else None
    ht = np.zeros((nh, dk, dv), np.float64) if want_ht else None
    rc = _load().oracle_gdn_fwd(*[_ptr(x) for x in arrs], int(f64), B, T, Hk, Hv, dk, dv,
                                float(scale), int(l2norm), int(gates_given), n_sel, sel_p,
                                _ptr(o), _ptr(ht), int(threads or max_threads()))
    _check(rc, "oracle_gdn_fwd")
    del sel_arr
    if heads is None:
        if o is not None:
            o = o.reshape(B, Hv, T, dv).transpose(0, 2, 1, 3).copy()
        if ht is not None:
            ht = ht.reshape(B, Hv, dk, dv)
    return o, ht


def gate_prep(q, k, a, b, A_log, dt_bias, *, scale=None):
    """Gate + L2-norm prologue: returns (q_hat, k_hat, g, beta), float64."""
    B, T, Hk, d = q.shape
    Hv = a.shape[2]
    f64 = _is_f64(q, k, a, b, A_log, dt_bias)
    arrs = [_arr(x, f64) for x in (q, k, a, b, A_log, dt_bias)]
    if scale is None:
        scale = d ** -0.5
    qh = np.zeros((B, T, Hk, d)); kh = np.zeros((B, T, Hk, d))
    g = np.zeros((B, T, Hv)); beta = np.zeros((B, T, Hv))
    rc = _load().oracle_gate_prep(*[_ptr(x) for x in arrs], int(f64), B, T, Hk, Hv, d,
                                  float(scale), _ptr(qh), _ptr(kh), _ptr(g), _ptr(beta))
    _check(rc, "oracle_gate_prep")
    return qh, kh, g, beta


def conv_step(x, conv_w, conv_state):
    """Causal depthwise conv1d (k=4) + SiLU for one new input per channel.

    x: [N, Cc]; conv_w: [Cc, 4]; conv_state: float64 [N, Cc, 3] updated IN PLACE.
    Returns y [N, Cc] float64.
    """
    N, Cc = x.shape
    f64 = _is_f64(x, conv_w)
    xa, wa = _arr(x, f64), _arr(conv_w, f64)
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert conv_state.shape == (N, Cc, 3)
    y = np.zeros((N, Cc))
    rc = _load().oracle_conv_step(_ptr(xa), _ptr(wa), int(f64), N, Cc, _ptr(conv_state), _ptr(y))
    _check(rc, "oracle_conv_step")
    return y


def conv_prefill(x, conv_w, conv_state):
    """The conv step over a whole prefill, token after token.

    x: [B, T, Cc]; conv_w: [Cc, 4]; conv_state: float64 [B, Cc, 3] updated IN
    PLACE (it ends holding the last three inputs).  Returns y [B, T, Cc] float64.
    """
    B, T, Cc = x.shape
    f64 = _is_f64(x, conv_w)
    xa, wa = _arr(x, f64), _arr(conv_w, f64)
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert conv_state.shape == (B, Cc, 3)
    y = np.zeros((B, T, Cc))
    rc = _load().oracle_conv_prefill(_ptr(xa), _ptr(wa), int(f64), B, T, Cc, _ptr(conv_state),
                                     _ptr(y))
    _check(rc, "oracle_conv_prefill")
    return y


def gdn_bwd(q, k, v, a, b, A_log, dt_bias, h0, do, dht=None, *, scale=None, l2norm=True,
            gates_given=False):
    """Gradients of sum(o * do) + sum(ht * dht) for gdn_fwd's (o, ht), by reverse-mode
    differentiation of the token recurrence (float64 throughout).

    Shapes as for gdn_fwd; do [B,T,Hv,dv]; dht [B,Hv,dk,dv] or None.  Returns a dict
    with dq, dk, dv, da, db, dA_log, ddt_bias, dh0 (with gates_given, da / db are the
    gradients with respect to g and beta, and dA_log / ddt_bias are None).
    """
    B, T, Hk, dk = q.shape
    Hv, dv = v.shape[2], v.shape[3]
    f = lambda x: None if x is None else _arr(x, True)
    arrs = [f(x) for x in (q, k, v, a, b, A_log, dt_bias, h0, do, dht)]
    if scale is None:
        scale = dk ** -0.5
    out = {"dq": np.zeros((B, T, Hk, dk)), "dk": np.zeros((B, T, Hk, dk)),
           "dv": np.zeros((B, T, Hv, dv)), "da": np.zeros((B, T, Hv)), "db": np.zeros((B, T, Hv)),
           "dA_log": None if gates_given else np.zeros(Hv),
           "ddt_bias": None if gates_given else np.zeros(Hv), "dh0": np.zeros((B, Hv, dk, dv))}
    rc = _load().oracle_gdn_bwd(*[_ptr(x) for x in arrs], B, T, Hk, Hv, dk, dv, float(scale),
                                int(l2norm), int(gates_given),
                                *[_ptr(out[n]) for n in ("dq", "dk", "dv", "da", "db", "dA_log",
                                                         "ddt_bias", "dh0")])
    _check(rc, "oracle_gdn_bwd")
    return out


def gdn2_bwd(q, k, v, a, b_logit, w_logit, A_log, dt_bias, h0, do, dht=None, *, scale=None,
             l2norm=True, gates_given=False):
    """Gradients of sum(o * do) + sum(ht * dht) for gdn2_fwd's (o, ht) (float64).

    Returns a dict with dq, dk, dv, da, db, dw, dA_log, ddt_bias, dh0 (with
    gates_given: da, db, dw with respect to g, b, w; dA_log / ddt_bias None).
    """
    B, T, H, dk = q.shape
    dv = v.shape[3]
    f = lambda x: None if x is None else _arr(x, True)
    arrs = [f(x) for x in (q, k, v, a, b_logit, w_logit, A_log, dt_bias, h0, do, dht)]
    if scale is None:
        scale = dk ** -0.5
    out = {"dq": np.zeros((B, T, H, dk)), "dk": np.zeros((B, T, H, dk)),
           "dv": np.zeros((B, T, H, dv)), "da": np.zeros((B, T, H, dk)),
           "db": np.zeros((B, T, H, dk)), "dw": np.zeros((B, T, H, dv)),
           "dA_log": None if gates_given else np.zeros((H, dk)),
           "ddt_bias": None if gates_given else np.zeros((H, dk)),
           "dh0": np.zeros((B, H, dk, dv))}
    rc = _load().oracle_gdn2_bwd(*[_ptr(x) for x in arrs], B, T, H, dk, dv, float(scale),
                                 int(l2norm), int(gates_given),
                                 *[_ptr(out[n]) for n in ("dq", "dk", "dv", "da", "db", "dw",
                                                          "dA_log", "ddt_bias", "dh0")])
    _check(rc, "oracle_gdn2_bwd")
    return out


def kda_fwd(q, k, v, a, b, A_log, dt_bias, h0=None, *, scale=None, l2norm=True,
            threads=None):
    """Token-by-token KDA forward, the literal matrix form of its update.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; a: [B,T,H,dk] (per-channel decay input);
    b: [B,T,H] (beta logit); A_log, dt_bias: [H,dk]; h0: [B,H,dk,dv] or None.
    Returns (o [B,T,H,dv], ht [B,H,dk,dv]) float64.
    """
    B, T, H, dk = q.shape
    dv = v.shape[3]
    f64 = _is_f64(q, k, v, a, b, A_log, dt_bias, h0)
    arrs = [_arr(x, f64) for x in (q, k, v, a, b, A_log, dt_bias, h0)]
    scale = dk ** -0.5 if scale is None else scale
    o = np.zeros((B * H, T, dv))
    ht = np.zeros((B * H, dk, dv))
    rc = _load().oracle_kda_fwd(*[_ptr(x) for x in arrs], int(f64), B, T, H, dk, dv,
                                float(scale), int(l2norm), _ptr(o), _ptr(ht),
                                int(threads or max_threads()))
    _check(rc, "oracle_kda_fwd")
    return o.reshape(B, H, T, dv).transpose(0, 2, 1, 3).copy(), ht.reshape(B, H, dk, dv)


def rmsnorm_gated(o, z, weight, *, eps=1e-6):
    """Gated RMSNorm of the core output: per row of the last axis (d_v),
    y = o / sqrt(mean(o^2) + eps) * weight * SiLU(z).

    o, z: [..., dv] (same shape); weight: [dv].  Returns y float64, o's shape.
    """
    f64 = _is_f64(o, z, weight)
    oa, za, wa = _arr(o, f64), _arr(z, f64), _arr(weight, f64)
    assert oa.shape == za.shape and wa.shape == (oa.shape[-1],)
    dv = oa.shape[-1]
    N = oa.size // dv
    y = np.zeros(oa.shape)
    rc = _load().oracle_rmsnorm_gated(_ptr(oa), _ptr(za), _ptr(wa), int(f64), N, dv, float(eps),
                                      _ptr(y))
    _check(rc, "oracle_rmsnorm_gated")
    return y


def decode_step(x, conv_w, a, b, A_log, dt_bias, conv_state, state, *, Hk, Hv,
                dk, dv, scale=None, seqs=None, threads=None):
    """One fused conv1d + GDN decode step.

    x: [N, Cc]; conv_w: [Cc,4] or None (x already post-conv); a, b: [N,Hv].
    conv_state [n_sel,Cc,3] and state [n_sel,Hv,dk,dv] are float64 numpy arrays,
    updated IN PLACE (compact over ``seqs``; all N when seqs is None).
    Returns o [n_sel,Hv,dv] float64.
    """
    N = x.shape[0]
    f64 = _is_f64(x, conv_w, a, b, A_log, dt_bias)
    arrs = [_arr(t, f64) for t in (x, conv_w, a, b, A_log, dt_bias)]
    if scale is None:
        scale = dk ** -0.5
    n_sel, sel_arr, sel_p = _sel(seqs)
    ns = n_sel if n_sel else N
    assert conv_state.dtype == np.float64 and conv_state.flags.c_contiguous
    assert state.dtype == np.float64 and state.flags.c_contiguous
    assert conv_state.shape == (ns, 2 * Hk * dk + Hv * dv, 3)
    assert state.shape == (ns, Hv, dk, dv)
    o = np.zeros((ns, Hv, dv))
    rc = _load().oracle_gdn_decode_step(*[_ptr(t) for t in arrs], int(f64), N, Hk, Hv, dk, dv,
                                        float(scale), n_sel, sel_p, _ptr(conv_state),
                                        _ptr(state), _ptr(o), int(threads or max_threads()))
    _check(rc, "oracle_gdn_decode_step")
    del sel_arr
    return o


def gdn2_fwd(q, k, v, a, b_logit, w_logit, A_log=None, dt_bias=None, h0=None, *,
             scale=None, l2norm=True, gates_given=False, heads=None, want_o=True,
             want_ht=True, threads=None):
    """Token-by-token Gated DeltaNet-2 forward.

    q, k: [B,T,H,dk]; v: [B,T,H,dv]; a, b_logit: [B,T,H,dk]; w_logit: [B,T,H,dv];
    A_log, dt_bias: [H,dk]; h0: [B,H,dk,dv] or None.  With ``gates_given``, a is
    the per-channel log-decay and b_logit / w_logit are the gate values.
    Returns (o, ht) shaped like ``gdn_fwd``'s.
    """
    B, T, H, dk = q.shape
    dv = v.shape[3]
    f64 = _is_f64(q, k, v, a, b_logit, w_logit, A_log, dt_bias, h0)
    arrs = [_arr(x, f64) for x in (q, k, v, a, b_logit, w_logit, A_log, dt_bias, h0)]
    if gates_given:
        arrs[6] = arrs[7] = None
    if scale is None:
        scale = dk ** -0.5
    n_sel, sel_arr, sel_p = _sel(heads)
    nh = n_sel if n_sel else B * H
    o = np.zeros((nh, T, dv)) if want_o else None
    ht = np.zeros((nh, dk, dv)) if want_ht else None
    rc = _load().oracle_gdn2_fwd(*[_ptr(x) for x in arrs], int(f64), B, T, H, dk, dv,
                                 float(scale), int(l2norm), int(gates_given), n_sel, sel_p,
                                 _ptr(o), _ptr(ht), int(threads or max_threads()))
    _check(rc, "oracle_gdn2_fwd")
    del sel_arr
    if heads is None:
        if o is not None:
            o = o.reshape(B, H, T, dv).transpose(0, 2, 1, 3).copy()
        if ht is not None:
            ht = ht.reshape(B, H, dk, dv)
    return o, ht
