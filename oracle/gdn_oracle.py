"""ctypes front of the fp64 C oracle (gdn_oracle.c) -- test infrastructure only.

The sequential fp64 recurrence is the reference every GPU result is checked
against.  Its passages: the Agnes-3.0-Flash model card, "Architecture" table,
row "Delta-rule layers" (16 key / 48 value heads, head dim 128, causal conv
kernel 4 in front, gated RMS-norm after, fp32 state), and "Agnes-3.0-Flash Deep
Dive: A 33B Hybrid-Attention Multimodal Model", section "Feed-Forward and
Positional Encoding", paragraph on the Gated Delta Rule (erase the key's old
association, then write; a forget gate decays the memory).  The recurrence itself, S_t = a_t S_{t-1}(I - b_t k_t k_t^T)
+ b_t v_t k_t^T with o_t = S_t q_t, is the standard gated delta rule those
passages name.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libgdn_oracle.so")
_lock = threading.Lock()
_lib = None

_dp = ctypes.POINTER(ctypes.c_double)
_i64p = ctypes.POINTER(ctypes.c_int64)
_u16p = ctypes.POINTER(ctypes.c_uint16)
_f32p = ctypes.POINTER(ctypes.c_float)
_i32p = ctypes.POINTER(ctypes.c_int)


def build(force: bool = False) -> str:
    """Compile gdn_oracle.c into libgdn_oracle.so (gcc, OpenMP, -O2, no fast-math)."""
    stale = (not os.path.exists(_LIB_PATH)) or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC)
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(
            ["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11", "-o", tmp, _SRC, "-lm"],
            check=True,
        )
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            lib.gdn_oracle_conv.argtypes = [ctypes.c_int, _i64p, ctypes.c_int, _dp, _dp, _dp, ctypes.c_int, _dp]
            lib.gdn_oracle_l2norm.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, _dp]
            lib.gdn_oracle_gates.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, _dp, _dp, _dp, _dp, _dp]
            lib.gdn_oracle_recurrence.argtypes = [
                ctypes.c_int, _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _dp, _dp, _dp, _dp, _dp, _dp, _dp, _dp,
            ]
            lib.gdn_oracle_gated_rmsnorm.argtypes = [ctypes.c_int64, ctypes.c_int, _dp, _dp, _dp, _dp]
            lib.gdn_oracle_mixer.argtypes = [
                ctypes.c_int, _i64p, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                _u16p, _u16p, _u16p, _u16p, _u16p, _u16p, _u16p, _f32p, _u16p, ctypes.c_double,
                _f32p, _u16p, _i32p, ctypes.c_int, _dp, _dp, _dp, _dp, ctypes.c_int,
            ]
            lib.gdn_oracle_mixer.restype = ctypes.c_int
            lib.gdn_oracle_num_threads.restype = ctypes.c_int
            _lib = lib
    return _lib


def _ptr(arr, ctype):
    if arr is None:
        return None
    return arr.ctypes.data_as(ctypes.POINTER(ctype))


def _f64(x):
    return None if x is None else np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _cu(cu_seqlens):
    return np.ascontiguousarray(np.asarray(cu_seqlens, dtype=np.int64))


def _bf16_bits(t):
    """A torch bf16 tensor (CPU) or a uint16 array of bf16 bit patterns -> uint16 array."""
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        assert t.dtype == np.uint16
        return np.ascontiguousarray(t)
    import torch

    assert t.dtype == torch.bfloat16, t.dtype
    return np.ascontiguousarray(t.detach().cpu().contiguous().view(torch.int16).numpy().view(np.uint16))


def _f32(t):
    if t is None:
        return None
    if isinstance(t, np.ndarray):
        return np.ascontiguousarray(t, dtype=np.float32)
    return np.ascontiguousarray(t.detach().cpu().float().contiguous().numpy())


def num_threads() -> int:
    return int(_load().gdn_oracle_num_threads())


def conv(x, w, cu_seqlens, hist=None, silu=True):
    """Causal depthwise conv (4 taps, tap 3 = current token) + optional SiLU; fp64.
    x [T][C], w [C][4], hist [N][3][C] (oldest first) or None."""
    lib = _load()
    x, w, hist = _f64(x), _f64(w), _f64(hist)
    cu = _cu(cu_seqlens)
    T, C = x.shape
    y = np.zeros((T, C), dtype=np.float64)
    lib.gdn_oracle_conv(len(cu) - 1, _ptr(cu, ctypes.c_int64), C, _ptr(x, ctypes.c_double),
                        _ptr(w, ctypes.c_double), _ptr(hist, ctypes.c_double), int(silu),
                        _ptr(y, ctypes.c_double))
    return y


def l2norm(x):
    lib = _load()
    x = _f64(x)
    y = np.empty_like(x)
    n = x.shape[-1]
    lib.gdn_oracle_l2norm(x.size // n, n, _ptr(x, ctypes.c_double), _ptr(y, ctypes.c_double))
    return y


def gates(A_log, a, b):
    """g = -exp(A_log) softplus(a), alpha = exp(g), beta = sigmoid(b); a, b [T][H]."""
    lib = _load()
    A_log, a, b = _f64(A_log), _f64(a), _f64(b)
    T, H = a.shape
    g, alpha, beta = (np.empty((T, H)) for _ in range(3))
    lib.gdn_oracle_gates(T, H, _ptr(A_log, ctypes.c_double), _ptr(a, ctypes.c_double),
                         _ptr(b, ctypes.c_double), _ptr(g, ctypes.c_double),
                         _ptr(alpha, ctypes.c_double), _ptr(beta, ctypes.c_double))
    return g, alpha, beta


def recurrence(q, k, v, alpha, beta, cu_seqlens, S0=None):
    """The gated delta rule on post-front-end inputs; q, k [T][H_k][dk], v [T][H_v][dv],
    alpha, beta [T][H_v], S0 [N][H_v][dv][dk] or None.  Returns (o [T][H_v][dv], S [N][H_v][dv][dk])."""
    lib = _load()
    q, k, v, alpha, beta, S0 = map(_f64, (q, k, v, alpha, beta, S0))
    cu = _cu(cu_seqlens)
    T, H_k, dk = q.shape
    _, H_v, dv = v.shape
    n = len(cu) - 1
    o = np.zeros((T, H_v, dv))
    S = np.zeros((n, H_v, dv, dk))
    lib.gdn_oracle_recurrence(n, _ptr(cu, ctypes.c_int64), H_k, H_v, dk, dv,
                              *(_ptr(t, ctypes.c_double) for t in (q, k, v, alpha, beta, S0, o, S)))
    return o, S


def gated_rmsnorm(o, z, w):
    lib = _load()
    o, z, w = _f64(o), _f64(z), _f64(w)
    n = o.shape[-1]
    y = np.empty_like(o)
    lib.gdn_oracle_gated_rmsnorm(o.size // n, n, _ptr(o, ctypes.c_double), _ptr(z, ctypes.c_double),
                                 _ptr(w, ctypes.c_double), _ptr(y, ctypes.c_double))
    return y


def mixer(inp, cu_seqlens, state_in=None, conv_in=None, heads=None, want_state=True,
          want_conv=True, want_pre_norm=False, n_threads=0):
    """The whole mixer in fp64 on the exact bf16/fp32 inputs.

    ``inp`` holds q, k, v, a, b, z (bf16 [T_tot, H, D] / [T_tot, H]), conv_w (bf16
    [C_conv, 4]), A_log (fp32 [H_v]), norm_w (bf16 [D]) and scale (float).
    ``heads`` limits the work to some value heads (outputs of the others stay 0).
    Returns a dict with out [T, H_v, D], state [N, H_v, D, D], conv [N, 3, C_conv],
    pre_norm [T, H_v, D] (each fp64, or None when not asked for).
    """
    lib = _load()
    cu = _cu(cu_seqlens)
    q, k, v = _bf16_bits(inp["q"]), _bf16_bits(inp["k"]), _bf16_bits(inp["v"])
    T, H_k, D = q.shape
    H_v = v.shape[1]
    n = len(cu) - 1
    C_conv = (2 * H_k + H_v) * D
    a, b, z = _bf16_bits(inp["a"]), _bf16_bits(inp["b"]), _bf16_bits(inp["z"])
    conv_w, norm_w = _bf16_bits(inp["conv_w"]), _bf16_bits(inp["norm_w"])
    A_log = _f32(inp["A_log"])
    st_in = _f32(state_in)
    cv_in = _bf16_bits(conv_in)
    hs = None if heads is None else np.ascontiguousarray(np.asarray(heads, dtype=np.int32))
    out = np.zeros((T, H_v, D))
    state = np.zeros((n, H_v, D, D)) if want_state else None
    conv_o = np.zeros((n, 3, C_conv)) if want_conv else None
    pre = np.zeros((T, H_v, D)) if want_pre_norm else None
    rc = lib.gdn_oracle_mixer(
        n, _ptr(cu, ctypes.c_int64), H_k, H_v, D,
        _ptr(q, ctypes.c_uint16), _ptr(k, ctypes.c_uint16), _ptr(v, ctypes.c_uint16),
        _ptr(a, ctypes.c_uint16), _ptr(b, ctypes.c_uint16), _ptr(z, ctypes.c_uint16),
        _ptr(conv_w, ctypes.c_uint16), _ptr(A_log, ctypes.c_float), _ptr(norm_w, ctypes.c_uint16),
        float(inp.get("scale", 1.0)), _ptr(st_in, ctypes.c_float), _ptr(cv_in, ctypes.c_uint16),
        _ptr(hs, ctypes.c_int), 0 if hs is None else len(hs),
        _ptr(out, ctypes.c_double), _ptr(state, ctypes.c_double), _ptr(conv_o, ctypes.c_double),
        _ptr(pre, ctypes.c_double), int(n_threads),
    )
    if rc != 0:
        raise ValueError("oracle rejected its arguments")
    return {"out": out, "state": state, "conv": conv_o, "pre_norm": pre}
