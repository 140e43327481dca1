"""Thin ctypes binding of libgdn.so (the C ABI in include/gdn.h).

Argument marshalling only: every step of the mixer runs in the library's CUDA
kernels.  torch supplies device memory and the current stream.  There is no
fallback: if the library is missing or a call is rejected, an exception is
raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

from . import build as _build

HEAD_DIM = 128
CHUNK = 64

_STATUS = {
    0: "GDN_OK", 1: "GDN_ERR_INVALID_ARG", 2: "GDN_ERR_UNSUPPORTED", 3: "GDN_ERR_MISALIGNED",
    4: "GDN_ERR_ALIAS", 5: "GDN_ERR_CUDA", 6: "GDN_ERR_DEVICE_TIMEOUT", 7: "GDN_ERR_WORKSPACE",
}


class GdnError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {_STATUS.get(status, status)}")


class GdnInputs(ctypes.Structure):
    _fields_ = [
        ("q", ctypes.c_void_p), ("k", ctypes.c_void_p), ("v", ctypes.c_void_p),
        ("a", ctypes.c_void_p), ("b", ctypes.c_void_p), ("z", ctypes.c_void_p),
        ("stride_q", ctypes.c_longlong), ("stride_k", ctypes.c_longlong), ("stride_v", ctypes.c_longlong),
        ("stride_z", ctypes.c_longlong), ("stride_a", ctypes.c_longlong), ("stride_b", ctypes.c_longlong),
        ("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p), ("norm_w", ctypes.c_void_p),
        ("H_k", ctypes.c_int), ("H_v", ctypes.c_int), ("scale", ctypes.c_float),
        ("events", ctypes.c_void_p),
        ("schedule", ctypes.c_int),
    ]

class GdnLayer(ctypes.Structure):
    """gdn_layer: the weights of one delta-rule layer (device pointers)."""
    _fields_ = [
        ("w_in", ctypes.c_void_p), ("ld_w_in", ctypes.c_longlong),
        ("w_out", ctypes.c_void_p), ("ld_w_out", ctypes.c_longlong),
        ("conv_w", ctypes.c_void_p), ("A_log", ctypes.c_void_p), ("norm_w", ctypes.c_void_p),
        ("H_k", ctypes.c_int), ("H_v", ctypes.c_int), ("hidden", ctypes.c_int),
        ("scale", ctypes.c_float), ("schedule", ctypes.c_int),
        ("events", ctypes.c_void_p),
    ]


class GdnAttnLayer(ctypes.Structure):
    """gdn_attn_layer: the weights of one global-attention layer (device pointers)."""
    _fields_ = [
        ("w_in", ctypes.c_void_p), ("ld_w_in", ctypes.c_longlong),
        ("w_out", ctypes.c_void_p), ("ld_w_out", ctypes.c_longlong),
        ("q_norm_w", ctypes.c_void_p), ("k_norm_w", ctypes.c_void_p),
        ("hidden", ctypes.c_int),
        ("events", ctypes.c_void_p),
    ]


ATTN_Q_HEADS, ATTN_KV_HEADS, ATTN_HEAD_DIM = 24, 4, 256
ATTN_N_IN = 2 * 24 * 256 + 2 * 4 * 256


SCHEDULE_AUTO = 0          # one overlapped launch when it pays (few scan units, many prep items)
SCHEDULE_TWO_LAUNCHES = 1  # prep kernel, then scan kernel
SCHEDULE_FUSED = 2         # one overlapped launch whenever the scan units fit in half the SMs


_lib = None
_vp, _sz, _i, _ll = ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_longlong

EXPORTS = ("gdn_prefill_workspace_size", "gdn_prefill", "gdn_prefill_varlen", "gdn_prefill_host_workspace_size",
           "gdn_prefill_host", "gdn_decode_step",
           "gdn_decode_multi", "gdn_gemm_bf16", "gdn_layer_n_in", "gdn_layer_workspace_size", "gdn_layer_prefill",
           "gdn_layer_decode_workspace_size", "gdn_layer_decode",
           "gdn_attn_layer_workspace_size", "gdn_attn_layer_prefill", "gdn_attention_prefill",
           "gdn_attn_decode_workspace_size", "gdn_attn_layer_decode_step", "gdn_status_string",
           "gdn_err_status", "gdn_prefill_fused_plan")
MAX_DECODE_TOKENS = 8


def load(path: str | None = None, fresh: bool = False):
    """Load libgdn.so from the package directory (it must have been built).  The first library
    loaded is kept for every later call; `fresh` loads `path` (e.g. libgdn_debug.so) and
    returns it without making it that library."""
    global _lib
    if _lib is not None and not fresh:
        return _lib
    path = path or _build.lib_path("libgdn.so")
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: run gated_delta_rule_81_b200.build.build() first")
    lib = ctypes.CDLL(path)
    P = ctypes.POINTER(GdnInputs)
    lib.gdn_prefill_workspace_size.argtypes = [_i, _i, _i, _ll]
    lib.gdn_prefill_workspace_size.restype = _sz
    lib.gdn_prefill.argtypes = [P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.gdn_prefill.restype = _i
    lib.gdn_prefill_host_workspace_size.argtypes = [_i, _i, _i, _i]
    lib.gdn_prefill_host_workspace_size.restype = _sz
    lib.gdn_prefill_host.argtypes = [P, _i, _i, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.gdn_prefill_host.restype = _i
    lib.gdn_prefill_varlen.argtypes = [P, _i, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _vp, _sz, _vp, _vp]
    lib.gdn_prefill_varlen.restype = _i
    lib.gdn_decode_step.argtypes = [P, _i, _vp, _vp, _vp, _vp, _vp]
    lib.gdn_decode_step.restype = _i
    lib.gdn_decode_multi.argtypes = [P, _i, _i, _vp, _vp, _vp, _i, _vp, _vp, _vp]
    lib.gdn_decode_multi.restype = _i
    lib.gdn_gemm_bf16.argtypes = [_vp, _ll, _vp, _ll, _vp, _ll, _i, _i, _i, _vp, _vp]
    lib.gdn_gemm_bf16.restype = _i
    lib.gdn_layer_n_in.argtypes = [_i, _i]
    lib.gdn_layer_n_in.restype = _ll
    lib.gdn_layer_workspace_size.argtypes = [_i, _i, _i, _i]
    lib.gdn_layer_workspace_size.restype = _sz
    lib.gdn_layer_prefill.argtypes = [ctypes.POINTER(GdnLayer), _i, _i, _vp, _ll, _vp, _vp, _vp, _vp, _vp, _ll, _vp,
                                      _sz, _vp, _vp]
    lib.gdn_layer_prefill.restype = _i
    lib.gdn_layer_decode_workspace_size.argtypes = [_i, _i, _i, _i]
    lib.gdn_layer_decode_workspace_size.restype = _sz
    lib.gdn_layer_decode.argtypes = [ctypes.POINTER(GdnLayer), _i, _i, _vp, _ll, _vp, _vp, _vp, _i, _vp, _ll, _vp, _sz,
                                     _vp, _vp]
    lib.gdn_layer_decode.restype = _i
    lib.gdn_attn_layer_workspace_size.argtypes = [_i, _i]
    lib.gdn_attn_layer_workspace_size.restype = _sz
    lib.gdn_attn_layer_prefill.argtypes = [ctypes.POINTER(GdnAttnLayer), _i, _i, _vp, _ll, _vp, _vp, _i, _vp, _ll,
                                           _vp, _sz, _vp, _vp]
    lib.gdn_attn_decode_workspace_size.argtypes = [_i, _i]
    lib.gdn_attn_decode_workspace_size.restype = _sz
    lib.gdn_attn_layer_decode_step.argtypes = [ctypes.POINTER(GdnAttnLayer), _i, _vp, _ll, _vp, _vp, _i, _vp, _vp,
                                               _ll, _vp, _sz, _vp, _vp]
    lib.gdn_attn_layer_decode_step.restype = _i
    lib.gdn_attn_layer_prefill.restype = _i
    lib.gdn_attention_prefill.argtypes = [_vp, _vp, _vp, _vp, _ll, _i, _i, _vp, _vp, _vp]
    lib.gdn_attention_prefill.restype = _i
    lib.gdn_status_string.argtypes = [_i]
    lib.gdn_status_string.restype = ctypes.c_char_p
    lib.gdn_err_status.argtypes = [_i]
    lib.gdn_err_status.restype = _i
    lib.gdn_prefill_fused_plan.argtypes = [_i, _i, _i, _ll, _i, _i]
    lib.gdn_prefill_fused_plan.restype = _i
    if not fresh:
        _lib = lib
    return lib


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _tok_stride(t, T_tot):
    """Token stride (elements) of a [T_tot, ...] tensor whose per-token channels are contiguous."""
    if t.dim() == 1:
        return t.numel() // max(T_tot, 1)
    inner = t[0] if t.shape[0] > 0 else t
    if t.shape[0] > 0 and not inner.is_contiguous():
        raise ValueError("per-token channels must be contiguous")
    return t.stride(0)


def make_inputs(q, k, v, a, b, z, conv_w, A_log, norm_w, scale=1.0, schedule=SCHEDULE_AUTO) -> GdnInputs:
    T_tot = q.shape[0]
    H_k = q.shape[1] if q.dim() == 3 else q.shape[-1] // HEAD_DIM
    H_v = v.shape[1] if v.dim() == 3 else v.shape[-1] // HEAD_DIM
    for name, t in (("q", q), ("k", k), ("v", v), ("a", a), ("b", b), ("z", z), ("conv_w", conv_w),
                    ("norm_w", norm_w)):
        if t.dtype != torch.bfloat16:
            raise TypeError(f"{name} must be bf16")
    if A_log.dtype != torch.float32:
        raise TypeError("A_log must be fp32")
    s = GdnInputs()
    s.q, s.k, s.v, s.a, s.b, s.z = (t.data_ptr() for t in (q, k, v, a, b, z))
    s.stride_q, s.stride_k, s.stride_v = (_tok_stride(t, T_tot) for t in (q, k, v))
    s.stride_z, s.stride_a, s.stride_b = (_tok_stride(t, T_tot) for t in (z, a, b))
    s.conv_w, s.A_log, s.norm_w = conv_w.data_ptr(), A_log.data_ptr(), norm_w.data_ptr()
    s.H_k, s.H_v, s.scale = int(H_k), int(H_v), float(scale)
    s.schedule = int(schedule)
    return s


def set_timing_events(inp: GdnInputs, events):
    """Attach torch.cuda.Event objects (enable_timing=True) that the library records
    around its kernels (3 for prefill, 2 for decode); None detaches.  Returns the
    ctypes array, which must stay alive while the call is in use."""
    if events is None:
        inp.events = None
        return None
    for ev in events:
        if not ev.cuda_event:
            ev.record()  # materialise the handle
    arr = (ctypes.c_void_p * len(events))(*[ev.cuda_event for ev in events])
    inp.events = ctypes.cast(arr, ctypes.c_void_p)
    return arr


def _check(status, where):
    if status != 0:
        raise GdnError(status, where)


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def workspace_size(H_k: int, H_v: int, N: int, n_chunks: int) -> int:
    return int(load().gdn_prefill_workspace_size(H_k, H_v, N, n_chunks))


def chunk_count(lengths) -> int:
    return sum((int(L) + CHUNK - 1) // CHUNK for L in lengths)


def _outputs(dev, T_tot, H_k, H_v, N, want_state, want_conv, out, state_out, conv_out):
    C_conv = (2 * H_k + H_v) * HEAD_DIM
    if out is None:
        out = torch.empty(T_tot, H_v, HEAD_DIM, dtype=torch.bfloat16, device=dev)
    if state_out is None and want_state:
        state_out = torch.empty(N, H_v, HEAD_DIM, HEAD_DIM, dtype=torch.float32, device=dev)
    if conv_out is None and want_conv:
        conv_out = torch.empty(N, 3, C_conv, dtype=torch.bfloat16, device=dev)
    return out, state_out, conv_out


def prefill(inp: GdnInputs, B: int, T: int, state_in=None, conv_in=None, *, want_state=True, want_conv=True,
            out=None, state_out=None, conv_out=None, workspace=None, err=None, device=None):
    """gdn_prefill: B sequences of T tokens, packed [B*T].  Returns (out, state_out, conv_out)."""
    lib = load()
    dev = device or torch.device("cuda", torch.cuda.current_device())
    out, state_out, conv_out = _outputs(dev, B * T, inp.H_k, inp.H_v, B, want_state, want_conv, out, state_out,
                                        conv_out)
    n_chunks = B * ((T + CHUNK - 1) // CHUNK)
    need = lib.gdn_prefill_workspace_size(inp.H_k, inp.H_v, B, n_chunks)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    _check(lib.gdn_prefill(ctypes.byref(inp), B, T, _ptr(state_in), _ptr(state_out), _ptr(conv_in),
                           _ptr(conv_out), _ptr(out), _ptr(workspace), workspace.numel(), _ptr(err), _stream()),
           "gdn_prefill")
    return out, state_out, conv_out


def prefill_host_workspace_size(H_k: int, H_v: int, B: int, T: int) -> int:
    return int(load().gdn_prefill_host_workspace_size(H_k, H_v, B, T))


def prefill_host(inp: GdnInputs, B: int, T: int, out, state_in=None, state_out=None, conv_in=None, conv_out=None, *,
                 workspace=None, err=None, stream=None):
    """gdn_prefill_host: `inp` built from pinned host tensors (q, k, v, a, b, z) and device
    weights; out, state_in / state_out, conv_in / conv_out are pinned host tensors (or None).
    Asynchronous on `stream` (a torch.cuda.Stream, default the current one); returns out."""
    lib = load()
    if workspace is None:
        workspace = torch.empty(prefill_host_workspace_size(inp.H_k, inp.H_v, B, T), dtype=torch.uint8,
                                device=torch.device("cuda", torch.cuda.current_device()))
    st = ctypes.c_void_p(stream.cuda_stream) if stream is not None else _stream()
    _check(lib.gdn_prefill_host(ctypes.byref(inp), B, T, _ptr(state_in), _ptr(state_out), _ptr(conv_in),
                                _ptr(conv_out), _ptr(out), _ptr(workspace), workspace.numel(), _ptr(err), st),
           "gdn_prefill_host")
    return out


def prefill_varlen(inp: GdnInputs, cu_seqlens, cu_seqlens_host, state_in=None, conv_in=None, *, want_state=True,
                   want_conv=True, out=None, state_out=None, conv_out=None, workspace=None, err=None):
    """gdn_prefill_varlen.  cu_seqlens: device int32 [N+1]; cu_seqlens_host: CPU int32 [N+1]."""
    lib = load()
    dev = cu_seqlens.device
    host = cu_seqlens_host.to(torch.int32).contiguous()
    N = host.numel() - 1
    T_tot = int(host[-1])
    out, state_out, conv_out = _outputs(dev, T_tot, inp.H_k, inp.H_v, N, want_state, want_conv, out, state_out,
                                        conv_out)
    n_chunks = chunk_count((host[1:] - host[:-1]).tolist())
    need = lib.gdn_prefill_workspace_size(inp.H_k, inp.H_v, N, n_chunks)
    if workspace is None:
        workspace = torch.empty(need, dtype=torch.uint8, device=dev)
    host_ptr = ctypes.cast(host.data_ptr(), ctypes.c_void_p)
    _check(lib.gdn_prefill_varlen(ctypes.byref(inp), N, _ptr(cu_seqlens), host_ptr, _ptr(state_in),
                                  _ptr(state_out), _ptr(conv_in), _ptr(conv_out), _ptr(out), _ptr(workspace),
                                  workspace.numel(), _ptr(err), _stream()),
           "gdn_prefill_varlen")
    return out, state_out, conv_out


def decode_step(inp: GdnInputs, N: int, state, conv_state, out=None, err=None):
    """gdn_decode_step: one token per sequence; state and conv_state updated in place.  Returns out."""
    lib = load()
    if out is None:
        out = torch.empty(N, inp.H_v, HEAD_DIM, dtype=torch.bfloat16, device=state.device)
    _check(lib.gdn_decode_step(ctypes.byref(inp), N, _ptr(state), _ptr(conv_state), _ptr(out), _ptr(err),
                               _stream()),
           "gdn_decode_step")
    return out


def decode_multi(inp: GdnInputs, N: int, T: int, state, conv_state, state_slot=None, out=None, err=None):
    """gdn_decode_multi: T new tokens per sequence (token n*T + t), states in pool slots.

    state [n_slots][H_v][128][128] fp32 and conv_state [n_slots][3][C_conv] bf16 are
    updated in place; state_slot is a device int32 [N] (None: sequence n uses slot n).
    Returns out [N*T][H_v][128] bf16."""
    lib = load()
    if out is None:
        out = torch.empty(N * T, inp.H_v, HEAD_DIM, dtype=torch.bfloat16, device=state.device)
    n_slots = state.shape[0]
    _check(lib.gdn_decode_multi(ctypes.byref(inp), N, T, _ptr(state), _ptr(conv_state), _ptr(state_slot), n_slots,
                                _ptr(out), _ptr(err), _stream()),
           "gdn_decode_multi")
    return out


def gemm_bf16(a, b, out=None, err=None):
    """gdn_gemm_bf16: out[M][N] = a[M][K] @ b[N][K]^T (bf16, fp32 accumulation).  a and b may be
    row-strided views (last dimension contiguous)."""
    lib = load()
    M, K = a.shape
    N = b.shape[0]
    if b.shape[1] != K:
        raise ValueError("a and b disagree on K")
    for name, t in (("a", a), ("b", b)):
        if t.dtype != torch.bfloat16 or t.stride(1) != 1:
            raise TypeError(f"{name} must be bf16 with a contiguous last dimension")
    if out is None:
        out = torch.empty(M, N, dtype=torch.bfloat16, device=a.device)
    _check(lib.gdn_gemm_bf16(_ptr(a), a.stride(0), _ptr(b), b.stride(0), _ptr(out), out.stride(0), M, N, K,
                             _ptr(err), _stream()), "gdn_gemm_bf16")
    return out


def make_layer(w_in, w_out, conv_w, A_log, norm_w, H_k, H_v, scale=1.0, schedule=SCHEDULE_AUTO) -> GdnLayer:
    """gdn_layer from device tensors: w_in bf16 [n_in][hidden], w_out bf16 [hidden][H_v*128]."""
    for name, t in (("w_in", w_in), ("w_out", w_out), ("conv_w", conv_w), ("norm_w", norm_w)):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise TypeError(f"{name} must be bf16 with a contiguous last dimension")
    L = GdnLayer()
    L.w_in, L.ld_w_in = w_in.data_ptr(), w_in.stride(0)
    L.w_out, L.ld_w_out = w_out.data_ptr(), w_out.stride(0)
    L.conv_w, L.A_log, L.norm_w = conv_w.data_ptr(), A_log.data_ptr(), norm_w.data_ptr()
    L.H_k, L.H_v, L.hidden = int(H_k), int(H_v), int(w_in.shape[1])
    L.scale, L.schedule = float(scale), int(schedule)
    return L


def layer_workspace_size(H_k, H_v, B, T) -> int:
    return int(load().gdn_layer_workspace_size(H_k, H_v, B, T))


def layer_prefill(L: GdnLayer, B: int, T: int, x, state_in=None, conv_in=None, *, want_state=True, want_conv=True,
                  y=None, state_out=None, conv_out=None, workspace=None, err=None):
    """gdn_layer_prefill: y = out_proj(mixer(in_proj(x))) for B sequences of T tokens.
    Returns (y, state_out, conv_out)."""
    lib = load()
    dev = x.device
    _, state_out, conv_out = _outputs(dev, 0, L.H_k, L.H_v, B, want_state, want_conv, torch.empty(0), state_out,
                                      conv_out)
    if y is None:
        y = torch.empty(B * T, L.hidden, dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = torch.empty(layer_workspace_size(L.H_k, L.H_v, B, T), dtype=torch.uint8, device=dev)
    _check(lib.gdn_layer_prefill(ctypes.byref(L), B, T, _ptr(x), x.stride(0), _ptr(state_in), _ptr(state_out),
                                 _ptr(conv_in), _ptr(conv_out), _ptr(y), y.stride(0), _ptr(workspace),
                                 workspace.numel(), _ptr(err), _stream()), "gdn_layer_prefill")
    return y, state_out, conv_out


def layer_decode(L: GdnLayer, N: int, T: int, x, state, conv_state, state_slot=None, n_slots=None, *, y=None,
                 workspace=None, err=None):
    """gdn_layer_decode: T new tokens for each of N sequences (x [N*T][hidden]); state and
    conv_state (the pool, or one slot per sequence) are updated in place.  Returns y."""
    lib = load()
    if y is None:
        y = torch.empty(N * T, L.hidden, dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(int(lib.gdn_layer_decode_workspace_size(L.H_k, L.H_v, N, T)), dtype=torch.uint8,
                                device=x.device)
    if n_slots is None:
        n_slots = state.shape[0]
    _check(lib.gdn_layer_decode(ctypes.byref(L), N, T, _ptr(x), x.stride(0), _ptr(state), _ptr(conv_state),
                                _ptr(state_slot), int(n_slots), _ptr(y), y.stride(0), _ptr(workspace),
                                workspace.numel(), _ptr(err), _stream()), "gdn_layer_decode")
    return y


def make_attn_layer(w_in, w_out, q_norm_w, k_norm_w) -> GdnAttnLayer:
    """gdn_attn_layer from device tensors: w_in bf16 [ATTN_N_IN][hidden], w_out bf16 [hidden][24*256]."""
    for name, t in (("w_in", w_in), ("w_out", w_out), ("q_norm_w", q_norm_w), ("k_norm_w", k_norm_w)):
        if t.dtype != torch.bfloat16 or t.stride(-1) != 1:
            raise TypeError(f"{name} must be bf16 with a contiguous last dimension")
    L = GdnAttnLayer()
    L.w_in, L.ld_w_in = w_in.data_ptr(), w_in.stride(0)
    L.w_out, L.ld_w_out = w_out.data_ptr(), w_out.stride(0)
    L.q_norm_w, L.k_norm_w = q_norm_w.data_ptr(), k_norm_w.data_ptr()
    L.hidden = int(w_in.shape[1])
    return L


def attn_layer_prefill(L: GdnAttnLayer, B: int, T: int, x, *, y=None, k_cache=None, v_cache=None, cache_cap=0,
                       workspace=None, err=None):
    """gdn_attn_layer_prefill.  Caches are [B][cache_cap or T][4][256].  Returns (y, k_cache, v_cache)."""
    lib = load()
    dev = x.device
    cap = cache_cap or T
    if y is None:
        y = torch.empty(B * T, L.hidden, dtype=torch.bfloat16, device=dev)
    if k_cache is None:
        k_cache = torch.empty(B, cap, ATTN_KV_HEADS, ATTN_HEAD_DIM, dtype=torch.bfloat16, device=dev)
    if v_cache is None:
        v_cache = torch.empty(B, cap, ATTN_KV_HEADS, ATTN_HEAD_DIM, dtype=torch.bfloat16, device=dev)
    if workspace is None:
        workspace = torch.empty(int(lib.gdn_attn_layer_workspace_size(B, T)), dtype=torch.uint8, device=dev)
    _check(lib.gdn_attn_layer_prefill(ctypes.byref(L), B, T, _ptr(x), x.stride(0), _ptr(k_cache), _ptr(v_cache),
                                      int(cache_cap), _ptr(y), y.stride(0), _ptr(workspace), workspace.numel(),
                                      _ptr(err), _stream()), "gdn_attn_layer_prefill")
    return y, k_cache, v_cache


def attn_layer_decode_step(L: GdnAttnLayer, x, k_cache, v_cache, cache_len, *, y=None, workspace=None, err=None):
    """gdn_attn_layer_decode_step: one new token per sequence (x [N][hidden]); the caches
    [N][cap][4][256] and cache_len (device int32 [N]) are updated in place.  Returns y."""
    lib = load()
    N, cap = x.shape[0], k_cache.shape[1]
    if y is None:
        y = torch.empty(N, L.hidden, dtype=torch.bfloat16, device=x.device)
    if workspace is None:
        workspace = torch.empty(int(lib.gdn_attn_decode_workspace_size(N, cap)), dtype=torch.uint8, device=x.device)
    _check(lib.gdn_attn_layer_decode_step(ctypes.byref(L), N, _ptr(x), x.stride(0), _ptr(k_cache), _ptr(v_cache),
                                          cap, _ptr(cache_len), _ptr(y), y.stride(0), _ptr(workspace),
                                          workspace.numel(), _ptr(err), _stream()), "gdn_attn_layer_decode_step")
    return y


def attention_prefill(q_hat, k, v, g, B: int, T: int, out=None, err=None):
    """gdn_attention_prefill on device tensors q_hat [B*T,24,256], k, v [B*T,4,256], g (rows of >= 24*256)."""
    lib = load()
    if out is None:
        out = torch.empty(B * T, ATTN_Q_HEADS * ATTN_HEAD_DIM, dtype=torch.bfloat16, device=q_hat.device)
    g2 = g.reshape(g.shape[0], -1) if g.dim() == 3 else g
    _check(lib.gdn_attention_prefill(_ptr(q_hat), _ptr(k), _ptr(v), _ptr(g2), g2.stride(0), B, T, _ptr(out),
                                     _ptr(err), _stream()), "gdn_attention_prefill")
    return out


def status_string(status: int) -> str:
    return load().gdn_status_string(status).decode()


def err_status(err_word: int) -> int:
    """gdn_err_status: the gdn_status an error word read back from the device stands for."""
    return load().gdn_err_status(int(err_word))
