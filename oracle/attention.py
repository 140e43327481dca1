"""The global-attention layer of the hybrid decoder, in fp64 -- test infrastructure only.

Passages: Agnes-3.0-Flash model card, "Architecture" table, rows "Global attention"
(24 query heads / 4 KV heads, 6 : 1 GQA, head dim 256, RMS-norm on q and k,
sigmoid-gated output) and "Positions" (3-axis rotary, interleaved mrope sections
11 : 11 : 10, base 1e7, on the first 25 % of each head dim = 64 dims); "Agnes-3.0-Flash
Deep Dive: A 33B Hybrid-Attention Multimodal Model", sections "Attention Layer
Details" and the paragraph on multimodal rotary encoding (32 rotation frequencies,
text / height / width each about a third of them, interleaved).

Readings where the pages are silent (listed in the design notes):
  * text tokens: the three rotary axes all carry the token's position in its
    sequence, so every frequency rotates by position * theta_i -- plain rotary
    embedding on the first 64 dims;
  * rotation pairs: dim i with dim i + 32 of the 64 rotary dims ("rotate half"),
    theta_i = 1e7 ** (-i / 32), i = 0 .. 31;
  * RMS-norm on each head's 256 dims of q and of k, eps 1e-6, one learned weight
    vector for q and one for k (shared by the heads), before the rotation;
  * scores scaled by 1/sqrt(256), causal within each sequence, query head h reads
    KV head h // 6;
  * output gate: o * sigmoid(g) per channel, g from the same input projection;
  * input projection channels: q (24*256) | g (24*256) | k (4*256) | v (4*256), no bias.
"""
from __future__ import annotations

import numpy as np
import torch

from .projections import gemm, round_bf16

ROPE_DIMS = 64
ROPE_BASE = 1e7
EPS = 1e-6


def _f64(x) -> np.ndarray:
    return np.asarray(torch.as_tensor(x).double().cpu().numpy())


def rms_norm(x, w, eps: float = EPS) -> np.ndarray:
    """x [..., D] / sqrt(mean(x^2) + eps) * w [D]."""
    x = _f64(x)
    return x / np.sqrt(np.mean(x * x, axis=-1, keepdims=True) + eps) * _f64(w)


def rope(x, pos) -> np.ndarray:
    """Rotate the first 64 dims of x [T, H, D] by positions pos [T]: pairs (i, i + 32)."""
    x = _f64(x).copy()
    half = ROPE_DIMS // 2
    inv = ROPE_BASE ** (-np.arange(half, dtype=np.float64) / half)
    ang = np.asarray(pos, dtype=np.float64)[:, None] * inv[None, :]  # [T, 32]
    c, s = np.cos(ang)[:, None, :], np.sin(ang)[:, None, :]
    x1, x2 = x[..., :half].copy(), x[..., half:ROPE_DIMS].copy()
    x[..., :half] = x1 * c - x2 * s
    x[..., half:ROPE_DIMS] = x2 * c + x1 * s
    return x


def positions(cu_seqlens) -> np.ndarray:
    """Position of every packed token within its own sequence."""
    cu = list(cu_seqlens)
    return np.concatenate([np.arange(cu[n + 1] - cu[n]) for n in range(len(cu) - 1)]) if cu[-1] else np.zeros(0)


def attention(q, k, v, cu_seqlens, scale=None) -> np.ndarray:
    """Causal softmax attention per sequence with GQA: q [T, Hq, D], k/v [T, Hkv, D]."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    T, Hq, D = q.shape
    Hkv = k.shape[1]
    grp = Hq // Hkv
    scale = D ** -0.5 if scale is None else scale
    out = np.zeros_like(q)
    cu = list(cu_seqlens)
    for n in range(len(cu) - 1):
        s0, s1 = cu[n], cu[n + 1]
        L = s1 - s0
        if L == 0:
            continue
        mask = np.tril(np.ones((L, L), dtype=bool))
        for h in range(Hq):
            kv = h // grp
            sc = (q[s0:s1, h] @ k[s0:s1, kv].T) * scale
            sc = np.where(mask, sc, -np.inf)
            sc = sc - sc.max(axis=1, keepdims=True)
            p = np.exp(sc)
            p /= p.sum(axis=1, keepdims=True)
            out[s0:s1, h] = p @ v[s0:s1, kv]
    return out


def attn_mixer(q, g, k, v, q_norm_w, k_norm_w, cu_seqlens) -> dict:
    """The attention layer between its projections, on bf16 inputs q, g [T, 24, 256] and
    k, v [T, 4, 256]: q_hat = rope(rms(q)) in fp64, k_hat = rope(rms(k)) rounded to bf16
    (the KV cache, a bf16 output of the layer that later steps read back),
    o = attention(q_hat, k_hat, v), out = o * sigmoid(g).  Returns fp64 out, the fp64
    q_hat and the bf16-rounded k_hat (cache) values."""
    pos = positions(cu_seqlens)
    qh = rope(rms_norm(q, q_norm_w), pos)
    kh = round_bf16(rope(rms_norm(k, k_norm_w), pos))
    o = attention(qh, kh, v, cu_seqlens)
    gate = 1.0 / (1.0 + np.exp(-_f64(g)))
    return {"out": o * gate, "q_hat": qh, "k_hat": kh}


def attn_in_proj_layout(Hq: int = 24, Hkv: int = 4, D: int = 256) -> dict:
    widths = [("q", Hq * D), ("g", Hq * D), ("k", Hkv * D), ("v", Hkv * D)]
    out, c = {}, 0
    for name, w in widths:
        out[name] = (c, c + w)
        c += w
    out["total"] = (0, c)
    return out


def attn_layer(x, w_in, w_out, q_norm_w, k_norm_w, cu_seqlens, Hq: int = 24, Hkv: int = 4, D: int = 256) -> dict:
    """y = (attn_mixer on the bf16 input projection) rounded to bf16, times W_out^T."""
    T = x.shape[0]
    proj = round_bf16(gemm(x, w_in))
    lay = attn_in_proj_layout(Hq, Hkv, D)
    parts = {n: proj[:, lay[n][0]:lay[n][1]].reshape(T, -1, D) for n in ("q", "g", "k", "v")}
    m = attn_mixer(parts["q"], parts["g"], parts["k"], parts["v"], q_norm_w, k_norm_w, cu_seqlens)
    o = round_bf16(m["out"]).reshape(T, Hq * D)
    y = o @ _f64(w_out).T
    return {"y": y, "proj": proj, "out": m["out"], "q_hat": m["q_hat"], "k_hat": m["k_hat"], "v": parts["v"]}
