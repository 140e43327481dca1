"""The dense projections around the mixer, in fp64 -- test infrastructure only.

Agnes-3.0-Flash model card, "Architecture" table: hidden size 5120; row
"Delta-rule layers": 16 key heads / 48 value heads of dimension 128.  A delta-rule
layer maps the hidden state to the mixer's inputs with one input projection and
the mixer's 48 x 128 outputs back to the hidden size with one output projection.
The pages give no bias and no layout for these projections; the readings taken
here are: no bias, one weight matrix each, and the input projection's output
channels in the order q (H_k*128) | k (H_k*128) | v (H_v*128) | z (H_v*128) |
a (H_v) | b (H_v).  Both products are computed exactly in fp64 from the bf16
values; the two intermediate tensors that the layer stores in bf16 (the
projection output and the mixer output) are rounded to bf16 at those points.
"""
from __future__ import annotations

import numpy as np
import torch

from .gdn_oracle import mixer


def gemm(a, b) -> np.ndarray:
    """C = A B^T in fp64 for A [M][K], B [N][K] (any float dtype; bf16 values are exact in fp64)."""
    a64 = np.asarray(torch.as_tensor(a).double().cpu().numpy())
    b64 = np.asarray(torch.as_tensor(b).double().cpu().numpy())
    return a64 @ b64.T


def round_bf16(x) -> np.ndarray:
    """fp64 -> nearest bf16 value (ties to even), returned as fp64.  Goes through fp32
    (round to nearest), then keeps the upper 16 bits of the fp32 pattern rounded to
    nearest-even on the 16 dropped bits."""
    x32 = np.ascontiguousarray(np.asarray(x, dtype=np.float64).astype(np.float32))
    u = x32.view(np.uint32).astype(np.uint64)
    finite = np.isfinite(x32)
    u = np.where(finite, (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000, u & 0xFFFF0000)
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def in_proj_layout(H_k: int, H_v: int, D: int = 128) -> dict:
    """Column ranges of the input projection's output: name -> (start, stop)."""
    widths = [("q", H_k * D), ("k", H_k * D), ("v", H_v * D), ("z", H_v * D), ("a", H_v), ("b", H_v)]
    out, c = {}, 0
    for name, w in widths:
        out[name] = (c, c + w)
        c += w
    out["total"] = (0, c)
    return out


def layer(x, w_in, w_out, conv_w, A_log, norm_w, cu_seqlens, H_k: int, H_v: int, scale: float = 1.0,
          state_in=None, conv_in=None, D: int = 128) -> dict:
    """One delta-rule layer on hidden states x [T_tot][hidden] (bf16 values):
    proj = bf16(x W_in^T); the mixer on its q|k|v|z|a|b columns; y = bf16(mixer out) W_out^T.
    Returns dict(y=fp64 [T_tot][hidden], proj=fp64 [T_tot][N_in], out=fp64 mixer output,
    state, conv)."""
    T = x.shape[0]
    proj = round_bf16(gemm(x, w_in))
    lay = in_proj_layout(H_k, H_v, D)
    pb = torch.from_numpy(proj).to(torch.bfloat16)  # exact: proj already holds bf16 values
    inp = {}
    for name in ("q", "k", "v", "z"):
        s0, s1 = lay[name]
        inp[name] = pb[:, s0:s1].reshape(T, -1, D).contiguous()
    for name in ("a", "b"):
        s0, s1 = lay[name]
        inp[name] = pb[:, s0:s1].contiguous()
    inp.update({"conv_w": conv_w, "A_log": A_log, "norm_w": norm_w, "scale": scale})
    m = mixer(inp, cu_seqlens, state_in=state_in, conv_in=conv_in)
    o = round_bf16(m["out"]).reshape(T, H_v * D)
    y = o @ np.asarray(torch.as_tensor(w_out).double().numpy()).T
    return {"y": y, "proj": proj, "out": m["out"], "state": m["state"], "conv": m["conv"]}
