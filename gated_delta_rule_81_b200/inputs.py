"""Seeded synthetic inputs for the gated-delta-rule mixer.

This module holds no arithmetic of the method: it only draws random tensors.
Both the CUDA path and the fp64 oracle are fed from it.

Recipe (the workloads of the mixer's benchmark configurations):
  * every tensor, and every head slice of it, comes from its own CPU
    ``torch.Generator`` seeded by ``_seed(seed, tensor, head)``, so any head
    can be regenerated alone and the draw does not depend on the order in which
    tensors are built;
  * q, k, v, z and the output-gate logits: bf16 N(0, 1); a (decay logit): bf16
    N(a_mean, 1) (a_mean = 0, or 2 for the full-context case); b (beta logit):
    bf16 N(0, 1); A_log: fp32 U(ln 1, ln 16) per value head; conv weights: bf16
    N(0, 1/4) (std 0.5); norm weight: bf16 ones; recurrent state (when not
    zero): fp32 N(0, 0.01) (std 0.1); decode conv state: bf16 N(0, 1);
  * packed lengths: integers U[1024, 32768].
"""
from __future__ import annotations

import math
from concurrent.futures import ThreadPoolExecutor

import torch

D = 128  # head dim of both keys and values

_TENSOR_IDS = {
    "q": 1, "k": 2, "v": 3, "a": 4, "b": 5, "z": 6, "A_log": 7, "conv_w": 8,
    "state": 9, "conv_state": 10, "lengths": 11,
}

# The five workloads (name, shapes, distributions).
CONFIGS = {
    0: dict(name="tiny-prefill-T512-2x6", kind="prefill", N=1, T=512, H_k=2, H_v=6,
            state="zero", a_mean=0.0),
    1: dict(name="layer-prefill-T4096-16x48", kind="prefill", N=1, T=4096, H_k=16, H_v=48,
            state="normal", a_mean=0.0),
    2: dict(name="full-context-prefill-T262144-16x48", kind="prefill", N=1, T=262144, H_k=16,
            H_v=48, state="zero", a_mean=2.0),
    3: dict(name="varlen-prefill-8seq-U1024-32768-16x48", kind="varlen", N=8, H_k=16, H_v=48,
            len_lo=1024, len_hi=32768, state="zero", a_mean=0.0),
    4: dict(name="decode-256seq-64steps-16x48", kind="decode", N=256, steps=64, H_k=16, H_v=48,
            state="normal", a_mean=0.0),
}


def _seed(seed: int, tensor: str, head: int = 0) -> int:
    return (seed * 1_000_003 + _TENSOR_IDS[tensor] * 65_537 + head * 257 + 17) % (2**63 - 1)


def _gen(seed, tensor, head=0):
    return torch.Generator().manual_seed(_seed(seed, tensor, head))


def _normal_heads(seed, tensor, rows, H, width, mean=0.0, std=1.0, dtype=torch.bfloat16):
    """[rows, H, width] (or [rows, H] when width is None), one generator per head."""
    shape = (rows, H) if width is None else (rows, H, width)
    out = torch.empty(shape, dtype=dtype)

    def one(h):
        n = (rows,) if width is None else (rows, width)
        x = torch.randn(n, generator=_gen(seed, tensor, h), dtype=torch.float32)
        if std != 1.0:
            x.mul_(std)
        if mean != 0.0:
            x.add_(mean)
        out[:, h] = x.to(dtype)

    with ThreadPoolExecutor(max_workers=min(8, H)) as ex:
        list(ex.map(one, range(H)))
    return out


def varlen_lengths(n: int, lo: int, hi: int, seed: int = 0) -> list[int]:
    g = _gen(seed, "lengths")
    return [int(x) for x in torch.randint(lo, hi + 1, (n,), generator=g)]


def cu_from_lengths(lengths) -> torch.Tensor:
    cu = [0]
    for L in lengths:
        cu.append(cu[-1] + int(L))
    return torch.tensor(cu, dtype=torch.int32)


def weights(H_k: int, H_v: int, seed: int = 0) -> dict:
    """Per-layer parameters: conv weights, A_log, norm weight."""
    C_conv = (2 * H_k + H_v) * D
    conv_w = (torch.randn(C_conv, 4, generator=_gen(seed, "conv_w"), dtype=torch.float32) * 0.5).to(
        torch.bfloat16)
    u = torch.rand(H_v, generator=_gen(seed, "A_log"), dtype=torch.float64)
    A_log = (math.log(1.0) + u * (math.log(16.0) - math.log(1.0))).to(torch.float32)
    norm_w = torch.ones(D, dtype=torch.bfloat16)
    return {"conv_w": conv_w, "A_log": A_log, "norm_w": norm_w}


def token_inputs(T: int, H_k: int, H_v: int, seed: int = 0, a_mean: float = 0.0) -> dict:
    """Per-token inputs of the mixer: pre-conv q, k, v, the gate logits a, b and z."""
    return {
        "q": _normal_heads(seed, "q", T, H_k, D),
        "k": _normal_heads(seed, "k", T, H_k, D),
        "v": _normal_heads(seed, "v", T, H_v, D),
        "a": _normal_heads(seed, "a", T, H_v, None, mean=a_mean),
        "b": _normal_heads(seed, "b", T, H_v, None),
        "z": _normal_heads(seed, "z", T, H_v, D),
    }


def recurrent_state(N: int, H_v: int, seed: int = 0, kind: str = "normal") -> torch.Tensor | None:
    if kind == "zero":
        return None
    out = torch.empty(N, H_v, D, D, dtype=torch.float32)
    for h in range(H_v):
        g = _gen(seed, "state", h)
        out[:, h] = torch.randn(N, D, D, generator=g, dtype=torch.float32) * 0.1
    return out


def conv_state(N: int, H_k: int, H_v: int, seed: int = 0) -> torch.Tensor:
    C_conv = (2 * H_k + H_v) * D
    return torch.randn(N, 3, C_conv, generator=_gen(seed, "conv_state"), dtype=torch.float32).to(
        torch.bfloat16)


def prefill_case(cfg_id: int, seed: int = 0, T: int | None = None, lengths=None) -> dict:
    """Inputs of a prefill workload (config 0-3), all on the CPU.

    Returns dict(inp=..., cu_seqlens=int32 [N+1], state_in=fp32 or None, N, T_tot).
    ``T`` overrides the length of a uniform case and ``lengths`` the packed lengths
    (both for smaller test variants of the same distributions).
    """
    cfg = CONFIGS[cfg_id]
    H_k, H_v = cfg["H_k"], cfg["H_v"]
    if cfg["kind"] == "varlen":
        if lengths is None:
            lengths = varlen_lengths(cfg["N"], cfg["len_lo"], cfg["len_hi"], seed)
    else:
        lengths = [T if T is not None else cfg["T"]] * cfg["N"]
    cu = cu_from_lengths(lengths)
    T_tot = int(cu[-1])
    inp = token_inputs(T_tot, H_k, H_v, seed, cfg["a_mean"])
    inp.update(weights(H_k, H_v, seed))
    inp["scale"] = 1.0
    st = recurrent_state(len(lengths), H_v, seed, cfg["state"])
    return {"inp": inp, "cu_seqlens": cu, "state_in": st, "N": len(lengths), "T_tot": T_tot,
            "lengths": list(lengths), "H_k": H_k, "H_v": H_v, "name": cfg["name"]}


def decode_case(cfg_id: int = 4, seed: int = 0, N: int | None = None, steps: int | None = None,
                H_k: int | None = None, H_v: int | None = None) -> dict:
    """Inputs of the batched decode workload: initial state and conv state, and the
    per-step token inputs laid out [steps * N, ...] (step-major)."""
    cfg = CONFIGS[cfg_id]
    N = N if N is not None else cfg["N"]
    steps = steps if steps is not None else cfg["steps"]
    H_k = H_k if H_k is not None else cfg["H_k"]
    H_v = H_v if H_v is not None else cfg["H_v"]
    tok = token_inputs(steps * N, H_k, H_v, seed, cfg["a_mean"])
    w = weights(H_k, H_v, seed)
    return {"tok": tok, "w": w, "scale": 1.0, "state": recurrent_state(N, H_v, seed, "normal"),
            "conv_state": conv_state(N, H_k, H_v, seed), "N": N, "steps": steps, "H_k": H_k,
            "H_v": H_v}
