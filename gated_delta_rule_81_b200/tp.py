"""Head-sharded tensor parallelism of the delta-rule layer: tp ranks, one GPU each.

Model card "Agnes-3.0-Flash Preview", section "Hardware Requirements", row "Tensor parallel":
the model serves on one GPU, or with tensor parallelism 2 for the longest contexts and the most
concurrent requests.  The pages do not say how a layer is split.  The reading taken here is the
split that the mixer allows with no exchange inside it: the conv, the gates, the recurrence and
the gated RMS-norm all act per channel or per head, so rank r takes the key heads
[r H_k / tp, (r + 1) H_k / tp) together with their value heads (value head h belongs to key head
h // G).  The rank's input projection is the rows of those heads' channels, kept in the layer's
q | k | v | z | a | b order; its output projection is the columns of its value heads; the layer's
output is the sum over ranks of the partial output products, one all-reduce per layer (NCCL over
NVLink between GPUs).  The rank's recurrent and conv states are the slices of its heads.

This module only selects rows, columns and slices: every step of the layer runs in the CUDA
library (gdn.layer_prefill), and the sum over ranks is torch.distributed's all-reduce.
"""
from __future__ import annotations

from dataclasses import dataclass

import torch
import torch.distributed as dist

from . import gdn

D = 128  # head dim of the delta-rule layer


@dataclass(frozen=True)
class HeadRange:
    k0: int  # key heads [k0, k1)
    k1: int
    v0: int  # value heads [v0, v1)
    v1: int

    @property
    def H_k(self) -> int:
        return self.k1 - self.k0

    @property
    def H_v(self) -> int:
        return self.v1 - self.v0


def head_range(H_k: int, H_v: int, tp: int, rank: int) -> HeadRange:
    """The heads of rank `rank` out of `tp`: H_k / tp key heads and their value heads."""
    if tp <= 0 or not 0 <= rank < tp:
        raise ValueError(f"rank {rank} out of tp {tp}")
    if H_k % tp or H_v % H_k:
        raise ValueError(f"H_k = {H_k} must split evenly over tp = {tp}, and H_v = {H_v} over H_k")
    G, per = H_v // H_k, H_k // tp
    return HeadRange(rank * per, (rank + 1) * per, rank * per * G, (rank + 1) * per * G)


def in_proj_rows(H_k: int, H_v: int, r: HeadRange) -> torch.Tensor:
    """Rows of the full input projection (output channels q | k | v | z | a | b of H_k key and
    H_v value heads) that form the shard's own q | k | v | z | a | b projection."""
    q0, k0, v0 = 0, H_k * D, 2 * H_k * D
    z0 = v0 + H_v * D
    a0 = z0 + H_v * D
    b0 = a0 + H_v
    parts = [
        torch.arange(q0 + r.k0 * D, q0 + r.k1 * D),
        torch.arange(k0 + r.k0 * D, k0 + r.k1 * D),
        torch.arange(v0 + r.v0 * D, v0 + r.v1 * D),
        torch.arange(z0 + r.v0 * D, z0 + r.v1 * D),
        torch.arange(a0 + r.v0, a0 + r.v1),
        torch.arange(b0 + r.v0, b0 + r.v1),
    ]
    return torch.cat(parts)


def conv_channels(H_k: int, H_v: int, r: HeadRange) -> torch.Tensor:
    """Channels of the full conv (q | k | v, C_conv = (2 H_k + H_v) * 128) that the shard owns,
    in the shard's own q | k | v order: indices into conv_w's rows and conv state's last dim."""
    return torch.cat([
        torch.arange(r.k0 * D, r.k1 * D),
        torch.arange(H_k * D + r.k0 * D, H_k * D + r.k1 * D),
        torch.arange(2 * H_k * D + r.v0 * D, 2 * H_k * D + r.v1 * D),
    ])


def shard_weights(w_in, w_out, conv_w, A_log, H_k: int, H_v: int, tp: int, rank: int) -> dict:
    """The rank's weights: w_in [n_in][hidden] -> its rows; w_out [hidden][H_v*128] -> its value
    heads' columns; conv_w [C_conv][4] -> its channels; A_log [H_v] -> its value heads."""
    r = head_range(H_k, H_v, tp, rank)
    rows = in_proj_rows(H_k, H_v, r).to(w_in.device)
    chans = conv_channels(H_k, H_v, r).to(conv_w.device)
    return {
        "w_in": w_in.index_select(0, rows).contiguous(),
        "w_out": w_out[:, r.v0 * D:r.v1 * D].contiguous(),
        "conv_w": conv_w.index_select(0, chans).contiguous(),
        "A_log": A_log[r.v0:r.v1].contiguous(),
        "H_k": r.H_k,
        "H_v": r.H_v,
    }


def shard_state(state, H_k: int, H_v: int, tp: int, rank: int):
    """Recurrent state [B][H_v][128][128] -> the rank's value heads (None stays None)."""
    if state is None:
        return None
    r = head_range(H_k, H_v, tp, rank)
    return state[:, r.v0:r.v1].contiguous()


def shard_conv_state(conv, H_k: int, H_v: int, tp: int, rank: int):
    """Conv state [B][3][C_conv] -> the rank's channels (None stays None)."""
    if conv is None:
        return None
    r = head_range(H_k, H_v, tp, rank)
    return conv.index_select(2, conv_channels(H_k, H_v, r).to(conv.device)).contiguous()


class TPDeltaLayer:
    """One rank's shard of a delta-rule layer.  Built from the full weights (identical on every
    rank); keeps only its slice, on the current CUDA device.  `tp` and `rank` default to the
    process group's; `partial_prefill` is the rank's own out_proj product, `prefill` adds the
    all-reduce over the group."""

    def __init__(self, w_in, w_out, conv_w, A_log, norm_w, H_k: int, H_v: int, *, group=None, tp=None,
                 rank=None, scale: float = 1.0, schedule: int = gdn.SCHEDULE_AUTO, device=None):
        if tp is None or rank is None:
            if not dist.is_initialized():
                raise RuntimeError("TPDeltaLayer: give tp and rank, or initialise torch.distributed")
            tp = dist.get_world_size(group) if tp is None else tp
            rank = dist.get_rank(group) if rank is None else rank
        self.group, self.tp, self.rank = group, int(tp), int(rank)
        self.H_k_full, self.H_v_full = int(H_k), int(H_v)
        dev = torch.device(device) if device is not None else torch.device("cuda", torch.cuda.current_device())
        w = shard_weights(w_in, w_out, conv_w, A_log, H_k, H_v, self.tp, self.rank)
        self.w = {k: (v.to(dev) if torch.is_tensor(v) else v) for k, v in w.items()}
        self.norm_w = norm_w.to(dev)
        self.heads = head_range(H_k, H_v, self.tp, self.rank)
        self.L = gdn.make_layer(self.w["w_in"], self.w["w_out"], self.w["conv_w"], self.w["A_log"], self.norm_w,
                                self.w["H_k"], self.w["H_v"], scale=scale, schedule=schedule)

    def shard_state(self, state):
        return shard_state(state, self.H_k_full, self.H_v_full, self.tp, self.rank)

    def shard_conv_state(self, conv):
        return shard_conv_state(conv, self.H_k_full, self.H_v_full, self.tp, self.rank)

    def partial_prefill(self, B: int, T: int, x, state_in=None, conv_in=None, **kw):
        """This rank's y partial [B*T][hidden] (bf16) with its heads' final states; state_in /
        conv_in are this rank's slices (see shard_state / shard_conv_state)."""
        return gdn.layer_prefill(self.L, B, T, x, state_in, conv_in, **kw)

    def prefill(self, B: int, T: int, x, state_in=None, conv_in=None, **kw):
        """The layer output, summed over the group's ranks in place; the states stay sharded."""
        y, S, C = self.partial_prefill(B, T, x, state_in, conv_in, **kw)
        if self.tp > 1:
            dist.all_reduce(y, op=dist.ReduceOp.SUM, group=self.group)
        return y, S, C
