"""Head-sharded tensor parallelism of the delta-rule layer, host side (no GPU).

The shard index sets must partition the layer: every input-projection row, conv channel and
value head belongs to exactly one rank, in the layer's own q | k | v | z | a | b order within
the rank.  Then two gloo ranks each run the fp64 oracle layer on their shard (their weights and
state slices from gated_delta_rule_81_b200.tp) and all-reduce the partial outputs: the sum must
equal the oracle's unsharded layer output (up to the order of the fp64 sums), and each rank's
final recurrent and conv states must equal the unsharded layer's slices exactly, since the mixer
computes every head on its own."""
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

import oracle
from gated_delta_rule_81_b200 import inputs as gin
from gated_delta_rule_81_b200 import tp

D = 128


@pytest.mark.parametrize("H_k,H_v,n", [(16, 48, 2), (16, 48, 4), (16, 48, 16), (4, 12, 2), (2, 6, 2)])
def test_shards_partition_the_layer(H_k, H_v, n):
    lay = oracle.in_proj_layout(H_k, H_v)
    n_in = lay["total"][1]
    rows = [tp.in_proj_rows(H_k, H_v, tp.head_range(H_k, H_v, n, r)) for r in range(n)]
    assert sorted(torch.cat(rows).tolist()) == list(range(n_in))
    chans = [tp.conv_channels(H_k, H_v, tp.head_range(H_k, H_v, n, r)) for r in range(n)]
    assert sorted(torch.cat(chans).tolist()) == list(range((2 * H_k + H_v) * D))
    for r in range(n):
        hr = tp.head_range(H_k, H_v, n, r)
        assert hr.H_k == H_k // n and hr.H_v == H_v // n
        # within the rank, the rows follow the shard's own layout, field by field
        own = oracle.in_proj_layout(hr.H_k, hr.H_v)
        assert len(rows[r]) == own["total"][1]
        for name, width in (("q", D), ("k", D), ("v", D), ("z", D), ("a", 1), ("b", 1)):
            first = hr.k0 if name in ("q", "k") else hr.v0
            s0, s1 = own[name]
            expect = torch.arange(lay[name][0] + first * width, lay[name][0] + first * width + (s1 - s0))
            assert torch.equal(rows[r][s0:s1], expect), name
        # value head h of the rank belongs to key head h // G of the rank
        assert hr.v0 == hr.k0 * (H_v // H_k)


def test_head_range_rejects_uneven_splits():
    with pytest.raises(ValueError):
        tp.head_range(16, 48, 3, 0)
    with pytest.raises(ValueError):
        tp.head_range(16, 48, 2, 2)


def _case(H_k, H_v, hidden, B, T, seed):
    g = torch.Generator().manual_seed(seed)
    n_in = oracle.in_proj_layout(H_k, H_v)["total"][1]
    x = torch.randn(B * T, hidden, generator=g).to(torch.bfloat16)
    w_in = (torch.randn(n_in, hidden, generator=g) * hidden ** -0.5).to(torch.bfloat16)
    w_out = (torch.randn(hidden, H_v * D, generator=g) * (H_v * D) ** -0.5).to(torch.bfloat16)
    w = gin.weights(H_k, H_v, seed=seed)
    st = gin.recurrent_state(B, H_v, seed + 1)
    cv = gin.conv_state(B, H_k, H_v, seed + 2)
    return dict(x=x, w_in=w_in, w_out=w_out, w=w, state=st, conv=cv)


def _oracle_layer(c, w_in, w_out, conv_w, A_log, H_k, H_v, B, T, state, conv):
    return oracle.layer(c["x"], w_in, w_out, conv_w, A_log, c["w"]["norm_w"], [i * T for i in range(B + 1)],
                        H_k, H_v, state_in=state, conv_in=conv)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _worker(rank, world, port, q, H_k, H_v, hidden, B, T):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        c = _case(H_k, H_v, hidden, B, T, seed=5)  # the same full weights on every rank
        w = tp.shard_weights(c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], H_k, H_v, world, rank)
        st = tp.shard_state(c["state"], H_k, H_v, world, rank)
        cv = tp.shard_conv_state(c["conv"], H_k, H_v, world, rank)
        part = _oracle_layer(c, w["w_in"], w["w_out"], w["conv_w"], w["A_log"], w["H_k"], w["H_v"], B, T, st, cv)
        y = torch.from_numpy(np.ascontiguousarray(part["y"]))
        dist.all_reduce(y, op=dist.ReduceOp.SUM)
        q.put((rank, y.numpy(), part["state"], part["conv"]))
    finally:
        dist.destroy_process_group()


def test_two_gloo_ranks_sum_to_the_unsharded_layer():
    H_k, H_v, hidden, B, T = 4, 12, 256, 2, 70
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(r, 2, port, q, H_k, H_v, hidden, B, T)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    c = _case(H_k, H_v, hidden, B, T, seed=5)
    full = _oracle_layer(c, c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], H_k, H_v, B, T, c["state"],
                         c["conv"])
    for rank, y, S, C in res:
        np.testing.assert_allclose(y, full["y"], rtol=0, atol=1e-12 * np.max(np.abs(full["y"])))
        hr = tp.head_range(H_k, H_v, 2, rank)
        np.testing.assert_array_equal(S, full["state"][:, hr.v0:hr.v1])
        np.testing.assert_array_equal(C, full["conv"][:, :, tp.conv_channels(H_k, H_v, hr).numpy()])


def test_layer_needs_a_group_or_explicit_rank():
    """Without torch.distributed initialised, TPDeltaLayer must be told tp and rank; the shard
    helpers pass absent states through."""
    assert not dist.is_initialized()
    w = torch.zeros(1)
    with pytest.raises(RuntimeError):
        tp.TPDeltaLayer(w, w, w, w, w, 16, 48)
    assert tp.shard_state(None, 16, 48, 2, 0) is None and tp.shard_conv_state(None, 16, 48, 2, 1) is None
    st = torch.arange(2 * 48 * 2 * 2, dtype=torch.float32).reshape(2, 48, 2, 2)
    assert torch.equal(tp.shard_state(st, 16, 48, 2, 1), st[:, 24:])


def _prefill_worker(rank, world, port, q, H_k, H_v, hidden, B, T):
    """One rank of TPDeltaLayer.prefill with the library's layer call replaced by the fp64 oracle
    on the rank's own shard (rounded to bf16, the layer's output format), so that the layer's own
    plumbing runs on the CPU: the shard it keeps, the group it was given, and the in-place bf16
    all-reduce of its partial output over that group."""
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        group = dist.new_group(list(range(world)))
        c = _case(H_k, H_v, hidden, B, T, seed=9)
        layer = tp.TPDeltaLayer(c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], c["w"]["norm_w"], H_k, H_v,
                                group=group, device="cpu")
        assert (layer.tp, layer.rank) == (world, rank)
        partials = {}

        def stand_in(L, B_, T_, x, state_in=None, conv_in=None, **kw):
            assert L is layer.L
            w = layer.w
            res = oracle.layer(x, w["w_in"], w["w_out"], w["conv_w"], w["A_log"], layer.norm_w,
                               [i * T_ for i in range(B_ + 1)], w["H_k"], w["H_v"], state_in=state_in, conv_in=conv_in)
            y = torch.from_numpy(np.ascontiguousarray(res["y"])).to(torch.bfloat16)
            partials["y"] = y.clone()
            return y, torch.from_numpy(res["state"]), torch.from_numpy(res["conv"])

        tp.gdn.layer_prefill = stand_in
        y, S, C = layer.prefill(B, T, c["x"], layer.shard_state(c["state"]), layer.shard_conv_state(c["conv"]))
        q.put((rank, partials["y"].float().numpy(), y.float().numpy(), S.numpy(), C.numpy()))
    finally:
        dist.destroy_process_group()


def test_tp_layer_prefill_all_reduces_its_partials_over_the_group():
    H_k, H_v, hidden, B, T = 4, 12, 128, 1, 40
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_prefill_worker, args=(r, 2, port, q, H_k, H_v, hidden, B, T)) for r in range(2)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in procs), key=lambda r: r[0])
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    (_, y0, out0, S0, C0), (_, y1, out1, S1, C1) = res
    # both ranks hold the same sum, the bf16 rounding of the two bf16 partials' sum
    np.testing.assert_array_equal(out0, out1)
    want = torch.from_numpy(y0 + y1).to(torch.bfloat16).float().numpy()
    np.testing.assert_array_equal(out0, want)
    # and it is the unsharded layer up to the bf16 roundings of the partials and of the sum
    c = _case(H_k, H_v, hidden, B, T, seed=9)
    full = _oracle_layer(c, c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], H_k, H_v, B, T, c["state"],
                         c["conv"])
    bound = 2.0 ** -8 * (np.abs(y0) + np.abs(y1)) + 2.0 ** -8 * np.abs(full["y"]) + 1e-6
    assert np.all(np.abs(out0 - full["y"]) <= bound)
    # the states stay sharded: each rank's are the unsharded layer's slices
    for rank, S, C in ((0, S0, C0), (1, S1, C1)):
        hr = tp.head_range(H_k, H_v, 2, rank)
        np.testing.assert_array_equal(S, full["state"][:, hr.v0:hr.v1])
        np.testing.assert_array_equal(C, full["conv"][:, :, tp.conv_channels(H_k, H_v, hr).numpy()])
