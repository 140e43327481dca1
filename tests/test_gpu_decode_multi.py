"""gdn_decode_multi (CUDA, through the C ABI): T new tokens per sequence in one call,
with the states in slots of a pool.  Checked against the fp64 oracle run over the
same tokens, against T single-token decode steps (bitwise), across the two launch
grids (bitwise), and for the slot indirection (permuted slots, untouched slots, a
slot outside the pool)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import OUT_TOL, STATE_TOL, err_word, out_error, raw_out_error, state_error

pytestmark = pytest.mark.gpu

TOKEN_KEYS = ("q", "k", "v", "z", "a", "b")
BAD_SLOT_BIT = 8


def seq_major(case, T):
    """The case's first T steps reordered so that token n * T + t is step t of sequence n."""
    N = case["N"]
    idx = torch.tensor([t * N + n for n in range(N) for t in range(T)])
    return {k: case["tok"][k][idx] for k in TOKEN_KEYS}


def make_dev_inputs(tok, w, scale):
    dev_tok = {k: v.cuda() for k, v in tok.items()}
    dev_w = {k: v.cuda() for k, v in w.items()}
    inp = gdn.make_inputs(*(dev_tok[k] for k in ("q", "k", "v", "a", "b", "z")), dev_w["conv_w"], dev_w["A_log"],
                          dev_w["norm_w"], scale=scale)
    return (dev_tok, dev_w), inp


def oracle_multi(case, tok, T, seqs):
    inp = {k: torch.cat([tok[k][n * T:(n + 1) * T] for n in seqs]) for k in TOKEN_KEYS}
    inp.update(case["w"])
    inp["scale"] = case["scale"]
    cu = [i * T for i in range(len(seqs) + 1)]
    return oracle.mixer(inp, cu, state_in=case["state"][seqs], conv_in=case["conv_state"][seqs])


@pytest.mark.parametrize("T", [1, 2, 3, 4, 8])
@pytest.mark.parametrize("heads", [(2, 6), (1, 8)])
def test_decode_multi_matches_oracle(T, heads):
    H_k, H_v = heads
    N = 5
    case = gin.decode_case(N=N, steps=T, H_k=H_k, H_v=H_v, seed=30 + T)
    tok = seq_major(case, T)
    keep, inp = make_dev_inputs(tok, case["w"], case["scale"])
    state = case["state"].cuda().clone()
    conv = case["conv_state"].cuda().clone()
    err = err_word()
    out = gdn.decode_multi(inp, N, T, state, conv, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_multi(case, tok, T, list(range(N)))
    print(f"[parity] decode_multi T={T} H={H_k}/{H_v}: out_err={out_error(out, ref['out']):.3e} "
          f"raw={raw_out_error(out, ref['out']):.3e} state_err={state_error(state, ref['state']):.3e}")
    assert out_error(out, ref["out"]) <= OUT_TOL
    assert state_error(state, ref["state"]) <= STATE_TOL
    np.testing.assert_array_equal(conv.float().cpu().numpy(), ref["conv"])


@pytest.mark.parametrize("T", [2, 5, 8])
def test_decode_multi_bitwise_equals_single_steps(T):
    """One call with T tokens applies exactly the arithmetic of T single-token steps."""
    N, H_k, H_v = 6, 2, 6
    case = gin.decode_case(N=N, steps=T, H_k=H_k, H_v=H_v, seed=50 + T)
    tok = seq_major(case, T)
    keep, inp = make_dev_inputs(tok, case["w"], case["scale"])
    S_multi = case["state"].cuda().clone()
    C_multi = case["conv_state"].cuda().clone()
    y_multi = gdn.decode_multi(inp, N, T, S_multi, C_multi)
    S_one = case["state"].cuda().clone()
    C_one = case["conv_state"].cuda().clone()
    dev_w = keep[1]
    ys = []
    for t in range(T):
        step = {k: case["tok"][k][t * N:(t + 1) * N].cuda() for k in TOKEN_KEYS}
        st = gdn.make_inputs(*(step[k] for k in ("q", "k", "v", "a", "b", "z")), dev_w["conv_w"], dev_w["A_log"],
                             dev_w["norm_w"], scale=case["scale"])
        ys.append(gdn.decode_step(st, N, S_one, C_one))
    torch.cuda.synchronize()
    y_one = torch.stack(ys, 1).reshape(N * T, H_v, 128)  # [seq][step]
    assert torch.equal(y_multi, y_one)
    assert torch.equal(S_multi, S_one)
    assert torch.equal(C_multi, C_one)


@pytest.mark.parametrize("T,heads", [(1, (2, 6)), (3, (1, 8))])
def test_decode_multi_value_head_grid_bitwise_equals_key_head_grid(T, heads):
    """Few sequences run one CTA per value head (the G CTAs of a key head in a cluster),
    a batch that fills the SMs one CTA per key head: the same sequences give bitwise
    equal outputs, states and conv states either way."""
    H_k, H_v = heads
    n_sm = torch.cuda.get_device_properties(0).multi_processor_count
    N_big, N_small = -(-n_sm // H_k) + 1, 3
    assert N_big * H_k >= n_sm and N_small * H_k < n_sm  # the two calls take different grids
    case = gin.decode_case(N=N_big, steps=T, H_k=H_k, H_v=H_v, seed=90 + T)
    tok = seq_major(case, T)
    keep, inp = make_dev_inputs(tok, case["w"], case["scale"])
    S_big = case["state"].cuda().clone()
    C_big = case["conv_state"].cuda().clone()
    y_big = gdn.decode_multi(inp, N_big, T, S_big, C_big)
    dev_w = keep[1]
    for n0 in range(0, N_big, N_small):
        seqs = list(range(n0, min(n0 + N_small, N_big)))
        rows = [n * T + t for n in seqs for t in range(T)]
        part = {k: tok[k][rows].cuda() for k in TOKEN_KEYS}
        pin = gdn.make_inputs(*(part[k] for k in ("q", "k", "v", "a", "b", "z")), dev_w["conv_w"], dev_w["A_log"],
                              dev_w["norm_w"], scale=case["scale"])
        S = case["state"][seqs].cuda()
        C = case["conv_state"][seqs].cuda()
        y = gdn.decode_multi(pin, len(seqs), T, S, C)
        torch.cuda.synchronize()
        assert torch.equal(y, y_big[rows[0]:rows[-1] + 1])
        assert torch.equal(S, S_big[seqs])
        assert torch.equal(C, C_big[seqs])


def test_decode_multi_state_slots():
    """Sequences read and write their own slot of a larger pool; the other slots stay as they were."""
    N, T, H_k, H_v, n_slots = 4, 3, 2, 6, 9
    slots = [7, 0, 4, 2]
    case = gin.decode_case(N=N, steps=T, H_k=H_k, H_v=H_v, seed=71)
    tok = seq_major(case, T)
    keep, inp = make_dev_inputs(tok, case["w"], case["scale"])
    pool_S = gin.recurrent_state(n_slots, H_v, seed=72, kind="normal")
    pool_C = gin.conv_state(n_slots, H_k, H_v, seed=73)
    pool_S[slots] = case["state"]
    pool_C[slots] = case["conv_state"]
    S = pool_S.cuda()
    C = pool_C.cuda()
    slot_dev = torch.tensor(slots, dtype=torch.int32, device="cuda")
    err = err_word()
    out = gdn.decode_multi(inp, N, T, S, C, state_slot=slot_dev, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_multi(case, tok, T, list(range(N)))
    assert out_error(out, ref["out"]) <= OUT_TOL
    assert state_error(S[slots], ref["state"]) <= STATE_TOL
    np.testing.assert_array_equal(C[slots].float().cpu().numpy(), ref["conv"])
    rest = [i for i in range(n_slots) if i not in slots]
    assert torch.equal(S[rest].cpu(), pool_S[rest])
    assert torch.equal(C[rest].cpu(), pool_C[rest])


def test_decode_multi_slot_outside_pool_is_reported():
    """A slot outside [0, n_slots) sets the error bit and leaves that sequence alone;
    the other sequences are still advanced."""
    N, T, H_k, H_v, n_slots = 3, 2, 2, 6, 3
    case = gin.decode_case(N=N, steps=T, H_k=H_k, H_v=H_v, seed=81)
    tok = seq_major(case, T)
    keep, inp = make_dev_inputs(tok, case["w"], case["scale"])
    S = case["state"].cuda().clone()
    C = case["conv_state"].cuda().clone()
    slot_dev = torch.tensor([0, n_slots, 2], dtype=torch.int32, device="cuda")
    err = err_word()
    out = gdn.decode_multi(inp, N, T, S, C, state_slot=slot_dev, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & BAD_SLOT_BIT
    ref = oracle_multi(case, tok, T, [0, 2])
    y = torch.cat([out[0:T], out[2 * T:3 * T]])
    assert out_error(y, ref["out"]) <= OUT_TOL
    assert state_error(S[[0, 2]], ref["state"]) <= STATE_TOL
    assert torch.equal(S[1].cpu(), case["state"][1])
    assert torch.equal(C[1].cpu(), case["conv_state"][1])
