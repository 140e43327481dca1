"""Parity of gdn_decode_step (CUDA, through the C ABI) with the fp64 oracle run
token by token, and the prefill -> decode hand-off."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import OUT_TOL, STATE_TOL, device_inputs, err_word, out_error, raw_out_error, state_error

pytestmark = pytest.mark.gpu

TOKEN_KEYS = ("q", "k", "v", "z", "a", "b")


def run_decode(case, record_steps=()):
    N, steps = case["N"], case["steps"]
    state = case["state"].cuda().clone()
    conv = case["conv_state"].cuda().clone()
    dev_tok = {k: case["tok"][k].cuda() for k in TOKEN_KEYS}
    w = {k: v.cuda() for k, v in case["w"].items()}
    err = err_word()
    outs, snaps = [], {}
    for s in range(steps):
        sl = slice(s * N, (s + 1) * N)
        inp = gdn.make_inputs(*(dev_tok[k][sl] for k in ("q", "k", "v", "a", "b", "z")), w["conv_w"], w["A_log"],
                              w["norm_w"], scale=case["scale"])
        outs.append(gdn.decode_step(inp, N, state, conv, err=err))
        if s + 1 in record_steps:
            snaps[s + 1] = (state.clone(), conv.clone())
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return torch.stack(outs), state, conv, snaps


def oracle_decode(case, seqs, steps):
    """Oracle over the first `steps` tokens of the chosen sequences, each run as one
    sequence that starts from its own state and conv history."""
    N = case["N"]
    tok = case["tok"]
    idx = torch.tensor([s * N + n for n in seqs for s in range(steps)])
    inp = {k: tok[k][idx] for k in TOKEN_KEYS}
    inp.update(case["w"])
    inp["scale"] = case["scale"]
    cu = [i * steps for i in range(len(seqs) + 1)]
    return oracle.mixer(inp, cu, state_in=case["state"][seqs], conv_in=case["conv_state"][seqs])


def test_decode_small_all_sequences():
    case = gin.decode_case(N=5, steps=9, H_k=2, H_v=6)
    outs, S, C, _ = run_decode(case)
    ref = oracle_decode(case, list(range(5)), 9)
    y = outs.permute(1, 0, 2, 3).reshape(5 * 9, 6, 128)  # [seq][step] order like the oracle
    print(f"[parity] decode small: out_err={out_error(y, ref['out']):.3e} raw={raw_out_error(y, ref['out']):.3e} "
          f"state_err={state_error(S, ref['state']):.3e}")
    assert out_error(y, ref["out"]) <= OUT_TOL
    assert state_error(S, ref["state"]) <= STATE_TOL
    np.testing.assert_array_equal(C.float().cpu().numpy(), ref["conv"])


def test_decode_config4_sampled_sequences():
    case = gin.decode_case(4)
    outs, S, C, snaps = run_decode(case, record_steps=(1, 8))
    seqs = [0, 77, 255]
    for steps in (1, 8, 64):
        ref = oracle_decode(case, seqs, steps)
        st, cv = (S, C) if steps == 64 else snaps[steps]
        assert state_error(st[seqs], ref["state"]) <= STATE_TOL
        np.testing.assert_array_equal(cv[seqs].float().cpu().numpy(), ref["conv"])
        y = outs[:steps, seqs].permute(1, 0, 2, 3).reshape(len(seqs) * steps, 48, 128)
        assert out_error(y, ref["out"]) <= OUT_TOL
    # the whole batch stays finite
    assert torch.isfinite(S).all() and torch.isfinite(outs.float()).all()


def test_prefill_then_decode_matches_longer_prefill():
    H_k, H_v, T0, n_dec = 2, 6, 70, 6
    inp = gin.token_inputs(T0 + n_dec, H_k, H_v, seed=21)
    inp.update(gin.weights(H_k, H_v, seed=21))
    inp["scale"] = 1.0
    st0 = gin.recurrent_state(1, H_v, seed=22)
    ref = oracle.mixer(inp, [0, T0 + n_dec], state_in=st0)
    keep, s = device_inputs({k: (v[:T0] if k in TOKEN_KEYS else v) for k, v in inp.items()})
    out0, S, C = gdn.prefill(s, 1, T0, st0.cuda(), None)
    ys = [out0]
    for t in range(T0, T0 + n_dec):
        kt, st = device_inputs({k: (v[t:t + 1] if k in TOKEN_KEYS else v) for k, v in inp.items()})
        ys.append(gdn.decode_step(st, 1, S, C))
    torch.cuda.synchronize()
    y = torch.cat(ys)
    assert out_error(y, ref["out"]) <= OUT_TOL
    assert state_error(S, ref["state"]) <= STATE_TOL
