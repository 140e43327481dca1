"""gdn_layer_prefill (in_proj GEMM -> mixer on the projection's columns -> out_proj GEMM,
through the C ABI) against the fp64 oracle layer.

The input projection is chosen exact in bf16 (two power-of-two weights per output
channel, inputs on a 1/8 grid): the GPU's fp32 accumulation and the oracle's fp64
product then give the same bf16 projection, so the layer output is held to the
mixer's own bounds: |y - y_ref| <= 1e-2 rms(y_ref) + 2^-8 |y_ref| per element, and
the final state to ||S - S_ref||_F <= 5e-3 ||S_ref||_F.  The dense GEMM itself is
checked on random data in test_gpu_gemm.py."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import OUT_TOL, STATE_TOL, err_word, out_error, state_error

pytestmark = pytest.mark.gpu


def exact_layer_case(H_k, H_v, hidden, B, T, seed, with_state=True, with_conv=True):
    g = torch.Generator().manual_seed(seed)
    n_in = int(gdn.load().gdn_layer_n_in(H_k, H_v))
    x = (torch.randint(-16, 17, (B * T, hidden), generator=g).float() / 8).to(torch.bfloat16)
    w_in = torch.zeros(n_in, hidden)
    cols = torch.stack([torch.randperm(hidden, generator=g)[:2] for _ in range(n_in)])
    vals = torch.tensor([1.0, -1.0, 0.5, -0.5, 0.25, -0.25])[torch.randint(0, 6, (n_in, 2), generator=g)]
    w_in.scatter_(1, cols, vals)
    w_in = w_in.to(torch.bfloat16)
    w_out = (torch.randn(hidden, H_v * 128, generator=g) * (H_v * 128) ** -0.5).to(torch.bfloat16)
    w = gin.weights(H_k, H_v, seed=seed)
    st = gin.recurrent_state(B, H_v, seed + 1) if with_state else None
    cv = gin.conv_state(B, H_k, H_v, seed + 2) if with_conv else None
    return dict(x=x, w_in=w_in, w_out=w_out, w=w, state=st, conv=cv, H_k=H_k, H_v=H_v, B=B, T=T)


def run_layer(c, schedule=gdn.SCHEDULE_AUTO):
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out")}
    w = {k: v.cuda() for k, v in c["w"].items()}
    L = gdn.make_layer(d["w_in"], d["w_out"], w["conv_w"], w["A_log"], w["norm_w"], c["H_k"], c["H_v"],
                       schedule=schedule)
    st = c["state"].cuda() if c["state"] is not None else None
    cv = c["conv"].cuda() if c["conv"] is not None else None
    err = err_word()
    y, S, C = gdn.layer_prefill(L, c["B"], c["T"], d["x"], st, cv, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    return y, S, C


def oracle_layer(c):
    B, T = c["B"], c["T"]
    return oracle.layer(c["x"], c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], c["w"]["norm_w"],
                        [i * T for i in range(B + 1)], c["H_k"], c["H_v"], state_in=c["state"],
                        conv_in=c["conv"])


@pytest.mark.parametrize("H_k,H_v,hidden,B,T", [(2, 6, 256, 1, 130), (2, 6, 512, 2, 70), (16, 48, 5120, 1, 256)])
def test_layer_matches_oracle(H_k, H_v, hidden, B, T):
    c = exact_layer_case(H_k, H_v, hidden, B, T, seed=hidden + T)
    y, S, C = run_layer(c)
    ref = oracle_layer(c)
    e_y, e_s = out_error(y, ref["y"]), state_error(S, ref["state"])
    print(f"[parity] layer {H_k}/{H_v} hidden {hidden} B {B} T {T}: y_err={e_y:.3e} state_err={e_s:.3e}")
    assert e_y <= OUT_TOL
    assert e_s <= STATE_TOL
    np.testing.assert_array_equal(C.float().cpu().numpy(), ref["conv"])


def test_layer_schedules_bitwise_equal():
    c = exact_layer_case(2, 6, 256, 1, 300, seed=3)
    a = run_layer(c, gdn.SCHEDULE_FUSED)
    b = run_layer(c, gdn.SCHEDULE_TWO_LAUNCHES)
    for x, y in zip(a, b):
        assert torch.equal(x, y)


@pytest.mark.parametrize("T_dec", [1, 3])
def test_layer_decode_continues_the_layer_prefill(T_dec):
    """gdn_layer_prefill of a prompt, then two gdn_layer_decode calls of T_dec tokens each on
    the prefill's own final state and conv buffers (the handoff is the same buffers): the
    decoded tokens' outputs and the final states match the oracle layer run over the whole
    sequences."""
    H_k, H_v, hidden, B, T0, calls = 2, 6, 256, 2, 70, 2
    T = T0 + calls * T_dec
    c = exact_layer_case(H_k, H_v, hidden, B, T, seed=40 + T_dec)
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out")}
    w = {k: v.cuda() for k, v in c["w"].items()}
    L = gdn.make_layer(d["w_in"], d["w_out"], w["conv_w"], w["A_log"], w["norm_w"], H_k, H_v)
    err = err_word()
    xs = d["x"].reshape(B, T, hidden)
    _, S, C = gdn.layer_prefill(L, B, T0, xs[:, :T0].reshape(B * T0, hidden).contiguous(), c["state"].cuda(),
                                c["conv"].cuda(), err=err)
    ys = []
    for i in range(calls):
        xi = xs[:, T0 + i * T_dec:T0 + (i + 1) * T_dec].reshape(B * T_dec, hidden).contiguous()
        ys.append(gdn.layer_decode(L, B, T_dec, xi, S, C, err=err).reshape(B, T_dec, hidden))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    ref = oracle_layer(c)
    y_ref = ref["y"].reshape(B, T, hidden)[:, T0:]
    y = torch.cat(ys, dim=1)
    e_y, e_s = out_error(y.reshape(-1, hidden), y_ref.reshape(-1, hidden)), state_error(S, ref["state"])
    print(f"[parity] layer decode after a {T0}-token layer prefill, {calls} x {T_dec} tokens: y_err={e_y:.3e} "
          f"state_err={e_s:.3e}")
    assert e_y <= OUT_TOL and e_s <= STATE_TOL
    np.testing.assert_array_equal(C.float().cpu().numpy(), ref["conv"])
