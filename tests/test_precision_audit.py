"""The precision audit behind the prefill's operand formats, on the CPU (no GPU): with every
tensor-core operand a bf16 hi/lo pair the chunk algebra stays far inside the parity bounds; with
the first operand of [Q;K]K^T in plain bf16 it breaks the output bound (the keys of a chunk are
strongly correlated after the conv and SiLU, so I + A is ill-conditioned); and the transfer form
of the chunk step (S <- S M + N) keeps the accuracy of the WY form the kernels use."""
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import inputs as gin
from precision_emulation import emulate, errors

OUT_BOUND, STATE_BOUND = 1e-2, 5e-3
T, H_k, H_v, HEADS = 256, 1, 3, [0, 2]


def case(seed, a_mean):
    inp = gin.token_inputs(T, H_k, H_v, seed=seed, a_mean=a_mean)
    inp.update(gin.weights(H_k, H_v, seed=seed))
    inp["scale"] = 1.0
    st0 = torch.zeros(1, H_v, 128, 128)
    return inp, st0, oracle.mixer(inp, [0, T], state_in=st0)


@pytest.fixture(scope="module", params=[(3, 0.0), (7, -6.0)], ids=["a~N(0,1)", "slow decay a~N(-6,1)"])
def audit_case(request):
    return case(*request.param)


def test_all_split_operands_stay_inside_the_bounds(audit_case):
    inp, st0, ref = audit_case
    out_err, st_err = errors(*emulate(inp, T, st0, H_k, H_v, HEADS), ref, HEADS)
    print(f"[audit] all split: out {out_err:.2e} state {st_err:.2e}")
    assert out_err <= 0.1 * OUT_BOUND and st_err <= 0.1 * STATE_BOUND


def test_plain_bf16_keys_in_the_gram_product_break_the_output_bound(audit_case):
    inp, st0, ref = audit_case
    out_err, _ = errors(*emulate(inp, T, st0, H_k, H_v, HEADS, prec={"qk": "bs"}), ref, HEADS)
    print(f"[audit] [Q;K]K^T first operand bf16: out {out_err:.2e}")
    assert out_err > OUT_BOUND


def test_transfer_form_keeps_the_wy_form_accuracy(audit_case):
    inp, st0, ref = audit_case
    wy = errors(*emulate(inp, T, st0, H_k, H_v, HEADS), ref, HEADS)
    tr = errors(*emulate(inp, T, st0, H_k, H_v, HEADS, form="transfer"), ref, HEADS)
    print(f"[audit] WY out {wy[0]:.2e} state {wy[1]:.2e}; transfer out {tr[0]:.2e} state {tr[1]:.2e}")
    assert tr[0] <= max(2 * wy[0], 1e-4) and tr[1] <= max(2 * wy[1], 1e-5)
