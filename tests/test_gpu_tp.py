"""Head-sharded tensor parallelism of the delta-rule layer on the GPU (through the C ABI).

This run has one GPU, so the two ranks of tp = 2 run one after the other in one process
(TPDeltaLayer with explicit tp and rank); the all-reduce of their bf16 partial outputs is
emulated by summing them in fp32 and rounding once to bf16, as a two-rank bf16 sum does.
Checks: (1) the summed output against the fp64 oracle's unsharded layer, within the layer
bound plus the rounding of the two partials (2^-8 |partial| each); (2) each rank's final
recurrent state and conv state equal, bit for bit, the unsharded GPU layer's slices of its
heads (the kernels compute every head on its own, and the exact input projection makes the
projection GEMM's output the same whatever its width)."""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn, tp
from gpu_helpers import OUT_TOL, STATE_TOL, err_word, state_error
from test_gpu_layer import exact_layer_case

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("H_k,H_v,hidden,B,T", [(4, 12, 256, 2, 130), (16, 48, 1024, 1, 200)])
def test_two_shards_sum_to_the_layer(H_k, H_v, hidden, B, T):
    c = exact_layer_case(H_k, H_v, hidden, B, T, seed=T + H_k)
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out")}
    w = {k: v.cuda() for k, v in c["w"].items()}
    st, cv = c["state"].cuda(), c["conv"].cuda()
    err = err_word()
    L_full = gdn.make_layer(d["w_in"], d["w_out"], w["conv_w"], w["A_log"], w["norm_w"], H_k, H_v)
    y_full, S_full, C_full = gdn.layer_prefill(L_full, B, T, d["x"], st, cv, err=err)
    parts, states, convs = [], [], []
    for rank in range(2):
        layer = tp.TPDeltaLayer(d["w_in"], d["w_out"], w["conv_w"], w["A_log"], w["norm_w"], H_k, H_v, tp=2,
                                rank=rank)
        y, S, C = layer.partial_prefill(B, T, d["x"], layer.shard_state(st), layer.shard_conv_state(cv), err=err)
        parts.append(y)
        states.append(S)
        convs.append(C)
        hr = layer.heads
        torch.cuda.synchronize()
        assert torch.equal(S, S_full[:, hr.v0:hr.v1]), f"rank {rank} state"
        assert torch.equal(C, C_full[:, :, tp.conv_channels(H_k, H_v, hr).cuda()]), f"rank {rank} conv"
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    y = (parts[0].float() + parts[1].float()).to(torch.bfloat16)
    ref = oracle.layer(c["x"], c["w_in"], c["w_out"], c["w"]["conv_w"], c["w"]["A_log"], c["w"]["norm_w"],
                       [i * T for i in range(B + 1)], H_k, H_v, state_in=c["state"], conv_in=c["conv"])
    y_ref = ref["y"]
    p_abs = np.abs(parts[0].double().cpu().numpy()) + np.abs(parts[1].double().cpu().numpy())
    bound = OUT_TOL * np.sqrt(np.mean(y_ref ** 2)) + 2.0 ** -8 * (np.abs(y_ref) + p_abs)
    ratio = float(np.max(np.abs(y.double().cpu().numpy() - y_ref) / bound))
    e_s = state_error(torch.cat(states, dim=1), ref["state"])
    print(f"[parity] tp=2 layer {H_k}/{H_v} hidden {hidden} B {B} T {T}: y err/bound={ratio:.3f} state_err={e_s:.3e}")
    assert ratio <= 1.0
    assert e_s <= STATE_TOL
