"""gdn_prefill_host (host tensors in and out, staged through the caller's device workspace)
against gdn_prefill on the same values: outputs, final state and conv state must be bitwise
equal, with strided host inputs (all six per-token tensors as column slices of one pinned
projection-like buffer), a recurrent state and conv history in, and a length that ends
inside a chunk.  Two calls on two streams with two workspaces give the same results too."""
import pytest
import torch

from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import err_word

pytestmark = pytest.mark.gpu


def test_prefill_host_equals_device_prefill():
    H_k, H_v, B, T = 4, 12, 2, 150
    w = gin.weights(H_k, H_v, seed=9)
    g = torch.Generator().manual_seed(9)
    T_tot = B * T
    widths = [H_k * 128, H_k * 128, H_v * 128, H_v * 128, H_v, H_v]  # q k v z a b
    ld = (sum(widths) + 7) // 8 * 8
    buf = torch.randn(T_tot, ld, generator=g).to(torch.bfloat16).pin_memory()
    offs = [sum(widths[:i]) for i in range(6)]
    q, k, v, z, a, b = (buf[:, o:o + wd] for o, wd in zip(offs, widths))
    st_in = (torch.randn(B, H_v, 128, 128, generator=g) * 0.1).pin_memory()
    cv_in = torch.randn(B, 3, (2 * H_k + H_v) * 128, generator=g).to(torch.bfloat16).pin_memory()
    wd = {kk: vv.cuda() for kk, vv in w.items()}

    # device reference
    dbuf = buf.cuda()
    dq, dk, dv, dz, da, db = (dbuf[:, o:o + wd_] for o, wd_ in zip(offs, widths))
    s_dev = gdn.make_inputs(dq, dk, dv, da, db, dz, wd["conv_w"], wd["A_log"], wd["norm_w"])
    err = err_word()
    out_ref, S_ref, C_ref = gdn.prefill(s_dev, B, T, st_in.cuda(), cv_in.cuda(), err=err)

    s_host = gdn.make_inputs(q, k, v, a, b, z, wd["conv_w"], wd["A_log"], wd["norm_w"])
    results = []
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    for j in range(2):
        out_h = torch.empty(T_tot, H_v, 128, dtype=torch.bfloat16).pin_memory()
        S_h = torch.empty(B, H_v, 128, 128).pin_memory()
        C_h = torch.empty(B, 3, (2 * H_k + H_v) * 128, dtype=torch.bfloat16).pin_memory()
        gdn.prefill_host(s_host, B, T, out_h, state_in=st_in, state_out=S_h, conv_in=cv_in, conv_out=C_h, err=err,
                         stream=streams[j])
        results.append((out_h, S_h, C_h))
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    for out_h, S_h, C_h in results:
        assert torch.equal(out_h, out_ref.cpu())
        assert torch.equal(S_h, S_ref.cpu())
        assert torch.equal(C_h, C_ref.cpu())
