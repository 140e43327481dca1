"""The debug build (libgdn_debug.so, compiled with GDN_DEBUG): every workspace access of the
prefill kernels is checked against the workspace's bounds, and one outside sets error bit 64
and is skipped instead of trapping.  On valid calls it must report nothing and compute exactly
what libgdn.so computes (the checks change no arithmetic): tiny, ragged, packed and fused cases.
"""
import pytest
import torch

from gated_delta_rule_81_b200 import build, gdn
from gated_delta_rule_81_b200 import inputs as gin

pytestmark = pytest.mark.gpu


def run(lib, case, schedule):
    prev = gdn._lib
    gdn._lib = lib
    try:
        d = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case["inp"].items()}
        s = gdn.make_inputs(d["q"], d["k"], d["v"], d["a"], d["b"], d["z"], d["conv_w"], d["A_log"], d["norm_w"],
                            scale=d["scale"], schedule=schedule)
        st = case["state_in"].cuda() if case["state_in"] is not None else None
        err = torch.zeros(1, dtype=torch.int32, device="cuda")
        if case["N"] > 1:
            cu = case["cu_seqlens"]
            out, S, C = gdn.prefill_varlen(s, cu.cuda(), cu, st, None, err=err)
        else:
            out, S, C = gdn.prefill(s, 1, case["lengths"][0], st, None, err=err)
        torch.cuda.synchronize()
        return out, S, C, int(err.item())
    finally:
        gdn._lib = prev


CASES = {
    "tiny": (lambda: gin.prefill_case(0), gdn.SCHEDULE_AUTO),
    "ragged": (lambda: gin.prefill_case(0, T=389), gdn.SCHEDULE_AUTO),
    "packed": (lambda: gin.prefill_case(3, lengths=[130, 64, 1, 257, 96]), gdn.SCHEDULE_AUTO),
    "fused": (lambda: gin.prefill_case(1, T=1024), 2),
}


@pytest.mark.parametrize("kind", sorted(CASES))
def test_debug_build_reports_nothing_and_matches_the_product_build(kind):
    build.build()
    prod = gdn.load()
    dbg = gdn.load(build.lib_path("libgdn_debug.so"), fresh=True)
    make, schedule = CASES[kind]
    case = make()
    o1, S1, C1, e1 = run(prod, case, schedule)
    o2, S2, C2, e2 = run(dbg, case, schedule)
    assert e1 == 0 and e2 == 0, (e1, e2)
    assert torch.equal(o1, o2) and torch.equal(S1, S2) and torch.equal(C1, C2)
