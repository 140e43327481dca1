"""Failure detection on the device without a fault: every wait in the library's kernels is
bounded (about 2^31 SM cycles, a little over a second), after which it ORs error bit 1 into the
caller's error word and returns false so that the kernel unwinds.  A test kernel in the test
library waits on an mbarrier that nothing arrives on and on a ready flag that nothing sets:
each wait must give up after the limit and report bit 1; a second waiter of the same block must
leave as soon as the first has given up (the block's abort flag) instead of running out its own
limit; and the context must stay usable afterwards (a prefill runs and matches its own earlier
result bit for bit)."""
import ctypes

import pytest
import torch

from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import err_word, selftest_lib

pytestmark = pytest.mark.gpu


def _lib():
    lib = selftest_lib()
    lib.gdn_selftest_wait.argtypes = [ctypes.c_int, ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    lib.gdn_selftest_wait.restype = ctypes.c_int
    lib.gdn_selftest_wait_limit_cycles.restype = ctypes.c_longlong
    return lib


def _small_prefill():
    case = gin.prefill_case(0, seed=3, T=130)
    inp = {k: (v.cuda() if torch.is_tensor(v) else v) for k, v in case["inp"].items()}
    s = gdn.make_inputs(inp["q"], inp["k"], inp["v"], inp["a"], inp["b"], inp["z"], inp["conv_w"], inp["A_log"],
                        inp["norm_w"], scale=inp["scale"])
    err = err_word()
    out, S, _ = gdn.prefill(s, case["N"], case["lengths"][0], None, None, err=err)
    torch.cuda.synchronize()
    return out, S, int(err.item())


def test_bounded_waits_give_up_report_and_unwind():
    lib = _lib()
    limit = lib.gdn_selftest_wait_limit_cycles()
    out_before, S_before, e0 = _small_prefill()
    assert e0 == 0
    flag = torch.zeros(1, dtype=torch.int32, device="cuda")  # nothing ever sets it

    # an mbarrier nothing arrives on: warp 0 gives up after the limit; warp 1, which started
    # waiting 2^30 cycles later, leaves when warp 0 raises the block's abort
    err = err_word()
    res = torch.zeros(4, dtype=torch.int64, device="cuda")
    assert lib.gdn_selftest_wait(0, ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(flag.data_ptr()),
                                 ctypes.c_void_p(res.data_ptr())) == 0
    torch.cuda.synchronize()
    ok0, waited0, ok1, waited1 = res.tolist()
    print(f"[waits] mbarrier: warp 0 ok={ok0} waited {waited0 / limit:.3f} limits; warp 1 ok={ok1} "
          f"waited {waited1 / limit:.3f} limits; err={int(err.item())}")
    assert ok0 == 0 and ok1 == 0
    assert int(err.item()) & 1
    assert waited0 >= limit
    assert waited1 < 0.75 * limit  # left on the abort, not on its own limit

    # a ready flag nothing sets
    err = err_word()
    res.zero_()
    assert lib.gdn_selftest_wait(1, ctypes.c_void_p(err.data_ptr()), ctypes.c_void_p(flag.data_ptr()),
                                 ctypes.c_void_p(res.data_ptr())) == 0
    torch.cuda.synchronize()
    ok0, waited0 = res.tolist()[:2]
    print(f"[waits] ready flag: ok={ok0} waited {waited0 / limit:.3f} limits; err={int(err.item())}")
    assert ok0 == 0 and waited0 >= limit and int(err.item()) & 1

    # the context is still usable, and gives the same result as before
    out_after, S_after, e1 = _small_prefill()
    assert e1 == 0
    assert torch.equal(out_after, out_before) and torch.equal(S_after, S_before)
