"""Parity of gdn_prefill / gdn_prefill_varlen (CUDA, through the C ABI) with the
fp64 oracle, plus the bitwise properties of the varlen path.

Tolerances (gpu_helpers): element-wise |y_gpu - y_ref| <= 1e-2 rms(y_ref) + 2^-8 |y_ref|
over the compared outputs -- the mixer's arithmetic bound plus the bf16 output's own
rounding, which no bf16 result can avoid (outputs reach ~20 rms) -- with the plain
max |y_gpu - y_ref| / rms(y_ref) printed beside it; and
||S_gpu - S_ref||_F / ||S_ref||_F <= 5e-3 per sequence.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gated_delta_rule_81_b200 import inputs as gin
from gpu_helpers import OUT_TOL, STATE_TOL, device_inputs, err_word, out_error, raw_out_error, state_error

pytestmark = pytest.mark.gpu


def small_case(lengths, H_k=2, H_v=6, seed=11, a_mean=0.0, with_state=True, with_conv=False):
    T = sum(lengths)
    inp = gin.token_inputs(T, H_k, H_v, seed, a_mean)
    inp.update(gin.weights(H_k, H_v, seed))
    inp["scale"] = 1.0
    N = len(lengths)
    return {"inp": inp, "cu_seqlens": gin.cu_from_lengths(lengths), "lengths": list(lengths), "N": N,
            "H_k": H_k, "H_v": H_v,
            "state_in": gin.recurrent_state(N, H_v, seed + 1) if with_state else None,
            "conv_in": gin.conv_state(N, H_k, H_v, seed + 2) if with_conv else None}


def run_gpu(case, uniform=False, conv_in=None, schedule=gdn.SCHEDULE_AUTO):
    keep, s = device_inputs(case["inp"])
    s.schedule = schedule
    st = case.get("state_in")
    st = st.cuda() if st is not None else None
    cv = conv_in if conv_in is not None else case.get("conv_in")
    cv = cv.cuda() if cv is not None else None
    err = err_word()
    if uniform:
        N = case["N"]
        T = case["lengths"][0]
        out, S, C = gdn.prefill(s, N, T, st, cv, err=err)
    else:
        cu = case["cu_seqlens"]
        out, S, C = gdn.prefill_varlen(s, cu.cuda(), cu, st, cv, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, f"device error word {int(err.item())}"
    del keep
    return out, S, C


def run_oracle(case, heads=None):
    return oracle.mixer(case["inp"], case["cu_seqlens"].tolist(), state_in=case.get("state_in"),
                        conv_in=case.get("conv_in"), heads=heads)


def check(case, out, S, C, ref, heads=None):
    eo = out_error(out, ref["out"], heads)
    es = state_error(S, ref["state"], heads)
    print(f"[parity] out_err={eo:.3e} raw_max_abs/rms={raw_out_error(out, ref['out'], heads):.3e} "
          f"state_err={es:.3e}")
    assert eo <= OUT_TOL, f"output error {eo:.3e}"
    assert es <= STATE_TOL, f"state error {es:.3e}"
    np.testing.assert_array_equal(C.float().cpu().numpy(), ref["conv"])
    return eo, es


# ------------------------------------------------------------------ oracle parity


def test_config0_tiny():
    case = gin.prefill_case(0)
    case["conv_in"] = None
    out, S, C = run_gpu(case, uniform=True)
    check(case, out, S, C, run_oracle(case))


@pytest.mark.parametrize("lengths", [[1], [2], [3], [63], [64], [65], [127], [200], [1, 64, 0, 65, 130, 3]])
def test_ragged_lengths(lengths):
    case = small_case(lengths, with_conv=True)
    out, S, C = run_gpu(case)
    check(case, out, S, C, run_oracle(case))


def test_config1_layer_prefill():
    case = gin.prefill_case(1)
    out, S, C = run_gpu(case, uniform=True)
    check(case, out, S, C, run_oracle(case))


def test_config3_varlen_sampled_heads():
    case = gin.prefill_case(3)
    heads = [0, 7, 29, 47]
    out, S, C = run_gpu(case)
    check(case, out, S, C, run_oracle(case, heads), heads)


@pytest.mark.slow
def test_config2_full_context_sampled_heads():
    case = gin.prefill_case(2)
    heads = [3, 44]
    out, S, C = run_gpu(case, uniform=True)
    ref = run_oracle(case, heads)
    check(case, out, S, C, ref, heads)
    # every head: finite output, bounded by the gated norm (|y| <= sqrt(128) |w silu(z)|)
    assert torch.isfinite(out.float()).all()


@pytest.mark.slow
def test_full_context_slow_decay_stress():
    """The long-horizon stress case at full length: T = 262,144 tokens, 16 / 48 heads, zero
    initial state, a ~ N(-6, 1) so that alpha = e^g stays close to 1 (0.96 .. 0.998 per
    token) and the state carries information over thousands of chunks; two sampled heads
    against the oracle, the state at the 5e-3 bound."""
    cfg = gin.CONFIGS[2]
    T, H_k, H_v = cfg["T"], cfg["H_k"], cfg["H_v"]
    inp = gin.token_inputs(T, H_k, H_v, seed=0, a_mean=-6.0)
    inp.update(gin.weights(H_k, H_v, seed=0))
    inp["scale"] = 1.0
    case = {"inp": inp, "cu_seqlens": gin.cu_from_lengths([T]), "lengths": [T], "N": 1, "H_k": H_k, "H_v": H_v,
            "state_in": None, "conv_in": None}
    heads = [5, 40]
    out, S, C = run_gpu(case, uniform=True)
    ref = run_oracle(case, heads)
    check(case, out, S, C, ref, heads)
    assert torch.isfinite(out.float()).all() and torch.isfinite(S).all()


def test_config3_packed_equals_solo_bitwise():
    """The packed 8-sequence workload at 16 / 48 heads: the shortest and the longest
    sequence, run alone, give bitwise the same outputs, final states and conv states as
    their slices of the packed call."""
    case = gin.prefill_case(3)
    out, S, C = run_gpu(case)
    cu = case["cu_seqlens"].tolist()
    lengths = case["lengths"]
    for n in (min(range(len(lengths)), key=lambda i: lengths[i]), max(range(len(lengths)), key=lambda i: lengths[i])):
        sub = {k: (v[cu[n]:cu[n + 1]] if k in ("q", "k", "v", "z", "a", "b") else v) for k, v in case["inp"].items()}
        solo = {"inp": sub, "cu_seqlens": gin.cu_from_lengths([lengths[n]]), "lengths": [lengths[n]], "N": 1,
                "H_k": case["H_k"], "H_v": case["H_v"], "state_in": None, "conv_in": None}
        o1, S1, C1 = run_gpu(solo)
        print(f"[parity] config 3 sequence {n} ({lengths[n]} tokens) alone vs packed: "
              f"out equal {torch.equal(o1, out[cu[n]:cu[n + 1]])}, state equal {torch.equal(S1[0], S[n])}")
        assert torch.equal(o1, out[cu[n]:cu[n + 1]])
        assert torch.equal(S1[0], S[n])
        assert torch.equal(C1[0], C[n])


def test_long_decay_variant():
    """a ~ N(-6, 1): alpha close to 1, the long-horizon accumulation case."""
    case = small_case([3000], H_k=2, H_v=6, a_mean=-6.0, with_state=True)
    out, S, C = run_gpu(case)
    check(case, out, S, C, run_oracle(case))


def test_scale_and_conv_history():
    case = small_case([90, 40], with_conv=True)
    case["inp"]["scale"] = 128 ** -0.5
    out, S, C = run_gpu(case)
    check(case, out, S, C, run_oracle(case))


def test_identity_gates_keep_state_bitwise():
    case = small_case([150], H_k=1, H_v=3)
    case["inp"]["a"] = torch.full_like(case["inp"]["a"], float("-inf"))
    case["inp"]["b"] = torch.full_like(case["inp"]["b"], float("-inf"))
    out, S, C = run_gpu(case)
    assert torch.equal(S.cpu(), case["state_in"])
    check(case, out, S, C, run_oracle(case))


# ------------------------------------------------------------------ bitwise properties


def test_repeat_calls_are_bitwise_identical():
    case = small_case([300, 77])
    res = [run_gpu(case) for _ in range(2)]
    assert torch.equal(res[1][0], res[0][0])
    assert torch.equal(res[1][1], res[0][1])


def test_varlen_equals_solo_bitwise():
    lengths = [1, 64, 65, 200, 3, 0, 130]
    case = small_case(lengths, with_conv=True)
    out, S, C = run_gpu(case)
    cu = case["cu_seqlens"].tolist()
    for n, L in enumerate(lengths):
        sub = {k: (v[cu[n]:cu[n + 1]] if k in ("q", "k", "v", "z", "a", "b") else v) for k, v in case["inp"].items()}
        solo = {"inp": sub, "cu_seqlens": gin.cu_from_lengths([L]), "lengths": [L], "N": 1, "H_k": 2, "H_v": 6,
                "state_in": case["state_in"][n:n + 1], "conv_in": case["conv_in"][n:n + 1]}
        o1, S1, C1 = run_gpu(solo)
        assert torch.equal(o1, out[cu[n]:cu[n + 1]])
        assert torch.equal(S1[0], S[n])
        assert torch.equal(C1[0], C[n])


def test_pack_order_invariance_bitwise():
    lengths = [70, 5, 128]
    case = small_case(lengths)
    out, S, _ = run_gpu(case)
    perm = [2, 0, 1]
    cu = case["cu_seqlens"].tolist()
    segs = {k: [v[cu[n]:cu[n + 1]] for n in perm] for k, v in case["inp"].items() if k in ("q", "k", "v", "z", "a", "b")}
    inp2 = dict(case["inp"])
    for k, parts in segs.items():
        inp2[k] = torch.cat(parts)
    case2 = dict(case, inp=inp2, lengths=[lengths[n] for n in perm], cu_seqlens=gin.cu_from_lengths([lengths[n] for n in perm]),
                 state_in=case["state_in"][perm])
    out2, S2, _ = run_gpu(case2)
    cu2 = case2["cu_seqlens"].tolist()
    for j, n in enumerate(perm):
        assert torch.equal(out2[cu2[j]:cu2[j + 1]], out[cu[n]:cu[n + 1]])
        assert torch.equal(S2[j], S[n])


@pytest.mark.parametrize("T1", [128, 100])
def test_split_prefill_resumes(T1):
    """prefill(T1) then prefill(T2) from the returned state and conv state equals
    prefill(T1 + T2): bitwise when T1 is a multiple of 64, within tolerance otherwise."""
    T = 200
    case = small_case([T], with_conv=True)
    out, S, C = run_gpu(case)
    a = {k: (v[:T1] if k in ("q", "k", "v", "z", "a", "b") else v) for k, v in case["inp"].items()}
    b = {k: (v[T1:] if k in ("q", "k", "v", "z", "a", "b") else v) for k, v in case["inp"].items()}
    ca = dict(case, inp=a, lengths=[T1], cu_seqlens=gin.cu_from_lengths([T1]))
    oa, Sa, Ca = run_gpu(ca)
    cb = dict(case, inp=b, lengths=[T - T1], cu_seqlens=gin.cu_from_lengths([T - T1]), state_in=Sa.cpu(),
              conv_in=Ca.cpu())
    ob, Sb, Cb = run_gpu(cb)
    joined = torch.cat([oa, ob])
    assert torch.equal(Cb, C)
    if T1 % 64 == 0:
        assert torch.equal(joined, out)
        assert torch.equal(Sb, S)
    else:
        ref = run_oracle(case)
        assert out_error(joined, ref["out"]) <= OUT_TOL
        assert state_error(Sb, ref["state"]) <= STATE_TOL


def test_empty_batch_and_empty_sequences():
    case = small_case([0, 0], with_conv=True)
    out, S, C = run_gpu(case)
    assert out.numel() == 0
    assert torch.equal(S.cpu(), case["state_in"])
    ref = run_oracle(case)
    np.testing.assert_array_equal(C.float().cpu().numpy(), ref["conv"])


# ------------------------------------------------------------------ layouts, head groupings, failure detection


def test_strided_inputs_from_one_projection_buffer():
    """q, k, v, z, a, b as column slices of one [T, proj] buffer (token stride = proj width)."""
    H_k, H_v, T = 2, 6, 150
    case = small_case([T], H_k=H_k, H_v=H_v, with_conv=True)
    inp = case["inp"]
    parts = [inp["q"].reshape(T, -1), inp["k"].reshape(T, -1), inp["v"].reshape(T, -1), inp["z"].reshape(T, -1),
             inp["a"], inp["b"], torch.zeros(T, 4, dtype=torch.bfloat16)]  # pad the row to a 16-byte multiple
    proj = torch.cat(parts, dim=1).cuda()
    assert (proj.shape[1] * 2) % 16 == 0
    o = 0
    views = {}
    for name, t in zip(("q", "k", "v", "z", "a", "b"), parts):
        views[name] = proj[:, o:o + t.shape[1]]
        o += t.shape[1]
    views["q"] = views["q"].unflatten(1, (H_k, 128))
    views["k"] = views["k"].unflatten(1, (H_k, 128))
    views["v"] = views["v"].unflatten(1, (H_v, 128))
    views["z"] = views["z"].unflatten(1, (H_v, 128))
    w = {k: inp[k].cuda() for k in ("conv_w", "A_log", "norm_w")}
    s = gdn.make_inputs(views["q"], views["k"], views["v"], views["a"], views["b"], views["z"], w["conv_w"],
                        w["A_log"], w["norm_w"])
    assert s.stride_q == proj.shape[1] and s.stride_a == proj.shape[1]
    err = err_word()
    out, S, C = gdn.prefill(s, 1, T, case["state_in"].cuda(), case["conv_in"].cuda(), err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check(case, out, S, C, run_oracle(case))


@pytest.mark.parametrize("H_k,H_v", [(4, 8), (1, 8), (3, 3)])
def test_other_head_groupings(H_k, H_v):
    case = small_case([70, 129], H_k=H_k, H_v=H_v, with_conv=True)
    out, S, C = run_gpu(case)
    check(case, out, S, C, run_oracle(case))


@pytest.mark.parametrize("schedule", [gdn.SCHEDULE_TWO_LAUNCHES, gdn.SCHEDULE_FUSED])
def test_device_cu_seqlens_mismatch_is_reported_not_computed(schedule):
    """The device copy of cu_seqlens disagrees with the host copy: the setup kernel
    detects it, sets error bit 4 and every other kernel skips its work."""
    case = small_case([64, 64])
    keep, s = device_inputs(case["inp"])
    s.schedule = schedule
    cu_host = case["cu_seqlens"]
    cu_bad = torch.tensor([0, 64, 100], dtype=torch.int32, device="cuda")  # host says 128 tokens
    err = err_word()
    out = torch.full((128, case["H_v"], 128), 7.0, dtype=torch.bfloat16, device="cuda")
    gdn.prefill_varlen(s, cu_bad, cu_host, None, None, out=out, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 4
    assert torch.all(out == 7.0)  # nothing was written


@pytest.mark.parametrize("kind", ["uniform-200-2x6", "varlen-2x6", "uniform-300-4x8", "layer-4096-16x48"])
def test_fused_and_two_launch_schedules_bitwise_equal(kind):
    """The fused schedule (prep and scan overlapped in one launch) and the plain
    two-launch schedule run the same arithmetic."""
    if kind == "uniform-200-2x6":
        case, uniform = small_case([200], seed=41), True
    elif kind == "varlen-2x6":
        case, uniform = small_case([1, 64, 0, 65, 130, 3], seed=42, with_conv=True), False
    elif kind == "uniform-300-4x8":
        case, uniform = small_case([300], H_k=4, H_v=8, seed=43), True
    else:
        case, uniform = gin.prefill_case(1), True
    a = run_gpu(case, uniform=uniform, schedule=gdn.SCHEDULE_FUSED)
    b = run_gpu(case, uniform=uniform, schedule=gdn.SCHEDULE_TWO_LAUNCHES)
    for x, y in zip(a, b):
        assert torch.equal(x, y)
    if kind != "layer-4096-16x48":
        check(case, *a, run_oracle(case))
