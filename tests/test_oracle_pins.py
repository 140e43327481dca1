"""Pins of the fp64 oracle against facts that do not come from the oracle itself:
a hand-worked example, closed forms, library routines (torch conv1d, rms_norm,
softplus, a linear solve), brute force on tiny inputs, and invariants.

The recurrence pinned here is the gated delta rule named on the Agnes-3.0-Flash
pages (model card, "Architecture" table, row "Delta-rule layers"; "Agnes-3.0-Flash
Deep Dive: A 33B Hybrid-Attention Multimodal Model", section "Feed-Forward and
Positional Encoding", paragraph on the Gated Delta Rule):
    S_t = a_t S_{t-1} (I - b_t k_t k_t^T) + b_t v_t k_t^T,  o_t = S_t q_t.
"""
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from gated_delta_rule_81_b200 import inputs as gin

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(1234)


def unit_rows(x):
    return x / np.linalg.norm(x, axis=-1, keepdims=True)


# ---------------------------------------------------------------- recurrence


def test_worked_example_from_golden():
    rows = np.loadtxt(os.path.join(GOLDEN, "recurrence_worked_example.txt"))
    T = rows.shape[0]
    k = rows[:, 1:3].reshape(T, 1, 2)
    v = rows[:, 3:5].reshape(T, 1, 2)
    q = rows[:, 5:7].reshape(T, 1, 2)
    alpha, beta = rows[:, 7:8], rows[:, 8:9]
    o, S = oracle.recurrence(q, k, v, alpha, beta, [0, T])
    np.testing.assert_allclose(o[:, 0], rows[:, 9:11], rtol=0, atol=1e-14)
    # state after the last step
    np.testing.assert_allclose(S[0, 0].reshape(-1), rows[-1, 11:15], rtol=0, atol=1e-14)
    # state after every step: run prefixes
    for t in range(1, T + 1):
        _, St = oracle.recurrence(q[:t], k[:t], v[:t], alpha[:t], beta[:t], [0, t])
        np.testing.assert_allclose(St[0, 0].reshape(-1), rows[t - 1, 11:15], atol=1e-14)


def test_identity_gate_keeps_state():
    """alpha = 1, beta = 0: S_t = S_0 for all t and o_t = S_0 q_t."""
    T, D = 37, 16
    q = RNG.standard_normal((T, 1, D))
    k = unit_rows(RNG.standard_normal((T, 1, D)))
    v = RNG.standard_normal((T, 1, D))
    S0 = RNG.standard_normal((1, 1, D, D))
    o, S = oracle.recurrence(q, k, v, np.ones((T, 1)), np.zeros((T, 1)), [0, T], S0)
    np.testing.assert_array_equal(S, S0)
    np.testing.assert_allclose(o[:, 0], q[:, 0] @ S0[0, 0].T, rtol=1e-13, atol=1e-13)


def test_orthonormal_keys_retrieve_values():
    """alpha = 1, beta = 1, orthonormal keys: after writing (k_i, v_i), querying k_j
    returns v_j (S (I - k k^T) + v k^T maps k to v and leaves orthogonal keys alone)."""
    D, n = 128, 48
    Qm, _ = np.linalg.qr(RNG.standard_normal((D, D)))
    keys = Qm[:, :n].T  # n orthonormal rows
    vals = RNG.standard_normal((n, D))
    # n writes (query = own key), then n read-only queries (beta = 0) in shuffled order
    order = RNG.permutation(n)
    k = np.concatenate([keys, keys[order]])[:, None, :]
    v = np.concatenate([vals, np.zeros((n, D))])[:, None, :]
    q = np.concatenate([keys, keys[order]])[:, None, :]
    beta = np.concatenate([np.ones(n), np.zeros(n)])[:, None]
    o, _ = oracle.recurrence(q, k, v, np.ones((2 * n, 1)), beta, [0, 2 * n])
    np.testing.assert_allclose(o[:n, 0], vals, atol=1e-13)
    np.testing.assert_allclose(o[n:, 0], vals[order], atol=1e-13)


def test_single_step_projector_form():
    """T = 1: S_1 = alpha S_0 (I - beta k k^T) + beta v k^T (matrix form), o = S_1 q."""
    D = 32
    S0 = RNG.standard_normal((1, 1, D, D))
    q, k, v = (RNG.standard_normal((1, 1, D)) for _ in range(3))
    k = unit_rows(k)
    alpha, beta = np.array([[0.37]]), np.array([[0.81]])
    o, S = oracle.recurrence(q, k, v, alpha, beta, [0, 1], S0)
    kk = np.outer(k[0, 0], k[0, 0])
    S1 = 0.37 * S0[0, 0] @ (np.eye(D) - 0.81 * kk) + 0.81 * np.outer(v[0, 0], k[0, 0])
    np.testing.assert_allclose(S[0, 0], S1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o[0, 0], S1 @ q[0, 0], rtol=1e-13, atol=1e-13)


def test_brute_force_products():
    """T <= 8: S_T = S0 prod_t alpha_t (I - beta_t k_t k_t^T)
    + sum_t beta_t v_t k_t^T prod_{tau > t} alpha_tau (I - beta_tau k_tau k_tau^T)."""
    D = 24
    for T in range(1, 9):
        q = RNG.standard_normal((T, 1, D))
        k = unit_rows(RNG.standard_normal((T, 1, D)))
        v = RNG.standard_normal((T, 1, D))
        alpha = RNG.uniform(0.2, 1.0, (T, 1))
        beta = RNG.uniform(0.0, 1.0, (T, 1))
        S0 = RNG.standard_normal((1, 1, D, D))
        o, S = oracle.recurrence(q, k, v, alpha, beta, [0, T], S0)
        P = [alpha[t, 0] * (np.eye(D) - beta[t, 0] * np.outer(k[t, 0], k[t, 0])) for t in range(T)]
        for tt in range(1, T + 1):  # state after tt steps, as explicit products
            St = S0[0, 0].copy()
            for t in range(tt):
                St = St @ P[t]
            for t in range(tt):
                term = beta[t, 0] * np.outer(v[t, 0], k[t, 0])
                for tau in range(t + 1, tt):
                    term = term @ P[tau]
                St = St + term
            np.testing.assert_allclose(o[tt - 1, 0], St @ q[tt - 1, 0], rtol=1e-11, atol=1e-11)
        np.testing.assert_allclose(S[0, 0], St, rtol=1e-11, atol=1e-11)


def test_memoryless_when_alpha_zero():
    """alpha -> 0: S_t = beta_t v_t k_t^T, o_t = beta_t (k_t . q_t) v_t."""
    T, D = 20, 16
    q = RNG.standard_normal((T, 1, D))
    k = unit_rows(RNG.standard_normal((T, 1, D)))
    v = RNG.standard_normal((T, 1, D))
    beta = RNG.uniform(0, 1, (T, 1))
    o, S = oracle.recurrence(q, k, v, np.zeros((T, 1)), beta, [0, T], RNG.standard_normal((1, 1, D, D)))
    want = beta * np.sum(k[:, 0] * q[:, 0], axis=1, keepdims=True) * v[:, 0]
    np.testing.assert_allclose(o[:, 0], want, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(S[0, 0], beta[-1, 0] * np.outer(v[-1, 0], k[-1, 0]), atol=1e-14)


@pytest.mark.parametrize("chunk", [1, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 64, 65, 200])
def test_chunked_form_agrees(chunk, T):
    """The UT-transform chunked form (library solve + matmuls) equals the sequential
    recurrence to 1e-12, including partial chunks; chunk = 1 is the recurrence."""
    D = 128
    q = RNG.standard_normal((T, 1, D))
    k = unit_rows(np.abs(RNG.standard_normal((T, 1, D))) + 0.3)  # correlated keys, as after SiLU
    v = RNG.standard_normal((T, 1, D))
    g = -RNG.uniform(0.0, 1.5, (T, 1))
    beta = RNG.uniform(0, 1, (T, 1))
    S0 = 0.1 * RNG.standard_normal((1, 1, D, D))
    o_seq, S_seq = oracle.recurrence(q, k, v, np.exp(g), beta, [0, T], S0)
    o_ch, S_ch = oracle.chunked_recurrence(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0], chunk)
    scale_o = max(1.0, np.sqrt(np.mean(o_seq**2)))
    scale_s = max(1.0, np.sqrt(np.mean(S_seq**2)))
    assert np.max(np.abs(o_ch - o_seq[:, 0])) <= 1e-12 * scale_o
    assert np.max(np.abs(S_ch - S_seq[0, 0])) <= 1e-12 * scale_s


@pytest.mark.parametrize("chunk", [1, 16, 64])
@pytest.mark.parametrize("T", [1, 63, 65, 200])
def test_chunked_transfer_form_agrees(chunk, T):
    """The chunk step with the state dependence gathered into S_0 M + N (transfer matrix
    and drive per chunk) equals the sequential recurrence to 1e-12, slow and fast decay."""
    D = 128
    for g_hi in (0.05, 1.5):
        q = RNG.standard_normal((T, 1, D))
        k = unit_rows(np.abs(RNG.standard_normal((T, 1, D))) + 0.3)
        v = RNG.standard_normal((T, 1, D))
        g = -RNG.uniform(0.0, g_hi, (T, 1))
        beta = RNG.uniform(0, 1, (T, 1))
        S0 = 0.1 * RNG.standard_normal((1, 1, D, D))
        o_seq, S_seq = oracle.recurrence(q, k, v, np.exp(g), beta, [0, T], S0)
        o_tr, S_tr = oracle.chunked_transfer_recurrence(q[:, 0], k[:, 0], v[:, 0], g[:, 0], beta[:, 0], S0[0, 0],
                                                        chunk)
        scale_o = max(1.0, np.sqrt(np.mean(o_seq**2)))
        scale_s = max(1.0, np.sqrt(np.mean(S_seq**2)))
        assert np.max(np.abs(o_tr - o_seq[:, 0])) <= 1e-12 * scale_o
        assert np.max(np.abs(S_tr - S_seq[0, 0])) <= 1e-12 * scale_s


def test_value_rows_are_independent():
    """Changing value channel r of head h changes only output channel r of head h
    and state row r (the state is d_v x d_k and o = S q)."""
    T, D = 30, 16
    q = RNG.standard_normal((T, 1, D))
    k = unit_rows(RNG.standard_normal((T, 1, D)))
    v = RNG.standard_normal((T, 2, D))
    alpha, beta = RNG.uniform(0.5, 1, (T, 2)), RNG.uniform(0, 1, (T, 2))
    o1, S1 = oracle.recurrence(q, k, v, alpha, beta, [0, T])
    v2 = v.copy()
    v2[:, 1, 5] += 1.0
    o2, S2 = oracle.recurrence(q, k, v2, alpha, beta, [0, T])
    diff_o = np.abs(o2 - o1).max(axis=0)
    assert diff_o[1, 5] > 0
    diff_o[1, 5] = 0
    assert diff_o.max() == 0
    diff_s = np.abs(S2 - S1)[0].max(axis=2)
    assert diff_s[1, 5] > 0
    diff_s[1, 5] = 0
    assert diff_s.max() == 0


# ---------------------------------------------------------------- front end / norm / gates


def test_conv_identity_taps():
    T, C = 50, 7
    x = RNG.standard_normal((T, C))
    w = np.zeros((C, 4))
    w[:, 3] = 1.0
    np.testing.assert_array_equal(oracle.conv(x, w, [0, T], silu=False), x)


def test_conv_matches_torch_conv1d():
    """Causal depthwise conv against torch.conv1d (fp64) on [history; x]."""
    C = 9
    cu = [0, 13, 14, 40]
    x = RNG.standard_normal((cu[-1], C))
    w = RNG.standard_normal((C, 4))
    hist = RNG.standard_normal((3, 3, C))
    for use_hist in (False, True):
        y = oracle.conv(x, w, cu, hist if use_hist else None, silu=True)
        for n in range(3):
            seg = x[cu[n]:cu[n + 1]]
            pre = hist[n] if use_hist else np.zeros((3, C))
            full = torch.from_numpy(np.concatenate([pre, seg]).T[None])  # [1, C, 3 + L]
            ref = F.conv1d(full, torch.from_numpy(w)[:, None, :], groups=C)[0].T  # [L, C]
            ref = F.silu(ref).numpy()
            np.testing.assert_allclose(y[cu[n]:cu[n + 1]], ref, rtol=1e-13, atol=1e-13)


def test_l2norm_unit_and_library():
    x = RNG.standard_normal((40, 128)) * 3
    y = oracle.l2norm(x)
    np.testing.assert_allclose(np.linalg.norm(y, axis=1), 1.0, atol=1e-9)
    ref = F.normalize(torch.from_numpy(x), dim=-1).numpy()
    np.testing.assert_allclose(y, ref, rtol=1e-9, atol=1e-12)


def test_gated_rmsnorm_matches_library():
    o = RNG.standard_normal((25, 128))
    z = RNG.standard_normal((25, 128)) * 2
    w = RNG.uniform(0.5, 1.5, 128)
    y = oracle.gated_rmsnorm(o, z, w)
    ot, zt, wt = (torch.from_numpy(t) for t in (o, z, w))
    ref = F.rms_norm(ot, (128,), weight=wt, eps=1e-6) * F.silu(zt)
    np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-13)


def test_gates_match_library_and_limits():
    H = 3
    A_log = np.log([1.0, 4.0, 16.0])
    a = RNG.standard_normal((10, H)) * 3
    b = RNG.standard_normal((10, H)) * 3
    g, alpha, beta = oracle.gates(A_log, a, b)
    ref_g = -np.exp(A_log)[None] * F.softplus(torch.from_numpy(a)).numpy()
    np.testing.assert_allclose(g, ref_g, rtol=1e-13)
    np.testing.assert_allclose(alpha, np.exp(ref_g), rtol=1e-13)
    np.testing.assert_allclose(beta, torch.sigmoid(torch.from_numpy(b)).numpy(), rtol=1e-13)
    lim = np.array([[-np.inf, -np.inf, np.inf]])
    _, al, be = oracle.gates(np.zeros(3), lim, lim)
    assert al[0, 0] == 1.0 and al[0, 1] == 1.0 and al[0, 2] == 0.0
    assert be[0, 0] == 0.0 and be[0, 2] == 1.0


def test_softplus_large_argument_branch():
    """a > 30 takes softplus(a) = a + log1p(e^-a): compare with the library's log(1 + e^a)
    (torch.logaddexp(0, a), exact for any a) at a in {31, 50, 100, 700}; g, alpha follow."""
    A_log = np.log([1.0, 2.0, 16.0, 3.0])
    a = np.array([[31.0, 50.0, 100.0, 700.0]])
    b = np.zeros_like(a)
    g, alpha, _ = oracle.gates(A_log, a, b)
    sp = torch.logaddexp(torch.zeros(1, 4, dtype=torch.float64), torch.from_numpy(a)).numpy()
    np.testing.assert_allclose(g, -np.exp(A_log)[None] * sp, rtol=1e-15)
    # torch's softplus, told not to switch to the identity, computes log1p(e^a) directly
    ref = F.softplus(torch.from_numpy(a[:, :3]), threshold=1e9).numpy()
    np.testing.assert_allclose(-g[:, :3] / np.exp(A_log)[None, :3], ref, rtol=1e-15)
    np.testing.assert_allclose(alpha, np.exp(-np.exp(A_log)[None] * sp), rtol=1e-13)
    # the branch boundary: 30 and 30 + 1e-9 agree with the library on both sides
    g2, _, _ = oracle.gates(np.zeros(2), np.array([[30.0, 30.0 + 1e-9]]), np.zeros((1, 2)))
    sp2 = torch.logaddexp(torch.zeros(1, 2, dtype=torch.float64), torch.tensor([[30.0, 30.0 + 1e-9]],
                                                                                 dtype=torch.float64)).numpy()
    np.testing.assert_allclose(g2, -sp2, rtol=1e-15)


# ---------------------------------------------------------------- whole mixer


def _torch_composition(case, state_in=None, conv_in=None):
    """The mixer rebuilt from library pieces (torch conv1d, normalize, softplus,
    sigmoid, rms_norm) around the independent chunked form."""
    inp, cu = case["inp"], case["cu_seqlens"].tolist()
    H_k, H_v = case["H_k"], case["H_v"]
    D = gin.D
    G = H_v // H_k
    f64 = lambda t: t.to(torch.float64)  # noqa: E731
    x = torch.cat([f64(inp["q"]).reshape(-1, H_k * D), f64(inp["k"]).reshape(-1, H_k * D),
                   f64(inp["v"]).reshape(-1, H_v * D)], dim=1)
    C = x.shape[1]
    w = f64(inp["conv_w"])
    out = np.zeros((cu[-1], H_v, D))
    S_fin = np.zeros((len(cu) - 1, H_v, D, D))
    for n in range(len(cu) - 1):
        seg = x[cu[n]:cu[n + 1]]
        pre = f64(conv_in[n]) if conv_in is not None else torch.zeros(3, C, dtype=torch.float64)
        y = F.conv1d(torch.cat([pre, seg]).T[None], w[:, None, :], groups=C)[0].T
        y = F.silu(y)
        L = seg.shape[0]
        qh = y[:, :H_k * D].reshape(L, H_k, D)
        kh = y[:, H_k * D:2 * H_k * D].reshape(L, H_k, D)
        vh = y[:, 2 * H_k * D:].reshape(L, H_v, D)
        qh = qh / torch.sqrt((qh * qh).sum(-1, keepdim=True) + 1e-6) * inp["scale"]
        kh = kh / torch.sqrt((kh * kh).sum(-1, keepdim=True) + 1e-6)
        a = f64(inp["a"][cu[n]:cu[n + 1]])
        b = f64(inp["b"][cu[n]:cu[n + 1]])
        g = -torch.exp(f64(inp["A_log"]))[None] * F.softplus(a)
        beta = torch.sigmoid(b)
        z = f64(inp["z"][cu[n]:cu[n + 1]])
        for h in range(H_v):
            S0 = None if state_in is None else state_in[n, h].double().numpy()
            o, S = oracle.chunked_recurrence(qh[:, h // G].numpy(), kh[:, h // G].numpy(),
                                             vh[:, h].numpy(), g[:, h].numpy(), beta[:, h].numpy(),
                                             S0, chunk=64)
            yv = F.rms_norm(torch.from_numpy(o), (D,), weight=f64(inp["norm_w"]), eps=1e-6) * F.silu(z[:, h])
            out[cu[n]:cu[n + 1], h] = yv.numpy()
            S_fin[n, h] = S
    return out, S_fin


def _small_case(lengths, H_k=2, H_v=6, seed=3):
    case = gin.prefill_case(3, seed=seed, lengths=lengths)
    # re-draw at the small head counts with the same recipe
    T = sum(lengths)
    inp = gin.token_inputs(T, H_k, H_v, seed)
    inp.update(gin.weights(H_k, H_v, seed))
    inp["scale"] = 1.0
    case.update(inp=inp, H_k=H_k, H_v=H_v)
    return case


def test_mixer_matches_library_composition():
    case = _small_case([70, 1, 130])
    N, H_v = 3, case["H_v"]
    st = gin.recurrent_state(N, H_v, seed=5)
    cv = gin.conv_state(N, case["H_k"], H_v, seed=5)
    res = oracle.mixer(case["inp"], case["cu_seqlens"], state_in=st, conv_in=cv)
    ref_out, ref_S = _torch_composition(case, st, cv)
    np.testing.assert_allclose(res["out"], ref_out, rtol=1e-10, atol=1e-11)
    np.testing.assert_allclose(res["state"], ref_S, rtol=1e-10, atol=1e-12)


def test_mixer_scale_multiplies_the_query_only():
    """scale multiplies the normalised query: o_t = S_t (s q_t) is linear in q_t and the state
    S_t does not involve q at all, so the pre-norm output at scale s is s times the output at
    scale 1 and the final state is the same.  (Applying s before the L2-norm would cancel it,
    and applying it to k would change the state: both fail here.)"""
    case = _small_case([70, 1, 130])
    st = gin.recurrent_state(3, case["H_v"], seed=9)
    inp1 = dict(case["inp"], scale=1.0)
    ref = oracle.mixer(inp1, case["cu_seqlens"], state_in=st, want_pre_norm=True)
    for s_ in (0.5, 128 ** -0.5, 3.0):
        res = oracle.mixer(dict(case["inp"], scale=s_), case["cu_seqlens"], state_in=st, want_pre_norm=True)
        np.testing.assert_allclose(res["pre_norm"], s_ * ref["pre_norm"], rtol=1e-12, atol=1e-14)
        np.testing.assert_array_equal(res["state"], ref["state"])
        assert np.max(np.abs(res["pre_norm"] - ref["pre_norm"])) > 1e-3 * np.max(np.abs(ref["pre_norm"]))


def test_mixer_conv_out_is_last_three_raw_tokens():
    case = _small_case([5, 1, 2])
    H_k, H_v = case["H_k"], case["H_v"]
    cv = gin.conv_state(3, H_k, H_v, seed=9)
    res = oracle.mixer(case["inp"], case["cu_seqlens"], conv_in=cv)
    inp = case["inp"]
    x = torch.cat([inp["q"].reshape(8, -1), inp["k"].reshape(8, -1), inp["v"].reshape(8, -1)], 1).double()
    hist = cv.double()
    np.testing.assert_array_equal(res["conv"][0], x[2:5].numpy())
    np.testing.assert_array_equal(res["conv"][1], torch.cat([hist[1, 1:], x[5:6]]).numpy())
    np.testing.assert_array_equal(res["conv"][2], torch.cat([hist[2, 2:], x[6:8]]).numpy())


def test_mixer_causal():
    case = _small_case([90])
    base = oracle.mixer(case["inp"], case["cu_seqlens"])["out"]
    inp = dict(case["inp"])
    for key in ("q", "k", "v", "z", "a", "b"):
        inp[key] = inp[key].clone()
        inp[key][60] = inp[key][60] + 1.0
    pert = oracle.mixer(inp, case["cu_seqlens"])["out"]
    np.testing.assert_array_equal(pert[:60], base[:60])
    assert np.abs(pert[60:] - base[60:]).max() > 0


def test_mixer_varlen_equals_solo_runs():
    case = _small_case([33, 64, 2])
    st = gin.recurrent_state(3, case["H_v"], seed=2)
    packed = oracle.mixer(case["inp"], case["cu_seqlens"], state_in=st)
    cu = case["cu_seqlens"].tolist()
    for n in range(3):
        sl = slice(cu[n], cu[n + 1])
        sub = {k: (v[sl] if k in ("q", "k", "v", "z", "a", "b") else v) for k, v in case["inp"].items()}
        solo = oracle.mixer(sub, [0, cu[n + 1] - cu[n]], state_in=st[n:n + 1])
        np.testing.assert_array_equal(packed["out"][sl], solo["out"])
        np.testing.assert_array_equal(packed["state"][n], solo["state"][0])


def test_mixer_identity_gate_through_full_path():
    """a = -inf, b = -inf (bf16 can hold them): alpha = 1, beta = 0 on every token, so
    the state is returned unchanged and the pre-norm output is S_0 q_hat."""
    case = _small_case([40], H_k=1, H_v=3)
    inp = dict(case["inp"])
    inp["a"] = torch.full_like(inp["a"], float("-inf"))
    inp["b"] = torch.full_like(inp["b"], float("-inf"))
    st = gin.recurrent_state(1, 3, seed=4)
    res = oracle.mixer(inp, case["cu_seqlens"], state_in=st, want_pre_norm=True)
    np.testing.assert_array_equal(res["state"], st.double().numpy())
    # q_hat from library pieces
    D = gin.D
    qraw = inp["q"].double().reshape(40, D)
    w = inp["conv_w"].double()[:D]
    y = F.silu(F.conv1d(torch.cat([torch.zeros(3, D, dtype=torch.float64), qraw]).T[None], w[:, None, :],
                        groups=D)[0].T)
    qh = (y / torch.sqrt((y * y).sum(-1, keepdim=True) + 1e-6)).numpy()
    for h in range(3):
        np.testing.assert_allclose(res["pre_norm"][:, h], qh @ st[0, h].double().numpy().T,
                                   rtol=1e-12, atol=1e-12)


# ------------------------------------------------------------------ projections around the mixer


def test_gemm_small_exact_and_orientation():
    """C = A B^T: a hand-computed 2x2 product pins the orientation (B holds one output channel per row)."""
    a = torch.tensor([[1.0, 2.0, 3.0], [4.0, 5.0, 6.0]], dtype=torch.bfloat16)
    b = torch.tensor([[1.0, 0.0, 1.0], [0.0, 1.0, 0.0]], dtype=torch.bfloat16)
    np.testing.assert_array_equal(oracle.gemm(a, b), np.array([[4.0, 2.0], [10.0, 5.0]]))


def test_round_bf16_ties_and_library():
    """Round to nearest bf16 with ties to even: values with a known answer, then agreement
    with torch's own float32 -> bfloat16 conversion on random fp32 values."""
    x = np.array([1 + 2.0**-8, 1 + 3 * 2.0**-9, 1 + 2.0**-7 + 2.0**-8, -2.5, 0.0, 3 * 2.0**-130])
    want = np.array([1.0, 1 + 2.0**-7, 1 + 2.0**-6, -2.5, 0.0, 3 * 2.0**-130])
    np.testing.assert_array_equal(oracle.round_bf16(x), want)
    r = torch.randn(4096, generator=torch.Generator().manual_seed(3)) * 7.0
    np.testing.assert_array_equal(oracle.round_bf16(r.double().numpy()), r.to(torch.bfloat16).double().numpy())


def test_layer_routes_projection_columns():
    """With permutation weights the layer is the mixer on permuted hidden channels: this pins
    the q|k|v|z|a|b column order of the input projection and the output projection's
    orientation, independently of the layer function's own bookkeeping."""
    H_k, H_v, D, T = 1, 2, 128, 9
    lay = oracle.in_proj_layout(H_k, H_v, D)
    n_in = lay["total"][1]
    hidden = n_in
    g = torch.Generator().manual_seed(5)
    x = torch.randn(T, hidden, generator=g).to(torch.bfloat16)
    perm = torch.randperm(n_in, generator=g)
    w_in = torch.zeros(n_in, hidden, dtype=torch.bfloat16)
    w_in[torch.arange(n_in), perm] = 1.0  # proj[:, j] = x[:, perm[j]]
    w_out = torch.zeros(hidden, H_v * D, dtype=torch.bfloat16)
    rows = torch.arange(H_v * D)
    w_out[rows, rows] = 1.0  # y[:, c] = out[:, c] for c < H_v*D, zero above
    w = gin.weights(H_k, H_v, seed=5)
    res = oracle.layer(x, w_in, w_out, w["conv_w"], w["A_log"], w["norm_w"], [0, T], H_k, H_v)
    xp = x[:, perm]
    inp = {n: xp[:, lay[n][0]:lay[n][1]].reshape(T, -1, D) for n in ("q", "k", "v", "z")}
    inp.update({n: xp[:, lay[n][0]:lay[n][1]] for n in ("a", "b")})
    inp.update(w)
    inp["scale"] = 1.0
    ref = oracle.mixer(inp, [0, T])
    np.testing.assert_array_equal(res["out"], ref["out"])
    o16 = torch.from_numpy(ref["out"]).to(torch.bfloat16).double().numpy().reshape(T, H_v * D)
    np.testing.assert_array_equal(res["y"][:, :H_v * D], o16)
    assert np.all(res["y"][:, H_v * D:] == 0)


# ------------------------------------------------------------------ global-attention layer


def test_rope_closed_forms():
    """Position 0 is the identity; a basis vector e_i (i < 32) at position p turns into
    cos(p theta_i) e_i + sin(p theta_i) e_{i+32} with theta_0 = 1; dims 64.. never move."""
    A = oracle.attn
    x = torch.randn(5, 2, 256, generator=torch.Generator().manual_seed(1), dtype=torch.float64)
    np.testing.assert_allclose(A.rope(x, np.zeros(5)), x.numpy(), atol=0, rtol=0)
    e = np.zeros((1, 1, 256))
    e[0, 0, 0] = 1.0
    for p in (1.0, 7.0, 1000.0):
        r = A.rope(e, [p])
        assert abs(r[0, 0, 0] - np.cos(p)) < 1e-12 and abs(r[0, 0, 32] - np.sin(p)) < 1e-12
        assert np.count_nonzero(np.abs(r) > 1e-15) == 2
    e2 = np.zeros((1, 1, 256))
    e2[0, 0, 5] = 1.0
    th = 1e7 ** (-5 / 32)
    r = A.rope(e2, [3.0])
    assert abs(r[0, 0, 5] - np.cos(3 * th)) < 1e-12 and abs(r[0, 0, 37] - np.sin(3 * th)) < 1e-12
    r = A.rope(x, np.arange(5) * 11.0)
    np.testing.assert_array_equal(r[..., 64:], x.numpy()[..., 64:])


def test_rope_norm_and_relative_position():
    """Rotations keep every pair's norm, and q_m . k_n depends on m - n only."""
    A = oracle.attn
    g = torch.Generator().manual_seed(2)
    q = torch.randn(1, 1, 256, generator=g, dtype=torch.float64).numpy()
    k = torch.randn(1, 1, 256, generator=g, dtype=torch.float64).numpy()
    r = A.rope(q, [123.0])
    np.testing.assert_allclose(r[..., :32] ** 2 + r[..., 32:64] ** 2, q[..., :32] ** 2 + q[..., 32:64] ** 2,
                               rtol=1e-12)
    d1 = (A.rope(q, [10.0]) * A.rope(k, [3.0])).sum()
    d2 = (A.rope(q, [507.0]) * A.rope(k, [500.0])).sum()
    assert abs(d1 - d2) < 1e-9 * abs(d1)


def test_rms_norm_matches_library():
    A = oracle.attn
    x = torch.randn(7, 3, 256, generator=torch.Generator().manual_seed(3), dtype=torch.float64)
    w = torch.rand(256, generator=torch.Generator().manual_seed(4), dtype=torch.float64) + 0.5
    ref = F.rms_norm(x, (256,), w, eps=1e-6)
    np.testing.assert_allclose(A.rms_norm(x, w), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_attention_matches_library_gqa_and_varlen():
    """Causal GQA attention equals torch's scaled_dot_product_attention with the KV heads
    repeated for their 6 query heads, per sequence; a packed call equals solo calls."""
    A = oracle.attn
    g = torch.Generator().manual_seed(5)
    lens = [9, 1, 14]
    T = sum(lens)
    q = torch.randn(T, 24, 32, generator=g, dtype=torch.float64)
    k = torch.randn(T, 4, 32, generator=g, dtype=torch.float64)
    v = torch.randn(T, 4, 32, generator=g, dtype=torch.float64)
    cu = [0, 9, 10, 24]
    out = A.attention(q, k, v, cu)
    for n in range(3):
        s0, s1 = cu[n], cu[n + 1]
        qq = q[s0:s1].transpose(0, 1)[None]
        kk = k[s0:s1].repeat_interleave(6, dim=1).transpose(0, 1)[None]
        vv = v[s0:s1].repeat_interleave(6, dim=1).transpose(0, 1)[None]
        ref = F.scaled_dot_product_attention(qq, kk, vv, is_causal=True)[0].transpose(0, 1)
        np.testing.assert_allclose(out[s0:s1], ref.numpy(), rtol=1e-10, atol=1e-12)
        np.testing.assert_allclose(A.attention(q[s0:s1], k[s0:s1], v[s0:s1], [0, s1 - s0]), out[s0:s1],
                                   rtol=0, atol=0)


def test_attention_closed_forms():
    """One token attends only to itself (output = v); with all keys equal the weights are
    uniform, so each output is the mean of the values up to and including its position."""
    A = oracle.attn
    g = torch.Generator().manual_seed(6)
    v = torch.randn(6, 4, 16, generator=g, dtype=torch.float64)
    q = torch.randn(6, 24, 16, generator=g, dtype=torch.float64)
    k1 = torch.randn(1, 4, 16, generator=g, dtype=torch.float64)
    np.testing.assert_allclose(A.attention(q[:1], k1, v[:1], [0, 1])[0, 7], v[0, 1].numpy(), rtol=1e-14)
    kc = k1.expand(6, 4, 16)
    out = A.attention(q, kc, v, [0, 6])
    prefix = np.cumsum(v.numpy(), axis=0) / np.arange(1, 7)[:, None, None]
    for h in range(24):
        np.testing.assert_allclose(out[:, h], prefix[:, h // 6], rtol=1e-12)


def test_attn_mixer_gate_limits():
    """A large positive gate passes the attention output, a zero gate halves it."""
    A = oracle.attn
    g = torch.Generator().manual_seed(7)
    T = 5
    q = torch.randn(T, 24, 256, generator=g).to(torch.bfloat16)
    k = torch.randn(T, 4, 256, generator=g).to(torch.bfloat16)
    v = torch.randn(T, 4, 256, generator=g).to(torch.bfloat16)
    w = torch.ones(256, dtype=torch.bfloat16)
    open_g = torch.full((T, 24, 256), 40.0).to(torch.bfloat16)
    half_g = torch.zeros(T, 24, 256, dtype=torch.bfloat16)
    a = A.attn_mixer(q, open_g, k, v, w, w, [0, T])
    b = A.attn_mixer(q, half_g, k, v, w, w, [0, T])
    o = A.attention(a["q_hat"], a["k_hat"], v, [0, T])
    np.testing.assert_allclose(a["out"], o, rtol=1e-15)
    np.testing.assert_allclose(b["out"], o / 2, rtol=1e-15)


def test_attn_layer_closed_form_routing():
    """The attention layer end to end on a case with a closed-form answer.  Hidden states are
    one-hot (x_t = e_t), so token t's projection is column t of W_in, chosen here: token 1's
    query equals its own key r (a +-1 vector: both RMS-norms leave it as it is, and the two
    rotations at the same position keep q.k = 256, a score of +16), token 0's key is -r (a score
    near -16), so token 1 attends to itself alone up to e^-32; token 0 sees only itself.  The
    values differ per KV head, so query head h must read KV head h // 6: out_t = v_t[h // 6] *
    sigmoid(g_t[h]) and y_t = bf16(out_t) W_out^T (both products exact in fp64)."""
    A = oracle.attn
    Hq, Hkv, D, hidden = 24, 4, 256, 8
    g = torch.Generator().manual_seed(11)
    lay = A.attn_in_proj_layout()
    r = (torch.randint(0, 2, (D,), generator=g) * 2 - 1).double()
    cols = torch.zeros(lay["total"][1], hidden, dtype=torch.float64)
    v = (torch.randn(2, Hkv, D, generator=g) * 0.5).to(torch.bfloat16).double()
    gate = torch.randn(2, Hq, D, generator=g).to(torch.bfloat16).double()
    for t in range(2):
        col = cols[:, t]
        col[lay["q"][0]:lay["q"][1]] = r.repeat(Hq)
        col[lay["g"][0]:lay["g"][1]] = gate[t].reshape(-1)
        col[lay["k"][0]:lay["k"][1]] = (r if t == 1 else -r).repeat(Hkv)
        col[lay["v"][0]:lay["v"][1]] = v[t].reshape(-1)
    w_in = cols.to(torch.bfloat16)  # every entry is exactly representable
    assert torch.equal(w_in.double(), cols)
    w_out = torch.randn(hidden, Hq * D, generator=g).to(torch.bfloat16)
    x = torch.eye(2, hidden).to(torch.bfloat16)
    ones = torch.ones(D, dtype=torch.bfloat16)
    ref = A.attn_layer(x, w_in, w_out, ones, ones, [0, 2])
    kv_of = torch.arange(Hq) // (Hq // Hkv)
    out = np.stack([(v[t][kv_of] * torch.sigmoid(gate[t])).numpy() for t in range(2)])  # [2, 24, 256]
    np.testing.assert_allclose(ref["out"].reshape(2, Hq, D), out, rtol=1e-12, atol=1e-13)
    y = oracle.round_bf16(out).reshape(2, -1) @ w_out.double().numpy().T
    np.testing.assert_allclose(ref["y"], y, rtol=1e-12, atol=1e-12)
