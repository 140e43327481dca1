"""The global-attention layer (through the C ABI) against the fp64 oracle.

gdn_attention_prefill -- the tcgen05 flash attention on given bf16 operands -- is held to
an element-wise bound from its arithmetic: the probabilities enter the tensor cores as
bf16 (relative error <= 2^-8 each, the unit roundoff of an 8-bit significand), so
|o - o_ref| <= 2^-8 sum_j p_j |v_j| / l (the
oracle's attention over |v|), times sigmoid(g), plus the bf16 rounding of the output.

gdn_attn_layer_prefill (in_proj GEMM, q/k norm + rotary, attention, out_proj GEMM) uses
an input projection that is exact in bf16 (two power-of-two weights per output channel,
inputs on a 1/8 grid), so both sides start from the same q, g, k, v.  q_hat and the K
cache must be within one bf16 ulp of the oracle's normalised, rotated values (2^-7 |x|:
the kernel stores them in bf16, and its fp32 rotation may land on the neighbouring value),
the V cache equal to the projected values.  The oracle keeps q_hat in fp64 (only the K
cache, an output, is rounded), so the kernel's scores differ from the oracle's by
d_ij = (q'_i . k'_j - q_i . k_j) / 16 (q', k' the kernel's bf16 operands); with
E_i = max_j |d_ij| every softmax weight moves by a factor within [e^{-2 E_i}, e^{2 E_i}],
so |o' - o| <= (e^{2 E_i} - 1) sum_j p_ij |v_j| for that row, and the kernel's own bf16
probabilities add 2^-8 e^{2 E_i} of the same sum.  E is measured from the operands the
kernel stored, which are themselves checked against the oracle's to one ulp.  The
attention output is held to that bound, and the layer output to it carried through
|W_out| plus the bf16 rounding of the stored attention output and of y.
"""
import numpy as np
import pytest
import torch

import oracle
from gated_delta_rule_81_b200 import gdn
from gpu_helpers import err_word, out_error

pytestmark = pytest.mark.gpu


def exact_attn_case(hidden, B, T, seed, extra=0):
    """extra: further tokens per sequence (for decode), generated after the prompt's."""
    g = torch.Generator().manual_seed(seed)
    n_in = gdn.ATTN_N_IN
    x = (torch.randint(-16, 17, (B * T, hidden), generator=g).float() / 8).to(torch.bfloat16)
    x_more = (torch.randint(-16, 17, (max(extra, 1), B, hidden), generator=g).float() / 8).to(torch.bfloat16)
    w_in = torch.zeros(n_in, hidden)
    cols = torch.stack([torch.randperm(hidden, generator=g)[:2] for _ in range(n_in)])
    vals = torch.tensor([1.0, -1.0, 0.5, -0.5, 0.25, -0.25])[torch.randint(0, 6, (n_in, 2), generator=g)]
    w_in.scatter_(1, cols, vals)
    w_in = w_in.to(torch.bfloat16)
    w_out = (torch.randn(hidden, 24 * 256, generator=g) * (24 * 256) ** -0.5).to(torch.bfloat16)
    qn = (1.0 + 0.1 * torch.randn(256, generator=g)).to(torch.bfloat16)
    kn = (1.0 + 0.1 * torch.randn(256, generator=g)).to(torch.bfloat16)
    return dict(x=x, w_in=w_in, w_out=w_out, qn=qn, kn=kn, B=B, T=T, x_more=x_more[:extra])


def score_shift(q_gpu, k_gpu, q_ref, k_ref, cu, rows=None):
    """Per (query row, head): e^{2 E} - 1 and e^{2 E}, with E the largest change of a causal
    score q_i . k_j / 16 between the kernel's operands (q_gpu [T, 24, 256], k_gpu [T, 4, 256])
    and the oracle's (q_ref fp64, k_ref); rows: the query rows wanted (default all)."""
    q_gpu, k_gpu, q_ref, k_ref = (np.asarray(x, dtype=np.float64) for x in (q_gpu, k_gpu, q_ref, k_ref))
    T, Hq = q_gpu.shape[0], q_gpu.shape[1]
    E = np.zeros((T, Hq, 1))
    for n in range(len(cu) - 1):
        s0, s1 = cu[n], cu[n + 1]
        want = [i for i in range(s0, s1) if rows is None or i in rows]
        if not want:
            continue
        for h in range(Hq):
            kv = h // (Hq // k_gpu.shape[1])
            qi = np.array(want)
            d = (q_gpu[qi, h] @ k_gpu[s0:s1, kv].T - q_ref[qi, h] @ k_ref[s0:s1, kv].T) / 16.0
            causal = (np.arange(s0, s1)[None, :] <= qi[:, None])
            E[qi, h, 0] = np.max(np.where(causal, np.abs(d), 0.0), axis=1)
    return np.expm1(2 * E), np.exp(2 * E)


def run_attn(c):
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out", "qn", "kn")}
    L = gdn.make_attn_layer(d["w_in"], d["w_out"], d["qn"], d["kn"])
    err = err_word()
    B, T = c["B"], c["T"]
    ws = torch.empty(int(gdn.load().gdn_attn_layer_workspace_size(B, T)), dtype=torch.uint8, device="cuda")
    y, kc, vc = gdn.attn_layer_prefill(L, B, T, d["x"], err=err, workspace=ws)
    kc, vc = kc.reshape(B * T, 4, 256), vc.reshape(B * T, 4, 256)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, int(err.item())
    # the workspace holds [projection | q_hat | attention output], each 1 KiB aligned
    T_tot = B * T
    up = lambda n: -(-n // 1024) * 1024
    off = up(T_tot * gdn.ATTN_N_IN * 2) + up(T_tot * 24 * 256 * 2)
    att = ws[off:off + T_tot * 24 * 256 * 2].view(torch.bfloat16).view(T_tot, 24 * 256)
    q0 = up(T_tot * gdn.ATTN_N_IN * 2)
    q_hat = ws[q0:q0 + T_tot * 24 * 256 * 2].view(torch.bfloat16).view(T_tot, 24, 256)
    return y, kc, vc, att.clone(), q_hat.clone()


@pytest.mark.parametrize("B,T,q_scale", [(2, 100, 1.0), (1, 200, 1.0), (1, 1024, 1.0), (3, 513, 4.0),
                                         (1, 1024, 4.0)])
def test_attention_core_matches_oracle(B, T, q_scale):
    """Random bf16 operands; q_scale 4 makes scores ~N(0, 16), so running maxima grow by
    more than the lazy threshold across key tiles and the rescale path runs."""
    A = oracle.attn
    g0 = torch.Generator().manual_seed(B * 1000 + T)
    T_tot = B * T
    q = (torch.randn(T_tot, 24, 256, generator=g0) * q_scale).to(torch.bfloat16)
    k = torch.randn(T_tot, 4, 256, generator=g0).to(torch.bfloat16)
    v = torch.randn(T_tot, 4, 256, generator=g0).to(torch.bfloat16)
    g = torch.randn(T_tot, 24, 256, generator=g0).to(torch.bfloat16)
    err = err_word()
    out = gdn.attention_prefill(q.cuda(), k.cuda(), v.cuda(), g.cuda(), B, T, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    cu = [i * T for i in range(B + 1)]
    sig = 1.0 / (1.0 + np.exp(-g.double().numpy()))
    ref = A.attention(q, k, v, cu) * sig
    o_abs = A.attention(q, k, np.abs(v.double().numpy()), cu) * sig
    bound = 2.0 ** -8 * o_abs + 2.0 ** -8 * np.abs(ref) + 1e-6
    d = np.abs(out.double().cpu().numpy().reshape(T_tot, 24, 256) - ref)
    r = float(np.max(d / bound))
    print(f"[parity] attention B {B} T {T} q_scale {q_scale}: max err / bound = {r:.3f}")
    assert r <= 1.0


@pytest.mark.parametrize("hidden,B,T", [(256, 2, 100), (512, 1, 200), (256, 1, 1024)])
def test_attn_layer_matches_oracle(hidden, B, T):
    A = oracle.attn
    c = exact_attn_case(hidden, B, T, seed=hidden + T)
    y, kc, vc, att, q_hat = run_attn(c)
    cu = [i * T for i in range(B + 1)]
    ref = A.attn_layer(c["x"], c["w_in"], c["w_out"], c["qn"], c["kn"], cu)
    T_tot = B * T
    q_ref = ref["q_hat"]  # fp64
    one_ulp = lambda gpu, r: float(np.max(np.abs(gpu.double().cpu().numpy().reshape(r.shape) - r) - 2.0 ** -7 * np.abs(r)))
    q_excess, k_excess = one_ulp(q_hat, q_ref), one_ulp(kc, ref["k_hat"])
    np.testing.assert_array_equal(vc.double().cpu().numpy(), ref["v"])
    # element-wise bounds: attention output, then through |W_out|
    lay = A.attn_in_proj_layout()
    sig = 1.0 / (1.0 + np.exp(-ref["proj"][:, lay["g"][0]:lay["g"][1]].reshape(T_tot, 24, 256)))
    o_abs = A.attention(q_ref, ref["k_hat"], np.abs(ref["v"]), cu) * sig
    att_ref = ref["out"]
    shift, grow = score_shift(q_hat.double().cpu().numpy(), kc.double().cpu().numpy(), q_ref, ref["k_hat"], cu)
    bound_att = (shift + 2.0 ** -8 * grow) * o_abs + 2.0 ** -8 * np.abs(att_ref) + 1e-6
    r_att = float(np.max(np.abs(att.double().cpu().numpy().reshape(T_tot, 24, 256) - att_ref) / bound_att))
    bound_y = (bound_att + 2.0 ** -8 * np.abs(att_ref)).reshape(T_tot, -1) @ np.abs(c["w_out"].double().numpy()).T \
        + 2.0 ** -8 * np.abs(ref["y"]) + 1e-6
    r_y = float(np.max(np.abs(y.double().cpu().numpy() - ref["y"]) / bound_y))
    e_y = out_error(y, ref["y"])
    print(f"[parity] attention layer hidden {hidden} B {B} T {T}: att/bound={r_att:.3f} y/bound={r_y:.3f} "
          f"(y_err rms form {e_y:.3e}); q_hat / K cache excess over 1 ulp {q_excess:.1e} / {k_excess:.1e}")
    assert q_excess <= 1e-6 and k_excess <= 1e-6
    assert r_att <= 1.0 and r_y <= 1.0


def test_attn_decode_steps_continue_the_prefill():
    """Prefill N prompts into caches with room for 3 more rows, then 3 decode steps: each
    step's output and attention output match the oracle layer over the whole sequence at
    its last position, the new cache rows match the oracle's, cache_len advances, and a 4th
    step finds the caches full (error bit 16, zero rows of y, caches unchanged).  The decode attention's
    scores are fp32 and its weights a bf16 hi + lo pair, so its bound is the score-shift term of the
    kernel's bf16 q_hat and cache rows against the oracle's (module docstring) plus 2^-12 e^{2E}
    sum p|v| / l and the output roundings."""
    A = oracle.attn
    N, T0, steps, hidden = 3, 150, 3, 256
    c = exact_attn_case(hidden, N, T0, seed=77, extra=steps)
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out", "qn", "kn")}
    L = gdn.make_attn_layer(d["w_in"], d["w_out"], d["qn"], d["kn"])
    err = err_word()
    cap = T0 + steps
    _, kc, vc = gdn.attn_layer_prefill(L, N, T0, d["x"], cache_cap=cap, err=err)
    cache_len = torch.full((N,), T0, dtype=torch.int32, device="cuda")
    ws = torch.empty(int(gdn.load().gdn_attn_decode_workspace_size(N, cap)), dtype=torch.uint8, device="cuda")
    xs = [c["x"].reshape(N, T0, hidden)]
    for st in range(steps):
        xn = c["x_more"][st]
        y = gdn.attn_layer_decode_step(L, xn.cuda(), kc, vc, cache_len, workspace=ws, err=err)
        torch.cuda.synchronize()
        assert int(err.item()) == 0
        assert torch.equal(cache_len.cpu(), torch.full((N,), T0 + st + 1, dtype=torch.int32))
        xs.append(xn[:, None])
        T = T0 + st + 1
        x_full = torch.cat(xs, dim=1).reshape(N * T, hidden)
        cu = [i * T for i in range(N + 1)]
        ref = A.attn_layer(x_full, c["w_in"], c["w_out"], c["qn"], c["kn"], cu)
        last = [i * T + T - 1 for i in range(N)]
        # attention output from the workspace: [projection | q_hat | attention], 1 KiB aligned
        up = lambda n: -(-n // 1024) * 1024
        off = up(N * gdn.ATTN_N_IN * 2) + up(N * 24 * 256 * 2)
        att = ws[off:off + N * 24 * 256 * 2].view(torch.bfloat16).view(N, 24, 256).double().cpu().numpy()
        lay = A.attn_in_proj_layout()
        sig = 1.0 / (1.0 + np.exp(-ref["proj"][:, lay["g"][0]:lay["g"][1]].reshape(N * T, 24, 256)))
        q_ref = ref["q_hat"]  # fp64
        o_abs = (A.attention(q_ref, ref["k_hat"], np.abs(ref["v"]), cu) * sig)[last]
        att_ref = ref["out"][last]
        # the kernel's operands: its q_hat of the new token (workspace) and its cache rows
        q_dec = ws[up(N * gdn.ATTN_N_IN * 2):up(N * gdn.ATTN_N_IN * 2) + N * 24 * 256 * 2].view(torch.bfloat16)
        q_gpu = np.zeros((N * T, 24, 256))
        q_gpu[last] = q_dec.view(N, 24, 256).double().cpu().numpy()
        k_gpu = kc[:, :T].reshape(N * T, 4, 256).double().cpu().numpy()
        shift, grow = score_shift(q_gpu, k_gpu, q_ref, ref["k_hat"], cu, rows=set(last))
        bound_att = (shift[last] + 2.0 ** -12 * grow[last]) * o_abs + 2.0 ** -8 * np.abs(att_ref) + 1e-6
        r_att = float(np.max(np.abs(att - att_ref) / bound_att))
        bound_y = (bound_att + 2.0 ** -8 * np.abs(att_ref)).reshape(N, -1) @ np.abs(c["w_out"].double().numpy()).T \
            + 2.0 ** -8 * np.abs(ref["y"][last]) + 1e-6
        r_y = float(np.max(np.abs(y.double().cpu().numpy() - ref["y"][last]) / bound_y))
        k_new = kc[:, T - 1].double().cpu().numpy()
        k_ref = ref["k_hat"][last]
        k_excess = float(np.max(np.abs(k_new - k_ref) - 2.0 ** -7 * np.abs(k_ref)))
        np.testing.assert_array_equal(vc[:, T - 1].double().cpu().numpy(), ref["v"][last])
        print(f"[parity] attention decode step {st + 1} (cache {T} rows): att/bound={r_att:.3f} y/bound={r_y:.3f} "
              f"new K row excess over 1 ulp {k_excess:.1e}")
        assert r_att <= 1.0 and r_y <= 1.0 and k_excess <= 1e-6
    # the caches are full now
    k_before = kc.clone()
    y_full = torch.full((N, hidden), 5.0, dtype=torch.bfloat16, device="cuda")
    gdn.attn_layer_decode_step(L, c["x_more"][0].cuda(), kc, vc, cache_len, y=y_full, workspace=ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) & 16
    assert torch.equal(cache_len.cpu(), torch.full((N,), cap, dtype=torch.int32))
    assert torch.all(y_full == 0)
    assert torch.equal(kc, k_before)


def test_attn_decode_long_ragged_caches():
    """Decode over caches filled with seeded rows, cache_len = 0, 511, 1023 and 1300 (1, 512,
    1024 and 1301 attended rows: one row, one full split, two full splits, three splits with a
    ragged last one), so the split-K partials and their merge are all exercised.  q_hat and the
    new K row must be within one bf16 ulp of the oracle's; the attention output is compared
    with the oracle's causal attention over the whole sequence (last row) on the kernel's own
    q_hat, where the fp32 scores and the p_hi + p_lo weights leave an error far below
    2^-12 sum p|v| / l, plus the bf16 rounding of the stored output."""
    A = oracle.attn
    lens = [0, 511, 1023, 1300]
    N, cap, hidden = len(lens), 1400, 256
    c = exact_attn_case(hidden, N, 1, seed=91)
    g = torch.Generator().manual_seed(92)
    kc = torch.randn(N, cap, 4, 256, generator=g).to(torch.bfloat16)
    vc = torch.randn(N, cap, 4, 256, generator=g).to(torch.bfloat16)
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out", "qn", "kn")}
    L = gdn.make_attn_layer(d["w_in"], d["w_out"], d["qn"], d["kn"])
    err = err_word()
    kcd, vcd = kc.cuda(), vc.cuda()
    cache_len = torch.tensor(lens, dtype=torch.int32, device="cuda")
    ws = torch.empty(int(gdn.load().gdn_attn_decode_workspace_size(N, cap)), dtype=torch.uint8, device="cuda")
    gdn.attn_layer_decode_step(L, d["x"], kcd, vcd, cache_len, workspace=ws, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert cache_len.cpu().tolist() == [n + 1 for n in lens]
    up = lambda n: -(-n // 1024) * 1024
    off_q = up(N * gdn.ATTN_N_IN * 2)
    off_att = off_q + up(N * 24 * 256 * 2)
    q_gpu = ws[off_q:off_q + N * 24 * 256 * 2].view(torch.bfloat16).view(N, 24, 256).double().cpu().numpy()
    att = ws[off_att:off_att + N * 24 * 256 * 2].view(torch.bfloat16).view(N, 24, 256).double().cpu().numpy()
    proj = oracle.round_bf16(oracle.gemm(c["x"], c["w_in"]))
    lay = A.attn_in_proj_layout()
    part = lambda name: proj[:, lay[name][0]:lay[name][1]]
    worst_att = worst_q = worst_k = 0.0
    for n, ln in enumerate(lens):
        pos = np.array([ln])
        q_ref = A.rope(A.rms_norm(part("q")[n].reshape(1, 24, 256), c["qn"]), pos)[0]  # fp64
        k_ref = oracle.round_bf16(A.rope(A.rms_norm(part("k")[n].reshape(1, 4, 256), c["kn"]), pos))[0]
        v_new = part("v")[n].reshape(4, 256)
        worst_q = max(worst_q, float(np.max(np.abs(q_gpu[n] - q_ref) - 2.0 ** -7 * np.abs(q_ref))))
        k_row = kcd[n, ln].double().cpu().numpy()
        worst_k = max(worst_k, float(np.max(np.abs(k_row - k_ref) - 2.0 ** -7 * np.abs(k_ref))))
        np.testing.assert_array_equal(vcd[n, ln].double().cpu().numpy(), v_new)
        # the sequence as the oracle sees it: the cache rows, then the new token (the GPU's own
        # new K row, checked above), whose query is the last row
        T = ln + 1
        keys = np.concatenate([kc[n, :ln].double().numpy(), k_row[None]], axis=0)
        vals = np.concatenate([vc[n, :ln].double().numpy(), v_new[None]], axis=0)
        qs = np.zeros((T, 24, 256))
        qs[-1] = q_gpu[n]
        sig = 1.0 / (1.0 + np.exp(-part("g")[n].reshape(24, 256)))
        ref = A.attention(qs, keys, vals, [0, T])[-1] * sig
        o_abs = A.attention(qs, keys, np.abs(vals), [0, T])[-1] * sig
        bound = 2.0 ** -12 * o_abs + 2.0 ** -8 * np.abs(ref) + 1e-6
        worst_att = max(worst_att, float(np.max(np.abs(att[n] - ref) / bound)))
    print(f"[parity] attention decode over caches {lens}: att/bound={worst_att:.3f}; q_hat / new K row excess "
          f"over 1 ulp {worst_q:.1e} / {worst_k:.1e}")
    assert worst_q <= 1e-6 and worst_k <= 1e-6
    assert worst_att <= 1.0
    # rows other than the new ones are untouched
    for n, ln in enumerate(lens):
        assert torch.equal(kcd[n, :ln].cpu(), kc[n, :ln]) and torch.equal(kcd[n, ln + 1:].cpu(), kc[n, ln + 1:])


def test_attn_decode_rejects_a_negative_cache_length():
    """A cache_len outside [0, cache_cap] is treated like a full cache: no cache row is written
    (in particular not the previous sequence's last row, which a negative length would reach),
    that sequence's row of y is zero, its cache_len is left alone and bit 32 of *err is set; the
    other sequences step normally."""
    N, T0, hidden = 3, 40, 256
    c = exact_attn_case(hidden, N, T0, seed=31, extra=1)
    d = {k: c[k].cuda() for k in ("x", "w_in", "w_out", "qn", "kn")}
    L = gdn.make_attn_layer(d["w_in"], d["w_out"], d["qn"], d["kn"])
    err = err_word()
    cap = T0 + 2
    _, kc, vc = gdn.attn_layer_prefill(L, N, T0, d["x"], cache_cap=cap, err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    # fill the unused rows with a marker, so that any write shows
    kc.view(N, cap, -1)[:, T0:] = 7.0
    vc.view(N, cap, -1)[:, T0:] = 7.0
    k_before, v_before = kc.clone(), vc.clone()
    cache_len = torch.tensor([T0, -1, T0], dtype=torch.int32, device="cuda")
    ws = torch.empty(int(gdn.load().gdn_attn_decode_workspace_size(N, cap)), dtype=torch.uint8, device="cuda")
    y = torch.full((N, hidden), 5.0, dtype=torch.bfloat16, device="cuda")
    gdn.attn_layer_decode_step(L, c["x_more"][0].cuda(), kc, vc, cache_len, y=y, workspace=ws, err=err)
    torch.cuda.synchronize()
    e = int(err.item())
    print(f"[parity] attention decode with cache_len -1: err word {e}, y finite {bool(torch.isfinite(y).all())}")
    assert e & 32 and not e & 16
    assert cache_len.cpu().tolist() == [T0 + 1, -1, T0 + 1]
    assert torch.isfinite(y).all()
    assert torch.all(y[1] == 0) and not torch.all(y[0] == 0) and not torch.all(y[2] == 0)
    kv = lambda t: t.view(N, cap, -1)
    # sequence 1 untouched, and so is sequence 0's last row (where row -1 of sequence 1 would land)
    assert torch.equal(kv(kc)[1], kv(k_before)[1]) and torch.equal(kv(vc)[1], kv(v_before)[1])
    assert torch.equal(kv(kc)[0, cap - 1], kv(k_before)[0, cap - 1])
    assert torch.equal(kv(vc)[0, cap - 1], kv(v_before)[0, cap - 1])
    # the valid sequences wrote their new row T0 only
    for n in (0, 2):
        assert not torch.equal(kv(kc)[n, T0], kv(k_before)[n, T0])
        assert torch.equal(kv(kc)[n, :T0], kv(k_before)[n, :T0])
