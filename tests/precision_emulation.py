"""CPU emulation of the prefill's chunk algebra with the tensor-core operand formats -- test
infrastructure only (imports the oracle for the front end's reference values; nothing here is
product code).

Every product X @ Y takes each operand either as a bf16 hi/lo pair ("s": hi = bf16(x),
lo = bf16(x - hi), the lo.lo term dropped, as the kernels do) or as plain bf16 ("b"), and
accumulates in fp64; every stored intermediate is rounded to fp32.  Two chunk steps:

  WY form (as built):  U = U0 - W S^T,  O = diag(gamma) Q S^T + P U,
                       S <- gamma_C S + U^T diag(e^{G_C - G_j}) K
  transfer form:       O = (diag(gamma) Q - P W) S^T + P U0,  S <- S M + N,
                       M = gamma_C I - W^T D K,  N = U0^T D K

with W = T diag(beta gamma) K, U0 = T diag(beta) V, T = (I + A)^{-1}, P = M_ij (Q K^T) as in
oracle/chunked.py.  The front end (conv, SiLU, L2-norm, gates) is computed in fp64 and the
q, k, v features rounded to fp32, as the prep kernel holds them.
"""
import numpy as np
import torch

PRODUCTS = ("qk", "w", "u0", "ws", "qs", "pu", "uk")
ALL_SPLIT = {name: "ss" for name in PRODUCTS}


def _bf(x):
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16).double().numpy()


def _f32(x):
    return np.asarray(x, dtype=np.float32).astype(np.float64)


def _parts(x, mode):
    x = _f32(x)
    hi = _bf(x)
    return (hi, None) if mode == "b" else (hi, _bf(x - hi))


def mm(X, Y, mx="s", my="s"):
    xh, xl = _parts(X, mx)
    yh, yl = _parts(Y, my)
    r = xh @ yh
    if yl is not None:
        r = r + xh @ yl
    if xl is not None:
        r = r + xl @ yh
    return _f32(r)


def _features(inp, T, H_k, H_v):
    D = 128
    x = torch.cat([inp["q"].double().reshape(T, -1), inp["k"].double().reshape(T, -1),
                   inp["v"].double().reshape(T, -1)], 1).numpy()
    w = inp["conv_w"].double().numpy()
    xp = np.concatenate([np.zeros((3, x.shape[1])), x])
    y = sum(w[:, j][None] * xp[j:j + T] for j in range(4))
    y = y / (1 + np.exp(-y))
    q = y[:, :H_k * D].reshape(T, H_k, D)
    k = y[:, H_k * D:2 * H_k * D].reshape(T, H_k, D)
    v = _f32(y[:, 2 * H_k * D:].reshape(T, H_v, D))
    q = _f32(q / np.sqrt((q * q).sum(-1, keepdims=True) + 1e-6) * float(inp.get("scale", 1.0)))
    k = _f32(k / np.sqrt((k * k).sum(-1, keepdims=True) + 1e-6))
    a = inp["a"].double().numpy()
    b = inp["b"].double().numpy()
    g = -np.exp(inp["A_log"].double().numpy())[None] * np.log1p(np.exp(a))
    beta = 1 / (1 + np.exp(-b))
    return q, k, v, g, beta, inp["z"].double().numpy()


def emulate(inp, T, state_in, H_k, H_v, heads, prec=None, form="wy"):
    """Outputs [T][H_v][128] (fp64, before the bf16 output rounding) and final states of the
    given value heads; prec maps each product of PRODUCTS to its two operands' formats."""
    p = dict(ALL_SPLIT)
    p.update(prec or {})
    D = 128
    G = H_v // H_k
    q, k, v, g, beta, z = _features(inp, T, H_k, H_v)
    out = np.zeros((T, H_v, D))
    S_fin = np.zeros((H_v, D, D))
    for h in heads:
        kh = h // G
        S = _f32(state_in[0, h].double().numpy())
        for c0 in range(0, T, 64):
            sl = slice(c0, min(c0 + 64, T))
            L = sl.stop - sl.start
            Q, K, V, bt = q[sl, kh], k[sl, kh], v[sl, h], beta[sl, h]
            Gc = np.cumsum(g[sl, h])
            gam = np.exp(Gc)
            ii, jj = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
            Mij = np.exp(np.where(jj <= ii, Gc[:, None] - Gc[None, :], -np.inf))
            QK = mm(Q, K.T, *p["qk"])
            KK = mm(K, K.T, *p["qk"])
            A = _f32(bt[:, None] * np.where(jj < ii, Mij, 0) * KK)
            P = _f32(Mij * QK)
            Tinv = _f32(np.linalg.inv(np.eye(L) + A))
            W = mm(_f32(Tinv * (bt * gam)[None, :]), K, *p["w"])
            U0 = mm(_f32(Tinv * bt[None, :]), V, *p["u0"])
            gQ = _f32(gam[:, None] * Q)
            DK = _f32(np.exp(Gc[-1] - Gc)[:, None] * K)
            if form == "wy":
                U = _f32(U0 - mm(W, S.T, *p["ws"]))
                O = _f32(mm(gQ, S.T, *p["qs"]) + mm(P, U, *p["pu"]))
                Ud = _f32(np.exp(Gc[-1] - Gc)[:, None] * U)
                S = _f32(np.exp(Gc[-1]) * S + mm(K.T, Ud, *p["uk"]).T)
            else:
                Mc = _f32(np.exp(Gc[-1]) * np.eye(D) - mm(W.T, DK))
                Qp = _f32(gQ - mm(P, W))
                O = _f32(mm(Qp, S.T) + mm(P, U0))
                S = _f32(mm(S, Mc) + mm(U0.T, DK))
            out[sl, h] = O / np.sqrt((O * O).mean(-1, keepdims=True) + 1e-6) * (z[sl, h] / (1 + np.exp(-z[sl, h])))
        S_fin[h] = S
    return out, S_fin


def errors(out, S, ref, heads):
    """(element-wise output error beyond the bf16 output rounding, in rms units; worst relative
    Frobenius state error) of the bf16-rounded emulated outputs against the oracle."""
    o = _bf(out)[:, heads]
    r = np.asarray(ref["out"])[:, heads]
    rms = np.sqrt(np.mean(r * r))
    out_err = float(np.max(np.abs(o - r) - 2.0**-8 * np.abs(r)) / rms)
    st = max(float(np.linalg.norm(S[h] - ref["state"][0, h]) / max(np.linalg.norm(ref["state"][0, h]), 1e-30))
             for h in heads)
    return out_err, st
