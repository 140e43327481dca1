"""Independent fp64 chunked form of the gated delta rule -- test infrastructure only.

It validates the chunk algebra that the GPU path uses; it is not the reference
(the sequential recurrence in gdn_oracle.c is).  Derivation, written out from
the recurrence the Agnes-3.0-Flash pages name (model card, "Architecture" table,
row "Delta-rule layers"; "Agnes-3.0-Flash Deep Dive: A 33B Hybrid-Attention
Multimodal Model", section "Feed-Forward and Positional Encoding", paragraph on
the Gated Delta Rule):

  S_i = alpha_i S_{i-1} + u_i k_i^T   with   u_i = beta_i (v_i - alpha_i S_{i-1} k_i).

Unrolling inside one chunk that starts from S_0, with gamma_i = prod_{j<=i} alpha_j
= exp(G_i), G the inclusive cumulative sum of g = log(alpha):

  S_i = gamma_i S_0 + sum_{j<=i} (gamma_i / gamma_j) u_j k_j^T
  (I + A) U = diag(beta) V - diag(beta gamma) K S_0^T,
        A_ij = beta_i exp(G_i - G_j) (k_i . k_j) for j < i, else 0
  O = diag(gamma) Q S_0^T + (M * Q K^T) U,  M_ij = exp(G_i - G_j) for j <= i, else 0
  S_C = gamma_C S_0 + U^T diag(exp(G_C - G_j)) K

This is the chunkwise (UT-transform) form of the published Gated Delta Networks
and DeltaNet-parallelisation papers, re-derived here.  A library triangular
solve and matmuls are its only primitives.

chunked_transfer_recurrence writes the same chunk step with the state dependence
gathered into one product per chunk.  With T = (I + A)^{-1}, W = T diag(beta gamma) K,
U0 = T diag(beta) V, P = M * Q K^T and D = diag(exp(G_C - G_j)), the solve above is
U = U0 - W S_0^T, so

  O   = (diag(gamma) Q - P W) S_0^T + P U0
  S_C = S_0 (gamma_C I - W^T D K) + U0^T D K

i.e. S_C = S_0 M + N with M and N independent of the state (a transfer matrix and a
drive per chunk).
"""
from __future__ import annotations

import numpy as np


def chunked_recurrence(q, k, v, g, beta, S0=None, chunk=64):
    """One head, one sequence: q, k [T][dk], v [T][dv], g, beta [T] (g = log alpha,
    finite).  Returns (o [T][dv], S [dv][dk]) in fp64."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        Q, K, V, b = q[sl], k[sl], v[sl], beta[sl]
        L = K.shape[0]
        G = np.cumsum(g[sl])
        gam = np.exp(G)
        ii, jj = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
        expo = np.where(jj <= ii, G[:, None] - G[None, :], -np.inf)
        M = np.exp(expo)  # exp(G_i - G_j) on and below the diagonal, 0 above
        strict = np.where(jj < ii, M, 0.0)
        A = b[:, None] * strict * (K @ K.T)
        rhs = b[:, None] * V - (b * gam)[:, None] * (K @ S.T)
        U = np.linalg.solve(np.eye(L) + A, rhs)
        o[sl] = gam[:, None] * (Q @ S.T) + (M * (Q @ K.T)) @ U
        dec = np.exp(G[-1] - G)
        S = gam[-1] * S + U.T @ (dec[:, None] * K)
    return o, S


def chunked_transfer_recurrence(q, k, v, g, beta, S0=None, chunk=64):
    """The same chunk step as chunked_recurrence, written as O = Q' S_0^T + P U0 and
    S_C = S_0 M + N (module docstring).  Arguments and results as chunked_recurrence."""
    q, k, v, g, beta = (np.asarray(x, dtype=np.float64) for x in (q, k, v, g, beta))
    T, dk = k.shape
    dv = v.shape[1]
    S = np.zeros((dv, dk)) if S0 is None else np.array(S0, dtype=np.float64)
    o = np.zeros((T, dv))
    for c0 in range(0, T, chunk):
        sl = slice(c0, min(c0 + chunk, T))
        Q, K, V, b = q[sl], k[sl], v[sl], beta[sl]
        L = K.shape[0]
        G = np.cumsum(g[sl])
        gam = np.exp(G)
        ii, jj = np.meshgrid(np.arange(L), np.arange(L), indexing="ij")
        M_ij = np.exp(np.where(jj <= ii, G[:, None] - G[None, :], -np.inf))
        A = b[:, None] * np.where(jj < ii, M_ij, 0.0) * (K @ K.T)
        Tinv = np.linalg.inv(np.eye(L) + A)
        W = Tinv @ ((b * gam)[:, None] * K)
        U0 = Tinv @ (b[:, None] * V)
        P = M_ij * (Q @ K.T)
        DK = np.exp(G[-1] - G)[:, None] * K
        transfer = gam[-1] * np.eye(dk) - W.T @ DK
        drive = U0.T @ DK
        o[sl] = (gam[:, None] * Q - P @ W) @ S.T + P @ U0
        S = S @ transfer + drive
    return o, S
