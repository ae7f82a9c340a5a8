"""Chunked reverse pass of KDA in fp64 numpy: a debug aid for a chunked backward.

Test code only. It differentiates the chunk algebra of ``chunked_form.kda_chunked_fp64``
(the UT-transform form of the blog.gzher.com review, section 4, built on the
Proposition of the mokono.cn explainer, section 2.1) and is checked against the
token-by-token reverse-pass oracle, which differentiates eq. (1) directly.

Per chunk of L tokens, with the state S at its start and g the chunk-local cumulative
sum of log_alpha:

    D[r,i,c] = exp(g_rc - g_ic) (i <= r)     Gam = exp(g)      E = exp(g_L - g)
    A_kk = Diag(beta) (sum_c K_rc K_ic D[r,i,c]) strictly lower
    A_qk = (sum_c Q_rc K_ic D[r,i,c]) lower, diagonal included
    T = (I + A_kk)^-1     W = T Diag(beta) (Gam * K)     U = T Diag(beta) V
    V_new = U - W S       O = (Q * Gam) S + A_qk V_new
    S_next = Diag(exp(g_L)) S + (K * E)^T V_new

Going backwards over the chunks with G = dLoss/dS_next, each line is differentiated in
reverse; the gradient of T = (I + A)^-1 is -T^T dT T^T restricted to A's strictly
lower support, and log_alpha's gradient is the reverse cumulative sum of g's.
"""
from __future__ import annotations

import numpy as np


def _pairwise_decay(g):
    L = g.shape[0]
    lower = np.tril(np.ones((L, L), dtype=bool))[:, :, None]
    diff = g[:, None, :] - g[None, :, :]
    return np.where(lower, np.exp(np.where(lower, diff, 0.0)), 0.0)


def _gram_backward(dA, X, K, D, g_grad, dX, dK):
    """A[r,i] = sum_c X_rc K_ic D[r,i,c] on A's support (dA already restricted to it):
    adds the gradients of X, K and g (through D = exp(g_r - g_i))."""
    dX += np.einsum("ri,ic,ric->rc", dA, K, D)
    dK += np.einsum("ri,rc,ric->ic", dA, X, D)
    dD = dA[:, :, None] * X[:, None, :] * K[None, :, :] * D
    g_grad += dD.sum(axis=1) - dD.sum(axis=0)


def kda_chunked_bwd_fp64(q, k, v, log_alpha, beta, S0, do, dS_T, C=64):
    """Gradients of sum(o do) + sum(S_T dS_T) for ``[B, T, H, d]`` inputs (fp64).

    Returns a dict like the reverse-pass oracle: dq, dk, dv, dlog_alpha, dbeta, dS0.
    """
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    out = {"dq": np.zeros_like(q), "dk": np.zeros_like(k), "dv": np.zeros_like(v),
           "dlog_alpha": np.zeros_like(log_alpha), "dbeta": np.zeros_like(beta),
           "dS0": np.zeros((B, H, dk, dv))}
    for b in range(B):
        for h in range(H):
            # forward over the chunks, keeping what the reverse pass needs
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            saved = []
            for c0 in range(0, T, C):
                L = min(C, T - c0)
                Q, K, V = q[b, c0:c0 + L, h], k[b, c0:c0 + L, h], v[b, c0:c0 + L, h]
                bt = beta[b, c0:c0 + L, h]
                g = np.cumsum(log_alpha[b, c0:c0 + L, h], axis=0)
                D = _pairwise_decay(g)
                strict = np.tril(np.ones((L, L)), -1)
                incl = np.tril(np.ones((L, L)))
                P = np.einsum("rc,ic,ric->ri", K, K, D) * strict
                A_kk = bt[:, None] * P
                A_qk = np.einsum("rc,ic,ric->ri", Q, K, D) * incl
                Tinv = np.linalg.inv(np.eye(L) + A_kk)
                Gam, E = np.exp(g), np.exp(g[-1] - g)
                W = Tinv @ (bt[:, None] * Gam * K)
                U = Tinv @ (bt[:, None] * V)
                Vn = U - W @ S
                saved.append((c0, L, S, g, D, strict, incl, P, A_qk, Tinv, Gam, E, W, Vn))
                S = np.exp(g[-1])[:, None] * S + (K * E).T @ Vn
            # reverse over the chunks
            G = dS_T[b, h].copy()
            for c0, L, S, g, D, strict, incl, P, A_qk, Tinv, Gam, E, W, Vn in reversed(saved):
                sl = slice(c0, c0 + L)
                Q, K, V = q[b, sl, h], k[b, sl, h], v[b, sl, h]
                bt = beta[b, sl, h]
                dO = do[b, sl, h]
                dQ, dK, dV = np.zeros_like(Q), np.zeros_like(K), np.zeros_like(V)
                dbt, dg = np.zeros(L), np.zeros_like(g)
                # O = (Q * Gam) S + A_qk V_new
                dQG = dO @ S.T
                dQ += dQG * Gam
                dg += dQG * Q * Gam
                dS = (Q * Gam).T @ dO
                dA_qk = (dO @ Vn.T) * incl
                dVn = A_qk.T @ dO
                # S_next = Diag(exp(g_L)) S + (K * E)^T V_new
                gamL = np.exp(g[-1])
                dS += gamL[:, None] * G
                dg_L = np.sum(G * S, axis=1) * gamL
                dKE = Vn @ G.T
                dVn += (K * E) @ G
                dK += dKE * E
                dE = dKE * K * E
                dg_L += dE.sum(axis=0)
                dg -= dE
                # V_new = U - W S
                dU = dVn
                dW = -dVn @ S.T
                dS -= W.T @ dVn
                # U = T Diag(beta) V,  W = T Diag(beta) (Gam * K)
                dT = dU @ (bt[:, None] * V).T + dW @ (bt[:, None] * Gam * K).T
                dBV = Tinv.T @ dU
                dV += bt[:, None] * dBV
                dbt += np.sum(dBV * V, axis=1)
                dBGK = Tinv.T @ dW
                dK += dBGK * bt[:, None] * Gam
                dg += dBGK * bt[:, None] * K * Gam
                dbt += np.sum(dBGK * Gam * K, axis=1)
                # T = (I + A_kk)^-1, A_kk = Diag(beta) P (strictly lower)
                dA_kk = -(Tinv.T @ dT @ Tinv.T) * strict
                dbt += np.sum(dA_kk * P, axis=1)
                _gram_backward(dA_kk * bt[:, None], K, K, D, dg, dK, dK)
                _gram_backward(dA_qk, Q, K, D, dg, dQ, dK)
                # g = cumsum(log_alpha); g_L = g[L-1]
                dg[-1] += dg_L
                out["dlog_alpha"][b, sl, h] = np.cumsum(dg[::-1], axis=0)[::-1]
                out["dq"][b, sl, h] = dQ
                out["dk"][b, sl, h] = dK
                out["dv"][b, sl, h] = dV
                out["dbeta"][b, sl, h] = dbt
                G = dS
            out["dS0"][b, h] = G
    return out
