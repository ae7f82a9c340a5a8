"""Chunked forms of KDA in fp64 numpy, used only as pins for the oracle.

Both follow the chunked formulation in the mokono.cn explainer "Kimi
Linear：高效注意力机制在长序列处理中的创新应用" (section 2.1, Proposition:
S_r = P_r S_0 + H_r with P_r = Diag(gamma_r) - sum_i Diag(gamma_{i->r}) k_i w_i^T
and H_r = sum_i Diag(gamma_{i->r}) k_i u_i^T; section 2.2, WY auxiliaries w_r, u_r)
and the chunk-parallel algorithm of the blog.gzher.com review (section 4: WY
representation, UT transform with a strictly lower triangular matrix, state
passed between chunks). Within a chunk, g_r = sum_{j<=r} log_alpha_j,
gamma_r = exp(g_r) and gamma_{i->r} = exp(g_r - g_i) = prod_{j=i+1..r} alpha_j.
Working the Proposition through eq. (1) by induction on r gives

    w_r = beta_r (gamma_r * k_r - sum_{i<r} (k_r^T Diag(gamma_{i->r}) k_i) w_i)
    u_r = beta_r (v_r         - sum_{i<r} (k_r^T Diag(gamma_{i->r}) k_i) u_i)

which in matrix form is (I + A_kk) W = Diag(beta)(Gamma * K), (I + A_kk) U =
Diag(beta) V with A_kk[r, i] = beta_r k_r^T Diag(gamma_{i->r}) k_i for i < r.

``kda_proposition_fp64`` evaluates P_r and H_r position by position (tiny
sizes); ``kda_chunked_fp64`` evaluates the UT matrix form chunk by chunk.
"""
from __future__ import annotations

import numpy as np


def _pairwise_decay(g):
    """D[r, i, c] = exp(g[r, c] - g[i, c]) for i <= r, else 0."""
    L = g.shape[0]
    diff = g[:, None, :] - g[None, :, :]
    lower = np.tril(np.ones((L, L), dtype=bool))[:, :, None]
    return np.where(lower, np.exp(np.where(lower, diff, 0.0)), 0.0)


def kda_chunked_fp64(q, k, v, log_alpha, beta, S0=None, C=64):
    """UT-transform chunked form over ``[B, T, H, d]`` inputs; returns (o, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                L = min(C, T - c0)
                Q, K, V = q[b, c0:c0 + L, h], k[b, c0:c0 + L, h], v[b, c0:c0 + L, h]
                bt = beta[b, c0:c0 + L, h]
                g = np.cumsum(log_alpha[b, c0:c0 + L, h], axis=0)
                D = _pairwise_decay(g)
                strict = np.tril(np.ones((L, L)), -1)
                A_kk = bt[:, None] * np.einsum("rc,ic,ric->ri", K, K, D) * strict
                A_qk = np.einsum("rc,ic,ric->ri", Q, K, D)
                Tinv = np.linalg.inv(np.eye(L) + A_kk)
                Gam = np.exp(g)
                W = Tinv @ (bt[:, None] * Gam * K)
                U = Tinv @ (bt[:, None] * V)
                Vn = U - W @ S
                o[b, c0:c0 + L, h] = (Q * Gam) @ S + A_qk @ Vn
                S = np.exp(g[-1])[:, None] * S + (K * np.exp(g[-1] - g)).T @ Vn
            S_T[b, h] = S
    return o, S_T


def kda_proposition_fp64(q, k, v, log_alpha, beta, S0=None, C=64):
    """Position-by-position P_r / H_r evaluation of the Proposition; returns (o, S_T)."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else S0[b, h].copy()
            for c0 in range(0, T, C):
                L = min(C, T - c0)
                g = np.cumsum(log_alpha[b, c0:c0 + L, h], axis=0)
                K, V, Q = k[b, c0:c0 + L, h], v[b, c0:c0 + L, h], q[b, c0:c0 + L, h]
                bt = beta[b, c0:c0 + L, h]
                w, u = [], []
                for r in range(L):
                    a_ri = [K[r] @ (np.exp(g[r] - g[i]) * K[i]) for i in range(r)]
                    w.append(bt[r] * (np.exp(g[r]) * K[r] - sum((a * wi for a, wi in zip(a_ri, w)), np.zeros(dk))))
                    u.append(bt[r] * (V[r] - sum((a * ui for a, ui in zip(a_ri, u)), np.zeros(dv))))
                    P = np.diag(np.exp(g[r])) - sum(np.outer(np.exp(g[r] - g[i]) * K[i], w[i]) for i in range(r + 1))
                    Hm = sum(np.outer(np.exp(g[r] - g[i]) * K[i], u[i]) for i in range(r + 1))
                    S_r = P @ S + Hm
                    o[b, c0 + r, h] = S_r.T @ Q[r]
                S = S_r
            S_T[b, h] = S
    return o, S_T
