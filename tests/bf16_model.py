"""A numpy model of where the bf16 tensor-core path rounds, for error budgets.

Test code only. It runs the UT-transform chunk algebra of ``chunked_form`` (the
blog.gzher.com review, section 4; the mokono.cn explainer, section 2.1) with the
roundings of the bf16 path: every MMA operand is rounded to bf16 (round to nearest
even), every accumulation and the recurrent state stay fp32 (modelled in fp64, whose
extra precision is far below the bf16 steps), and the output is rounded to bf16.

Rounded to bf16 are:
- q e^g and k e^g (the Gram's A operand, and W's B operand);
- k e^-g (the Gram's B operand);
- k e^(g_L - g) (the state update's A operand);
- A_qk, T Diag(beta) and W (the stored operand images);
- the state image S (B operand of the chunk's first MMAs);
- V_new (B operand of the state update and the output MMA);
- o.

It does not model the factorised exponentials' own rounding or the order of fp32
sums, so it predicts the size of the path's error, not its exact values.
"""
from __future__ import annotations

import numpy as np


def bf16(x):
    """Round to the nearest bf16 value (ties to even), returned in float64."""
    f = np.asarray(x, dtype=np.float32)
    u = f.view(np.uint32).astype(np.uint64)
    u = (u + 0x7FFF + ((u >> 16) & 1)) & 0xFFFF0000
    return u.astype(np.uint32).view(np.float32).astype(np.float64)


def kda_bf16_model(q, k, v, log_alpha, beta, S0=None, C=64):
    """bf16-path model over ``[B, T, H, d]`` inputs; returns (o, S_T) in float64."""
    B, T, H, dk = q.shape
    dv = v.shape[-1]
    o = np.zeros((B, T, H, dv))
    S_T = np.zeros((B, H, dk, dv))
    for b in range(B):
        for h in range(H):
            S = np.zeros((dk, dv)) if S0 is None else np.array(S0[b, h], dtype=np.float64)
            for c0 in range(0, T, C):
                L = min(C, T - c0)
                Q, K, V = q[b, c0:c0 + L, h], k[b, c0:c0 + L, h], v[b, c0:c0 + L, h]
                bt = beta[b, c0:c0 + L, h]
                g = np.cumsum(log_alpha[b, c0:c0 + L, h], axis=0)
                Qg, Kg = bf16(Q * np.exp(g)), bf16(K * np.exp(g))
                Kinv, Kt = bf16(K * np.exp(-g)), bf16(K * np.exp(g[-1] - g))
                G = np.concatenate([Qg, Kg]) @ Kinv.T
                A_qk = bf16(np.tril(G[:L]))
                A_kk = bt[:, None] * np.tril(G[L:], -1)
                TB = bf16(np.linalg.inv(np.eye(L) + A_kk) * bt[None, :])
                W = bf16(TB @ Kg)
                S_img = bf16(S)
                Vn = bf16(TB @ V - W @ S_img)
                o[b, c0:c0 + L, h] = bf16(Qg @ S_img + A_qk @ Vn)
                S = np.exp(g[-1])[:, None] * S + Kt.T @ Vn
            S_T[b, h] = S
    return o, S_T
