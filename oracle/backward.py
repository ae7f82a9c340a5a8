"""KDA oracle, reverse pass: plain fp64 gradients of the recurrence.

TEST INFRASTRUCTURE ONLY, like the forward oracle: nothing in the product path may
import or call it. It shares no code with the CUDA library.

The forward step is eq. (1) of blog.gzher.com "Kimi K3论文：Kimi Linear", section 3,
written in the order the formula reads (and the forward oracle runs):

    a   = exp(log_alpha_t)                 S' = Diag(a) S_{t-1}
    u   = S'^T k_t                         d  = beta_t (v_t - u)
    S_t = S' + k_t d^T                     o_t = S_t^T q_t

Given the gradients of a scalar loss with respect to every o_t (do) and to the final
state (dS_T), this walks the tokens backwards and applies the chain rule to each line
in reverse, with G the gradient with respect to S_t:

    G  += q_t do_t^T            dq_t  = S_t do_t                 (o_t = S_t^T q_t)
    dk_t = G d                  dd    = G^T k_t                  (S_t = S' + k_t d^T)
    dbeta_t = dd . (v_t - u)    dv_t  = beta_t dd    du = -beta_t dd
    G' = G + k_t du^T           dk_t += S' du                    (u = S'^T k_t)
    dlog_alpha_t = a * rowsum(G' * S_{t-1})                      (S' = Diag(a) S_{t-1})
    G  = Diag(a) G'   (the gradient with respect to S_{t-1})

and finally dS0 = G. The states S_{t-1} of every step are kept from a forward sweep
run here; nothing is blocked, fused or reordered. Section 4 of the same page quotes
the per-head cost of training; these are the plain gradients that any training-time
(chunked) backward has to reproduce.

Layouts are those of the forward oracle: batched [B, T, H, .] or packed [n_tok, H, .]
with cu_seqlens; beta [.., H]; states [n_seqs, H, dk, dv].
"""
from __future__ import annotations

import numpy as np

from . import _f64


def _offsets(q, cu_seqlens):
    if cu_seqlens is None:
        B, T = q.shape[:2]
        return np.arange(B + 1, dtype=np.int64) * T
    cu = cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens
    return np.asarray(cu, dtype=np.int64)


def kda_bwd(q, k, v, log_alpha, beta, S0, do, dS_T, cu_seqlens=None):
    """Gradients of sum(o * do) + sum(S_T * dS_T) with respect to every input.

    Returns a dict of fp64 arrays shaped like the inputs: dq, dk, dv, dlog_alpha,
    dbeta, dS0 (dS0 is returned even when S0 is None, which means zeros). dS_T may be
    None (no loss on the final state).
    """
    q, k, v, la, b, do = (_f64(t) for t in (q, k, v, log_alpha, beta, do))
    cu = _offsets(q, cu_seqlens)
    H, dk = q.shape[-2:]
    dv = v.shape[-1]
    n_seqs = len(cu) - 1
    flat = lambda x, d: x.reshape(-1, H, d) if d else x.reshape(-1, H)
    qf, kf, vf, laf, dof = flat(q, dk), flat(k, dk), flat(v, dv), flat(la, dk), flat(do, dv)
    bf = flat(b, 0)
    s0 = np.zeros((n_seqs, H, dk, dv)) if S0 is None else _f64(S0)
    dST = np.zeros((n_seqs, H, dk, dv)) if dS_T is None else _f64(dS_T)
    out = {name: np.zeros_like(x) for name, x in
           (("dq", qf), ("dk", kf), ("dv", vf), ("dlog_alpha", laf), ("dbeta", bf))}
    dS0 = np.zeros((n_seqs, H, dk, dv))
    for s in range(n_seqs):
        t0, t1 = int(cu[s]), int(cu[s + 1])
        for h in range(H):
            # forward sweep, keeping S_{t-1}, S' and S_t of every token
            S = s0[s, h].copy()
            prev, decayed, after, us, ds = [], [], [], [], []
            for t in range(t0, t1):
                a = np.exp(laf[t, h])
                prev.append(S)
                Sp = a[:, None] * S
                u = Sp.T @ kf[t, h]
                d = bf[t, h] * (vf[t, h] - u)
                S = Sp + np.outer(kf[t, h], d)
                decayed.append(Sp)
                after.append(S)
                us.append(u)
                ds.append(d)
            # reverse sweep
            G = dST[s, h].copy()
            for i in range(t1 - t0 - 1, -1, -1):
                t = t0 + i
                a = np.exp(laf[t, h])
                G = G + np.outer(qf[t, h], dof[t, h])
                out["dq"][t, h] = after[i] @ dof[t, h]
                dkt = G @ ds[i]
                dd = G.T @ kf[t, h]
                out["dbeta"][t, h] = dd @ (vf[t, h] - us[i])
                out["dv"][t, h] = bf[t, h] * dd
                du = -bf[t, h] * dd
                Gp = G + np.outer(kf[t, h], du)
                dkt = dkt + decayed[i] @ du
                out["dk"][t, h] = dkt
                out["dlog_alpha"][t, h] = a * np.sum(Gp * prev[i], axis=1)
                G = a[:, None] * Gp
            dS0[s, h] = G
    shapes = {"dq": q.shape, "dk": k.shape, "dv": v.shape, "dlog_alpha": la.shape, "dbeta": b.shape}
    res = {name: out[name].reshape(shapes[name]) for name in shapes}
    res["dS0"] = dS0
    return res
