"""Pins for the fp64 oracle: checks against what the pages and the mathematics fix.

Each ``pin_*`` function takes ``fwd`` (a callable with the signature of
``oracle.kda_fwd``) and raises AssertionError when the oracle disagrees with
an independent computation. None of them re-runs the oracle's own loop:

* hand-worked values (tests/golden/kda_handworked.txt);
* explicit products of the dk x dk transition matrices written in the DPLR
  form of the blog.gzher.com review "Kimi K3论文：Kimi Linear", section 4;
* DeltaNet as online gradient descent on 1/2 ||S^T k - v||^2 (section 2),
  with the gradient taken by autograd, not written out;
* Gated DeltaNet's scalar-gate form (section 2);
* closed forms for beta = 0 (pure decay) and alpha = 0 (state reset);
* the delta-rule write identity S_t^T k_t = (1 - beta|k|^2) u + beta|k|^2 v;
* invariances: state carry across a split, linearity in (S0, V), column
  permutation equivariance, packed varlen = separate sequences;
* the chunked form of the mokono.cn explainer (section 2.1, S_r = P_r S_0 + H_r),
  evaluated in ``chunked_form``.

The same pins run against oracle builds with planted mistakes
(test_oracle_mutants.py) to show that each mistake is caught.
"""
from __future__ import annotations

import math
import os
from fractions import Fraction

import numpy as np

from chunked_form import kda_chunked_fp64, kda_proposition_fp64

GOLDEN = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden", "kda_handworked.txt")


def rand_case(seed, *, B=2, T=37, H=2, dk=16, dv=40, la_range=(0.001, 0.1), s0_std=0.3,
              unit=True, beta=None):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((B, T, H, dk))
    k = rng.standard_normal((B, T, H, dk))
    if unit:
        q /= np.linalg.norm(q, axis=-1, keepdims=True)
        k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal((B, T, H, dv))
    lo, hi = la_range
    la = -rng.uniform(lo, hi, (B, T, H, dk))
    b = 1.0 / (1.0 + np.exp(-rng.standard_normal((B, T, H)))) if beta is None else np.full((B, T, H), beta)
    S0 = s0_std * rng.standard_normal((B, H, dk, dv))
    return dict(q=q, k=k, v=v, log_alpha=la, beta=b, S0=S0)


def _close(a, b, tol, what):
    a = np.asarray(a, dtype=np.float64)
    b = np.asarray(b, dtype=np.float64)
    assert a.shape == b.shape, (what, a.shape, b.shape)
    err = np.max(np.abs(a - b)) if a.size else 0.0
    scale = max(1.0, np.max(np.abs(b)) if b.size else 0.0)
    assert err <= tol * scale, f"{what}: max abs err {err:.3e} > {tol:.1e} x {scale:.3e}"


# --------------------------------------------------------------------------
def _parse_golden(path=GOLDEN):
    cases, cur = [], None
    for raw in open(path, encoding="utf-8"):
        line = raw.split("#", 1)[0].strip()
        if not line:
            continue
        tok = line.split()
        if tok[0] == "case":
            cur = dict(name=tok[1], steps=[], o=[])
            cases.append(cur)
        elif tok[0] in ("dk", "dv"):
            cur[tok[0]] = int(tok[1])
        elif tok[0] in ("S0", "ST"):
            cur[tok[0]] = [float(x) for x in tok[1:]]
        elif tok[0] == "o":
            cur["o"].append([float(x) for x in tok[1:]])
        elif tok[0] == "t":
            st, key = {}, None
            for x in tok[1:]:
                if x in ("k", "v", "beta", "alpha", "q"):
                    key = x
                    st[key] = []
                else:
                    st[key].append(float(Fraction(x)))
            cur["steps"].append(st)
    return cases


def pin_golden(fwd):
    """Values worked by hand from eq. (1) (tests/golden/kda_handworked.txt)."""
    for c in _parse_golden():
        dk, dv, T = c["dk"], c["dv"], len(c["steps"])
        arr = lambda key, d: np.array([s[key] for s in c["steps"]]).reshape(1, T, 1, d)
        q, k, v = arr("q", dk), arr("k", dk), arr("v", dv)
        la = np.log(arr("alpha", dk))
        b = np.array([s["beta"][0] for s in c["steps"]]).reshape(1, T, 1)
        S0 = np.array(c["S0"]).reshape(1, 1, dk, dv)
        o, st = fwd(q, k, v, la, b, S0)
        _close(o.reshape(T, dv), np.array(c["o"]), 1e-12, f"golden {c['name']} o")
        _close(st.reshape(-1), np.array(c["ST"]), 1e-12, f"golden {c['name']} S_T")


def pin_transition_product(fwd):
    """Explicit products of the DPLR-form transition matrices, tiny T."""
    for seed, (dk, dv, T) in enumerate([(4, 3, 6), (8, 5, 8), (128, 4, 5)]):
        c = rand_case(100 + seed, B=1, T=T, H=1, dk=dk, dv=dv, la_range=(0.05, 0.7))
        o, st = fwd(**c)
        q, k, v = c["q"][0, :, 0], c["k"][0, :, 0], c["v"][0, :, 0]
        alpha, b, S0 = np.exp(c["log_alpha"][0, :, 0]), c["beta"][0, :, 0], c["S0"][0, 0]
        # section 4: S_t = (Diag(alpha_t) - beta_t k_t (k_t*alpha_t)^T) S_{t-1} + beta_t k_t v_t^T
        M = [np.diag(alpha[t]) - b[t] * np.outer(k[t], k[t] * alpha[t]) for t in range(T)]

        def prod(lo, hi):  # M_hi ... M_lo  (identity when empty)
            P = np.eye(dk)
            for t in range(lo, hi + 1):
                P = M[t] @ P
            return P

        for t in range(T):
            S_t = prod(0, t) @ S0 + sum(prod(i + 1, t) @ (b[i] * np.outer(k[i], v[i])) for i in range(t + 1))
            _close(o[0, t, 0], S_t.T @ q[t], 1e-12, f"transition product o[{t}] dk={dk}")
        _close(st[0, 0], S_t, 1e-12, f"transition product S_T dk={dk}")


def pin_deltanet_gradient_step(fwd):
    """alpha = 1: each step is one SGD step of rate beta on 1/2 ||S^T k - v||^2 (section 2)."""
    import torch

    c = rand_case(7, B=1, T=12, H=1, dk=16, dv=6)
    c["log_alpha"][:] = 0.0
    o, st = fwd(**c)
    S = torch.tensor(c["S0"][0, 0], dtype=torch.float64)
    for t in range(12):
        kt = torch.tensor(c["k"][0, t, 0])
        vt = torch.tensor(c["v"][0, t, 0])
        qt = torch.tensor(c["q"][0, t, 0])
        Sv = S.clone().requires_grad_(True)
        loss = 0.5 * ((Sv.T @ kt - vt) ** 2).sum()
        (grad,) = torch.autograd.grad(loss, Sv)
        S = (S - float(c["beta"][0, t, 0]) * grad).detach()
        _close(o[0, t, 0], (S.T @ qt).numpy(), 1e-12, f"deltanet o[{t}]")
    _close(st[0, 0], S.numpy(), 1e-12, "deltanet S_T")


def pin_gdn_scalar_gate(fwd):
    """alpha equal across channels: S_t = alpha_t (I - beta k k^T) S_{t-1} + beta k v^T (section 2)."""
    c = rand_case(11, B=1, T=15, H=1, dk=12, dv=7)
    rng = np.random.default_rng(12)
    a_scalar = -rng.uniform(0.01, 0.5, size=15)
    c["log_alpha"][0, :, 0, :] = a_scalar[:, None]
    o, st = fwd(**c)
    S = c["S0"][0, 0].copy()
    dk = 12
    for t in range(15):
        k, v, q, b = c["k"][0, t, 0], c["v"][0, t, 0], c["q"][0, t, 0], c["beta"][0, t, 0]
        S = math.exp(a_scalar[t]) * (np.eye(dk) - b * np.outer(k, k)) @ S + b * np.outer(k, v)
        _close(o[0, t, 0], S.T @ q, 1e-12, f"gdn o[{t}]")
    _close(st[0, 0], S, 1e-12, "gdn S_T")


def pin_pure_decay(fwd):
    """beta = 0: S_t = Diag(prod_s alpha_s) S0 and o_t = S0^T (exp(sum log_alpha) * q_t)."""
    c = rand_case(13, B=2, T=20, H=2, dk=16, dv=40, beta=0.0)
    o, st = fwd(**c)
    G = np.cumsum(c["log_alpha"], axis=1)  # [B, T, H, dk]
    want_o = np.einsum("bthc,bhcj->bthj", np.exp(G) * c["q"], c["S0"])
    _close(o, want_o, 1e-12, "pure decay o")
    _close(st, np.exp(G[:, -1])[..., None] * c["S0"], 1e-12, "pure decay S_T")


def pin_alpha_zero(fwd):
    """alpha = 0 (log_alpha = -1e4): S_t = beta_t k_t v_t^T, o_t = beta_t (k_t . q_t) v_t."""
    c = rand_case(17, B=2, T=9, H=2, dk=16, dv=40)
    c["log_alpha"][:] = -1e4
    o, st = fwd(**c)
    b = c["beta"][..., None]
    want_o = b * np.sum(c["k"] * c["q"], axis=-1, keepdims=True) * c["v"]
    _close(o, want_o, 1e-12, "alpha=0 o")
    want_st = c["beta"][:, -1, :, None, None] * np.einsum("bhc,bhj->bhcj", c["k"][:, -1], c["v"][:, -1])
    _close(st, want_st, 1e-12, "alpha=0 S_T")


def pin_write_identity(fwd):
    """beta = 1, |k| = 1, q = k gives o = v; in general S^T k = (1-b|k|^2) u + b|k|^2 v."""
    c = rand_case(19, B=1, T=10, H=2, dk=16, dv=40, beta=1.0)
    c["q"] = c["k"].copy()
    o, _ = fwd(**c)
    _close(o, c["v"], 1e-12, "write identity o = v")
    # one step, non-unit k, random beta: u = (Diag(alpha) S0)^T k
    c = rand_case(23, B=1, T=1, H=1, dk=16, dv=40, unit=False)
    c["q"] = c["k"].copy()
    o, _ = fwd(**c)
    k, v, b = c["k"][0, 0, 0], c["v"][0, 0, 0], c["beta"][0, 0, 0]
    u = (np.exp(c["log_alpha"][0, 0, 0])[:, None] * c["S0"][0, 0]).T @ k
    kk = float(k @ k)
    _close(o[0, 0, 0], (1 - b * kk) * u + b * kk * v, 1e-12, "write identity general")


def pin_state_carry(fwd):
    """Splitting a sequence anywhere and passing S_T on as S0 changes nothing."""
    c = rand_case(29, B=2, T=50, H=2, dk=16, dv=40)
    o, st = fwd(**c)
    cuts = [0, 1, 17, 33, 34, 50]
    S = c["S0"]
    for a, z in zip(cuts[:-1], cuts[1:]):
        part = {key: (val[:, a:z] if key != "S0" else S) for key, val in c.items()}
        o_p, S = fwd(**part)
        _close(o_p, o[:, a:z], 1e-12, f"state carry o[{a}:{z}]")
    _close(S, st, 1e-12, "state carry S_T")


def pin_linearity(fwd):
    """(o, S_T) is linear in the pair (S0, V) jointly."""
    c1 = rand_case(31, B=1, T=25, H=2, dk=16, dv=40)
    c2 = rand_case(37, B=1, T=25, H=2, dk=16, dv=40)
    for key in ("q", "k", "log_alpha", "beta"):
        c2[key] = c1[key]
    a, b = 0.75, -1.5
    o1, s1 = fwd(**c1)
    o2, s2 = fwd(**c2)
    c3 = dict(c1, v=a * c1["v"] + b * c2["v"], S0=a * c1["S0"] + b * c2["S0"])
    o3, s3 = fwd(**c3)
    _close(o3, a * o1 + b * o2, 1e-12, "linearity o")
    _close(s3, a * s1 + b * s2, 1e-12, "linearity S_T")


def pin_column_permutation(fwd):
    """Permuting the value columns of V and S0 permutes o and S_T the same way."""
    c = rand_case(41, B=1, T=21, H=2, dk=16, dv=40)
    perm = np.random.default_rng(43).permutation(40)
    o, st = fwd(**c)
    cp = dict(c, v=c["v"][..., perm], S0=c["S0"][..., perm])
    op, sp = fwd(**cp)
    _close(op, o[..., perm], 1e-13, "column permutation o")
    _close(sp, st[..., perm], 1e-13, "column permutation S_T")


def pin_varlen_equals_separate(fwd):
    """Packed sequences with offsets give the same result as separate calls."""
    lens = [5, 0, 23, 1, 64, 17]
    rng = np.random.default_rng(47)
    parts = [rand_case(int(rng.integers(1 << 30)), B=1, T=max(n, 1), H=2, dk=16, dv=40) for n in lens]
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int64)
    packed = {key: np.concatenate([p[key][0, :n] for p, n in zip(parts, lens)], axis=0)
              for key in ("q", "k", "v", "log_alpha", "beta")}
    S0 = np.stack([p["S0"][0] for p in parts])
    o, st = fwd(**packed, S0=S0, cu_seqlens=cu)
    for i, (p, n) in enumerate(zip(parts, lens)):
        if n == 0:
            _close(st[i], S0[i], 0.0, "empty sequence keeps S0")
            continue
        sub = {key: (val[:, :n] if key != "S0" else val) for key, val in p.items()}
        o_i, s_i = fwd(**sub)
        _close(o[cu[i]:cu[i + 1]], o_i[0], 1e-13, f"varlen o seq {i}")
        _close(st[i], s_i[0], 1e-13, f"varlen S_T seq {i}")


def pin_chunked_form(fwd):
    """The chunked form (Proposition: S_r = P_r S_0 + H_r; WY/UT matrix form) equals the recurrence."""
    for C, T in ((64, 150), (16, 37), (32, 100), (128, 300)):
        c = rand_case(53 + C, B=2, T=T, H=2, dk=32, dv=40, la_range=(0.001, 0.3))
        o, st = fwd(**c)
        o_c, st_c = kda_chunked_fp64(**c, C=C)
        _close(o_c, o, 1e-10, f"UT chunked form o (C={C})")
        _close(st_c, st, 1e-10, f"UT chunked form S_T (C={C})")
    c = rand_case(59, B=1, T=21, H=1, dk=8, dv=5, la_range=(0.01, 0.5))
    o, st = fwd(**c)
    o_p, st_p = kda_proposition_fp64(**c, C=8)
    _close(o_p, o, 1e-11, "proposition P_r/H_r form o")
    _close(st_p, st, 1e-11, "proposition P_r/H_r form S_T")


ALL_PINS = [pin_golden, pin_transition_product, pin_deltanet_gradient_step, pin_gdn_scalar_gate,
            pin_pure_decay, pin_alpha_zero, pin_write_identity, pin_state_carry, pin_linearity,
            pin_column_permutation, pin_varlen_equals_separate, pin_chunked_form]
