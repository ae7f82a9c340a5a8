"""Pins of the reverse-pass oracle (oracle/backward.py), no GPU needed.

Its gradients are checked against things other than its own derivation:
* reverse-mode automatic differentiation (torch.autograd) of a plain fp64 PyTorch
  recurrence written here from eq. (1) (blog.gzher.com "Kimi K3论文：Kimi Linear",
  section 3), batched and packed with an empty sequence;
* central finite differences of the C forward oracle in random directions;
* beta = 0: the state never sees k or v, so their gradients vanish;
* planted mistakes: each plausible slip in a copy of the reverse pass fails the
  autograd pin.
"""
import numpy as np
import pytest
import torch

import oracle
from oracle import backward
from oracle.backward import kda_bwd


def _case(seed, lead, H=2, dk=6, dv=5, n_seqs=None, la_range=(0.05, 0.8)):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal(lead + (H, dk))
    k = rng.standard_normal(lead + (H, dk))
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = rng.standard_normal(lead + (H, dv))
    la = -rng.uniform(*la_range, size=lead + (H, dk))
    beta = rng.uniform(0.1, 0.9, size=lead + (H,))
    n = lead[0] if n_seqs is None else n_seqs
    S0 = 0.5 * rng.standard_normal((n, H, dk, dv))
    do = rng.standard_normal(lead + (H, dv))
    dST = rng.standard_normal((n, H, dk, dv))
    return q, k, v, la, beta, S0, do, dST


def _autograd(q, k, v, la, beta, S0, do, dST, cu):
    """Gradients of sum(o do) + sum(S_T dS_T) by torch.autograd of the recurrence."""
    T = lambda x: torch.tensor(x, dtype=torch.float64, requires_grad=True)
    tq, tk, tv, tla, tb, tS0 = (T(x) for x in (q, k, v, la, beta, S0))
    H = q.shape[-2]
    loss = torch.zeros((), dtype=torch.float64)
    for s in range(len(cu) - 1):
        for h in range(H):
            S = tS0[s, h]
            for t in range(cu[s], cu[s + 1]):
                S = torch.exp(tla[t, h])[:, None] * S                      # decay
                u = S.T @ tk[t, h]                                         # recall
                S = S + torch.outer(tk[t, h], tb[t, h] * (tv[t, h] - u))   # delta write
                loss = loss + (S.T @ tq[t, h]) @ torch.from_numpy(do[t, h])
            loss = loss + (S * torch.from_numpy(dST[s, h])).sum()
    grads = torch.autograd.grad(loss, (tq, tk, tv, tla, tb, tS0))
    return dict(zip(("dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"), (g.numpy() for g in grads)))


def _assert_close(got, want, tol, what):
    for name in want:
        err = np.max(np.abs(got[name] - want[name]))
        scale = max(np.max(np.abs(want[name])), 1e-30)
        assert err <= tol * scale, f"{what} {name}: max-abs {err:.3e} vs scale {scale:.3e}"


def _packed(seed, lengths, **kw):
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int64)
    c = _case(seed, (int(cu[-1]),), n_seqs=len(lengths), **kw)
    return c, cu


def test_backward_equals_autograd_batched():
    B, T = 2, 13
    c = _case(1, (B, T))
    flat = tuple(x.reshape((-1,) + x.shape[2:]) for x in c[:5]) + (c[5], c[6].reshape((-1,) + c[6].shape[2:]), c[7])
    want = _autograd(*flat, np.arange(B + 1) * T)
    got = kda_bwd(*c)
    got = {k: (v.reshape(want[k].shape)) for k, v in got.items()}
    _assert_close(got, want, 1e-10, "batched")


def test_backward_equals_autograd_packed_with_an_empty_sequence():
    c, cu = _packed(2, [3, 0, 7, 1])
    want = _autograd(*c, cu)
    got = kda_bwd(*c, cu_seqlens=cu)
    _assert_close(got, want, 1e-10, "packed")
    assert np.array_equal(got["dS0"][1], c[7][1])  # empty sequence: dS0 = dS_T


def test_backward_matches_finite_differences_of_the_forward_oracle():
    B, T, H, dk, dv = 1, 5, 1, 4, 3
    q, k, v, la, beta, S0, do, dST = _case(3, (B, T), H=H, dk=dk, dv=dv)
    g = kda_bwd(q, k, v, la, beta, S0, do, dST)

    def loss(args):
        o, st = oracle.kda_fwd(*args)
        return float(np.sum(o * do) + np.sum(st * dST))

    base = [q, k, v, la, beta, S0]
    names = ["dq", "dk", "dv", "dlog_alpha", "dbeta", "dS0"]
    rng = np.random.default_rng(4)
    eps = 1e-6
    for i, name in enumerate(names):
        for _ in range(3):
            d = rng.standard_normal(base[i].shape)
            plus = [x.copy() for x in base]
            minus = [x.copy() for x in base]
            plus[i] = plus[i] + eps * d
            minus[i] = minus[i] - eps * d
            fd = (loss(plus) - loss(minus)) / (2 * eps)
            an = float(np.sum(g[name] * d))
            assert abs(fd - an) <= 1e-6 * max(1.0, abs(an)), f"{name}: fd {fd:.9g} vs {an:.9g}"


def test_beta_zero_makes_k_and_v_irrelevant():
    c = list(_case(5, (2, 9)))
    c[4] = np.zeros_like(c[4])
    g = kda_bwd(*c)
    assert np.all(g["dk"] == 0) and np.all(g["dv"] == 0)
    assert np.any(g["dbeta"] != 0)  # the write strength still matters


MUTANTS = [
    ("dkt = dkt + decayed[i] @ du", "dkt = dkt"),                                  # recall term dropped
    ("np.sum(Gp * prev[i], axis=1)", "np.sum(Gp * after[i], axis=1)"),             # wrong state
    ("du = -bf[t, h] * dd", "du = bf[t, h] * dd"),                                 # sign
    ("a * np.sum(Gp * prev[i], axis=1)", "np.sum(Gp * prev[i], axis=1)"),          # chain rule of exp
    ("G = G + np.outer(qf[t, h], dof[t, h])", "G = G + np.outer(kf[t, h], dof[t, h])"),  # q for k
    ("G = a[:, None] * Gp", "G = Gp"),                                             # decay not applied
    ("out[\"dq\"][t, h] = after[i] @ dof[t, h]", "out[\"dq\"][t, h] = decayed[i] @ dof[t, h]"),  # read before write
]


@pytest.mark.parametrize("old,new", MUTANTS)
def test_each_planted_mistake_fails_the_autograd_pin(old, new):
    import inspect
    import types

    src = inspect.getsource(backward)
    assert src.count(old) == 1, old
    mod = types.ModuleType("backward_mutant")
    mod.__dict__["_f64"] = oracle._f64
    exec(compile(src.replace(old, new).replace("from . import _f64", ""), "<mutant>", "exec"), mod.__dict__)
    c, cu = _packed(6, [4, 6])
    want = _autograd(*c, cu)
    got = mod.kda_bwd(*c, cu_seqlens=cu)
    with pytest.raises(AssertionError):
        _assert_close(got, want, 1e-10, "mutant")


@pytest.mark.parametrize("C", [1, 16, 64])
@pytest.mark.parametrize("la_range", [(0.05, 0.5), (2.0, 6.0)])
def test_chunked_backward_equals_the_reverse_pass_oracle(C, la_range):
    """The chunk algebra's reverse pass (tests/chunked_backward.py, the blueprint of a
    chunked backward) reproduces the token-by-token gradients, ragged last chunk and
    strong decay included."""
    from chunked_backward import kda_chunked_bwd_fp64

    c = _case(7, (2, 37), dk=8, dv=5, la_range=la_range)
    want = kda_bwd(*c)
    got = kda_chunked_bwd_fp64(*c, C=C)
    _assert_close(got, want, 1e-10, f"chunked C={C}")
