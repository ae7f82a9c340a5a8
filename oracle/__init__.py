"""KDA oracle: plain fp64 CPU recurrence, loaded from ``kda_oracle.c``.

TEST INFRASTRUCTURE ONLY. Only ``tests/``, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this package. The CUDA library
(``gated_delta_rule_101_b200``) never imports or links it, and the two share
no code: the only thing both sides use is the seeded input generator, which
holds none of the method's arithmetic.

``kda_fwd`` runs the recurrence; ``backward.kda_bwd`` gives its gradients (the
reverse pass, plain numpy). What is computed is Kimi Delta Attention's recurrence, eq. (1) of the
blog.gzher.com review "Kimi K3论文：Kimi Linear" (section 3):

    S_t = (I - beta_t k_t k_t^T) Diag(alpha_t) S_{t-1} + beta_t k_t v_t^T,
    o_t = S_t^T q_t,            alpha_t = exp(log_alpha_t).

It is evaluated token by token in fp64 (see the C file for the four steps).
Inputs are the exact values handed to the GPU, widened to fp64.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "kda_oracle.c")
_LIB = os.path.join(_HERE, "_kda_oracle.so")
_lock = threading.Lock()
_cache: dict[str, ctypes.CDLL] = {}


def compile_oracle(src: str = _SRC, out: str = _LIB, defines: tuple[str, ...] = ()) -> str:
    """Compile the C oracle into a shared library with gcc; return its path."""
    cmd = ["gcc", "-O2", "-std=c11", "-D_POSIX_C_SOURCE=200809L", "-shared", "-fPIC",
           *[f"-D{d}" for d in defines], "-o", out, src, "-lpthread", "-lm"]
    subprocess.run(cmd, check=True, capture_output=True, text=True)
    return out


def build() -> str:
    """Build ``_kda_oracle.so`` next to the source if it is missing or stale."""
    with _lock:
        if (not os.path.exists(_LIB)) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
            compile_oracle()
    return _LIB


def _bind(path: str) -> ctypes.CDLL:
    lib = ctypes.CDLL(path)
    dp = ctypes.POINTER(ctypes.c_double)
    lib.kda_oracle_fwd.restype = ctypes.c_int
    lib.kda_oracle_fwd.argtypes = [dp, dp, dp, dp, dp, dp, dp, dp,
                                   ctypes.POINTER(ctypes.c_int64), ctypes.c_int,
                                   ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int]
    lib.kda_oracle_default_threads.restype = ctypes.c_int
    lib.kda_oracle_default_threads.argtypes = []
    return lib


def load(path: str | None = None) -> ctypes.CDLL:
    """Return the ctypes handle of the oracle library (building it if needed)."""
    path = path or build()
    with _lock:
        if path not in _cache:
            _cache[path] = _bind(path)
        return _cache[path]


def default_threads() -> int:
    return int(load().kda_oracle_default_threads())


def _f64(x) -> np.ndarray:
    if x is None:
        return None
    if hasattr(x, "detach"):  # a torch tensor: take its exact values
        x = x.detach().to("cpu")
        import torch  # local: torch is only needed when torch tensors are passed

        x = x.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _ptr(a: np.ndarray | None):
    if a is None:
        return None
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def kda_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None, *, threads: int = 0,
            lib_path: str | None = None):
    """Run the fp64 recurrence.

    Shapes: either batched ``q, k, log_alpha [B, T, H, dk]``, ``v [B, T, H, dv]``,
    ``beta [B, T, H]`` (B sequences of length T), or packed ``[n_tok, H, .]``
    with ``cu_seqlens`` (``n_seqs + 1`` token offsets). ``S0`` is
    ``[n_seqs, H, dk, dv]`` or None (zeros).

    Returns ``(o, S_T)`` in fp64: ``o`` has the layout of ``v``; ``S_T`` is
    ``[n_seqs, H, dk, dv]``.
    """
    q, k, v, la, b = (_f64(t) for t in (q, k, v, log_alpha, beta))
    batched = cu_seqlens is None
    if batched:
        B, T, H, dk = q.shape
        cu = np.arange(B + 1, dtype=np.int64) * T
        lead = (B, T)
    else:
        cu = np.ascontiguousarray(np.asarray(
            cu_seqlens.cpu().numpy() if hasattr(cu_seqlens, "cpu") else cu_seqlens, dtype=np.int64))
        _, H, dk = q.shape
        lead = (q.shape[0],)
    dv = v.shape[-1]
    n_seqs = len(cu) - 1
    s0 = _f64(S0)
    if s0 is not None:
        assert s0.shape == (n_seqs, H, dk, dv), s0.shape
    o = np.empty(lead + (H, dv), dtype=np.float64)
    st = np.empty((n_seqs, H, dk, dv), dtype=np.float64)
    rc = load(lib_path).kda_oracle_fwd(
        _ptr(q), _ptr(k), _ptr(v), _ptr(la), _ptr(b), _ptr(s0), _ptr(o), _ptr(st),
        cu.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), n_seqs, H, dk, dv, int(threads))
    if rc != 0:
        raise RuntimeError(f"kda_oracle_fwd failed with status {rc}")
    return o, st
