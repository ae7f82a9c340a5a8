"""Parity metrics and the tolerances the CUDA path must meet against the oracle.

bf16 inputs: relative L2 error <= 1e-2 and max-abs error <= 2e-2 x max|ref|.
fp32 inputs: relative L2 error <= 1e-4.
Both apply to the output o and to the final state S_T.
"""
import numpy as np

TOL = {"bf16": dict(rel_l2=1e-2, max_abs_frac=2e-2), "f32": dict(rel_l2=1e-4, max_abs_frac=None)}


def as_f64(x):
    if hasattr(x, "detach"):
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def errors(x, ref):
    x, ref = as_f64(x), as_f64(ref)
    assert x.shape == ref.shape, (x.shape, ref.shape)
    diff = x - ref
    nref = np.linalg.norm(ref)
    rel = np.linalg.norm(diff) / nref if nref > 0 else np.linalg.norm(diff)
    mx = np.max(np.abs(ref)) if ref.size else 0.0
    return float(rel), float(np.max(np.abs(diff)) if diff.size else 0.0), float(mx)


def check(x, ref, kind, what):
    assert np.all(np.isfinite(as_f64(x))), f"{what}: non-finite values"
    rel, mabs, mx = errors(x, ref)
    tol = TOL[kind]
    assert rel <= tol["rel_l2"], f"{what}: rel-L2 {rel:.3e} > {tol['rel_l2']:.0e}"
    if tol["max_abs_frac"] is not None:
        assert mabs <= tol["max_abs_frac"] * mx, \
            f"{what}: max-abs {mabs:.3e} > {tol['max_abs_frac']:.0e} x {mx:.3e}"
    return rel, mabs


def per_channel_gate(log_alpha, gate, like):
    """The forget gate in the form the oracle takes: fp32 log rates, one per key channel,
    shaped like ``like`` (q). A head-wide rate (Gated DeltaNet) is the same rate on every
    channel, a bf16 gate is widened exactly, and no gate (DeltaNet) is log 1 = 0."""
    import torch

    if gate == "none":
        return torch.zeros(like.shape, dtype=torch.float32, device=like.device)
    if gate == "head":
        return log_alpha[..., None].expand(like.shape).float()
    return log_alpha.float()
