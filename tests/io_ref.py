"""fp64 definitions of the fused input and output transformations, for the oracle side.

The layer around the operator (blog.gzher.com "Kimi K3论文：Kimi Linear", section 3):
q and k are L2-normalised, beta = Sigmoid(.), the forget gate is alpha = f(z) of a
low-rank projection z (read here as f = sigmoid, so log alpha = log sigmoid(z)), and
the output goes through a head-wise RMSNorm and a sigmoid output gate. These are the
plain formulas, applied in fp64 to the exact values handed to the GPU, so that the
fp64 oracle sees the same transformed inputs and its output can be transformed the
same way.
"""
import numpy as np


def f64(x):
    if hasattr(x, "detach"):
        import torch

        return x.detach().to("cpu", torch.float64).numpy()
    return np.asarray(x, dtype=np.float64)


def log_sigmoid(z):
    """log(1 / (1 + exp(-z))) = -log(1 + exp(-z)), evaluated without overflow."""
    return -np.logaddexp(0.0, -f64(z))


def sigmoid(z):
    return 1.0 / (1.0 + np.exp(-f64(z)))


def l2norm_rows(x, eps):
    """Each row (last axis) divided by sqrt(sum of squares + eps)."""
    x = f64(x)
    return x / np.sqrt(np.sum(x * x, axis=-1, keepdims=True) + eps)


def rmsnorm_gate(o, gate, w, eps):
    """o / sqrt(mean(o^2) + eps) * w * sigmoid(gate) over the last axis."""
    o = f64(o)
    w = np.ones(o.shape[-1]) if w is None else f64(w)
    return o / np.sqrt(np.mean(o * o, axis=-1, keepdims=True) + eps) * w * sigmoid(gate)


def l2norm_rows_bwd(y, dx, eps):
    """Gradient through x = y / sqrt(|y|^2 + eps) (rows on the last axis): for x's
    gradient dx, y's is (dx - x (x . dx)) / sqrt(|y|^2 + eps)."""
    y, dx = f64(y), f64(dx)
    n = np.sqrt(np.sum(y * y, axis=-1, keepdims=True) + eps)
    x = y / n
    return (dx - x * np.sum(x * dx, axis=-1, keepdims=True)) / n
