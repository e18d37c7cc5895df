"""Fit of the GELU polynomial used by the CUDA kernels (common.cuh, gelu_q).

GELU(x) = x * Phi(x) = max(x, 0) - |x| * Phi(-|x|), and Phi(-u) = 2^q(u).
q is a degree-11 polynomial in u on [0, 6] with q(0) = -1 (Phi(0) = 1/2),
fitted to log2 Phi(-u) by least squares on Chebyshev nodes whose weights are
raised where the residual is large (iteratively reweighted least squares,
which drives the error toward equal ripple).  Running this file prints the
coefficients q_0 .. q_11 rounded to f32.
"""
import numpy as np
from scipy.special import log_ndtr

DEGREE = 11
UMAX = 6.0


def fit(n_nodes=6000, iters=40):
    u = UMAX * (1.0 - np.cos(np.pi * (np.arange(n_nodes) + 0.5) / n_nodes)) / 2.0
    target = log_ndtr(-u) / np.log(2.0) + 1.0  # q(u) - q(0)
    basis = np.stack([u ** k for k in range(1, DEGREE + 1)], axis=1)
    w = np.ones_like(u)
    for _ in range(iters):
        c, *_ = np.linalg.lstsq(basis * w[:, None], target * w, rcond=None)
        r = np.abs(basis @ c - target)
        w = w * (r / r.max() + 0.05)
        w /= w.max()
    return np.concatenate([[-1.0], c]).astype(np.float32)


if __name__ == "__main__":
    print(", ".join("%.9ef" % v for v in fit()))
