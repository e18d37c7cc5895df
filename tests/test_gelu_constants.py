"""The GELU polynomial compiled into the CUDA kernels, checked on the host.

The kernels evaluate GELU(x) = max(x, 0) - |x| * 2^q(min(|x|, 6)) with q a
degree-11 polynomial (common.cuh, gelu_q).  These tests read the coefficients
out of the source, evaluate them the way the kernel does (f32 Horner with
fused multiply-add, then 2^q), and compare with x * Phi(x) from scipy's
normal CDF, so that a mistyped or reordered coefficient fails here, without
a GPU.
"""
import importlib.util
import pathlib
import re

import numpy as np
from scipy.special import ndtr

CSRC = pathlib.Path(__file__).resolve().parents[1] / "jepa_video_encoder_b200" / "csrc"


def kernel_coefficients():
    src = (CSRC / "common.cuh").read_text()
    body = re.search(r"float gelu_q\(int k\)\s*\{\s*constexpr float c\[12\]\s*=\s*\{([^}]*)\}", src)
    assert body, "gelu_q table not found in common.cuh"
    vals = [float(t.strip().rstrip("f")) for t in body.group(1).split(",") if t.strip()]
    assert len(vals) == 12
    return np.array(vals, dtype=np.float32)


def gelu_as_kernel(x, c):
    x = np.asarray(x, dtype=np.float32)
    u = np.abs(x)
    cu = np.minimum(u, np.float32(6.0)).astype(np.float64)
    q = np.full(x.shape, np.float64(c[11]))
    for k in range(10, -1, -1):  # one rounding to f32 per fused multiply-add
        q = (q * cu + np.float64(c[k])).astype(np.float32).astype(np.float64)
    e = np.exp2(q)
    return np.maximum(x, 0).astype(np.float64) - u.astype(np.float64) * e


def test_gelu_polynomial_accuracy():
    c = kernel_coefficients()
    x = np.linspace(-8.0, 8.0, 400001).astype(np.float32).astype(np.float64)  # the kernel's inputs are f32
    ref = x * ndtr(x)
    err = np.abs(gelu_as_kernel(x, c) - ref)
    assert err.max() < 1e-7, err.max()


def test_gelu_special_values():
    c = kernel_coefficients()
    assert c[0] == np.float32(-1.0)  # Phi(0) = 1/2 exactly
    g = gelu_as_kernel(np.array([0.0, 1.0, -1.0, 3.0, -3.0, 20.0, -20.0]), c)
    ref = np.array([0.0, ndtr(1.0), -ndtr(-1.0), 3 * ndtr(3.0), -3 * ndtr(-3.0), 20.0, 0.0])
    assert np.abs(g - ref).max() < 1e-7
    # large negative inputs: below half the smallest f16 subnormal
    assert np.abs(gelu_as_kernel(np.array([-6.5, -10.0, -29.0]), c)).max() < 2.98e-8


def test_gelu_fit_reproduces_kernel_table():
    spec = importlib.util.spec_from_file_location("gelu_fit", CSRC / "gelu_fit.py")
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    fitted = mod.fit()
    c = kernel_coefficients()
    np.testing.assert_allclose(fitted, c, rtol=1e-5, atol=1e-12)


def test_gemm_constant_pairs_match_kernel_table():
    """The quantised-weight GEMMs evaluate the same polynomial from a table of
    coefficient pairs in constant memory (gemm.cu, kGeluPairs): both entries
    of every pair equal gelu_q's coefficient of the same degree."""
    src = (CSRC / "gemm.cu").read_text()
    body = re.search(r"__constant__ float2 kGeluPairs\[12\]\s*=\s*\{(.*?)\};", src, re.S)
    assert body, "kGeluPairs not found in gemm.cu"
    pairs = re.findall(r"\{\s*([^,{}]+?)f?\s*,\s*([^,{}]+?)f?\s*\}", body.group(1))
    assert len(pairs) == 12
    got = np.array([[float(a.rstrip("f")), float(b.rstrip("f"))] for a, b in pairs], dtype=np.float32)
    c = kernel_coefficients()
    assert np.array_equal(got[:, 0], c) and np.array_equal(got[:, 1], c)
