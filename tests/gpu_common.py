"""Shared helpers of the GPU parity tests (CUDA path vs the oracle)."""
import numpy as np
import pytest

torch = pytest.importorskip("torch")

from jepa_video_encoder_b200 import synth  # noqa: E402
from oracle import jepa_oracle as orc  # noqa: E402

# f16 / bf16 compute gates on last_hidden_state (per-token cosine of every
# token, and max|a-b| / max|b|), and the quantised-weight gate.
COS_F16 = 0.9999
REL_MAX_F16 = 2e-2
COS_QUANT = 0.9995


def need_cuda():
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")


def dev(x, dtype=None):
    t = torch.from_numpy(np.ascontiguousarray(x))
    if dtype is not None:
        t = t.to(dtype)
    return t.cuda()


def host(t) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_tokens_close(got, ref, cos_min=COS_F16, rel_max=REL_MAX_F16, what=""):
    got = np.asarray(got, np.float64)
    ref = np.asarray(ref, np.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    cos = orc.token_cosines(got, ref)
    rm = orc.rel_max(got, ref)
    assert cos.min() >= cos_min, f"{what}: worst token cosine {cos.min():.6f} (mean {cos.mean():.6f})"
    if rel_max is not None:
        assert rm <= rel_max, f"{what}: rel_max {rm:.3e}"
    return cos, rm


def f16_values(x) -> np.ndarray:
    """The value a float tensor takes once rounded to binary16."""
    return np.asarray(x, np.float32).astype(np.float16).astype(np.float64)
