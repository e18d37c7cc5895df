"""The allocation-free mean pooling entry point.

Some callers cannot call cudaMalloc: serving loops that run under a fixed
device-memory budget, code that must never stall the device (cudaMalloc may
synchronise it), and hosts whose device allocator belongs to another
framework.  jepa_b200_op_mean_pool_noalloc serves them with a fixed device
array instead of a grown buffer.  These tests check it against the
allocating entry point (jepa_b200_op_mean_pool) on two calls in a row, with
different inputs, and that oversized requests are refused before any device
work.  This file is collected last on purpose."""
import ctypes

import numpy as np
import pytest

from jepa_video_encoder_b200 import _abi, build


def _lib():
    build.build()
    return _abi.load_library()


def test_noalloc_rejects_sizes_beyond_its_array():
    lib = _lib()
    # B * D = 4 * 16384 > 32768: refused on the host, no device touched
    assert lib.jepa_b200_op_mean_pool_noalloc(ctypes.c_void_p(16), 4, 10, 16384, 0, ctypes.c_void_p(16),
                                              None) == _abi.ERR_SHAPE
    assert lib.jepa_b200_op_mean_pool_noalloc(None, 1, 10, 64, 0, None, None) == _abi.ERR_ARG


@pytest.mark.gpu
def test_noalloc_mean_pool_matches_allocating_entry_point():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("needs a CUDA device")
    import jepa_video_encoder_b200 as jb
    lib = _lib()
    rng = np.random.default_rng(2024)
    # two calls in a row, the second smaller, with different data
    for B, N, D, first in ((8, 3137, 1024, 1), (3, 2048, 1024, 0)):
        y = rng.standard_normal((B, N, D)).astype(np.float32)
        yd = torch.from_numpy(y).cuda()
        ref = torch.empty((B, D), dtype=torch.float32, device="cuda")
        got = torch.full((B, D), float("nan"), dtype=torch.float32, device="cuda")
        jb.mean_pool(yd, B, N, D, first, ref)
        st = lib.jepa_b200_op_mean_pool_noalloc(yd.data_ptr(), B, N, D, first, got.data_ptr(),
                                                torch.cuda.current_stream().cuda_stream)
        assert st == _abi.OK
        assert jb.op_sync_status() == 0
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        assert np.isfinite(g).all()
        # same tolerance as the mean-pool parity test, against both the
        # allocating entry point and the float64 mean
        assert np.abs(g - r).max() <= 1e-5
        assert np.abs(g - y[:, first:].astype(np.float64).mean(1)).max() <= 1e-5
