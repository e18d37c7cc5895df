"""The Python binding's argument checks, on the CPU: tensors that the library
would read as device memory (host tensors, wrong dtype, strided views, wrong
shape) are refused before any library call."""
import pytest
import torch

import jepa_video_encoder_b200 as jb
from jepa_video_encoder_b200 import synth

CFG = synth.small_config(synth.LEVJEPA_VIT_L, frames=2, batch=2)
SHAPE = (2, CFG.frames, 3, CFG.img_h, CFG.img_w)
assert CFG.img_h == CFG.img_w


def test_check_pixels_accepts_the_workload_shape():
    assert jb.check_pixels(CFG, torch.zeros(SHAPE), on_cuda=False) == 2
    assert jb.check_pixels(CFG, torch.zeros((1,) + SHAPE[1:]), on_cuda=False) == 1


@pytest.mark.parametrize("bad", [
    torch.zeros(SHAPE, dtype=torch.float16),                        # dtype
    torch.zeros(SHAPE, dtype=torch.float64),
    torch.zeros(SHAPE[:1] + (SHAPE[1] + 1,) + SHAPE[2:]),           # frames
    torch.zeros(SHAPE[:3] + (SHAPE[3], SHAPE[4] + 16)),             # width
    torch.zeros((0,) + SHAPE[1:]),                                  # empty batch
    torch.zeros(SHAPE[1:]),                                         # no batch axis
    torch.zeros(SHAPE).transpose(3, 4),                             # strided view (H = W)
])
def test_check_pixels_refuses(bad):
    with pytest.raises(ValueError):
        jb.check_pixels(CFG, bad, on_cuda=False)


def test_check_pixels_refuses_the_wrong_side():
    with pytest.raises(ValueError):
        jb.check_pixels(CFG, torch.zeros(SHAPE), on_cuda=True, device=0)   # host tensor for encode
    with pytest.raises(TypeError):
        jb.check_pixels(CFG, [0.0], on_cuda=False)


def test_check_out():
    jb.check_out(torch.zeros(4, 8), on_cuda=False)
    for bad in (torch.zeros(4, 8, dtype=torch.float16), torch.zeros(8, 4).t()):
        with pytest.raises(ValueError):
            jb.check_out(bad, on_cuda=False)
    with pytest.raises(ValueError):
        jb.check_out(torch.zeros(4, 8), on_cuda=True, device=0)


def test_model_encode_checks_before_the_library():
    """encode / encode_host / debug_stage validate their tensors before the
    handle is used (a Model shell without a loaded handle shows it)."""
    m = object.__new__(jb.Model)
    m.cfg, m.device, m._h = CFG, 0, None
    with pytest.raises(ValueError):
        m.encode(torch.zeros(SHAPE), pool="cls")                 # a host tensor
    with pytest.raises(ValueError):
        m.debug_stage(torch.zeros(SHAPE), 1)
    with pytest.raises(ValueError):
        m.encode_host(torch.zeros(SHAPE, dtype=torch.float16), pool="cls")


def test_op_wrappers_refuse_host_tensors():
    x = torch.zeros(4, 64)
    with pytest.raises(ValueError):
        jb.layernorm(x, torch.ones(64), torch.zeros(64), 1e-6, torch.zeros(4, 64))
    with pytest.raises(ValueError):
        jb.mean_pool(x, 1, 4, 64, 0, torch.zeros(1, 64))
    with pytest.raises(ValueError):
        jb.linear(torch.zeros(4, 64, dtype=torch.float16), torch.zeros(128, 64, dtype=torch.float16),
                  synth.DT_F16, 128, None, 0, torch.zeros(4, 128))


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """Without the built library nothing computes: loading it raises with the
    build command instead of falling back to anything."""
    from jepa_video_encoder_b200 import _abi
    monkeypatch.setattr(_abi, "_lib", None)
    with pytest.raises(RuntimeError, match="missing"):
        _abi.load_library(str(tmp_path / "libjepa_b200.so"))
