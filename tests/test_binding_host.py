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


def test_check_tokens():
    """The predictor's input must be [B, N, dim] of the loaded encoder: the
    library reads B * N * dim values through the pointer."""
    cfg = CFG
    good = torch.zeros((2, cfg.n_tokens, cfg.dim))
    assert jb.check_tokens(cfg, good, on_cuda=False) == 2
    for bad in (torch.zeros((2, cfg.n_tokens - 1, cfg.dim)),     # fewer tokens than the encoder's
                torch.zeros((2, cfg.n_tokens, cfg.dim + 64)),     # another width
                torch.zeros((0, cfg.n_tokens, cfg.dim)),          # empty batch
                torch.zeros((cfg.n_tokens, cfg.dim)),             # no batch axis
                torch.zeros((2, cfg.n_tokens, cfg.dim), dtype=torch.float16),
                torch.zeros((2, cfg.dim, cfg.n_tokens)).transpose(1, 2)):   # strided view
        with pytest.raises(ValueError):
            jb.check_tokens(cfg, bad, on_cuda=False)
    with pytest.raises(ValueError):
        jb.check_tokens(cfg, good, on_cuda=True, device=0)        # a host tensor where a device one is due


def test_check_world_model_inputs():
    """States [C, T, dim] and actions [C, T, A] for a predictor call, or
    [C, T + steps - 1, A] for a rollout: the library reads exactly those
    rows through the pointers."""
    wc = synth.LEWM_WM_STEP
    D, A = wc.dim, wc.action_dim
    st, ac = torch.zeros((5, 3, D)), torch.zeros((5, 3, A))
    assert jb.check_world_model_inputs(wc, st, ac, 0, on_cuda=False) == (5, 3)
    assert jb.check_world_model_inputs(wc, st[:, :1].contiguous(), torch.zeros((5, 20, A)), 20,
                                       on_cuda=False) == (5, 1)
    bad = [(st, torch.zeros((5, 2, A)), 0),            # fewer action rows than frames
           (st, torch.zeros((4, 3, A)), 0),            # candidates differ
           (st, torch.zeros((5, 3, A + 1)), 0),        # another action width
           (torch.zeros((5, 3, D + 64)), ac, 0),       # another state width
           (torch.zeros((0, 3, D)), torch.zeros((0, 3, A)), 0),   # no candidates
           (torch.zeros((5, 0, D)), torch.zeros((5, 0, A)), 0),   # no frames
           (st, ac, 2),                                # a 2-step rollout from 3 frames reads 4 action rows
           (st, ac, -1),
           (st, ac.to(torch.float16), 0)]
    for s_, a_, steps in bad:
        with pytest.raises(ValueError):
            jb.check_world_model_inputs(wc, s_, a_, steps, on_cuda=False)


def test_single_op_operand_sizes():
    """The single-op wrappers check each operand's bytes against what the
    call's dimensions address before handing the pointer over: a short
    tensor is refused on the host (here before the device check)."""
    with pytest.raises(ValueError, match="holds 40 bytes"):
        jb._buf(torch.zeros(10), 41, "x")
    with pytest.raises(ValueError, match="contiguous"):
        jb._buf(torch.zeros((4, 4)).t(), 4, "x")
    with pytest.raises(ValueError, match="CUDA"):
        jb._buf(torch.zeros(10), 40, "x")                     # big enough, but on the host
    # weight operands: f16 [N, K], q8_0 codes [N, K], q4_0 nibbles [N, K/2], f16 scales [N, K/32]
    assert jb._weight_bytes(synth.DT_F16, 128, 256) == 128 * 256 * 2
    assert jb._weight_bytes(synth.DT_Q8_0, 128, 256) == 128 * 256
    assert jb._weight_bytes(synth.DT_Q4_0, 128, 256) == 128 * 128
    assert jb._scale_bytes(synth.DT_Q4_0, 128, 256) == 128 * 8 * 2
    assert jb._scale_bytes(synth.DT_F16, 128, 256) == 0
    # mean pool of 2 clips x 10 tokens x 64 from a 9-token buffer
    with pytest.raises(ValueError, match="y holds"):
        jb.mean_pool(torch.zeros((2, 9, 64)), 2, 10, 64, 1, torch.zeros((2, 64)))
