"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every symbol include/jepa_b200.h declares, and rejects bad arguments and bad
tensor tables before any device work."""
import ctypes
import os
import re
import subprocess

import numpy as np
import pytest

from jepa_video_encoder_b200 import _abi, build, synth, make_config

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "jepa_b200.h")


@pytest.fixture(scope="module")
def lib():
    build.build()
    return _abi.load_library()


def header_functions():
    txt = open(HEADER).read()
    return sorted(set(re.findall(r"JEPA_B200_API\s+[^;(]*?\b(jepa_b200_\w+)\s*\(", txt)))


def test_header_declares_functions():
    names = header_functions()
    assert "jepa_b200_load_weights" in names and "jepa_b200_encode" in names
    assert len(names) >= 20


def test_library_exports_every_declared_symbol(lib):
    names = header_functions()
    out = subprocess.run(["nm", "-D", "--defined-only", _abi.LIB_PATH], capture_output=True, text=True).stdout
    exported = set(l.split()[-1] for l in out.splitlines() if " T " in l)
    missing = [n for n in names if n not in exported]
    assert not missing, missing
    for n in names:
        assert hasattr(lib, n)
    # the binding declares exactly the header's functions
    assert sorted(_abi.SIGNATURES) == names


def test_status_strings(lib):
    for s in range(0, -8, -1):
        assert _abi.status_str(s)
    assert _abi.status_str(_abi.ERR_TIMEOUT).startswith("a bounded")


def _tiny_cfg(**kw):
    base = synth.EncoderConfig(name="t", dim=128, depth=1, heads=2, mlp=256, patch=8, tubelet=1, img_h=16,
                               img_w=16, frames=2, has_cls=True, mask="block_causal", weights="f16", batch=1,
                               pool="cls")
    return base.with_(**kw)


def _load(lib, cfg, table, predictor=None, world_model=None):
    entries = (_abi.TensorEntry * len(table))()
    keep = []
    for i, t in enumerate(table):
        nm = t.name.encode()
        keep.append(nm)
        entries[i].name = nm
        entries[i].dtype = t.dtype
        entries[i].ndim = len(t.shape)
        for j, s in enumerate(t.shape):
            entries[i].shape[j] = s
        entries[i].data = t.data.ctypes.data
        entries[i].nbytes = t.nbytes
    c = make_config(cfg, predictor=predictor, world_model=world_model)
    h = ctypes.c_void_p()
    st = lib.jepa_b200_load_weights(ctypes.byref(c), entries, len(table), 0, ctypes.byref(h))
    if st == 0:
        lib.jepa_b200_free(h)
    return st


def _has_gpu():
    try:
        import torch
        return torch.cuda.is_available()
    except Exception:
        return False


def test_table_validation(lib):
    cfg = _tiny_cfg()
    table = synth.make_tensor_table(cfg)
    full = _load(lib, cfg, table)
    # a complete table passes validation; without a device the upload then fails
    assert full == (0 if _has_gpu() else _abi.ERR_CUDA)
    assert _load(lib, cfg, [t for t in table if t.name != "enc.blk.0.ffn_up.bias"]) == _abi.ERR_MISSING_TENSOR
    bad = list(table)
    i = [t.name for t in bad].index("enc.blk.0.ln1.weight")
    bad[i] = synth.Tensor(bad[i].name, synth.DT_Q8_0, bad[i].shape,
                          synth.quantize_q8_0(np.ones(cfg.dim, np.float32)))
    assert _load(lib, cfg, bad) == _abi.ERR_DTYPE
    bad = list(table)
    i = [t.name for t in bad].index("enc.pos_embed")
    bad[i] = synth.Tensor(bad[i].name, synth.DT_F32, (cfg.n_tokens - 1, cfg.dim),
                          np.zeros((cfg.n_tokens - 1, cfg.dim), np.float32))
    assert _load(lib, cfg, bad) == _abi.ERR_SHAPE
    bad = list(table)
    i = [t.name for t in bad].index("enc.blk.0.attn_out.weight")
    bad[i] = synth.Tensor(bad[i].name, bad[i].dtype, bad[i].shape, bad[i].data[:-1])   # nbytes off by one row
    assert _load(lib, cfg, bad) == _abi.ERR_SHAPE


def test_duplicate_and_extra_names(lib):
    cfg = _tiny_cfg()
    table = synth.make_tensor_table(cfg)
    ok = 0 if _has_gpu() else _abi.ERR_CUDA
    dup = list(table) + [table[3]]
    assert _load(lib, cfg, dup) == _abi.ERR_ARG                      # a name given twice
    extra = list(table) + [synth.Tensor("pred.blk.0.ln1.weight", synth.DT_F32, (cfg.dim,),
                                        np.ones(cfg.dim, np.float32))]
    assert _load(lib, cfg, extra) == ok                               # unused names are ignored


def test_quantised_table_validation(lib):
    cfg = _tiny_cfg(weights="q8_0")
    table = synth.make_tensor_table(cfg)
    assert _load(lib, cfg, table) == (0 if _has_gpu() else _abi.ERR_CUDA)
    # quantised blocks are refused outside the re-typed matrices
    bad = list(table)
    i = [t.name for t in bad].index("enc.patch_embed.weight")
    w = np.zeros((cfg.dim, 3 * 8 * 8), np.float32)
    bad[i] = synth.Tensor(bad[i].name, synth.DT_Q8_0, bad[i].shape, synth.quantize_q8_0(w))
    assert _load(lib, cfg, bad) == _abi.ERR_DTYPE


def test_bad_config(lib):
    cfg = _tiny_cfg()
    table = synth.make_tensor_table(cfg)
    assert _load(lib, cfg.with_(heads=3), table) == _abi.ERR_SHAPE       # dim != 64 * heads
    assert _load(lib, cfg.with_(img_h=20), table) == _abi.ERR_SHAPE      # not a multiple of the patch
    # shapes whose sizes would overflow 32-bit indexing are refused up front
    assert _load(lib, cfg.with_(patch=1, img_h=1 << 16, img_w=1 << 16), table) == _abi.ERR_SHAPE
    assert _load(lib, cfg.with_(patch=1, img_h=512, img_w=1024, frames=1), table) == _abi.ERR_SHAPE
    assert _load(lib, cfg.with_(patch=1 << 16, img_h=1 << 16, img_w=1 << 16), table) == _abi.ERR_SHAPE
    assert _load(lib, cfg.with_(patch=128, tubelet=1, img_h=128, img_w=128), table) == _abi.ERR_SHAPE
    c = make_config(cfg)
    c.mask = 7
    h = ctypes.c_void_p()
    assert lib.jepa_b200_load_weights(ctypes.byref(c), None, 0, 0, ctypes.byref(h)) == _abi.ERR_ARG


def test_rotary_config_validation(lib):
    """Rotary positions take one (slot, row, column) index per patch token:
    no CLS token, and at most 64 positions on each axis."""
    cfg = _tiny_cfg(has_cls=False, rope=True, pool="mean")
    table = synth.make_tensor_table(cfg)
    assert "enc.pos_embed" not in [t.name for t in table]
    assert _load(lib, cfg, table) == (0 if _has_gpu() else _abi.ERR_CUDA)
    assert _load(lib, cfg.with_(has_cls=True, pool="cls"), synth.make_tensor_table(cfg.with_(has_cls=True))) \
        == _abi.ERR_SHAPE
    edge = cfg.with_(frames=64, img_w=8 * 64)                              # 64 slots, 64 patch columns
    assert _load(lib, edge, synth.make_tensor_table(edge)) == (0 if _has_gpu() else _abi.ERR_CUDA)
    assert _load(lib, cfg.with_(frames=65), table) == _abi.ERR_SHAPE       # 65 slots
    assert _load(lib, cfg.with_(frames=130, tubelet=2), table) == _abi.ERR_SHAPE   # 65 slots of two frames
    assert _load(lib, cfg.with_(img_h=8 * 65), table) == _abi.ERR_SHAPE    # 65 patch rows
    assert _load(lib, cfg.with_(img_w=8 * 65), table) == _abi.ERR_SHAPE    # 65 patch columns
    c = make_config(cfg)
    c.rope = 2
    h = ctypes.c_void_p()
    assert lib.jepa_b200_load_weights(ctypes.byref(c), None, 0, 0, ctypes.byref(h)) == _abi.ERR_ARG
    # without rotary positions the additive table is required again
    assert _load(lib, cfg.with_(rope=False), table) == _abi.ERR_MISSING_TENSOR


def test_patch_embed_op_shape_limits(lib):
    """The single-kernel patch-embed refuses shapes beyond the model's limits
    before touching the device (the pointers are never dereferenced)."""
    buf = (ctypes.c_float * 64)()
    p = ctypes.cast(buf, ctypes.c_void_p)
    p = ctypes.c_void_p((p.value + 15) // 16 * 16) if p.value % 16 else p

    def call(B, T, H, W, patch, kt, D):
        return lib.jepa_b200_op_patch_embed(p, B, T, H, W, patch, kt, p, D, None, p, None, 0, p, None)

    assert call(1, 1, 128, 128, 128, 1, 128) == _abi.ERR_SHAPE           # K = 49152
    assert call(1, 1, 1 << 16, 1 << 16, 1, 1, 128) == _abi.ERR_SHAPE      # 2^32 patches
    assert call(3, 1, 512, 512, 1, 1, 128) == _abi.ERR_SHAPE              # 3 * 262144 rows
    assert call(1, 1, 64, 64, 16, 1, 8192) == _abi.ERR_SHAPE              # D > 4096
    assert call(1, 1, 20, 64, 16, 1, 128) == _abi.ERR_SHAPE               # H not a multiple of the patch


def test_null_arguments(lib):
    shp = (ctypes.c_int64 * 3)()
    assert lib.jepa_b200_out_shape(None, 1, 0, shp) == _abi.ERR_ARG
    assert lib.jepa_b200_encode(None, None, 1, 0, None, 0, None) == _abi.ERR_ARG
    assert lib.jepa_b200_encode_host(None, None, 1, 0, None, 0, None) == _abi.ERR_ARG
    assert lib.jepa_b200_debug_stage(None, None, 1, 0, 0, None, 0, None) == _abi.ERR_ARG
    assert lib.jepa_b200_op_layernorm(None, 4, 64, 1, None, None, 1e-6, None, 1, None) == _abi.ERR_ARG
    assert lib.jepa_b200_op_linear(None, 4, 64, None, None, 1, 128, None, 0, None, 128, None) == _abi.ERR_ARG
    assert lib.jepa_b200_op_linear(None, 4, 64, None, None, 5, 128, None, 0, None, 128, None) == _abi.ERR_ARG
    assert lib.jepa_b200_op_gemv(None, 1, 64, None, None, 1, 8, None, 7, None, 0, None, None) == _abi.ERR_ARG
    assert lib.jepa_b200_model_n_bytes(None) == 0
    assert lib.jepa_b200_last_ms(None) < 0
    lib.jepa_b200_free(None)


def test_predictor_config_and_table_validation(lib):
    """The predictor's shape limits (width a multiple of 64, head dim 32 or
    64, MLP a multiple of 64) and its tensors, checked on the host."""
    cfg = _tiny_cfg(mask="bidir", has_cls=False)
    ok = 0 if _has_gpu() else _abi.ERR_CUDA
    pc = synth.PredictorConfig(name="p", enc=cfg, dim=128, depth=1, heads=4, mlp=256)
    table = synth.make_tensor_table(cfg) + synth.make_predictor_table(pc)
    assert _load(lib, cfg, table, pc) == ok
    assert _load(lib, cfg, table, pc.with_(heads=2)) == ok                       # head dim 64
    assert _load(lib, cfg, table, pc.with_(heads=8)) == _abi.ERR_SHAPE           # head dim 16
    assert _load(lib, cfg, table, pc.with_(dim=96, heads=3)) == _abi.ERR_SHAPE    # width not a multiple of 64
    assert _load(lib, cfg, table, pc.with_(mlp=200)) == _abi.ERR_SHAPE
    assert _load(lib, cfg, table, pc.with_(depth=-1)) == _abi.ERR_ARG
    assert _load(lib, cfg, [t for t in table if t.name != "pred.mask_tokens"], pc) == _abi.ERR_MISSING_TENSOR
    assert _load(lib, cfg, [t for t in table if t.name != "pred.blk.0.ffn_down.bias"], pc) == \
        _abi.ERR_MISSING_TENSOR
    # pred.embed / pred.proj may be quantised (re-typed), pred.pos_embed may not
    q = synth.make_tensor_table(cfg) + synth.make_predictor_table(pc.with_(weights="q8_0"))
    assert {t.name: t.dtype for t in q}["pred.embed.weight"] == synth.DT_Q8_0
    assert _load(lib, cfg, q, pc) == ok
    bad = list(table)
    i = [t.name for t in bad].index("pred.pos_embed")
    bad[i] = synth.Tensor("pred.pos_embed", synth.DT_Q8_0, bad[i].shape,
                          synth.quantize_q8_0(np.zeros(bad[i].shape, np.float32)))
    assert _load(lib, cfg, bad, pc) == _abi.ERR_DTYPE


def test_world_model_config_and_table_validation(lib):
    """The world model's shape limits (state width at most 256 in heads of 64,
    MLP / output widths multiples of 64 up to 1024, window at most 32, a CLS
    row to project) and its tensors, checked on the host."""
    cfg = _tiny_cfg(dim=128, heads=2, mlp=256, mask="bidir")
    ok = 0 if _has_gpu() else _abi.ERR_CUDA
    wc = synth.WorldModelConfig(name="w", enc=cfg, dim=128, depth=2, heads=2, mlp=256, window=3, proj_hidden=256,
                                pred_hidden=256)
    table = synth.make_tensor_table(cfg) + synth.make_world_model_table(wc)
    assert _load(lib, cfg, table, world_model=wc) == ok
    assert _load(lib, cfg, table, world_model=wc.with_(heads=4)) == _abi.ERR_SHAPE        # head dim 32
    assert _load(lib, cfg, table, world_model=wc.with_(mlp=200)) == _abi.ERR_SHAPE
    assert _load(lib, cfg, table, world_model=wc.with_(mlp=2048)) == _abi.ERR_SHAPE       # above 1024
    assert _load(lib, cfg, table, world_model=wc.with_(pred_hidden=96)) == _abi.ERR_SHAPE
    assert _load(lib, cfg, table, world_model=wc.with_(window=33)) == _abi.ERR_SHAPE
    assert _load(lib, cfg, table, world_model=wc.with_(action_dim=65)) == _abi.ERR_SHAPE
    assert _load(lib, cfg, table, world_model=wc.with_(depth=-1)) == _abi.ERR_ARG
    no_cls = cfg.with_(has_cls=False)
    assert _load(lib, no_cls, synth.make_tensor_table(no_cls) + synth.make_world_model_table(wc),
                 world_model=wc) == _abi.ERR_SHAPE
    pc = synth.PredictorConfig(name="p", enc=cfg, dim=128, depth=1, heads=2, mlp=256)
    assert _load(lib, cfg, table + synth.make_predictor_table(pc), predictor=pc, world_model=wc) == _abi.ERR_ARG
    for gone in ("pred.blk.1.adaln.bias", "pred.action_embed.0.weight", "enc.proj.2.weight", "pred.proj.0.bias"):
        assert _load(lib, cfg, [t for t in table if t.name != gone], world_model=wc) == _abi.ERR_MISSING_TENSOR
    # the re-typed matrices may be quantised; adaLN and the action embedder stay f32 / f16
    q = synth.make_tensor_table(cfg) + synth.make_world_model_table(wc.with_(weights="q4_0"))
    dt = {t.name: t.dtype for t in q}
    assert dt["pred.proj.0.weight"] == synth.DT_Q4_0 and dt["pred.blk.0.adaln.weight"] == synth.DT_F32
    assert _load(lib, cfg, q, world_model=wc) == ok
    bad = list(table)
    i = [t.name for t in bad].index("pred.blk.0.adaln.weight")
    bad[i] = synth.Tensor(bad[i].name, synth.DT_Q8_0, bad[i].shape,
                          synth.quantize_q8_0(np.zeros(bad[i].shape, np.float32)))
    assert _load(lib, cfg, bad, world_model=wc) == _abi.ERR_DTYPE
