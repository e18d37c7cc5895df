"""End-to-end parity of the CUDA forward (jepa_b200_encode through the C ABI)
against the oracle on the same seeded tables and pixels.

* Shrunk copies of the five workloads run the whole forward in the oracle
  (seconds) and are compared element by element.
* The LeWM ViT-Ti/14 workload is small enough to run in full.
* At full size (ViT-L/16, the batch sizes the benchmark times) the oracle
  evaluates sampled rows of chosen blocks, fed with the GPU's own input to
  that block (jepa_b200_debug_stage), plus the pooled outputs / head."""
import numpy as np
import pytest

from tests.gpu_common import (COS_F16, COS_QUANT, REL_MAX_F16, assert_tokens_close, dev, host, need_cuda, orc,
                              synth, torch)

import jepa_video_encoder_b200 as jb

pytestmark = pytest.mark.gpu


def _small(base, **kw):
    return synth.small_config(base, **kw)


SMALL = {
    "lewm": _small(synth.LEWM_VIT_TI, dim=192, heads=3, mlp=768, img_h=56, img_w=56, frames=1, batch=3),
    "levjepa": _small(synth.LEVJEPA_VIT_L, frames=8, batch=3),                       # 129 tokens, block-causal
    "vjepa2_ssv2": _small(synth.VJEPA2_SSV2, frames=8, batch=3, head_sa_blocks=1),   # q8_0 + head
    "levjepa_q4": _small(synth.LEVJEPA_VIT_L_Q4, frames=8, batch=2),
    "vjepa2_long": _small(synth.VJEPA2_LONG, frames=16, batch=2),                    # 128 tokens, bidir
    # 3-D rotary positions: 128 tokens x 2 clips (CTA-pair GEMMs, TMA QKV epilogue) and,
    # with q8_0 and the head, 64 tokens x 3 clips (row-by-row QKV epilogue)
    "vjepa2_rope": _small(synth.VJEPA2_LONG, frames=16, batch=2, rope=True),
    "vjepa2_ssv2_rope": _small(synth.VJEPA2_SSV2, frames=8, batch=3, head_sa_blocks=1, rope=True),
}


def _gate(cfg):
    return (COS_QUANT, None) if cfg.weights in ("q8_0", "q4_0") else (COS_F16, REL_MAX_F16)


def _run(cfg, pool, table=None, pix=None):
    table = synth.make_tensor_table(cfg) if table is None else table
    pix = synth.make_pixels(cfg) if pix is None else pix
    m = jb.Model(cfg, table)
    out = m.encode(dev(pix), pool=pool)
    assert m.sync_status() == 0
    return m, table, pix, host(out)


@pytest.mark.parametrize("name", sorted(SMALL))
def test_small_workload_last_hidden_state(name):
    need_cuda()
    cfg = SMALL[name]
    m, table, pix, got = _run(cfg, "none")
    W = orc.weights_f64(table)
    ref = orc.encoder(cfg, W, pix.astype(np.float64))
    cos_min, rel = _gate(cfg)
    assert_tokens_close(got, ref, cos_min, rel, what=name)
    # the configured pooled output of the same forward
    if cfg.pool != "none":
        out = host(m.encode(dev(pix), pool=cfg.pool))
        assert m.sync_status() == 0
        if cfg.pool == "attentive":
            lref = orc.attentive_head(cfg, W, ref)
            assert_tokens_close(out, lref, cos_min, None, what=name + " logits")
            assert (out.argmax(1) == lref.argmax(1)).all()
        else:
            assert_tokens_close(out, orc.pool(cfg, ref, cfg.pool), cos_min, rel, what=name + " " + cfg.pool)
    m.close()


@pytest.mark.parametrize("name", ["lewm_vit_ti14_224_b1", "lewm_vit_ti14_224_b8"])
def test_lewm_full_size(name):
    """LeWM ViT-Ti/14, 224^2, 257 tokens, f32 weights, CLS output: the whole
    forward in the oracle, one clip and a batch of 8 (2056 rows)."""
    need_cuda()
    cfg = synth.WORKLOADS[name]
    m, table, pix, got = _run(cfg, "none")
    ref = orc.encoder(cfg, orc.weights_f64(table), pix.astype(np.float64))
    assert_tokens_close(got, ref, what="lewm full")
    cls = host(m.encode(dev(pix), pool="cls"))
    assert_tokens_close(cls, ref[:, 0], what="lewm cls")
    m.close()


def test_batch_invariance_bitwise():
    """Clip b of a batch-B forward equals the B=1 forward of that clip bit for bit."""
    need_cuda()
    cfg = SMALL["levjepa"]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    full = m.encode(dev(pix), pool="none").cpu().numpy()
    for b in range(cfg.batch):
        one = m.encode(dev(pix[b:b + 1]), pool="none").cpu().numpy()
        assert np.array_equal(one[0].view(np.uint32), full[b].view(np.uint32))
    assert m.sync_status() == 0
    m.close()


def test_graph_replay_matches_direct_launches():
    """The CUDA-graph replay of a forward gives the bits of the kernel-by-kernel
    forward; a new output buffer or a smaller batch recaptures (and the ops are
    rebuilt for the smaller batch)."""
    need_cuda()
    cfg = SMALL["levjepa"]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    m.set_graph(False)
    direct = m.encode(dev(pix), pool="none").cpu().numpy()
    m.set_graph(True)
    x = dev(pix)
    out = torch.empty(m.out_shape(cfg.batch, "none"), dtype=torch.float32, device="cuda")
    for _ in range(3):  # capture, then two replays
        m.encode(x, pool="none", out=out)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), direct.view(np.uint32))
    out2 = torch.empty_like(out)
    m.encode(x, pool="none", out=out2)
    assert np.array_equal(out2.cpu().numpy().view(np.uint32), direct.view(np.uint32))
    one = m.encode(dev(pix[1:2]), pool="none").cpu().numpy()
    assert np.array_equal(one[0].view(np.uint32), direct[1].view(np.uint32))
    # a larger batch reallocates the workspace: the graph bound to the old one
    # must not be replayed
    pix2 = np.concatenate([pix, pix], axis=0)
    big = m.encode(dev(pix2), pool="none").cpu().numpy()
    assert np.array_equal(big[cfg.batch:].view(np.uint32), direct.view(np.uint32))
    for _ in range(2):
        m.encode(x, pool="none", out=out)
        assert np.array_equal(out.cpu().numpy().view(np.uint32), direct.view(np.uint32))
    assert m.sync_status() == 0
    m.close()


def test_block_causal_perturbation_forward_bit_identical():
    """Perturbing the pixels of frame t+1 leaves every patch token of frames
    <= t bit-identical at the encoder output (GPU path)."""
    need_cuda()
    cfg = SMALL["levjepa"]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    base = m.encode(dev(pix), pool="none").cpu().numpy()
    pf = cfg.patches_per_slot
    for t in (0, 3, cfg.frames - 2):
        p2 = pix.copy()
        p2[:, t + 1] = np.random.default_rng(t).standard_normal(p2[:, t + 1].shape).astype(np.float32)
        out = m.encode(dev(p2), pool="none").cpu().numpy()
        keep = 1 + (t + 1) * pf
        assert np.array_equal(out[:, 1:keep].view(np.uint32), base[:, 1:keep].view(np.uint32))
        assert not np.array_equal(out[:, keep:], base[:, keep:])
        assert not np.array_equal(out[:, 0], base[:, 0])
    assert m.sync_status() == 0
    m.close()


def test_encode_host_matches_device():
    need_cuda()
    cfg = SMALL["vjepa2_ssv2"]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    d = m.encode(dev(pix), pool="attentive").cpu().numpy()
    h = m.encode_host(torch.from_numpy(pix).pin_memory(), pool="attentive").numpy()
    assert np.array_equal(d, h)
    m.close()


def test_encode_errors():
    need_cuda()
    cfg = SMALL["levjepa"]
    m = jb.Model(cfg, synth.make_tensor_table(cfg))
    pix = dev(synth.make_pixels(cfg))
    with pytest.raises(jb.JepaError) as e:
        m.encode(pix, pool="attentive")
    assert e.value.status == jb._abi.ERR_MISSING_TENSOR
    small = torch.empty(3, device="cuda")
    with pytest.raises(jb.JepaError) as e:
        m.encode(pix, pool="cls", out=small)
    assert e.value.status == jb._abi.ERR_SHAPE
    m.close()


def test_model_timeout_path():
    """A zero wait bound makes the forward's kernels give up at once and unwind;
    the model reports ERR_TIMEOUT and the next forward is correct again."""
    need_cuda()
    cfg = SMALL["levjepa"]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    good = m.encode(dev(pix), pool="cls").cpu().numpy()
    m.set_timeout_ns(0)
    m.encode(dev(pix), pool="cls")
    assert m.sync_status() == jb._abi.ERR_TIMEOUT
    m.set_timeout_ns(4_000_000_000)
    again = m.encode(dev(pix), pool="cls").cpu().numpy()
    assert m.sync_status() == 0
    assert np.array_equal(good, again)
    m.close()


# ---------------------------------------------------------------- full size --
def _increment_check(x_in, x_out, ref_out, rows, cos_min, what):
    """Compare a block's increment x_out - x_in on the sampled rows."""
    d_gpu = x_out[rows] - x_in[rows]
    d_ref = ref_out - x_in[rows]
    assert_tokens_close(d_gpu, d_ref, cos_min, REL_MAX_F16, what=what)


def _full_size_layers(cfg, layers, clips, rows_fn):
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    W = orc.weights_f64(table)
    m = jb.Model(cfg, table)
    pd = dev(pix)
    cos_min = COS_QUANT if cfg.weights in ("q8_0", "q4_0") else COS_F16
    x0 = host(m.debug_stage(pd, 0))
    emb = orc.embed(cfg, W, pix.astype(np.float64))
    for b in clips:
        assert_tokens_close(x0[b], emb[b], COS_F16, REL_MAX_F16, what=f"{cfg.name} embed clip {b}")
    allow = orc.encoder_allow(cfg)
    rope_pos = orc.rope_positions(cfg) if cfg.rope else None
    for l in layers:
        xin = host(m.debug_stage(pd, l))
        xout = host(m.debug_stage(pd, l + 1))
        assert m.sync_status() == 0
        for b in clips:
            rows = rows_fn(cfg)
            ref = orc.block_rows(xin[b], W, f"enc.blk.{l}.", cfg.heads, cfg.ln_eps, allow, rows, rope_pos)
            _increment_check(xin[b], xout[b], ref, rows, cos_min, f"{cfg.name} block {l} clip {b}")
    return m, table, pix, W


def _rows(cfg):
    N = cfg.n_tokens
    return np.unique(np.r_[0, 1, 2, 127, 128, 129, cfg.patches_per_slot, cfg.patches_per_slot + 1,
                           N // 2, N - 129, N - 2, N - 1])


def test_levjepa_full_size_sampled():
    """LeVJEPA ViT-L/16, 16 frames 224^2, B=4, f16, block-causal, CLS: the
    benchmark workload.  Blocks 0 and 23 on sampled rows, and the CLS output
    from the GPU's last residual."""
    need_cuda()
    cfg = synth.LEVJEPA_VIT_L
    m, table, pix, W = _full_size_layers(cfg, [0, 23], [0, 3], _rows)
    pd = dev(pix)
    x24 = host(m.debug_stage(pd, cfg.depth))
    cls = host(m.encode(pd, pool="cls"))
    assert m.sync_status() == 0
    ref = orc.layer_norm(x24[:, 0], W["enc.norm.weight"], W["enc.norm.bias"], cfg.ln_eps)
    assert_tokens_close(cls, ref, what="levjepa cls")
    m.close()


def test_vjepa2_ssv2_full_size_q8_head():
    """V-JEPA 2 ViT-L/16 + attentive head, q8_0, 16 frames 256^2, B=8: block 0
    on sampled rows of two clips; the head of clip 0 from the GPU's tokens."""
    need_cuda()
    cfg = synth.VJEPA2_SSV2
    m, table, pix, W = _full_size_layers(cfg, [0], [0, 7], _rows)
    pd = dev(pix)
    tokens = host(m.encode(pd, pool="none"))
    logits = host(m.encode(pd, pool="attentive"))
    assert m.sync_status() == 0
    ref = orc.attentive_head(cfg, W, tokens[:1])
    assert_tokens_close(logits[:1], ref, COS_QUANT, None, what="ssv2 logits clip 0")
    assert logits[0].argmax() == ref[0].argmax()
    m.close()


def test_levjepa_q4_full_size_mean():
    """The LeVJEPA encoder with q4_0 matrices, B=8, mean pooling: block 11 on
    sampled rows, and the mean pool from the GPU's last residual."""
    need_cuda()
    cfg = synth.LEVJEPA_VIT_L_Q4
    m, table, pix, W = _full_size_layers(cfg, [11], [0, 7], _rows)
    pd = dev(pix)
    x24 = host(m.debug_stage(pd, cfg.depth))
    mean = host(m.encode(pd, pool="mean"))
    assert m.sync_status() == 0
    y = orc.layer_norm(x24, W["enc.norm.weight"], W["enc.norm.bias"], cfg.ln_eps)
    assert_tokens_close(mean, orc.pool(cfg, y, "mean"), COS_QUANT, None, what="q4 mean")
    m.close()


def test_vjepa2_long_full_size_sampled():
    """V-JEPA 2 64-frame clip, 8192 tokens, B=2, f16, full token map: block 0
    on sampled rows, and the final LayerNorm on all rows."""
    need_cuda()
    cfg = synth.VJEPA2_LONG
    m, table, pix, W = _full_size_layers(cfg, [0], [1], _rows)
    pd = dev(pix)
    x24 = host(m.debug_stage(pd, cfg.depth))
    out = host(m.encode(pd, pool="none"))
    assert m.sync_status() == 0
    ref = orc.layer_norm(x24, W["enc.norm.weight"], W["enc.norm.bias"], cfg.ln_eps)
    assert_tokens_close(out, ref, what="long final norm")
    m.close()


def test_vjepa2_long_rope_full_size_sampled():
    """The 64-frame, 8192-token V-JEPA 2 clip with 3-D rotary positions in
    every encoder block (slots up to 31, patch rows and columns up to 15):
    blocks 0 and 23 on sampled rows."""
    need_cuda()
    cfg = synth.VJEPA2_LONG.with_(name="vjepa2_vit_l16_64f256_rope_b2", rope=True)
    m, table, pix, W = _full_size_layers(cfg, [0, 23], [0, 1], _rows)
    m.close()


@pytest.mark.parametrize("name", ["vjepa2_ssv2", "levjepa_q4"])
def test_quant_loader_unpack_matches_f16_copy_bitwise(name):
    """A q8_0 / q4_0 model keeps its blocks only (every GEMM unpacks them in
    its loader) or, on request, also an f16 copy for the large GEMMs: the
    copy holds exactly the unpacked values, so both forwards agree bit for
    bit, and the blocks-only model holds fewer bytes.  (Batches of 320 and
    258 rows: the CTA-pair GEMMs with and without the copy.)"""
    need_cuda()
    cfg = SMALL[name] if name != "vjepa2_ssv2" else SMALL[name].with_(batch=5)
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    outs, sizes = [], []
    for copy in (False, True):
        m = jb.Model(cfg, table, quant_f16_copy=copy)
        outs.append(m.encode(dev(pix), pool="none").cpu().numpy())
        if cfg.pool == "attentive":
            outs.append(m.encode(dev(pix), pool="attentive").cpu().numpy())
        assert m.sync_status() == 0
        sizes.append(m.n_bytes)
        m.close()
    half = len(outs) // 2
    for a, b in zip(outs[:half], outs[half:]):
        assert np.array_equal(a.view(np.uint32), b.view(np.uint32))
    assert sizes[0] < sizes[1]
