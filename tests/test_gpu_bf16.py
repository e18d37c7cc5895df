"""The bf16 activation option (jepa_b200_config.act_bf16): every 16-bit
activation and MMA operand in bf16 instead of f16, accumulations, softmax,
LayerNorm statistics and the residual stream in f32.  Checked against the
oracle at the gates the pages give for f16 / bf16 compute (per-token cosine
>= 0.9999 and max|a-b| / max|b| <= 2e-2 for 16-bit weights; cosine >= 0.9995
and the same top-1 for q8_0 / q4_0 weights), on shrunk copies of every
workload family, the full-size LeVJEPA forward from pixels, and the masked
predictor.  The oracle keeps the table's own weight values; the bf16 path
rounds 16-bit weights to bf16 once at load, so its error includes that
rounding."""
import numpy as np
import pytest

from tests.gpu_common import COS_F16, COS_QUANT, REL_MAX_F16, assert_tokens_close, dev, host, need_cuda, orc, synth

import jepa_video_encoder_b200 as jb

pytestmark = pytest.mark.gpu


def _small(base, **kw):
    return synth.small_config(base, act_bf16=True, **kw)


SMALL_BF16 = {
    "levjepa": _small(synth.LEVJEPA_VIT_L, frames=8, batch=3),                       # block-causal, CLS, 258+ rows
    "vjepa2_ssv2": _small(synth.VJEPA2_SSV2, frames=8, batch=5, head_sa_blocks=1),   # q8_0 + head, 320 rows
    "levjepa_q4": _small(synth.LEVJEPA_VIT_L_Q4, frames=8, batch=2),
    "vjepa2_long_rope": _small(synth.VJEPA2_LONG, frames=16, batch=2, rope=True),
    "lewm": _small(synth.LEWM_VIT_TI, dim=192, heads=3, mlp=768, img_h=56, img_w=56, frames=1, batch=3),
}


@pytest.mark.parametrize("name", sorted(SMALL_BF16))
def test_bf16_small_workloads(name):
    need_cuda()
    cfg = SMALL_BF16[name]
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    got = host(m.encode(dev(pix), pool="none"))
    pooled = host(m.encode(dev(pix), pool=cfg.pool)) if cfg.pool != "none" else None
    assert m.sync_status() == 0
    m.close()
    W = orc.weights_f64(table)
    ref = orc.encoder(cfg, W, pix.astype(np.float64))
    quant = cfg.weights in ("q8_0", "q4_0")
    assert_tokens_close(got, ref, COS_QUANT if quant else COS_F16, None if quant else REL_MAX_F16, what=name)
    if cfg.pool == "attentive":
        lref = orc.attentive_head(cfg, W, ref)
        assert_tokens_close(pooled, lref, COS_QUANT, None, what=name + " logits")
        assert (pooled.argmax(1) == lref.argmax(1)).all()
    elif pooled is not None:
        assert_tokens_close(pooled, orc.pool(cfg, ref, cfg.pool), COS_QUANT if quant else COS_F16, None,
                            what=name + " " + cfg.pool)


def test_bf16_differs_from_f16():
    """The option changes the arithmetic: the same table and pixels give
    other bits in bf16 than in f16."""
    need_cuda()
    cfg = SMALL_BF16["levjepa"]
    table = synth.make_tensor_table(cfg)
    pix = dev(synth.make_pixels(cfg))
    outs = []
    for bf in (False, True):
        m = jb.Model(cfg.with_(act_bf16=bf), table)
        outs.append(m.encode(pix, pool="none").cpu().numpy())
        assert m.sync_status() == 0
        m.close()
    assert not np.array_equal(outs[0], outs[1])


def test_bf16_levjepa_full_forward(capsys):
    """LeVJEPA ViT-L/16, 16 frames 224^2, B=4, bf16 activations: every token
    of clip 0 from pixels against the oracle's forward from the same pixels."""
    need_cuda()
    cfg = synth.LEVJEPA_VIT_L_BF16
    table = synth.make_tensor_table(cfg)
    pix = synth.make_pixels(cfg)
    m = jb.Model(cfg, table)
    tokens = host(m.encode(dev(pix), pool="none")[:1])
    assert m.sync_status() == 0
    m.close()
    ref = orc.encoder(cfg, orc.weights_f64(table), pix[:1].astype(np.float64))
    cos = orc.token_cosines(tokens, ref)
    with capsys.disabled():
        print(f"\n[bf16 parity] {cfg.name} clip 0: worst-token cos {cos.min():.7f}, "
              f"rel_max {orc.rel_max(tokens, ref):.3e}")
    assert_tokens_close(tokens, ref, COS_F16, REL_MAX_F16, what="levjepa bf16 clip 0")


def test_bf16_predictor():
    need_cuda()
    enc = synth.small_config(synth.VJEPA2_SSV2, frames=16, img_h=80, img_w=80, depth=1, head_sa_blocks=0, n_classes=0,
                             pool="none", weights="f16", act_bf16=True)
    pc = synth.PredictorConfig(name="pred_bf16", enc=enc, dim=128, depth=2, heads=4, mlp=256, ctx="all", tgt="all",
                               batch=2, random_ln_affine=True)
    table = synth.make_tensor_table(enc) + synth.make_predictor_table(pc)
    m = jb.Model(enc, table, predictor=pc)
    tok = synth.make_predictor_tokens(pc)
    got = host(m.predict(dev(tok), pc.ctx_idx, pc.tgt_idx))
    assert m.sync_status() == 0
    m.close()
    W = orc.weights_f64([t for t in table if t.name.startswith("pred.")])
    ref = orc.predictor(pc, W, tok.astype(np.float64), pc.ctx_idx, pc.tgt_idx)
    assert_tokens_close(got, ref, COS_F16, REL_MAX_F16, what="predictor bf16")
