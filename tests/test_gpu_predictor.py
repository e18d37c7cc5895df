"""The masked predictor on the GPU (jepa_b200_predict through the C ABI)
against the oracle's predictor on the same seeded tables and tokens.

Head dim 32 (the V-JEPA 2 predictor's 384 / 12) runs through the 64-dim
attention kernel with dims 32..63 of Q, K and V^T zero, so these tests cover
the 32-dim QKV scatter, the softmax scale 1/sqrt(32) and the 32-dim output
rows; head dim 64 is covered too.  Gates as for the encoder: per-token cosine
>= 0.9999 and max|a-b| / max|b| <= 2e-2 (f16 weights), cosine >= 0.9995 for
q8_0 / q4_0 weights."""
import numpy as np
import pytest

from tests.gpu_common import COS_F16, COS_QUANT, REL_MAX_F16, assert_tokens_close, dev, host, need_cuda, orc, synth

import jepa_video_encoder_b200 as jb

pytestmark = pytest.mark.gpu


def _enc_small(frames=16, img=64, **kw):
    # a one-block encoder whose tables the model needs; the predictor reads given tokens
    return synth.small_config(synth.VJEPA2_SSV2, frames=frames, img_h=img, img_w=img, depth=1, head_sa_blocks=0,
                              n_classes=0, pool="none", weights="f16", **kw)


def _model(pc, quant_f16_copy=False):
    table = synth.make_tensor_table(pc.enc) + synth.make_predictor_table(pc)
    return jb.Model(pc.enc, table, predictor=pc, quant_f16_copy=quant_f16_copy), table


def _check(pc, tokens, what):
    m, table = _model(pc)
    got = host(m.predict(dev(tokens), pc.ctx_idx, pc.tgt_idx))
    assert m.sync_status() == 0
    m.close()
    W = orc.weights_f64([t for t in table if t.name.startswith("pred.")])
    ref = orc.predictor(pc, W, tokens.astype(np.float64), pc.ctx_idx, pc.tgt_idx)
    quant = pc.weights in ("q8_0", "q4_0")
    assert_tokens_close(got, ref, COS_QUANT if quant else COS_F16, None if quant else REL_MAX_F16, what=what)


CASES = {
    # name: (encoder tokens, heads of a 128-wide predictor, ctx, tgt, batch, weights)
    "hd32_even_odd": (dict(frames=16), 4, "even", "odd", 3, "f16"),          # L = 128
    "hd32_all_all": (dict(frames=16), 4, "all", "all", 3, "f16"),            # L = 256, 768 rows
    "hd32_ragged": (dict(frames=16, img=80), 4, "all", "all", 2, "f16"),     # N = 200, L = 400
    "hd32_halves": (dict(frames=16, img=80), 4, "first_half", "second_half", 2, "f16"),
    "hd64_all_all": (dict(frames=16), 2, "all", "all", 2, "f16"),
    "hd32_q8": (dict(frames=16), 4, "all", "all", 2, "q8_0"),
    "hd32_q4": (dict(frames=16, img=80), 4, "even", "all", 2, "q4_0"),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_predictor_small(name):
    need_cuda()
    enc_kw, heads, ctx, tgt, B, wdt = CASES[name]
    enc = _enc_small(**enc_kw)
    pc = synth.PredictorConfig(name="pred_" + name, enc=enc, dim=128, depth=2, heads=heads, mlp=256, ctx=ctx, tgt=tgt,
                               weights=wdt, batch=B, random_ln_affine=True)
    _check(pc, synth.make_predictor_tokens(pc), name)


def test_predictor_full_size_sampled(capsys):
    """The V-JEPA 2 ViT-L predictor (12 blocks, width 384, 12 heads of 32)
    on the 16-frame 256^2 clip, context = target = every token (a 4096-row
    sequence per clip, the pages' worst case), B = 8: clips 0 and 7 against
    the oracle."""
    need_cuda()
    pc = synth.VJEPA2_PREDICTOR
    tokens = synth.make_predictor_tokens(pc)
    m, table = _model(pc)
    out = m.predict(dev(tokens), pc.ctx_idx, pc.tgt_idx)
    assert m.sync_status() == 0
    got = host(out[[0, 7]])
    m.close()
    W = orc.weights_f64([t for t in table if t.name.startswith("pred.")])
    ref = orc.predictor(pc, W, tokens[[0, 7]].astype(np.float64), pc.ctx_idx, pc.tgt_idx)
    cos = orc.token_cosines(got, ref)
    with capsys.disabled():
        print(f"\n[predictor parity] {pc.name} clips 0, 7: worst-token cos {cos.min():.7f}, "
              f"rel_max {orc.rel_max(got, ref):.3e}")
    assert_tokens_close(got, ref, COS_F16, REL_MAX_F16, what="predictor full size")


def test_predictor_errors_and_batch_invariance():
    need_cuda()
    enc = _enc_small()
    pc = synth.PredictorConfig(name="pred_err", enc=enc, dim=128, depth=1, heads=4, mlp=256, batch=3)
    m, _ = _model(pc)
    tok = dev(synth.make_predictor_tokens(pc))
    with pytest.raises(jb.JepaError) as e:
        m.predict(tok, [0, enc.n_tokens], [1])
    assert e.value.status == jb._abi.ERR_ARG
    full = m.predict(tok, pc.ctx_idx, pc.tgt_idx).cpu().numpy()
    one = m.predict(tok[1:2].contiguous(), pc.ctx_idx, pc.tgt_idx).cpu().numpy()
    assert np.array_equal(one[0].view(np.uint32), full[1].view(np.uint32))
    assert m.sync_status() == 0
    m.close()
    m2 = jb.Model(enc, synth.make_tensor_table(enc))   # no predictor
    with pytest.raises(jb.JepaError) as e:
        m2.predict(tok, [0], [1])
    assert e.value.status == jb._abi.ERR_ARG
    m2.close()
