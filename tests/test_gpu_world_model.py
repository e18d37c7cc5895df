"""The LeWM world model on the GPU (jepa_b200_lewm_predict / _rollout and the
"lewm" pool, through the C ABI) against the oracle on the same seeded
tables and inputs.

Gates as for the encoder: per-row cosine >= 0.9999 and max|a-b| / max|b|
<= 2e-2 with f16 weights (cosine >= 0.9995 for q8_0 / q4_0).  A rollout
feeds its predictions back, so its later steps carry the error of the
earlier ones: the rollout gate is per-row cosine >= 0.999.  Causality is
checked bit for bit ("LeWorldModel Push-T", "Measured": perturbing step t
leaves every prediction before t bit-identical), and so is the independence
of candidates (a candidate alone gives the bits it gives in a batch)."""
import numpy as np
import pytest

from tests.gpu_common import COS_F16, COS_QUANT, REL_MAX_F16, assert_tokens_close, dev, host, need_cuda, orc, synth

import jepa_video_encoder_b200 as jb

pytestmark = pytest.mark.gpu

COS_ROLLOUT = 0.999


def _wc(weights="f16", **kw):
    enc = synth.small_config(synth.LEWM_VIT_TI, dim=128, heads=2, mlp=256, depth=1)
    d = dict(name="wm_small", enc=enc, dim=128, depth=2, heads=2, mlp=256, window=3, proj_hidden=256,
             pred_hidden=256, frames=3, candidates=3, weights=weights)
    d.update(kw)
    return synth.WorldModelConfig(**d)


def _model(wc, enc_weights=None):
    enc = wc.enc if enc_weights is None else wc.enc.with_(weights=enc_weights)
    table = synth.make_tensor_table(enc) + synth.make_world_model_table(wc)
    return jb.Model(enc, table, world_model=wc), table


def _W(table):
    return orc.weights_f64([t for t in table if t.name.startswith(("pred.", "enc.proj."))])


CASES = {
    # name: (config overrides, candidates)
    "t1_c1": (dict(frames=1), 1),
    "t2_c5": (dict(frames=2), 5),
    "t3_c13": (dict(frames=3), 13),            # 10 candidates a CTA: two CTAs, the second ragged
    "t3_c40_d64": (dict(dim=64, heads=1, frames=3,
                        enc=synth.small_config(synth.LEWM_VIT_TI, dim=64, heads=1, mlp=256, depth=1)), 40),
    "t3_w5_wide": (dict(window=5, frames=5, mlp=512, pred_hidden=1024), 7),
    "q8": (dict(weights="q8_0"), 4),
    "q4": (dict(weights="q4_0"), 4),
}


@pytest.mark.parametrize("name", sorted(CASES))
def test_lewm_predict_small(name):
    need_cuda()
    over, C = CASES[name]
    wc = _wc(**over)
    m, table = _model(wc)
    st, ac = synth.make_world_model_inputs(wc, candidates=C)
    got = host(m.lewm_predict(dev(st), dev(ac)))
    assert m.sync_status() == 0
    m.close()
    ref = orc.lewm_predict(wc, _W(table), st, ac)
    quant = wc.weights in ("q8_0", "q4_0")
    assert_tokens_close(got, ref, COS_QUANT if quant else COS_F16, None if quant else REL_MAX_F16, what=name)


@pytest.mark.parametrize("frames,steps,C", [(1, 6, 4), (2, 4, 11), (4, 3, 2)])
def test_lewm_rollout_small(frames, steps, C):
    need_cuda()
    wc = _wc(frames=frames, steps=steps)
    m, table = _model(wc)
    st, ac = synth.make_world_model_inputs(wc, candidates=C)
    got = host(m.lewm_rollout(dev(st), dev(ac), steps))
    assert m.sync_status() == 0
    m.close()
    ref = orc.lewm_rollout(wc, _W(table), st, ac, steps)
    assert_tokens_close(got, ref, COS_ROLLOUT, None, what=f"rollout {frames}/{steps}")
    # the first step alone is one predictor call: the f16 gate
    assert_tokens_close(got[:, :1], ref[:, :1], COS_F16, REL_MAX_F16, what="rollout step 0")


def test_lewm_causality_and_candidates_bit_exact():
    need_cuda()
    wc = _wc(frames=3)
    m, _ = _model(wc)
    st, ac = synth.make_world_model_inputs(wc, candidates=13)
    base = host(m.lewm_predict(dev(st), dev(ac)))
    rng = np.random.default_rng(1)
    for t in range(3):
        st2, ac2 = st.copy(), ac.copy()
        st2[:, t:] += rng.standard_normal(st2[:, t:].shape).astype(np.float32)
        ac2[:, t:] += rng.standard_normal(ac2[:, t:].shape).astype(np.float32)
        got = host(m.lewm_predict(dev(st2), dev(ac2)))
        assert np.array_equal(got[:, :t], base[:, :t]), f"frame {t} changed an earlier prediction"
        assert np.abs(got[:, t:] - base[:, t:]).max() > 0
    for c in (0, 9, 12):
        one = host(m.lewm_predict(dev(st[c:c + 1]), dev(ac[c:c + 1])))
        assert np.array_equal(one[0], base[c])
    # a rollout's first step equals the predictor call over the observed frames
    wr = _wc(frames=3, steps=2)
    st3, ac3 = st, np.concatenate([ac, ac[:, :1]], axis=1)
    roll = host(m.lewm_rollout(dev(st3), dev(np.ascontiguousarray(ac3)), 2))
    assert np.array_equal(roll[:, 0], base[:, 2])
    assert m.sync_status() == 0
    m.close()
    del wr


def test_lewm_full_size_step_and_rollout(capsys):
    """The LeWM Push-T world model at its size (D 192, 6 blocks, 3 heads,
    window 3): one predictor call over 3 frames of 64 candidates and a
    20-step rollout from one frame, sampled candidates against the oracle."""
    need_cuda()
    wc = synth.LEWM_WM_STEP
    table = synth.make_tensor_table(wc.enc) + synth.make_world_model_table(wc)
    m = jb.Model(wc.enc, table, world_model=wc)
    W = _W(table)
    st, ac = synth.make_world_model_inputs(wc, candidates=64)
    got = host(m.lewm_predict(dev(st), dev(ac)))
    idx = [0, 31, 63]
    ref = orc.lewm_predict(wc, W, st[idx], ac[idx])
    c1, _ = assert_tokens_close(got[idx], ref, COS_F16, REL_MAX_F16, what="lewm step")
    wr = synth.LEWM_WM_ROLLOUT
    st, ac = synth.make_world_model_inputs(wr, candidates=64)
    got = host(m.lewm_rollout(dev(st), dev(ac), wr.steps))
    ref = orc.lewm_rollout(wr, W, st[idx], ac[idx], wr.steps)
    c2, _ = assert_tokens_close(got[idx], ref, COS_ROLLOUT, None, what="lewm rollout")
    assert m.sync_status() == 0
    m.close()
    with capsys.disabled():
        print(f"\n[world model parity] step worst cos {c1.min():.7f}; 20-step rollout worst cos {c2.min():.7f} "
              f"(last step {orc.token_cosines(got[idx][:, -1], ref[:, -1]).min():.7f})")


def test_lewm_pool_projector():
    need_cuda()
    wc = _wc()
    m, table = _model(wc)
    px = synth.make_pixels(wc.enc, batch=3)
    got = host(m.encode(dev(px), pool="lewm"))
    assert m.sync_status() == 0
    m.close()
    W = orc.weights_f64(table)
    ref = orc.forward(wc.enc, W, px, pool_mode="lewm")
    assert_tokens_close(got, ref, COS_F16, REL_MAX_F16, what="lewm pool")


def test_lewm_bf16():
    need_cuda()
    wc = _wc()
    enc = wc.enc.with_(act_bf16=True)
    wc = wc.with_(enc=enc)
    table = synth.make_tensor_table(enc) + synth.make_world_model_table(wc)
    m = jb.Model(enc, table, world_model=wc)
    st, ac = synth.make_world_model_inputs(wc, candidates=5)
    got = host(m.lewm_predict(dev(st), dev(ac)))
    assert m.sync_status() == 0
    m.close()
    ref = orc.lewm_predict(wc, _W(table), st, ac)
    assert_tokens_close(got, ref, 0.9995, None, what="bf16")


def test_lewm_errors():
    need_cuda()
    wc = _wc(frames=3)
    m, _ = _model(wc)
    st, ac = synth.make_world_model_inputs(wc.with_(frames=4, window=4), candidates=2)
    with pytest.raises(jb.JepaError) as e:   # 4 frames > window 3
        m.lewm_predict(dev(st), dev(ac))
    assert e.value.status == jb._abi.ERR_SHAPE
    m.close()
    m2 = jb.Model(wc.enc, synth.make_tensor_table(wc.enc))   # no world model
    st, ac = synth.make_world_model_inputs(wc, candidates=2)
    with pytest.raises(jb.JepaError) as e:
        m2.lewm_predict(dev(st), dev(ac))
    assert e.value.status == jb._abi.ERR_ARG
    with pytest.raises(jb.JepaError) as e:
        m2.encode(dev(synth.make_pixels(wc.enc, batch=1)), pool="lewm")
    assert e.value.status == jb._abi.ERR_MISSING_TENSOR
    m2.close()


def test_lewm_timeout_path():
    """A zero wait bound makes the world-model kernel give up at its first
    wait and unwind (every role drains what it issued); the model reports
    ERR_TIMEOUT, and the next call with the normal bound gives the same bits
    as before."""
    need_cuda()
    wc = _wc(frames=1, steps=3)
    m, _ = _model(wc)
    st, ac = synth.make_world_model_inputs(wc, candidates=5)
    good = host(m.lewm_rollout(dev(st), dev(ac), wc.steps))
    assert m.sync_status() == 0
    m.set_timeout_ns(0)
    m.lewm_rollout(dev(st), dev(ac), wc.steps)
    assert m.sync_status() == jb._abi.ERR_TIMEOUT
    m.set_timeout_ns(4_000_000_000)
    again = host(m.lewm_rollout(dev(st), dev(ac), wc.steps))
    assert m.sync_status() == 0
    assert np.array_equal(good, again)
    m.close()


def test_lewm_largest_shape():
    """The largest shape the kernel accepts (state width 256 in four 64-dim
    heads, MLP and output hidden widths 1024, a 32-frame window: the shared
    memory the launch reserves): one predictor call over 32 frames, and a
    34-step rollout whose window fills up and then slides."""
    need_cuda()
    enc = synth.small_config(synth.LEWM_VIT_TI, dim=256, heads=4, mlp=256, depth=1)
    wc = _wc(enc=enc, dim=256, heads=4, mlp=1024, pred_hidden=1024, window=32, frames=32)
    m, table = _model(wc)
    W = _W(table)
    st, ac = synth.make_world_model_inputs(wc, candidates=3)
    got = host(m.lewm_predict(dev(st), dev(ac)))
    assert m.sync_status() == 0
    ref = orc.lewm_predict(wc, W, st, ac)
    assert_tokens_close(got, ref, COS_F16, REL_MAX_F16, what="largest shape, predict")
    wr = wc.with_(frames=1, steps=34)
    st, ac = synth.make_world_model_inputs(wr, candidates=2)
    got = host(m.lewm_rollout(dev(st), dev(ac), wr.steps))
    assert m.sync_status() == 0
    m.close()
    ref = orc.lewm_rollout(wr, W, st, ac, wr.steps)
    assert_tokens_close(got, ref, COS_ROLLOUT, None, what="largest shape, rollout")
    assert_tokens_close(got[:, :1], ref[:, :1], COS_F16, REL_MAX_F16, what="largest shape, rollout step 0")
