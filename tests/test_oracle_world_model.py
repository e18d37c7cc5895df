"""Pins of the oracle's LeWM world model (projector, action embedder,
AdaLN-zero causal predictor, rollout) against things other than itself:

* an independent float64 forward written with torch's library calls
  (F.layer_norm without affine, F.scaled_dot_product_attention with
  is_causal, F.silu, F.gelu, chunk(6)) -- a transposed operand, a wrong
  modulation order, a missing (1 + scale) or a mask off by one fails it;
* the AdaLN-zero closed form: with every adaLN weight and bias zero the
  gates are zero, every block is the identity, and the output is
  pred.proj(pred.norm(states + pos)) -- computed here with torch;
* exact causality (the pages' bit-exactness check, "LeWorldModel Push-T",
  "Measured"): perturbing frame t leaves every prediction of an earlier
  frame bit-identical, and candidates are independent;
* the rollout's window: a torch loop over independent torch predictor calls,
  through the growing and then sliding window."""
import numpy as np
import pytest
import torch
import torch.nn.functional as F

from jepa_video_encoder_b200 import synth
from oracle import jepa_oracle as orc


def _wc(**kw):
    enc = synth.small_config(synth.LEWM_VIT_TI, dim=128, heads=2, mlp=256, depth=1)
    d = dict(name="wm_small", enc=enc, dim=128, depth=2, heads=2, mlp=256, window=3, proj_hidden=256,
             pred_hidden=256, frames=3, candidates=3)
    d.update(kw)
    return synth.WorldModelConfig(**d)


def _W(wc):
    return orc.weights_f64(synth.make_world_model_table(wc))


def _t(a):
    return torch.tensor(np.asarray(a, np.float64), dtype=torch.float64)


def _torch_predict(wc, W, states, actions):
    D, H = wc.dim, wc.heads
    x = _t(states)
    B, T, _ = x.shape
    x = x + _t(W["pred.pos_embed"][:T])
    c = F.linear(F.silu(F.linear(_t(actions), _t(W["pred.action_embed.0.weight"]), _t(W["pred.action_embed.0.bias"]))),
                 _t(W["pred.action_embed.2.weight"]), _t(W["pred.action_embed.2.bias"]))
    for i in range(wc.depth):
        p = f"pred.blk.{i}."
        sh1, sc1, g1, sh2, sc2, g2 = F.linear(F.silu(c), _t(W[p + "adaln.weight"]), _t(W[p + "adaln.bias"])).chunk(6, -1)
        h = F.layer_norm(x, (D,), eps=wc.ln_eps) * (1 + sc1) + sh1
        q, k, v = F.linear(h, _t(W[p + "attn_qkv.weight"]), _t(W[p + "attn_qkv.bias"])).split(D, -1)
        q, k, v = (z.reshape(B, T, H, D // H).transpose(1, 2) for z in (q, k, v))
        o = F.scaled_dot_product_attention(q, k, v, is_causal=True).transpose(1, 2).reshape(B, T, D)
        x = x + g1 * F.linear(o, _t(W[p + "attn_out.weight"]), _t(W[p + "attn_out.bias"]))
        h = F.layer_norm(x, (D,), eps=wc.ln_eps) * (1 + sc2) + sh2
        u = F.gelu(F.linear(h, _t(W[p + "ffn_up.weight"]), _t(W[p + "ffn_up.bias"])))
        x = x + g2 * F.linear(u, _t(W[p + "ffn_down.weight"]), _t(W[p + "ffn_down.bias"]))
    return _torch_head(wc, W, x)


def _torch_head(wc, W, x):
    y = F.layer_norm(x, (wc.dim,), _t(W["pred.norm.weight"]), _t(W["pred.norm.bias"]), eps=wc.ln_eps)
    u = F.gelu(F.linear(y, _t(W["pred.proj.0.weight"]), _t(W["pred.proj.0.bias"])))
    return F.linear(u, _t(W["pred.proj.2.weight"]), _t(W["pred.proj.2.bias"])).numpy()


@pytest.mark.parametrize("T", [1, 2, 3])
def test_predict_matches_torch(T):
    wc = _wc(frames=T)
    W = _W(wc)
    st, ac = synth.make_world_model_inputs(wc)
    got = orc.lewm_predict(wc, W, st, ac)
    ref = _torch_predict(wc, W, st, ac)
    assert got.shape == (wc.candidates, T, wc.dim)
    np.testing.assert_allclose(got, ref, rtol=1e-11, atol=1e-11)
    # the blocks must move the state: the identity closed form is far off
    assert np.abs(got - _torch_head(wc, W, _t(st) + _t(W["pred.pos_embed"][:T]))).max() > 1e-2


def test_adaln_zero_blocks_are_identity():
    wc = _wc()
    W = dict(_W(wc))
    for i in range(wc.depth):
        W[f"pred.blk.{i}.adaln.weight"] = np.zeros_like(W[f"pred.blk.{i}.adaln.weight"])
        W[f"pred.blk.{i}.adaln.bias"] = np.zeros_like(W[f"pred.blk.{i}.adaln.bias"])
    st, ac = synth.make_world_model_inputs(wc)
    got = orc.lewm_predict(wc, W, st, ac)
    ref = _torch_head(wc, W, _t(st) + _t(W["pred.pos_embed"][:wc.frames]))
    np.testing.assert_allclose(got, ref, rtol=1e-12, atol=1e-12)


def test_causality_bit_exact_and_candidates_independent():
    wc = _wc(frames=3, candidates=2)
    W = _W(wc)
    st, ac = synth.make_world_model_inputs(wc)
    base = orc.lewm_predict(wc, W, st, ac)
    rng = np.random.default_rng(5)
    for t in range(3):
        st2, ac2 = st.copy(), ac.copy()
        st2[:, t:] += rng.standard_normal(st2[:, t:].shape).astype(np.float32)
        ac2[:, t:] += rng.standard_normal(ac2[:, t:].shape).astype(np.float32)
        got = orc.lewm_predict(wc, W, st2, ac2)
        assert np.array_equal(got[:, :t], base[:, :t])
        assert np.abs(got[:, t:] - base[:, t:]).min() > 0
    one = orc.lewm_predict(wc, W, st[1:2], ac[1:2])
    np.testing.assert_allclose(one[0], base[1], rtol=1e-13, atol=1e-13)


def test_rollout_window_against_torch_loop():
    wc = _wc(frames=1, steps=5, candidates=2)
    W = _W(wc)
    st, ac = synth.make_world_model_inputs(wc)
    got = orc.lewm_rollout(wc, W, st, ac, wc.steps)
    seq = [_t(st[:, 0]).numpy()]
    ref = []
    for s in range(wc.steps):
        lo = max(0, len(seq) - wc.window)
        win = np.stack(seq[lo:], axis=1)
        nxt = _torch_predict(wc, W, win, ac[:, lo:len(seq)])[:, -1]
        seq.append(nxt)
        ref.append(nxt)
    np.testing.assert_allclose(got, np.stack(ref, 1), rtol=1e-10, atol=1e-10)
    # step 0 is one predictor call over the single observed frame
    np.testing.assert_allclose(got[:, 0], orc.lewm_predict(wc, W, st, ac[:, :1])[:, 0], rtol=1e-13, atol=1e-13)


def test_projector_and_lewm_pool():
    wc = _wc()
    enc = wc.enc
    W = dict(orc.weights_f64(synth.make_tensor_table(enc)))
    W.update(_W(wc))
    px = synth.make_pixels(enc, batch=2)
    emb = orc.forward(enc, W, px, pool_mode="lewm")
    y = orc.encoder(enc, W, px)[:, 0]
    ref = F.linear(F.gelu(F.linear(_t(y), _t(W["enc.proj.0.weight"]), _t(W["enc.proj.0.bias"]))),
                   _t(W["enc.proj.2.weight"]), _t(W["enc.proj.2.bias"])).numpy()
    assert emb.shape == (2, wc.dim)
    np.testing.assert_allclose(emb, ref, rtol=1e-12, atol=1e-12)
