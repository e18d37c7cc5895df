"""Pins for the oracle: checks against what the pages and the mathematics fix.

Each test ties an oracle function to something other than itself -- printed
figures (tests/golden/), closed forms, library routines in float64
(torch.nn.functional on the CPU), or brute-force enumeration on tiny inputs --
so that a dropped term, a wrong sign or index or a transposed operand fails.
"""
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from jepa_video_encoder_b200 import synth
from oracle import jepa_oracle as orc

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _read_blocks(fname):
    out = []
    cur = None
    for line in open(os.path.join(GOLDEN, fname)):
        if line.startswith("bytes "):
            cur = bytes.fromhex(line.split()[1])
        elif line.startswith("values "):
            out.append((cur, [float(v) for v in line.split()[1:]]))
    return out


# ---------------------------------------------------------------- formats ----
def test_f16_decoder_all_bit_patterns():
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    raw = bits.view(np.uint8).reshape(-1, 2)
    ours = orc._f16_bits_to_f64(raw[:, 0], raw[:, 1])
    ref = bits.view(np.float16).astype(np.float64)
    same = (ours == ref) | (np.isnan(ours) & np.isnan(ref))
    assert same.all()


@pytest.mark.parametrize("fname,fn,bsz", [("q8_0_blocks.txt", orc.dequant_q8_0, 34),
                                          ("q4_0_blocks.txt", orc.dequant_q4_0, 18)])
def test_dequant_golden_blocks(fname, fn, bsz):
    blocks = _read_blocks(fname)
    assert len(blocks) >= 3
    for raw, vals in blocks:
        assert len(raw) == bsz and len(vals) == 32
        got = fn(np.frombuffer(raw, np.uint8), 32)
        assert np.array_equal(got, np.asarray(vals))


def test_block_sizes_bits_per_weight():
    gold = dict(l.split()[1:3:1] for l in open(os.path.join(GOLDEN, "levjepa_sizes.txt"))
                if l.startswith("bits_per_weight"))
    x = np.random.default_rng(0).standard_normal((3, 64)).astype(np.float32)
    q8 = synth.quantize_q8_0(x)
    q4 = synth.quantize_q4_0(x)
    assert q8.shape == (3, 2 * 34) and q4.shape == (3, 2 * 18)
    assert 34 * 8 / 32 == float(gold["q8_0"])
    assert 18 * 8 / 32 == float(gold["q4_0"])


def test_q8_0_roundtrip_error_bound():
    rng = np.random.default_rng(1)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.001, 10, (64, 1))).astype(np.float32)
    x[0, :32] = 0.0                     # all-zero block
    x[1, :32] = 0.75                    # constant block
    blocks = synth.quantize_q8_0(x)
    deq = orc.dequant_q8_0(blocks, x.size).reshape(x.shape)
    d = np.abs(x.reshape(-1, 32)).max(1) / 127.0
    err = np.abs(deq - x).reshape(-1, 32).max(1)
    # |q d16 - x| <= d/2 + 127 |d16 - d| and |d16 - d| <= d 2^-11
    assert (err <= d * (0.5 + 127 * 2.0 ** -11) + 1e-30).all()
    assert (deq[0, :32] == 0).all()
    assert np.allclose(deq[1, :32], 0.75, rtol=1e-3)


def test_q4_0_roundtrip_error_bound():
    rng = np.random.default_rng(2)
    x = (rng.standard_normal((64, 256)) * rng.uniform(0.001, 10, (64, 1))).astype(np.float32)
    blocks = synth.quantize_q4_0(x)
    deq = orc.dequant_q4_0(blocks, x.size).reshape(x.shape).reshape(-1, 32)
    xb = x.reshape(-1, 32).astype(np.float64)
    m = xb[np.arange(xb.shape[0]), np.abs(xb).argmax(1)]
    d = np.abs(m) / 8.0
    # q = floor(x/d + 8.5) is clamped to 15 only where x/d >= 7.5 (the element
    # of opposite sign to m); elsewhere the error is at most d/2 (+ fp16 scale).
    xd = xb / (m / -8.0)[:, None]
    unclamped = xd < 7.5
    err = np.abs(deq - xb)
    bound = (d * (0.5 + 8 * 2.0 ** -11))[:, None] + 1e-30
    assert (err[unclamped] <= np.broadcast_to(bound, err.shape)[unclamped]).all()
    # the largest-magnitude element is reproduced up to the fp16 rounding of d
    got_m = deq[np.arange(xb.shape[0]), np.abs(xb).argmax(1)]
    assert np.allclose(got_m, m, rtol=2.0 ** -10)


def test_levjepa_parameter_count_and_file_sizes():
    """303 M params and the published f32 / f16 / q8_0 / q4_0 file sizes of the
    LeVJEPA ViT-L/16 card follow from the tensor set (no learned pos table):
    patch_embed, cls_token, 24 x (ln1, attn_qkv, attn_out, ln2, ffn_up,
    ffn_down, with biases) and the final norm."""
    g = {}
    for l in open(os.path.join(GOLDEN, "levjepa_sizes.txt")):
        if l.startswith("#") or not l.strip():
            continue
        k, *v = l.split()
        g.setdefault(k, []).append(v)
    cfg = synth.LEVJEPA_VIT_L
    n = synth.param_count(cfg, with_pos=False)
    assert n == 303_099_904
    assert round(n / 1e6) == int(g["params_millions"][0][0])
    mib = lambda b: b / 2 ** 20
    sizes = {v[0]: float(v[1]) for v in g["file_mib"]}
    # f32 file: every tensor f32; GGUF metadata adds < 0.1 MiB on top
    assert 0 <= sizes["f32"] - mib(4 * n) < 0.1
    # f16 file: the 96 block matrices and patch_embed.weight in f16, the rest f32
    f16_params = 24 * (3 + 1 + 4 + 4) * 1024 * 1024 + 1024 * 3 * 16 * 16
    f16_bytes = 2 * f16_params + 4 * (n - f16_params)
    assert 0 <= sizes["f16"] - mib(f16_bytes) < 0.1
    for wdt in ("q8_0", "q4_0"):
        b = synth.table_bytes(cfg, wdt, with_pos=False, rest="f32")
        assert 0 <= sizes[wdt] - mib(b) < 0.1, (wdt, mib(b))
    rem = mib(4 * (n - 24 * 12 * 1024 * 1024))
    assert abs(rem - float(g["remainder_mib"][0][0])) < 0.05
    # tensor-type counts of the f16 and q8_0 files: 97 + 196 = 96 + 197 = 293 tensors
    specs = synth.tensor_specs(cfg, with_pos=False)
    assert len(specs) == 293
    n_retyped = sum(synth.is_retyped(nm) for nm, _, _ in specs)
    counts = {v[0]: dict(x.split(":") for x in v[1:]) for v in g["tensor_types"]}
    assert n_retyped == int(counts["q8_0"]["Q8_0"])
    assert len(specs) - n_retyped == int(counts["q8_0"]["F32"])
    assert n_retyped + 1 == int(counts["f16"]["F16"])          # + patch_embed.weight


# ------------------------------------------------------------- LayerNorm ----
def test_layernorm_closed_forms():
    eps = 1e-6
    D = 64
    g = np.linspace(0.5, 1.5, D)
    b = np.linspace(-0.2, 0.3, D)
    const = np.full((1, D), 3.25)
    assert np.array_equal(orc.layer_norm(const, g, b, eps), b[None, :])
    rng = np.random.default_rng(3)
    x = rng.standard_normal((5, D)) * 2.0 + 0.7
    y = orc.layer_norm(x, np.ones(D), np.zeros(D), eps)
    var = x.var(axis=1)
    assert np.allclose(y.mean(1), 0, atol=1e-14)
    assert np.allclose(y.var(1), var / (var + eps), rtol=1e-12)
    a = 0.37
    alt = np.array([[a if i % 2 == 0 else -a for i in range(D)]])
    want = np.array([[1 if i % 2 == 0 else -1 for i in range(D)]]) * a / math.sqrt(a * a + eps)
    assert np.allclose(orc.layer_norm(alt, np.ones(D), np.zeros(D), eps), want, rtol=1e-13)


def test_layernorm_vs_torch():
    rng = np.random.default_rng(4)
    x = rng.standard_normal((7, 96)) * 3
    g, b = rng.standard_normal(96), rng.standard_normal(96)
    ref = F.layer_norm(torch.from_numpy(x), (96,), torch.from_numpy(g), torch.from_numpy(b), 1e-6)
    assert np.allclose(orc.layer_norm(x, g, b, 1e-6), ref.numpy(), rtol=1e-12, atol=1e-12)


def test_gelu_exact_erf():
    x = np.linspace(-8, 8, 1001)
    ref = F.gelu(torch.from_numpy(x), approximate="none").numpy()
    assert np.allclose(orc.gelu(x), ref, rtol=1e-14, atol=1e-15)
    # x Phi(x) - (-x) Phi(-x) = x
    assert np.allclose(orc.gelu(x) - orc.gelu(-x), x, atol=1e-14)
    assert orc.gelu(np.array([0.0]))[0] == 0.0


# ------------------------------------------------------------- attention ----
def _sdpa(q, k, v, allow):
    m = None if allow is None else torch.from_numpy(allow)
    return F.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                          torch.from_numpy(v), attn_mask=m).numpy()


@pytest.mark.parametrize("mask", ["bidir", "block_causal"])
def test_attention_vs_sdpa(mask):
    rng = np.random.default_rng(5)
    n_p, pf = 12, 4
    allow = orc.allowed_keys(n_p, pf, True, mask)
    N = n_p + 1
    q, k, v = (rng.standard_normal((2, 3, N, 16)) for _ in range(3))
    got = orc.attention(q, k, v, allow)
    assert np.allclose(got, _sdpa(q, k, v, allow), rtol=1e-12, atol=1e-13)


def test_attention_explicit_loop():
    """Element by element from the definition on a tiny case."""
    rng = np.random.default_rng(6)
    N, d = 7, 4
    allow = orc.allowed_keys(6, 2, True, "block_causal")
    q, k, v = (rng.standard_normal((N, d)) for _ in range(3))
    got = orc.attention(q, k, v, allow)
    for i in range(N):
        w = [math.exp(sum(q[i, t] * k[j, t] for t in range(d)) / math.sqrt(d)) if allow[i, j] else 0.0
             for j in range(N)]
        z = sum(w)
        for c in range(d):
            assert abs(got[i, c] - sum(w[j] * v[j, c] for j in range(N)) / z) < 1e-12


def test_block_causal_predicate_enumeration():
    """The mask table equals the verbal rule, checked pair by pair."""
    T, pf = 3, 4
    for has_cls in (True, False):
        allow = orc.allowed_keys(T * pf, pf, has_cls, "block_causal")
        c = 1 if has_cls else 0
        N = T * pf + c
        for i in range(N):
            for j in range(N):
                if has_cls and i == 0:
                    want = True                       # CLS reads every token
                elif has_cls and j == 0:
                    want = False                      # no patch reads CLS
                else:
                    want = (j - c) // pf <= (i - c) // pf   # causal across slots
                assert allow[i, j] == want


# ----------------------------------------------------------- patch-embed ----
@pytest.mark.parametrize("kt,p", [(1, 4), (2, 4), (1, 3)])
def test_patch_embed_vs_conv3d(kt, p):
    rng = np.random.default_rng(7)
    B, T, H, W, D = 2, 4, 3 * p, 2 * p, 8
    pix = rng.standard_normal((B, T, 3, H, W))
    w = rng.standard_normal((D, 3, kt, p, p))
    b = rng.standard_normal(D)
    got = orc.patch_embed(pix, w, b, p, kt)
    x = torch.from_numpy(pix).permute(0, 2, 1, 3, 4)           # B, C, T, H, W
    ref = F.conv3d(x, torch.from_numpy(w), torch.from_numpy(b), stride=(kt, p, p))
    ref = ref.flatten(2).transpose(1, 2).numpy()                # B, (t', h, w), D
    assert np.allclose(got, ref, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------- whole forward ----
def _tiny(mask="block_causal", has_cls=True, frames=3, **kw):
    base = synth.EncoderConfig(
        name="tiny", dim=32, depth=2, heads=2, mlp=128, patch=4, tubelet=1,
        img_h=8, img_w=8, frames=frames, has_cls=has_cls, mask=mask, weights="f32",
        batch=2, pool="cls" if has_cls else "mean", seed=11, random_ln_affine=True)
    return base.with_(**kw)


def _torch_rotary(t, cfg):
    """3-D rotary positions on head vectors t [B, h, N, 64] (q or k), written
    as complex multiplication: the tokens' (slot, patch row, patch column)
    come from nested loops in token order; in axis group a (head dims
    20a .. 20a + 19) the complex number t[20a + 2i] + i t[20a + 2i + 1] is
    multiplied by exp(i pos_a / 10000^(i / 10)); dims 60..63 pass through."""
    pos = torch.tensor([(s, r, c) for s in range(cfg.slots) for r in range(cfg.img_h // cfg.patch)
                        for c in range(cfg.img_w // cfg.patch)], dtype=torch.float64)   # [N, 3]
    freq = 10000.0 ** (-torch.arange(10, dtype=torch.float64) / 10.0)                     # [10]
    ang = pos[:, :, None] * freq[None, None, :]                                           # [N, 3, 10]
    rot = torch.polar(torch.ones_like(ang), ang)                                          # e^{i ang}
    B, h, N, d = t.shape
    z = torch.view_as_complex(t[..., :60].reshape(B, h, N, 3, 10, 2).contiguous())
    turned = torch.view_as_real(z * rot).reshape(B, h, N, 60)
    return torch.cat([turned, t[..., 60:]], dim=-1)


def _torch_forward(cfg, W, pix):
    """An independent float64 forward from torch.nn.functional routines."""
    T = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in W.items()}
    x = torch.from_numpy(pix).permute(0, 2, 1, 3, 4)
    x = F.conv3d(x, T["enc.patch_embed.weight"], T["enc.patch_embed.bias"],
                 stride=(cfg.tubelet, cfg.patch, cfg.patch)).flatten(2).transpose(1, 2)
    if cfg.has_cls:
        x = torch.cat([T["enc.cls_token"].expand(x.shape[0], 1, -1), x], 1)
    if not cfg.rope:   # a rotary model's positions enter through q and k instead
        x = x + T["enc.pos_embed"]
    B, N, D = x.shape
    h = cfg.heads
    mask = None
    if cfg.mask == "block_causal":
        c = 1 if cfg.has_cls else 0
        idx = torch.arange(N)
        slot = torch.where(idx >= c, (idx - c) // cfg.patches_per_slot, torch.full_like(idx, -1))
        mask = (slot[None, :] <= slot[:, None]) & (slot[None, :] >= 0)
        if cfg.has_cls:
            mask[0, :] = True

    def blk(x, p):
        y = F.layer_norm(x, (D,), T[p + "ln1.weight"], T[p + "ln1.bias"], cfg.ln_eps)
        qkv = F.linear(y, T[p + "attn_qkv.weight"], T[p + "attn_qkv.bias"])
        qkv = qkv.reshape(B, -1, 3, h, D // h).permute(2, 0, 3, 1, 4)
        q, k = (_torch_rotary(qkv[0], cfg), _torch_rotary(qkv[1], cfg)) if cfg.rope else (qkv[0], qkv[1])
        o = F.scaled_dot_product_attention(q, k, qkv[2], attn_mask=mask)
        x = x + F.linear(o.transpose(1, 2).reshape(B, -1, D), T[p + "attn_out.weight"], T[p + "attn_out.bias"])
        y = F.layer_norm(x, (D,), T[p + "ln2.weight"], T[p + "ln2.bias"], cfg.ln_eps)
        y = F.gelu(F.linear(y, T[p + "ffn_up.weight"], T[p + "ffn_up.bias"]))
        return x + F.linear(y, T[p + "ffn_down.weight"], T[p + "ffn_down.bias"])

    for i in range(cfg.depth):
        x = blk(x, f"enc.blk.{i}.")
    return F.layer_norm(x, (D,), T["enc.norm.weight"], T["enc.norm.bias"], cfg.ln_eps).numpy()


@pytest.mark.parametrize("mask,has_cls,kt", [("block_causal", True, 1), ("bidir", False, 2),
                                             ("bidir", True, 1)])
def test_encoder_vs_torch_float64(mask, has_cls, kt):
    cfg = _tiny(mask=mask, has_cls=has_cls, tubelet=kt, frames=4 if kt == 2 else 3)
    W = orc.weights_f64(synth.make_tensor_table(cfg))
    pix = synth.make_pixels(cfg).astype(np.float64)
    got = orc.encoder(cfg, W, pix)
    ref = _torch_forward(cfg, W, pix)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-11)
    # pooling: CLS row, and the mean over the patch tokens only
    if has_cls:
        assert np.array_equal(orc.pool(cfg, got, "cls"), got[:, 0])
        assert np.allclose(orc.pool(cfg, got, "mean"), ref[:, 1:].mean(1), rtol=1e-12)
    else:
        assert np.allclose(orc.pool(cfg, got, "mean"), ref.mean(1), rtol=1e-12)


def test_block_causal_perturbation_bit_identical():
    """Perturbing the pixels of slot t+1 leaves every patch row of slots <= t
    bit-identical at the output; the CLS row (which reads every token) moves."""
    cfg = _tiny(frames=3)
    W = orc.weights_f64(synth.make_tensor_table(cfg))
    pix = synth.make_pixels(cfg).astype(np.float64)
    base = orc.encoder(cfg, W, pix)
    pf = cfg.patches_per_slot
    for t in range(cfg.frames - 1):
        p2 = pix.copy()
        p2[:, t + 1] += np.random.default_rng(t).standard_normal(p2[:, t + 1].shape)
        out = orc.encoder(cfg, W, p2)
        keep = 1 + (t + 1) * pf
        assert np.array_equal(out[:, 1:keep], base[:, 1:keep])
        assert not np.allclose(out[:, keep:], base[:, keep:])
        assert not np.allclose(out[:, 0], base[:, 0])


def test_single_frame_reduces_to_full_attention():
    """With one time slot the patch rows of the block-causal model with a CLS
    sink equal the bidirectional model run on the patches alone."""
    cfg = _tiny(frames=1)
    table = synth.make_tensor_table(cfg)
    W = orc.weights_f64(table)
    pix = synth.make_pixels(cfg).astype(np.float64)
    out = orc.encoder(cfg, W, pix)
    cfg2 = cfg.with_(has_cls=False, mask="bidir")
    W2 = dict(W)
    W2["enc.pos_embed"] = W["enc.pos_embed"][1:]
    del W2["enc.cls_token"]
    out2 = orc.encoder(cfg2, W2, pix)
    assert np.allclose(out[:, 1:], out2, rtol=1e-12, atol=1e-13)


def test_block_rows_matches_full_block():
    cfg = _tiny(frames=3)
    W = orc.weights_f64(synth.make_tensor_table(cfg))
    pix = synth.make_pixels(cfg).astype(np.float64)
    x = orc.embed(cfg, W, pix)
    allow = orc.encoder_allow(cfg)
    full = orc.block(x, W, "enc.blk.0.", cfg.heads, cfg.ln_eps, allow)
    rows = [0, 3, 7, 12]
    got = orc.block_rows(x[1], W, "enc.blk.0.", cfg.heads, cfg.ln_eps, allow, rows)
    assert np.allclose(got, full[1, rows], rtol=1e-12, atol=1e-13)


def _torch_head(cfg, W, tok):
    """The attentive-pool classifier from torch routines: pre-LN
    self-attention blocks (no positions), then nn.MultiheadAttention with the
    learned query, MLP and the linear classifier."""
    T = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in W.items()}
    x = torch.from_numpy(tok)
    B, N, D = x.shape
    h = cfg.heads
    for i in range(cfg.head_sa_blocks):
        p = f"head.blk.{i}."
        y = F.layer_norm(x, (D,), T[p + "ln1.weight"], T[p + "ln1.bias"], cfg.ln_eps)
        qkv = F.linear(y, T[p + "attn_qkv.weight"], T[p + "attn_qkv.bias"]).reshape(B, N, 3, h, D // h)
        qkv = qkv.permute(2, 0, 3, 1, 4)
        o = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2]).transpose(1, 2).reshape(B, N, D)
        x = x + F.linear(o, T[p + "attn_out.weight"], T[p + "attn_out.bias"])
        y = F.layer_norm(x, (D,), T[p + "ln2.weight"], T[p + "ln2.bias"], cfg.ln_eps)
        x = x + F.linear(F.gelu(F.linear(y, T[p + "ffn_up.weight"], T[p + "ffn_up.bias"])),
                         T[p + "ffn_down.weight"], T[p + "ffn_down.bias"])
    kv = F.layer_norm(x, (D,), T["head.ln_kv.weight"], T["head.ln_kv.bias"], cfg.ln_eps)
    mha = torch.nn.MultiheadAttention(D, h, batch_first=True, dtype=torch.float64)
    with torch.no_grad():
        mha.in_proj_weight.copy_(torch.cat([T["head.xattn.q.weight"], T["head.xattn.k.weight"],
                                            T["head.xattn.v.weight"]]))
        mha.in_proj_bias.copy_(torch.cat([T["head.xattn.q.bias"], T["head.xattn.k.bias"],
                                          T["head.xattn.v.bias"]]))
        mha.out_proj.weight.copy_(T["head.xattn.out.weight"])
        mha.out_proj.bias.copy_(T["head.xattn.out.bias"])
        q = T["head.query"].reshape(1, 1, D).expand(B, 1, D)
        z = q + mha(q, kv, kv, need_weights=False)[0]
        y = F.layer_norm(z, (D,), T["head.xattn.ln2.weight"], T["head.xattn.ln2.bias"], cfg.ln_eps)
        z = z + F.linear(F.gelu(F.linear(y, T["head.xattn.ffn_up.weight"], T["head.xattn.ffn_up.bias"])),
                         T["head.xattn.ffn_down.weight"], T["head.xattn.ffn_down.bias"])
        return F.linear(z[:, 0], T["head.cls.weight"], T["head.cls.bias"]).numpy()


def test_attentive_head_vs_torch_float64():
    cfg = _tiny(mask="bidir", has_cls=False, head_sa_blocks=2, n_classes=5, pool="attentive")
    W = orc.weights_f64(synth.make_tensor_table(cfg))
    rng = np.random.default_rng(9)
    tok = rng.standard_normal((2, cfg.n_tokens, cfg.dim))
    got = orc.attentive_head(cfg, W, tok)
    assert np.allclose(got, _torch_head(cfg, W, tok), rtol=1e-10, atol=1e-12)


def test_metrics_definitions():
    a = np.array([[1.0, 0.0], [0.0, 2.0]])
    b = np.array([[1.0, 1.0], [0.0, -2.0]])
    assert np.allclose(orc.token_cosines(a, b), [1 / math.sqrt(2), -1.0])
    assert orc.rel_max(a, b) == 4.0 / 2.0
    assert math.isclose(orc.rel_fro(a, b), math.sqrt(1 + 16) / math.sqrt(6))


# ------------------------------------------------ 3-D rotary positions (R18) --
def _rope_cfg():
    return synth.VJEPA2_LONG.with_(name="rope_pin", dim=128, depth=1, heads=2, mlp=256, frames=6,
                                   img_h=48, img_w=64, patch=16, rope=True)


def test_rope_positions_enumerate_slot_row_column():
    cfg = _rope_cfg()
    want = [(t, y, x) for t in range(cfg.slots) for y in range(cfg.img_h // cfg.patch)
            for x in range(cfg.img_w // cfg.patch)]
    assert np.array_equal(orc.rope_positions(cfg), np.array(want))


def test_rope_identity_at_origin_and_last_dims_untouched():
    rng = np.random.default_rng(30)
    x = rng.standard_normal((2, 7, 64))
    assert np.array_equal(orc.rope(x, np.zeros((7, 3), int)), x)
    pos = rng.integers(0, 40, (7, 3))
    y = orc.rope(x, pos)
    assert np.array_equal(y[..., 60:], x[..., 60:])  # 64 - 3 * 20 dimensions are not turned
    pairs = lambda t: np.hypot(t[..., 0:60:2], t[..., 1:60:2])
    assert np.allclose(pairs(y), pairs(x), rtol=1e-13, atol=0)  # every pair keeps its length


def test_rope_rotation_closed_forms():
    """Pair i = 0 of each axis turns by pos radians; pair i = 5 by pos / 100
    (10000^(-10/20) = 1/100); a unit vector on the pair's first dimension
    goes to (cos, sin) of that angle."""
    for a in range(3):
        for i, scale in ((0, 1.0), (5, 0.01)):
            j = 20 * a + 2 * i
            e = np.zeros((1, 64))
            e[0, j] = 1.0
            pos = np.zeros((1, 3), int)
            pos[0, a] = 7
            y = orc.rope(e, pos)
            assert y[0, j] == pytest.approx(math.cos(7 * scale), abs=1e-15)
            assert y[0, j + 1] == pytest.approx(math.sin(7 * scale), abs=1e-15)
            assert np.count_nonzero(np.abs(y) > 1e-15) <= 2


def test_rope_composition_adds_positions():
    rng = np.random.default_rng(31)
    x = rng.standard_normal((5, 64))
    p, q = rng.integers(0, 20, (5, 3)), rng.integers(0, 20, (5, 3))
    assert np.allclose(orc.rope(orc.rope(x, p), q), orc.rope(x, p + q), rtol=0, atol=1e-12)


def test_rope_scores_depend_on_position_differences_only():
    rng = np.random.default_rng(32)
    qv, kv = rng.standard_normal((1, 64)), rng.standard_normal((1, 64))
    for _ in range(5):
        p, pk, c = rng.integers(0, 30, (1, 3)), rng.integers(0, 30, (1, 3)), rng.integers(0, 30, (1, 3))
        s1 = (orc.rope(qv, p) @ orc.rope(kv, pk).T).item()
        s2 = (orc.rope(qv, p + c) @ orc.rope(kv, pk + c).T).item()
        assert s1 == pytest.approx(s2, rel=1e-11, abs=1e-12)


@pytest.mark.parametrize("mask", ["bidir", "block_causal"])
def test_rotary_encoder_vs_torch_float64(mask):
    """The whole rotary encoder (no positional table, q and k turned after
    their bias in every block, v untouched) against the torch forward whose
    rotation is a complex multiplication over enumerated positions."""
    cfg = _rope_cfg().with_(depth=2, mask=mask, random_ln_affine=True, batch=2)
    table = synth.make_tensor_table(cfg)
    assert "enc.pos_embed" not in synth.table_dict(table)
    W = orc.weights_f64(table)
    pix = synth.make_pixels(cfg).astype(np.float64)
    got = orc.encoder(cfg, W, pix)
    ref = _torch_forward(cfg, W, pix)
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-11)
    # the rotation matters: the same weights without it give another result
    assert not np.allclose(got, _torch_forward(cfg.with_(rope=False), dict(W, **{
        "enc.pos_embed": np.zeros((cfg.n_tokens, cfg.dim))}), pix), rtol=1e-6, atol=1e-8)


def test_rotary_model_head_has_no_positions():
    """A rotary encoder with the attentive head: the head's self-attention
    blocks and its cross-attention take no rotation."""
    cfg = _rope_cfg().with_(depth=1, head_sa_blocks=1, n_classes=5, pool="attentive",
                            random_ln_affine=True, batch=2)
    W = orc.weights_f64(synth.make_tensor_table(cfg))
    pix = synth.make_pixels(cfg).astype(np.float64)
    got = orc.forward(cfg, W, pix)
    ref = _torch_head(cfg, W, _torch_forward(cfg, W, pix))
    assert np.allclose(got, ref, rtol=1e-10, atol=1e-12)


# ------------------------------------------------------- masked predictor --
def _pred_cfg(**kw):
    enc = synth.small_config(synth.VJEPA2_SSV2, frames=4, img_h=32, img_w=48, dim=128, heads=2, mlp=256)
    base = synth.PredictorConfig(name="pred_pin", enc=enc, dim=64, depth=2, heads=2, mlp=128, ctx="even",
                                 tgt="odd", weights="f32", batch=2, random_ln_affine=True)
    return base.with_(**kw)


def _torch_predictor(pc, W, tokens, ctx_idx, tgt_idx):
    """The predictor from torch routines: rows assembled with index_select /
    cat, blocks with scaled_dot_product_attention (head dim 32 here)."""
    T = {k: torch.from_numpy(np.ascontiguousarray(v)) for k, v in W.items()}
    tok = torch.from_numpy(tokens)
    ci, ti = torch.from_numpy(np.asarray(ctx_idx)), torch.from_numpy(np.asarray(tgt_idx))
    D, h = pc.dim, pc.heads
    ctx = F.linear(tok.index_select(1, ci), T["pred.embed.weight"], T["pred.embed.bias"]) + \
        T["pred.pos_embed"].index_select(0, ci)
    tgt = (T["pred.mask_tokens"] + T["pred.pos_embed"].index_select(0, ti)).expand(tok.shape[0], -1, -1)
    x = torch.cat([ctx, tgt], 1)
    B, L, _ = x.shape
    for i in range(pc.depth):
        p = f"pred.blk.{i}."
        y = F.layer_norm(x, (D,), T[p + "ln1.weight"], T[p + "ln1.bias"], pc.ln_eps)
        qkv = F.linear(y, T[p + "attn_qkv.weight"], T[p + "attn_qkv.bias"]).reshape(B, L, 3, h, D // h)
        qkv = qkv.permute(2, 0, 3, 1, 4)
        o = F.scaled_dot_product_attention(qkv[0], qkv[1], qkv[2]).transpose(1, 2).reshape(B, L, D)
        x = x + F.linear(o, T[p + "attn_out.weight"], T[p + "attn_out.bias"])
        y = F.layer_norm(x, (D,), T[p + "ln2.weight"], T[p + "ln2.bias"], pc.ln_eps)
        x = x + F.linear(F.gelu(F.linear(y, T[p + "ffn_up.weight"], T[p + "ffn_up.bias"])),
                         T[p + "ffn_down.weight"], T[p + "ffn_down.bias"])
    y = F.layer_norm(x[:, len(ctx_idx):], (D,), T["pred.norm.weight"], T["pred.norm.bias"], pc.ln_eps)
    return F.linear(y, T["pred.proj.weight"], T["pred.proj.bias"]).numpy()


@pytest.mark.parametrize("ctx,tgt", [("even", "odd"), ("all", "all"), ("first_half", "second_half")])
def test_predictor_vs_torch_float64(ctx, tgt):
    pc = _pred_cfg(ctx=ctx, tgt=tgt)
    assert pc.head_dim == 32
    W = orc.weights_f64(synth.make_predictor_table(pc))
    tok = synth.make_predictor_tokens(pc).astype(np.float64)
    got = orc.predictor(pc, W, tok, pc.ctx_idx, pc.tgt_idx)
    assert got.shape == (pc.batch, len(pc.tgt_idx), pc.enc.dim)
    assert np.allclose(got, _torch_predictor(pc, W, tok, pc.ctx_idx, pc.tgt_idx), rtol=1e-10, atol=1e-12)


def test_predictor_permutation_properties():
    """Attention reads the rows as a set and every row carries its own
    position: shuffling the context list leaves the predictions unchanged,
    shuffling the target list shuffles them the same way."""
    pc = _pred_cfg()
    W = orc.weights_f64(synth.make_predictor_table(pc))
    tok = synth.make_predictor_tokens(pc).astype(np.float64)
    ctx, tgt = pc.ctx_idx, pc.tgt_idx
    base = orc.predictor(pc, W, tok, ctx, tgt)
    rng = np.random.default_rng(40)
    assert np.allclose(orc.predictor(pc, W, tok, rng.permutation(ctx), tgt), base, rtol=1e-11, atol=1e-13)
    perm = rng.permutation(len(tgt))
    assert np.allclose(orc.predictor(pc, W, tok, ctx, tgt[perm]), base[:, perm], rtol=1e-11, atol=1e-13)
    # a target's prediction depends on its own position row, not only on the mask token
    W2 = dict(W)
    W2["pred.pos_embed"] = W["pred.pos_embed"].copy()
    W2["pred.pos_embed"][tgt[0]] += 0.5 * rng.standard_normal(pc.dim)   # (a constant shift LayerNorm removes)
    moved = orc.predictor(pc, W2, tok, ctx, tgt)
    assert not np.allclose(moved[:, 0], base[:, 0])
    assert np.abs(moved[:, 1:] - base[:, 1:]).max() > 1e-9      # the other rows read that row


def test_predictor_with_zero_blocks_is_norm_and_projection():
    """With every block's projection weights and biases zero the blocks are
    the identity (each residual branch adds 0): a target's prediction is
    pred.proj(pred.norm(mask token + its position row)), whatever the
    context."""
    pc = _pred_cfg()
    W = orc.weights_f64(synth.make_predictor_table(pc))
    for n in list(W):
        if n.startswith("pred.blk.") and (n.endswith("attn_out.weight") or n.endswith("attn_out.bias") or
                                          n.endswith("ffn_down.weight") or n.endswith("ffn_down.bias")):
            W[n] = np.zeros_like(W[n])
    tok = synth.make_predictor_tokens(pc).astype(np.float64)
    got = orc.predictor(pc, W, tok, pc.ctx_idx, pc.tgt_idx)
    z = W["pred.mask_tokens"][0] + W["pred.pos_embed"][pc.tgt_idx]
    mu = z.mean(-1, keepdims=True)
    sd = np.sqrt(((z - mu) ** 2).mean(-1, keepdims=True) + pc.ln_eps)
    want = ((z - mu) / sd * W["pred.norm.weight"] + W["pred.norm.bias"]) @ W["pred.proj.weight"].T + \
        W["pred.proj.bias"]
    assert np.allclose(got, np.broadcast_to(want, got.shape), rtol=1e-12, atol=1e-13)
