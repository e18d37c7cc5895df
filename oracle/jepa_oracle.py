"""Oracle: a plain, slow, float64 CPU forward of the JEPA ViT encoder.

TEST INFRASTRUCTURE ONLY.  Nothing on the product path imports this module;
only ``tests/``, ``__graft_entry__.smoke()`` and the ``cpu_baseline`` /
``--impl reference`` legs of ``bench.py`` may call it.  It shares no code with
the CUDA path: it reads the same seeded tensor table and pixels and nothing
else.

Every step is the textbook definition written out in numpy float64 (library
matmul as the only primitive), in the order the pages describe the model:

* tubelet patch-embed: a conv with stride = kernel, i.e. unfold + matmul
  (model cards "LeVJEPA ViT-L/16" and "V-JEPA 2 ViT-L/16 SSv2 classifier":
  patch 16, tubelet 1 / 2; benchmarks page, "What the milliseconds are": the
  engine unfolds patches before the graph);
* an additive positional table and a CLS row where the model has one
  ("LeVJEPA" card, intro; "Quantization" page, "The rule": enc.pos_embed,
  enc.cls_token);
* pre-LN blocks ln1 -> attn_qkv -> attention -> attn_out -> +res, ln2 ->
  ffn_up -> GELU -> ffn_down -> +res ("Quantization" page, "The rule": the
  tensor set of a block);
* the block-causal mask of LeVJEPA: bidirectional inside a frame, causal
  across frames, CLS a read-only sink ("LeVJEPA" card, intro);
* the final ``norm`` before last_hidden_state ("Quantization" page, "Reading
  the numbers");
* pooling mean / cls / none / lewm ("LeVJEPA" card, "Run it": --pool) and the
  attentive-pool classifier: 3 self-attention blocks over the tokens, one
  cross-attention query, MLP, linear ("jepa.cpp — measured benchmarks",
  "Attentive-pool head");
* the LeWM world model: the projector of the CLS row and the AdaLN-zero
  causal predictor with its rollout ("LeWorldModel Push-T" card, intro;
  readings in its section below);
* q8_0 / q4_0 dequantisation: value = q*d and (q-8)*d per 32-element block
  with one fp16 scale (ggml's published block formats; the "Quantization"
  page, "File sizes", gives their 8.5 / 4.5 bits per weight).

Where the pages are silent this module takes the plainest reading: LayerNorm
eps from the config (1e-6 on every workload), GELU in its exact erf form, the
attention scale 1/sqrt(d_h), attn_qkv's output columns ordered [q | k | v]
with head h at columns h*d_h .. h*d_h + d_h - 1 of each, the mean pool over
the patch tokens only (CLS excluded), and an out-projection plus an ln2 in the
head's cross-attention block.
"""
from __future__ import annotations

import math
import os
import queue
from concurrent.futures import ThreadPoolExecutor
from typing import Dict, Iterable, Optional, Sequence

import numpy as np
from scipy.special import erf as _erf
from threadpoolctl import threadpool_limits

# ggml dtype ids (the tensor table's own numbering)
DT_F32, DT_F16, DT_Q4_0, DT_Q8_0 = 0, 1, 2, 8


# ---------------------------------------------------------------------------
# Weight decoding
# ---------------------------------------------------------------------------
def _f16_bits_to_f64(lo: np.ndarray, hi: np.ndarray) -> np.ndarray:
    """IEEE binary16 (little-endian byte pair) -> float64, decoded from the
    bit fields: sign, 5-bit exponent (bias 15), 10-bit fraction."""
    bits = lo.astype(np.uint32) | (hi.astype(np.uint32) << 8)
    sign = np.where(bits >> 15, -1.0, 1.0)
    e = ((bits >> 10) & 0x1F).astype(np.int64)
    f = (bits & 0x3FF).astype(np.float64)
    normal = sign * np.ldexp(1.0 + f / 1024.0, e - 15)
    sub = sign * np.ldexp(f / 1024.0, -14)
    out = np.where(e == 0, sub, normal)
    out = np.where(e == 31, np.where(f == 0, sign * np.inf, np.nan), out)
    return out


def dequant_q8_0(blocks: np.ndarray, n: int) -> np.ndarray:
    """q8_0: each 34-byte block = fp16 scale d, then 32 signed bytes q;
    element value q*d (ggml's published q8_0 block format; its 34 bytes per
    32 weights are the 8.5 bits per weight of the "Quantization" page, "File
    sizes")."""
    b = np.asarray(blocks, np.uint8).reshape(-1, 34)
    d = _f16_bits_to_f64(b[:, 0], b[:, 1])
    q = b[:, 2:].view(np.int8).astype(np.float64)
    out = (q * d[:, None]).reshape(-1)
    assert out.size == n
    return out


def dequant_q4_0(blocks: np.ndarray, n: int) -> np.ndarray:
    """q4_0 (ggml's published block format, value (q-8)*d; 18 bytes per 32
    weights = the 4.5 bits per weight of the "Quantization" page, "File
    sizes"): each 18-byte block = fp16 scale d, then 16 bytes; byte j carries
    element j (low nibble) and element j+16 (high nibble); value (q-8)*d."""
    b = np.asarray(blocks, np.uint8).reshape(-1, 18)
    d = _f16_bits_to_f64(b[:, 0], b[:, 1])
    nib = b[:, 2:]
    q = np.empty((b.shape[0], 32), np.float64)
    q[:, :16] = (nib & 0x0F).astype(np.float64)
    q[:, 16:] = (nib >> 4).astype(np.float64)
    out = ((q - 8.0) * d[:, None]).reshape(-1)
    assert out.size == n
    return out


def tensor_f64(t) -> np.ndarray:
    """A tensor-table entry -> float64 values in its PyTorch-order shape."""
    shape = tuple(t.shape)
    n = int(np.prod(shape))
    if t.dtype == DT_F32:
        return np.asarray(t.data, np.float32).astype(np.float64).reshape(shape)
    if t.dtype == DT_F16:
        raw = np.ascontiguousarray(t.data).view(np.uint8).reshape(-1, 2)
        return _f16_bits_to_f64(raw[:, 0], raw[:, 1]).reshape(shape)
    if t.dtype == DT_Q8_0:
        return dequant_q8_0(t.data, n).reshape(shape)
    if t.dtype == DT_Q4_0:
        return dequant_q4_0(t.data, n).reshape(shape)
    raise ValueError(f"unknown dtype {t.dtype} for {t.name}")


def weights_f64(table) -> Dict[str, np.ndarray]:
    return {t.name: tensor_f64(t) for t in table}


# ---------------------------------------------------------------------------
# Building blocks (each the plain definition)
# ---------------------------------------------------------------------------
def patchify(pixels: np.ndarray, patch: int, tubelet: int) -> np.ndarray:
    """[B, T, 3, H, W] -> [B, N_p, 3*kt*p*p].  Token order: time slot t',
    then patch row, then patch column.  Vector order (c, dt, kh, kw), the
    row-major flattening of a conv weight [D, 3, kt, p, p]."""
    B, T, C, H, W = pixels.shape
    kt, p = tubelet, patch
    x = np.asarray(pixels, np.float64).reshape(B, T // kt, kt, C, H // p, p, W // p, p)
    # axes: b, t', dt, c, hp, kh, wp, kw  ->  b, t', hp, wp, c, dt, kh, kw
    x = x.transpose(0, 1, 4, 6, 3, 2, 5, 7)
    return x.reshape(B, (T // kt) * (H // p) * (W // p), C * kt * p * p)


def patch_embed(pixels, w_pe, b_pe, patch, tubelet) -> np.ndarray:
    """Conv3d with stride = kernel = (kt, p, p) written as unfold + matmul
    (the cards' patch 16 / tubelet 1 or 2 embedding; the benchmarks page,
    "What the milliseconds are", unfolds patches before the graph)."""
    cols = patchify(pixels, patch, tubelet)
    D = w_pe.shape[0]
    return cols @ w_pe.reshape(D, -1).T + b_pe


def layer_norm(x: np.ndarray, gamma, beta, eps: float) -> np.ndarray:
    """(x - mean) / sqrt(var + eps) * gamma + beta over the last axis, with
    the biased variance: the ln1 / ln2 / norm tensors of the "Quantization"
    page, "The rule" (eps is a reading: the pages give none)."""
    x = np.asarray(x, np.float64)
    mu = x.mean(axis=-1, keepdims=True)
    var = ((x - mu) ** 2).mean(axis=-1, keepdims=True)
    return (x - mu) / np.sqrt(var + eps) * gamma + beta


def gelu(x: np.ndarray) -> np.ndarray:
    """Exact GELU: x * Phi(x) = 0.5 x (1 + erf(x / sqrt 2)), the activation
    between ffn_up and ffn_down (the pages name no variant; the erf form is
    the reading taken)."""
    return 0.5 * x * (1.0 + _erf(x / math.sqrt(2.0)))


def linear(x, w, b) -> np.ndarray:
    """y = x W^T + b with W in PyTorch [out, in] order."""
    y = np.asarray(x, np.float64) @ w.T
    return y + b if b is not None else y


def allowed_keys(n_patches: int, patches_per_slot: int, has_cls: bool,
                 mask: str) -> np.ndarray:
    """Boolean [N, N]: may query i read key j?

    bidir: every pair.  block_causal (LeVJEPA): a patch of time slot s reads
    the patches of slots <= s (bidirectional inside a slot, causal across
    slots); the CLS row, when present, reads every token including itself and
    no patch reads CLS (the read-only sink) -- "LeVJEPA ViT-L/16 (VideoMix)"
    card, intro."""
    c = 1 if has_cls else 0
    N = n_patches + c
    if mask == "bidir":
        return np.ones((N, N), bool)
    if mask != "block_causal":
        raise ValueError(mask)
    slot = np.arange(n_patches) // patches_per_slot
    allow = np.zeros((N, N), bool)
    allow[c:, c:] = slot[None, :] <= slot[:, None]
    if has_cls:
        allow[0, :] = True
    return allow


def _attention_slice(q, k, v, blocked, s):
    """One (clip, head) slice of the attention below, scores in buffer s."""
    np.matmul(q, np.swapaxes(k, -1, -2), out=s)
    s /= math.sqrt(q.shape[-1])
    if blocked is not None:
        np.copyto(s, -np.inf, where=blocked)
    s -= s.max(axis=-1, keepdims=True)
    np.exp(s, out=s)
    s /= s.sum(axis=-1, keepdims=True)
    return s @ v


def attention(q, k, v, allow: Optional[np.ndarray]) -> np.ndarray:
    """softmax(q k^T / sqrt(d) + mask) v for q [.., Nq, d], k/v [.., Nk, d];
    ``allow`` [Nq, Nk] boolean (None = every pair).  The row max is
    subtracted before exp (exact in the softmax's definition).

    Evaluated one (clip, head) slice at a time, each in a score buffer of its
    own thread, so that a long clip (8192 tokens: 512 MB per score matrix)
    holds only a few score matrices; the slices are independent, and every
    element goes through the same operations in the same order as the
    vectorised definition."""
    q, k, v = (np.asarray(t, np.float64) for t in (q, k, v))
    lead = q.shape[:-2]
    out = np.empty(lead + (q.shape[-2], v.shape[-1]))
    blocked = None if allow is None else ~np.asarray(allow, bool)
    idx = list(np.ndindex(*lead))
    nq, nk = q.shape[-2], k.shape[-2]
    workers = max(1, min(len(idx), os.cpu_count() or 1, (8 << 30) // max(1, 8 * nq * nk)))
    if workers == 1 or nq * nk < (1 << 20):
        s = np.empty((nq, nk))
        for i in idx:
            out[i] = _attention_slice(q[i], k[i], v[i], blocked, s)
        return out
    bufs = queue.SimpleQueue()
    for _ in range(workers):
        bufs.put(np.empty((nq, nk)))

    def one(i):
        s = bufs.get()
        out[i] = _attention_slice(q[i], k[i], v[i], blocked, s)
        bufs.put(s)

    # each slice's matrix products on one BLAS thread; the slices in parallel
    with threadpool_limits(limits=1, user_api="blas"):
        with ThreadPoolExecutor(max_workers=workers) as ex:
            list(ex.map(one, idx))
    return out


def split_heads(x, heads):
    """[B, N, h*d] -> [B, h, N, d]  (head hd owns columns hd*d .. hd*d+d-1)."""
    B, N, C = x.shape
    return x.reshape(B, N, heads, C // heads).transpose(0, 2, 1, 3)


def merge_heads(x):
    B, h, N, d = x.shape
    return x.transpose(0, 2, 1, 3).reshape(B, N, h * d)


# ---------------------------------------------------------------------------
# 3-D rotary position embedding of the V-JEPA 2 encoders (the "Quantization"
# page, "How the accuracy was measured", says that reference graph's encoder
# uses 3-D rotary embeddings;
# the pages give no formula, so the plainest 3-D extension of rotary
# embeddings is read here): the head dimensions are split into three groups
# of g = 2*floor(d_h/6), one per axis (time slot, patch row, patch column);
# in group a the pair of dimensions (a*g + 2i, a*g + 2i + 1) is turned by the
# angle pos_a * 10000^(-2i/g); the last d_h - 3g dimensions are not turned.
# ---------------------------------------------------------------------------
ROPE_BASE = 10000.0


def rope_positions(cfg) -> np.ndarray:
    """[N, 3] integer (slot, patch row, patch column) of every token; the
    rotary models have no CLS row."""
    pw = cfg.img_w // cfg.patch
    ppf = cfg.patches_per_slot
    n = np.arange(cfg.n_patches)
    return np.stack([n // ppf, (n % ppf) // pw, (n % ppf) % pw], axis=1)


def rope(x: np.ndarray, pos: np.ndarray, base: float = ROPE_BASE) -> np.ndarray:
    """Rotate the head vectors x [..., N, d_h] of tokens at positions pos [N, 3]
    (the 3-D rotary scheme read above for the V-JEPA 2 encoders)."""
    d = x.shape[-1]
    g = 2 * (d // 6)
    out = np.array(x, np.float64, copy=True)
    for a in range(3):
        for i in range(g // 2):
            th = pos[:, a].astype(np.float64) * base ** (-2.0 * i / g)
            c, s = np.cos(th), np.sin(th)
            j = a * g + 2 * i
            x0, x1 = x[..., j], x[..., j + 1]
            out[..., j] = x0 * c - x1 * s
            out[..., j + 1] = x0 * s + x1 * c
    return out


def block(x, W: Dict[str, np.ndarray], prefix: str, heads: int, eps: float,
          allow: Optional[np.ndarray], rope_pos: Optional[np.ndarray] = None) -> np.ndarray:
    """One pre-LN transformer block ("Quantization" page, "The rule": ln1,
    attn_qkv, attn_out, ln2, ffn_up, ffn_down).  attn_qkv's output columns are
    [q | k | v], each head-major (head hd at hd*d_h ...).  With rope_pos, q and
    k are rotated (after their bias) before the attention."""
    D = x.shape[-1]
    y = layer_norm(x, W[prefix + "ln1.weight"], W[prefix + "ln1.bias"], eps)
    qkv = linear(y, W[prefix + "attn_qkv.weight"], W[prefix + "attn_qkv.bias"])
    q, k, v = (split_heads(qkv[..., i * D:(i + 1) * D], heads) for i in range(3))
    if rope_pos is not None:
        q, k = rope(q, rope_pos), rope(k, rope_pos)
    o = merge_heads(attention(q, k, v, allow))
    x = x + linear(o, W[prefix + "attn_out.weight"], W[prefix + "attn_out.bias"])
    y = layer_norm(x, W[prefix + "ln2.weight"], W[prefix + "ln2.bias"], eps)
    h = gelu(linear(y, W[prefix + "ffn_up.weight"], W[prefix + "ffn_up.bias"]))
    return x + linear(h, W[prefix + "ffn_down.weight"], W[prefix + "ffn_down.bias"])


def embed(cfg, W, pixels) -> np.ndarray:
    """Patch-embed, prepend CLS (when the model has one), add pos_embed (the
    rotary models have none: their positions enter the attention); the
    enc.cls_token / enc.pos_embed tensors of the "Quantization" page, "The
    rule"."""
    x = patch_embed(pixels, W["enc.patch_embed.weight"], W["enc.patch_embed.bias"],
                    cfg.patch, cfg.tubelet)
    if cfg.has_cls:
        cls = np.broadcast_to(W["enc.cls_token"], (x.shape[0], 1, x.shape[-1]))
        x = np.concatenate([cls, x], axis=1)
    if getattr(cfg, "rope", False):
        return x
    return x + W["enc.pos_embed"][None]


def encoder_allow(cfg) -> Optional[np.ndarray]:
    if cfg.mask == "bidir":
        return None
    return allowed_keys(cfg.n_patches, cfg.patches_per_slot, cfg.has_cls, cfg.mask)


def encoder(cfg, W, pixels, layers: Optional[int] = None,
            return_residuals: bool = False):
    """Full encoder: embed, ``depth`` blocks, final LayerNorm ->
    last_hidden_state [B, N, D] (the final ``norm``: "Quantization" page,
    "Reading the numbers")."""
    allow = encoder_allow(cfg)
    rope_pos = rope_positions(cfg) if getattr(cfg, "rope", False) else None
    x = embed(cfg, W, pixels)
    res = [x]
    for i in range(cfg.depth if layers is None else layers):
        x = block(x, W, f"enc.blk.{i}.", cfg.heads, cfg.ln_eps, allow, rope_pos)
        res.append(x)
    y = layer_norm(x, W["enc.norm.weight"], W["enc.norm.bias"], cfg.ln_eps)
    return (y, res) if return_residuals else y


def pool(cfg, y: np.ndarray, mode: str) -> np.ndarray:
    """cls: the CLS row; mean: mean over the patch tokens (CLS excluded);
    none: the full token map ("LeVJEPA" card, "Run it": --pool; which tokens
    the mean covers is a reading)."""
    if mode == "none":
        return y
    if mode == "cls":
        if not cfg.has_cls:
            raise ValueError("cls pooling needs a CLS token")
        return y[:, 0]
    if mode == "mean":
        return y[:, 1 if cfg.has_cls else 0:].mean(axis=1)
    raise ValueError(mode)


def attentive_head(cfg, W, tokens: np.ndarray) -> np.ndarray:
    """Attentive-pool classifier: ``head_sa_blocks`` pre-LN self-attention
    blocks over the tokens, then one cross-attention block whose single query
    is the learned ``head.query`` (not normalised): q = W_q query + b_q;
    k, v = W_{k,v} LN_kv(tokens) + b; z = query + W_out attn + b_out;
    z += MLP(LN2(z)); logits = W_cls z + b_cls ("jepa.cpp — measured
    benchmarks", "Attentive-pool head": three self-attention blocks, one
    cross-attention query, MLP, linear; the tensors, head.query, ln_kv,
    head.xattn.{q,k,v,ffn_up,ffn_down} and head.cls, from the "Quantization"
    page, "The rule"; the cross-attention out-projection is a reading)."""
    x = tokens
    for i in range(cfg.head_sa_blocks):
        x = block(x, W, f"head.blk.{i}.", cfg.heads, cfg.ln_eps, None)
    B, N, D = x.shape
    kv_in = layer_norm(x, W["head.ln_kv.weight"], W["head.ln_kv.bias"], cfg.ln_eps)
    qv = linear(W["head.query"][None, None, :], W["head.xattn.q.weight"], W["head.xattn.q.bias"])
    qv = np.broadcast_to(qv, (B, 1, D))
    k = linear(kv_in, W["head.xattn.k.weight"], W["head.xattn.k.bias"])
    v = linear(kv_in, W["head.xattn.v.weight"], W["head.xattn.v.bias"])
    o = merge_heads(attention(split_heads(qv, cfg.heads), split_heads(k, cfg.heads),
                              split_heads(v, cfg.heads), None))
    z = W["head.query"][None, None, :] + linear(o, W["head.xattn.out.weight"],
                                                W["head.xattn.out.bias"])
    h = layer_norm(z, W["head.xattn.ln2.weight"], W["head.xattn.ln2.bias"], cfg.ln_eps)
    h = gelu(linear(h, W["head.xattn.ffn_up.weight"], W["head.xattn.ffn_up.bias"]))
    z = z + linear(h, W["head.xattn.ffn_down.weight"], W["head.xattn.ffn_down.bias"])
    return linear(z[:, 0], W["head.cls.weight"], W["head.cls.bias"])


def forward(cfg, W, pixels, pool_mode: Optional[str] = None) -> np.ndarray:
    """Encoder + output selected by ``pool_mode`` (default: the config's)."""
    mode = cfg.pool if pool_mode is None else pool_mode
    y = encoder(cfg, W, pixels)
    if mode == "attentive":
        return attentive_head(cfg, W, y)
    if mode == "lewm":
        return lewm_project(W, pool(cfg, y, "cls"))
    return pool(cfg, y, mode)


# ---------------------------------------------------------------------------
# Masked predictor of the V-JEPA 2 encoders ("jepa.cpp — measured
# benchmarks", "Masked predictor": a 12-layer, 384-wide predictor that reads
# context tokens and predicts target tokens, head dim 32; the "Quantization"
# page, "The rule", names its tensors: pred.embed (the context projection),
# pred.mask_tokens, pred.pos_embed, predictor blocks with the encoder
# block's tensor set, pred.proj).  Readings where the pages are silent: the
# sequence is [context rows | target rows]; a context row is
# pred.embed(token) plus the positional row of its token index; a target row
# is the mask token plus the positional row of its token index; attention is
# bidirectional over the whole sequence; the final norm (pred.norm) and
# pred.proj map the target rows back to the encoder's width.
# ---------------------------------------------------------------------------
def predictor(pc, W, tokens: np.ndarray, ctx_idx: Sequence[int], tgt_idx: Sequence[int]) -> np.ndarray:
    """tokens [B, N, D_enc] (the encoder's output) -> predictions [B, N_tgt,
    D_enc] for the target indices."""
    ctx_idx, tgt_idx = np.asarray(ctx_idx), np.asarray(tgt_idx)
    tokens = np.asarray(tokens, np.float64)
    B = tokens.shape[0]
    pos = W["pred.pos_embed"]
    ctx = linear(tokens[:, ctx_idx], W["pred.embed.weight"], W["pred.embed.bias"]) + pos[ctx_idx][None]
    tgt = np.broadcast_to(W["pred.mask_tokens"][0] + pos[tgt_idx], (B, len(tgt_idx), pos.shape[1]))
    x = np.concatenate([ctx, tgt], axis=1)
    for i in range(pc.depth):
        x = block(x, W, f"pred.blk.{i}.", pc.heads, pc.ln_eps, None)
    y = layer_norm(x[:, len(ctx_idx):], W["pred.norm.weight"], W["pred.norm.bias"], pc.ln_eps)
    return linear(y, W["pred.proj.weight"], W["pred.proj.bias"])


# ---------------------------------------------------------------------------
# LeWM world model ("LeWorldModel Push-T" card, intro: the encoder's CLS token
# is projected to a world-model state, and six AdaLN-zero causal blocks
# conditioned on a 10-d action roll that state forward; "Measured": the
# projector and predictor MLPs are BatchNorm-folded; "Quantization" page,
# "The rule": enc.proj.* (the projector) and pred.proj.0 / pred.proj.2 are
# re-typed matrices, pred.blk.*.adaln.* and pred.action_embed.* stay f32;
# benchmarks page, "LeWM world model": one predictor call covers a window of
# 3 frames of 192-d states, a rollout grows that window one predicted state
# per step).  Readings where the pages are silent:
#   * projector: emb = W2 GELU(W1 cls + b1) + b2 on the final-normed CLS row
#     (BatchNorm folded into W1, b1);
#   * action embedding: c_t = W2 SiLU(W1 a_t + b1) + b2 (pred.action_embed.0
#     / .2), one per frame;
#   * AdaLN-zero block (the diffusion-transformer form): [shift1, scale1,
#     gate1, shift2, scale2, gate2] = adaln(SiLU(c_t)) split in six; LayerNorms
#     without affine parameters; x += gate1 * attn_out(attention(LN(x) (1 +
#     scale1) + shift1)); x += gate2 * MLP(LN(x) (1 + scale2) + shift2); the
#     attention causal over the frames (frame t reads frames <= t), the MLP
#     ffn_up -> GELU -> ffn_down as in the encoder;
#   * the input states plus the predictor's positional rows pred.pos_embed
#     [window, D] (row t for the t-th frame of the window);
#   * output: pred.proj.2 GELU(pred.proj.0 pred.norm(x)): row t predicts the
#     state of frame t + 1;
#   * rollout: the window holds the last `window` states; each step appends
#     the prediction of its last row; the action of a state is the one taken
#     in that frame.
# ---------------------------------------------------------------------------
def silu(x: np.ndarray) -> np.ndarray:
    """x * sigmoid(x)."""
    x = np.asarray(x, np.float64)
    return x / (1.0 + np.exp(-x))


def lewm_project(W, cls: np.ndarray) -> np.ndarray:
    """The LeWM projector (enc.proj.0 / enc.proj.2) on final-normed CLS rows
    [B, D] -> world-model states [B, D_s]."""
    h = gelu(linear(cls, W["enc.proj.0.weight"], W["enc.proj.0.bias"]))
    return linear(h, W["enc.proj.2.weight"], W["enc.proj.2.bias"])


def lewm_action_embed(W, act: np.ndarray) -> np.ndarray:
    """Actions [.., A] -> conditioning vectors [.., D] (pred.action_embed)."""
    h = silu(linear(act, W["pred.action_embed.0.weight"], W["pred.action_embed.0.bias"]))
    return linear(h, W["pred.action_embed.2.weight"], W["pred.action_embed.2.bias"])


def causal_allow(T: int) -> np.ndarray:
    """Boolean [T, T]: frame i reads frames j <= i."""
    return np.tril(np.ones((T, T), bool))


def adaln_block(x, c, W, prefix: str, heads: int, eps: float) -> np.ndarray:
    """One AdaLN-zero block over x [B, T, D] conditioned on c [B, T, D]."""
    D = x.shape[-1]
    mod = linear(silu(c), W[prefix + "adaln.weight"], W[prefix + "adaln.bias"])
    shift1, scale1, gate1, shift2, scale2, gate2 = (mod[..., i * D:(i + 1) * D] for i in range(6))
    one, zero = np.ones(D), np.zeros(D)
    h = layer_norm(x, one, zero, eps) * (1.0 + scale1) + shift1
    qkv = linear(h, W[prefix + "attn_qkv.weight"], W[prefix + "attn_qkv.bias"])
    q, k, v = (split_heads(qkv[..., i * D:(i + 1) * D], heads) for i in range(3))
    o = merge_heads(attention(q, k, v, causal_allow(x.shape[1])))
    x = x + gate1 * linear(o, W[prefix + "attn_out.weight"], W[prefix + "attn_out.bias"])
    h = layer_norm(x, one, zero, eps) * (1.0 + scale2) + shift2
    u = gelu(linear(h, W[prefix + "ffn_up.weight"], W[prefix + "ffn_up.bias"]))
    return x + gate2 * linear(u, W[prefix + "ffn_down.weight"], W[prefix + "ffn_down.bias"])


def lewm_predict(wc, W, states: np.ndarray, actions: np.ndarray) -> np.ndarray:
    """One predictor call: states [B, T, D], actions [B, T, A] (T <= the
    window) -> predictions [B, T, D], row t the predicted state of frame
    t + 1."""
    states = np.asarray(states, np.float64)
    T = states.shape[1]
    if T > wc.window:
        raise ValueError("window")
    x = states + W["pred.pos_embed"][:T][None]
    c = lewm_action_embed(W, actions)
    for i in range(wc.depth):
        x = adaln_block(x, c, W, f"pred.blk.{i}.", wc.heads, wc.ln_eps)
    y = layer_norm(x, W["pred.norm.weight"], W["pred.norm.bias"], wc.ln_eps)
    h = gelu(linear(y, W["pred.proj.0.weight"], W["pred.proj.0.bias"]))
    return linear(h, W["pred.proj.2.weight"], W["pred.proj.2.bias"])


def lewm_rollout(wc, W, states0: np.ndarray, actions: np.ndarray, steps: int) -> np.ndarray:
    """Rollout: states0 [B, T0, D] (the observed frames), actions
    [B, T0 + steps - 1, A] (action t belongs to frame t) -> the predicted
    states of frames T0 .. T0 + steps - 1, [B, steps, D].  Each step runs the
    predictor on the last min(window, frames so far) frames and appends the
    prediction of the last one."""
    seq = [np.asarray(states0[:, t], np.float64) for t in range(states0.shape[1])]
    out = []
    for _ in range(steps):
        n = len(seq)
        lo = max(0, n - wc.window)
        win = np.stack(seq[lo:n], axis=1)
        nxt = lewm_predict(wc, W, win, actions[:, lo:n])[:, -1]
        seq.append(nxt)
        out.append(nxt)
    return np.stack(out, axis=1)


# ---------------------------------------------------------------------------
# Sampled rows of one block: the block's output for chosen query rows of one
# clip, given that clip's block input.  Same definitions, evaluated only where
# needed (K and V still come from every row).
# ---------------------------------------------------------------------------
def block_rows(x_clip: np.ndarray, W, prefix: str, heads: int, eps: float,
               allow: Optional[np.ndarray], rows: Sequence[int],
               rope_pos: Optional[np.ndarray] = None) -> np.ndarray:
    rows = np.asarray(rows)
    N, D = x_clip.shape
    y = layer_norm(x_clip, W[prefix + "ln1.weight"], W[prefix + "ln1.bias"], eps)
    wqkv, bqkv = W[prefix + "attn_qkv.weight"], W[prefix + "attn_qkv.bias"]
    q = linear(y[rows], wqkv[:D], bqkv[:D])
    k = linear(y, wqkv[D:2 * D], bqkv[D:2 * D])
    v = linear(y, wqkv[2 * D:], bqkv[2 * D:])
    qh, kh, vh = (split_heads(t[None], heads)[0] for t in (q, k, v))
    if rope_pos is not None:
        qh, kh = rope(qh, rope_pos[rows]), rope(kh, rope_pos)
    o = merge_heads(attention(qh, kh, vh, None if allow is None else allow[rows])[None])[0]
    xr = x_clip[rows] + linear(o, W[prefix + "attn_out.weight"], W[prefix + "attn_out.bias"])
    y2 = layer_norm(xr, W[prefix + "ln2.weight"], W[prefix + "ln2.bias"], eps)
    h = gelu(linear(y2, W[prefix + "ffn_up.weight"], W[prefix + "ffn_up.bias"]))
    return xr + linear(h, W[prefix + "ffn_down.weight"], W[prefix + "ffn_down.bias"])


# ---------------------------------------------------------------------------
# Comparison metrics ("Quantization" page, "How the accuracy was measured")
# ---------------------------------------------------------------------------
def token_cosines(a: np.ndarray, b: np.ndarray) -> np.ndarray:
    a = np.asarray(a, np.float64).reshape(-1, a.shape[-1])
    b = np.asarray(b, np.float64).reshape(-1, b.shape[-1])
    num = (a * b).sum(-1)
    den = np.sqrt((a * a).sum(-1) * (b * b).sum(-1))
    return np.where(den > 0, num / np.where(den > 0, den, 1), 1.0)


def rel_max(a, b) -> float:
    """max|a-b| / max|b| with b the reference."""
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.abs(a - b).max() / max(np.abs(b).max(), 1e-300))


def rel_fro(a, b) -> float:
    a = np.asarray(a, np.float64)
    b = np.asarray(b, np.float64)
    return float(np.linalg.norm(a - b) / max(np.linalg.norm(b), 1e-300))
