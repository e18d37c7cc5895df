"""Seeded synthetic inputs: model configurations, tensor tables and pixel clips.

This module holds no step of the encoder's arithmetic.  It only *makes inputs*:

* the five workload shapes of the JEPA model cards and benchmark pages
  (ViT-Ti/14 LeWM image encoder, LeVJEPA ViT-L/16 block-causal video encoder,
  V-JEPA 2 ViT-L/16 with its SSv2 attentive-pooler head, the same LeVJEPA
  encoder with q4_0 matrices, and the 64-frame V-JEPA 2 long clip), plus small
  shapes for tests;
* a tensor table of seeded N(0, 0.02) weights named as in the "Quantization"
  docs page, section "The rule" (``enc.blk.N.attn_qkv.weight`` ...), stored as
  f32, f16, or in the ggml block formats q8_0 / q4_0 that the LeVJEPA and V-JEPA 2
  model cards ship ("Files" tables);
* seeded uint8 frames put through a per-channel mean/std normalisation, the way
  the "jepa.cpp — measured benchmarks" page makes its synthetic input
  (section "jepa.cpp — measured benchmarks", first paragraph).

The block *quantiser* lives here because it only produces blocks; both the
oracle and the CUDA path consume the identical bytes and dequantise them with
their own code.  Random numbers come from numpy's PCG64 (``default_rng``).
"""
from __future__ import annotations

import dataclasses
from dataclasses import dataclass, field
from typing import Dict, List, Optional

import numpy as np

# dtype ids follow ggml's general.file_type / tensor type numbering
# ("Quantization" page, section "The rule": 0 f32, 1 f16, 2 q4_0, 8 q8_0 ...)
DT_F32, DT_F16, DT_Q4_0, DT_Q8_0 = 0, 1, 2, 8
DTYPE_NAMES = {DT_F32: "f32", DT_F16: "f16", DT_Q4_0: "q4_0", DT_Q8_0: "q8_0"}
DTYPE_IDS = {v: k for k, v in DTYPE_NAMES.items()}

QK = 32                 # elements per q8_0 / q4_0 block
Q8_0_BLOCK_BYTES = 34   # fp16 scale + 32 x int8
Q4_0_BLOCK_BYTES = 18   # fp16 scale + 16 bytes of nibbles

POOL_NONE, POOL_MEAN, POOL_CLS, POOL_ATTENTIVE = 0, 1, 2, 3
POOL_LEWM = 4
POOL_IDS = {"none": POOL_NONE, "mean": POOL_MEAN, "cls": POOL_CLS, "attentive": POOL_ATTENTIVE, "lewm": POOL_LEWM}
MASK_BIDIR, MASK_BLOCK_CAUSAL = 0, 1
MASK_IDS = {"bidir": MASK_BIDIR, "block_causal": MASK_BLOCK_CAUSAL}

IMAGENET_MEAN = (0.485, 0.456, 0.406)
IMAGENET_STD = (0.229, 0.224, 0.225)


@dataclass(frozen=True)
class EncoderConfig:
    """Shape of one JEPA ViT encoder (plus optional attentive head) workload."""
    name: str
    dim: int
    depth: int
    heads: int
    mlp: int
    patch: int
    tubelet: int
    img_h: int
    img_w: int
    frames: int
    has_cls: bool
    mask: str                 # "bidir" | "block_causal"
    weights: str              # "f32" | "f16" | "q8_0" | "q4_0"
    batch: int
    pool: str                 # "none" | "mean" | "cls" | "attentive"
    seed: int = 0
    head_sa_blocks: int = 0
    n_classes: int = 0
    ln_eps: float = 1e-6
    pix_mean: tuple = IMAGENET_MEAN
    pix_std: tuple = IMAGENET_STD
    random_ln_affine: bool = False   # tests: exercise gamma/beta instead of 1/0
    rope: bool = False               # 3-D rotary positions in the attention instead of pos_embed (no CLS)
    act_bf16: bool = False           # bf16 instead of f16 for the kernels' 16-bit activations and operands

    # -- derived shapes ---------------------------------------------------
    @property
    def head_dim(self) -> int:
        return self.dim // self.heads

    @property
    def patches_per_slot(self) -> int:        # P_f
        return (self.img_h // self.patch) * (self.img_w // self.patch)

    @property
    def slots(self) -> int:                   # T' = T / tubelet
        return self.frames // self.tubelet

    @property
    def n_patches(self) -> int:               # N_p
        return self.slots * self.patches_per_slot

    @property
    def n_tokens(self) -> int:                # N
        return self.n_patches + (1 if self.has_cls else 0)

    @property
    def patch_k(self) -> int:                 # 3 * kt * p * p
        return 3 * self.tubelet * self.patch * self.patch

    @property
    def has_head(self) -> bool:
        return self.n_classes > 0

    def with_(self, **kw) -> "EncoderConfig":
        return dataclasses.replace(self, **kw)


# ---------------------------------------------------------------------------
# The five model configurations (model cards: LeWorldModel Push-T, LeVJEPA
# ViT-L/16, V-JEPA 2 ViT-L/16 SSv2 classifier; benchmarks page: 64-frame long
# clip), then the batch sweeps and rotary variants built from them.
# ---------------------------------------------------------------------------
LEWM_VIT_TI = EncoderConfig(
    name="lewm_vit_ti14_224_b1", dim=192, depth=12, heads=3, mlp=768, patch=14,
    tubelet=1, img_h=224, img_w=224, frames=1, has_cls=True, mask="bidir",
    weights="f32", batch=1, pool="cls", seed=0, pix_mean=(0.5, 0.5, 0.5),
    pix_std=(0.5, 0.5, 0.5))
# the same model at the batch sizes the pages also time it at
LEWM_VIT_TI_B8 = LEWM_VIT_TI.with_(name="lewm_vit_ti14_224_b8", batch=8)
LEWM_VIT_TI_B32 = LEWM_VIT_TI.with_(name="lewm_vit_ti14_224_b32", batch=32)
LEVJEPA_VIT_L = EncoderConfig(
    name="levjepa_vit_l16_16f224_b4", dim=1024, depth=24, heads=16, mlp=4096,
    patch=16, tubelet=1, img_h=224, img_w=224, frames=16, has_cls=True,
    mask="block_causal", weights="f16", batch=4, pool="cls", seed=1)
VJEPA2_SSV2 = EncoderConfig(
    name="vjepa2_vit_l16_16f256_ssv2_q8_b8", dim=1024, depth=24, heads=16,
    mlp=4096, patch=16, tubelet=2, img_h=256, img_w=256, frames=16,
    has_cls=False, mask="bidir", weights="q8_0", batch=8, pool="attentive",
    seed=2, head_sa_blocks=3, n_classes=174)
LEVJEPA_VIT_L_Q4 = LEVJEPA_VIT_L.with_(
    name="levjepa_vit_l16_16f224_q4_b8", weights="q4_0", batch=8, pool="mean",
    seed=3)
# the same q4_0 model at one clip (where the weight stream is visible) and at 32
LEVJEPA_VIT_L_Q4_B1 = LEVJEPA_VIT_L_Q4.with_(name="levjepa_vit_l16_16f224_q4_b1", batch=1)
LEVJEPA_VIT_L_Q4_B32 = LEVJEPA_VIT_L_Q4.with_(name="levjepa_vit_l16_16f224_q4_b32", batch=32)
VJEPA2_LONG = EncoderConfig(
    name="vjepa2_vit_l16_64f256_b2", dim=1024, depth=24, heads=16, mlp=4096,
    patch=16, tubelet=2, img_h=256, img_w=256, frames=64, has_cls=False,
    mask="bidir", weights="f16", batch=2, pool="none", seed=4)

# The V-JEPA 2 workloads with the 3-D rotary positions of the real encoders
# (instead of an additive table).
VJEPA2_LONG_ROPE = VJEPA2_LONG.with_(name="vjepa2_vit_l16_64f256_rope_b2", rope=True)
VJEPA2_SSV2_ROPE = VJEPA2_SSV2.with_(name="vjepa2_vit_l16_16f256_ssv2_q8_rope_b8", rope=True)
# The LeVJEPA workload with bf16 activations (the same f16 weight table,
# rounded to bf16 at load).
LEVJEPA_VIT_L_BF16 = LEVJEPA_VIT_L.with_(name="levjepa_vit_l16_16f224_b4_bf16", act_bf16=True)

WORKLOADS: Dict[str, EncoderConfig] = {
    c.name: c for c in (LEWM_VIT_TI, LEWM_VIT_TI_B8, LEWM_VIT_TI_B32, LEVJEPA_VIT_L,
                        VJEPA2_SSV2, LEVJEPA_VIT_L_Q4, LEVJEPA_VIT_L_Q4_B1,
                        LEVJEPA_VIT_L_Q4_B32, VJEPA2_LONG, VJEPA2_LONG_ROPE, VJEPA2_SSV2_ROPE,
                        LEVJEPA_VIT_L_BF16)}


@dataclass(frozen=True)
class PredictorConfig:
    """The masked predictor of a V-JEPA 2 encoder ("jepa.cpp — measured
    benchmarks", "Masked predictor": a 12-layer, 384-wide predictor; head dim
    32): context tokens of the encoder output are projected to the
    predictor's width (pred.embed), one learned mask token stands at every
    target position, both get the predictor's positional table
    (pred.pos_embed), the sequence [context | targets] runs through pre-LN
    blocks with bidirectional attention, and the targets leave through the
    final norm and pred.proj back to the encoder's width.  ``ctx`` / ``tgt``
    select token indices of the encoder's N tokens (the same for every clip);
    "all" is every token, the pages' worst case (context = target = every
    token)."""
    name: str
    enc: EncoderConfig
    dim: int = 384
    depth: int = 12
    heads: int = 12
    mlp: int = 1536
    ctx: str = "all"          # "all" | "even" | "first_half"
    tgt: str = "all"          # "all" | "odd" | "second_half"
    weights: str = "f16"
    batch: int = 1
    seed: int = 7
    ln_eps: float = 1e-6
    random_ln_affine: bool = False

    @property
    def head_dim(self) -> int:
        return self.dim // self.heads

    @property
    def n_tokens(self) -> int:
        return self.enc.n_tokens

    def _sel(self, rule: str) -> np.ndarray:
        n = np.arange(self.n_tokens)
        return {"all": n, "even": n[0::2], "odd": n[1::2], "first_half": n[: self.n_tokens // 2],
                "second_half": n[self.n_tokens // 2:]}[rule]

    @property
    def ctx_idx(self) -> np.ndarray:
        return self._sel(self.ctx)

    @property
    def tgt_idx(self) -> np.ndarray:
        return self._sel(self.tgt)

    def with_(self, **kw) -> "PredictorConfig":
        return dataclasses.replace(self, **kw)


def predictor_specs(pc: PredictorConfig) -> List[tuple]:
    """(name, shape, kind) of the predictor's tensors in table order."""
    De, D, M = pc.enc.dim, pc.dim, pc.mlp
    s = [("pred.embed.weight", (D, De), "w"), ("pred.embed.bias", (D,), "b"),
         ("pred.mask_tokens", (1, D), "w"), ("pred.pos_embed", (pc.n_tokens, D), "w")]
    for i in range(pc.depth):
        s += _block_names(f"pred.blk.{i}.", D, M)
    s += [("pred.norm.weight", (D,), "ln_g"), ("pred.norm.bias", (D,), "ln_b"),
          ("pred.proj.weight", (De, D), "w"), ("pred.proj.bias", (De,), "b")]
    return s


def make_predictor_table(pc: PredictorConfig, std: float = 0.02) -> List["Tensor"]:
    """Seeded predictor tensors, drawn like make_tensor_table's."""
    rng = np.random.default_rng(pc.seed)
    table = []
    for name, shape, kind in predictor_specs(pc):
        if kind == "ln_g":
            v = (np.float32(1.0) + np.float32(0.1) * rng.standard_normal(shape, dtype=np.float32)
                 if pc.random_ln_affine else np.ones(shape, np.float32))
        elif kind == "ln_b":
            v = (np.float32(std) * rng.standard_normal(shape, dtype=np.float32)
                 if pc.random_ln_affine else np.zeros(shape, np.float32))
        else:
            v = np.float32(std) * rng.standard_normal(shape, dtype=np.float32)
        table.append(_store(name, shape, v, pc.weights))
    return table


def make_predictor_tokens(pc: PredictorConfig, batch: Optional[int] = None) -> np.ndarray:
    """Seeded encoder-output-like tokens [B, N, D_enc]: LayerNorm outputs
    (unit variance per token) stand in for the encoder's last_hidden_state."""
    B = pc.batch if batch is None else batch
    rng = np.random.default_rng(pc.seed + 2000)
    return rng.standard_normal((B, pc.n_tokens, pc.enc.dim), dtype=np.float32)


# The masked predictor of the V-JEPA 2 ViT-L encoder on the 16-frame 256^2
# clip (2048 tokens), context = target = every token: a 4096-row sequence,
# the pages' worst case ("Masked predictor").
VJEPA2_PREDICTOR = PredictorConfig(name="vjepa2_predictor_l16_16f256_all_b8", enc=VJEPA2_SSV2.with_(weights="f16"),
                                   batch=8)
PREDICTORS: Dict[str, "PredictorConfig"] = {VJEPA2_PREDICTOR.name: VJEPA2_PREDICTOR}

@dataclass(frozen=True)
class WorldModelConfig:
    """The LeWM world model ("LeWorldModel Push-T" card, intro: the ViT-Ti/14
    encoder's CLS row projected to a world-model state, six AdaLN-zero causal
    blocks conditioned on a 10-d action; benchmarks page, "LeWM world model":
    a 3-frame window of 192-d states).  ``dim`` is the state width (the
    encoder's width), ``window`` the frames one predictor call reads (the
    rows of pred.pos_embed); ``proj_hidden`` / ``pred_hidden`` the hidden
    widths of the projector (enc.proj) and of the output MLP (pred.proj),
    which the pages do not give (read as the blocks' MLP width).  A workload
    is ``candidates`` independent sequences: ``frames`` observed states, and
    ``steps`` rollout steps after them (0: one predictor call over the
    observed frames, every row an output)."""
    name: str
    enc: EncoderConfig
    dim: int = 192
    depth: int = 6
    heads: int = 3
    mlp: int = 768
    action_dim: int = 10
    window: int = 3
    proj_hidden: int = 768
    pred_hidden: int = 768
    weights: str = "f16"
    candidates: int = 1
    frames: int = 3
    steps: int = 0
    seed: int = 11
    ln_eps: float = 1e-6

    @property
    def n_actions(self) -> int:
        """Actions per candidate: one per observed frame, plus one per
        predicted frame that is read again (all but the last)."""
        return self.frames + max(0, self.steps - 1)

    def with_(self, **kw) -> "WorldModelConfig":
        return dataclasses.replace(self, **kw)


def world_model_specs(wc: WorldModelConfig) -> List[tuple]:
    """(name, shape, kind) of the world model's tensors in table order; the
    kind ``w32`` marks the matrices the pages keep in f32 (adaLN, action
    embedder)."""
    De, D, M, A = wc.enc.dim, wc.dim, wc.mlp, wc.action_dim
    s = [("enc.proj.0.weight", (wc.proj_hidden, De), "w"), ("enc.proj.0.bias", (wc.proj_hidden,), "b"),
         ("enc.proj.2.weight", (D, wc.proj_hidden), "w"), ("enc.proj.2.bias", (D,), "b"),
         ("pred.action_embed.0.weight", (D, A), "w32_act0"), ("pred.action_embed.0.bias", (D,), "b32"),
         ("pred.action_embed.2.weight", (D, D), "w32_act2"), ("pred.action_embed.2.bias", (D,), "b32"),
         ("pred.pos_embed", (wc.window, D), "pos")]
    for i in range(wc.depth):
        p = f"pred.blk.{i}."
        s += [(p + "adaln.weight", (6 * D, D), "w32_ada"), (p + "adaln.bias", (6 * D,), "b32_ada"),
              (p + "attn_qkv.weight", (3 * D, D), "w_in"), (p + "attn_qkv.bias", (3 * D,), "b"),
              (p + "attn_out.weight", (D, D), "w_in"), (p + "attn_out.bias", (D,), "b"),
              (p + "ffn_up.weight", (M, D), "w_in"), (p + "ffn_up.bias", (M,), "b"),
              (p + "ffn_down.weight", (D, M), "w_hid"), (p + "ffn_down.bias", (D,), "b")]
    s += [("pred.norm.weight", (D,), "ln_g"), ("pred.norm.bias", (D,), "ln_b"),
          ("pred.proj.0.weight", (wc.pred_hidden, D), "w_in"), ("pred.proj.0.bias", (wc.pred_hidden,), "b"),
          ("pred.proj.2.weight", (D, wc.pred_hidden), "w_hid"), ("pred.proj.2.bias", (D,), "b")]
    return s


def make_world_model_table(wc: WorldModelConfig) -> List["Tensor"]:
    """Seeded world-model tensors.  Scales are chosen so that every part of
    the computation moves the result: matrices ~ N(0, 0.7 / sqrt(fan_in))
    (0.3 / sqrt(fan_in) for the adaLN, whose shifts, scales and gates then
    have a spread of about 0.3), biases ~ N(0, 0.02), the action embedder
    ~ N(0, 1 / sqrt(fan_in)), pos_embed ~ N(0, 0.5), LayerNorm gamma ~
    1 + N(0, 0.1), beta ~ N(0, 0.02).  f32 for adaLN and the action embedder,
    the model's weight type for the re-typed matrices."""
    rng = np.random.default_rng(wc.seed)
    table = []
    for name, shape, kind in world_model_specs(wc):
        z = rng.standard_normal(shape, dtype=np.float32)
        fan_in = shape[-1]
        scale = {"w": 0.7 / np.sqrt(fan_in), "w_in": 0.7 / np.sqrt(fan_in), "w_hid": 0.7 / np.sqrt(fan_in),
                 "w32_ada": 0.3 / np.sqrt(fan_in), "w32_act0": 1.0 / np.sqrt(fan_in),
                 "w32_act2": 1.0 / np.sqrt(fan_in), "b": 0.02, "b32": 0.02, "b32_ada": 0.02, "pos": 0.5,
                 "ln_b": 0.02}.get(kind)
        if kind == "ln_g":
            v = np.float32(1.0) + np.float32(0.1) * z
        else:
            v = np.float32(scale) * z
        table.append(_store(name, shape, v, "f32" if kind.startswith(("w32", "b32")) else wc.weights))
    return table


def make_world_model_inputs(wc: WorldModelConfig, candidates: Optional[int] = None):
    """Seeded inputs: observed states [C, frames, D] ~ N(0, 1) (projector
    outputs stand-in) and actions [C, n_actions, A] ~ U(-1, 1)."""
    C = wc.candidates if candidates is None else candidates
    rng = np.random.default_rng(wc.seed + 3000)
    states = rng.standard_normal((C, wc.frames, wc.dim), dtype=np.float32)
    actions = rng.uniform(-1.0, 1.0, (C, wc.n_actions, wc.action_dim)).astype(np.float32)
    return states, actions


# LeWM world model workloads of the benchmarks page ("LeWM world model"):
# one predictor call over the full 3-frame window, and a 20-step rollout from
# one observed frame (the window grows to 3, then slides); plus a planner-sized
# batch of candidate action sequences (the axis the V-JEPA 2-AC planner rows
# of the same page scale on).
LEWM_WM_STEP = WorldModelConfig(name="lewm_wm_step_3f", enc=LEWM_VIT_TI, frames=3, steps=0, candidates=1)
LEWM_WM_ROLLOUT = WorldModelConfig(name="lewm_wm_rollout_20", enc=LEWM_VIT_TI, frames=1, steps=20, candidates=1)
LEWM_WM_PLAN = WorldModelConfig(name="lewm_wm_rollout_20_c1024", enc=LEWM_VIT_TI, frames=1, steps=20,
                                candidates=1024)
WORLD_MODELS: Dict[str, "WorldModelConfig"] = {w.name: w for w in (LEWM_WM_STEP, LEWM_WM_ROLLOUT, LEWM_WM_PLAN)}


def small_config(base: EncoderConfig, **kw) -> EncoderConfig:
    """A shrunk copy of a workload that the oracle runs in seconds."""
    d = dict(dim=256, depth=2, heads=4, mlp=1024, img_h=64, img_w=64,
             frames=min(base.frames, 4), batch=2, random_ln_affine=True)
    if base.tubelet == 2:
        d["frames"] = 4
    if 64 % base.patch:   # keep the image a whole number of patches (LeWM's 14)
        d["img_h"] = d["img_w"] = base.patch * (64 // base.patch)
    d.update(kw)
    return base.with_(name=base.name + "_small", **d)


# ---------------------------------------------------------------------------
# Tensor table
# ---------------------------------------------------------------------------
@dataclass
class Tensor:
    """One entry of the tensor table: PyTorch-order shape ([out, in] for a
    matrix), a ggml dtype id and the raw bytes as a contiguous numpy array
    (float32 / float16 values, or uint8 block bytes for q8_0 / q4_0)."""
    name: str
    dtype: int
    shape: tuple
    data: np.ndarray

    @property
    def nbytes(self) -> int:
        return int(self.data.nbytes)


# Matrices the "Quantization" page (section "The rule") re-types.
_RETYPED_SUFFIXES = ("attn_qkv.weight", "attn_out.weight", "ffn_up.weight",
                     "ffn_down.weight", "head.xattn.q.weight",
                     "head.xattn.k.weight", "head.xattn.v.weight",
                     "head.xattn.out.weight", "head.cls.weight",
                     "pred.embed.weight", "pred.proj.weight", "enc.proj.0.weight",
                     "enc.proj.2.weight", "pred.proj.0.weight", "pred.proj.2.weight")


def is_retyped(name: str) -> bool:
    return name.endswith(_RETYPED_SUFFIXES)


def _block_names(prefix: str, D: int, M: int) -> List[tuple]:
    return [
        (prefix + "ln1.weight", (D,), "ln_g"), (prefix + "ln1.bias", (D,), "ln_b"),
        (prefix + "attn_qkv.weight", (3 * D, D), "w"),
        (prefix + "attn_qkv.bias", (3 * D,), "b"),
        (prefix + "attn_out.weight", (D, D), "w"), (prefix + "attn_out.bias", (D,), "b"),
        (prefix + "ln2.weight", (D,), "ln_g"), (prefix + "ln2.bias", (D,), "ln_b"),
        (prefix + "ffn_up.weight", (M, D), "w"), (prefix + "ffn_up.bias", (M,), "b"),
        (prefix + "ffn_down.weight", (D, M), "w"), (prefix + "ffn_down.bias", (D,), "b"),
    ]


def tensor_specs(cfg: EncoderConfig, with_pos: Optional[bool] = None) -> List[tuple]:
    """(name, shape, kind) in table order (no pos_embed for a rotary model)."""
    if with_pos is None:
        with_pos = not cfg.rope
    D, M, kt, p = cfg.dim, cfg.mlp, cfg.tubelet, cfg.patch
    s = [("enc.patch_embed.weight", (D, 3, kt, p, p), "w"),
         ("enc.patch_embed.bias", (D,), "b")]
    if with_pos:
        s.append(("enc.pos_embed", (cfg.n_tokens, D), "w"))
    if cfg.has_cls:
        s.append(("enc.cls_token", (D,), "w"))
    for i in range(cfg.depth):
        s += _block_names(f"enc.blk.{i}.", D, M)
    s += [("enc.norm.weight", (D,), "ln_g"), ("enc.norm.bias", (D,), "ln_b")]
    if cfg.has_head:
        for i in range(cfg.head_sa_blocks):
            s += _block_names(f"head.blk.{i}.", D, M)
        s += [("head.query", (D,), "w"),
              ("head.ln_kv.weight", (D,), "ln_g"), ("head.ln_kv.bias", (D,), "ln_b")]
        for t in ("q", "k", "v", "out"):
            s += [(f"head.xattn.{t}.weight", (D, D), "w"), (f"head.xattn.{t}.bias", (D,), "b")]
        s += [("head.xattn.ln2.weight", (D,), "ln_g"), ("head.xattn.ln2.bias", (D,), "ln_b"),
              ("head.xattn.ffn_up.weight", (M, D), "w"), ("head.xattn.ffn_up.bias", (M,), "b"),
              ("head.xattn.ffn_down.weight", (D, M), "w"), ("head.xattn.ffn_down.bias", (D,), "b"),
              ("head.cls.weight", (cfg.n_classes, D), "w"),
              ("head.cls.bias", (cfg.n_classes,), "b")]
    return s


def quantize_q8_0(x: np.ndarray) -> np.ndarray:
    """Rows of float values -> q8_0 blocks (uint8 [..., K/32 * 34]).

    Per 32-element block: amax = max|x|, d = amax/127, q = round-half-away(x/d)
    clamped to [-127, 127], d stored as IEEE binary16 (round to nearest even),
    then 32 int8.  An all-zero block gets d = 0, q = 0."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    lead, K = x.shape[:-1], x.shape[-1]
    assert K % QK == 0, "q8_0 needs the row length to be a multiple of 32"
    b = x.reshape(-1, QK)
    amax = np.abs(b).max(axis=1)
    d = (amax / np.float32(127.0)).astype(np.float32)
    inv = np.where(d > 0, np.float32(1.0) / np.where(d > 0, d, 1), 0).astype(np.float32)
    v = b * inv[:, None]
    q = np.trunc(v + np.copysign(np.float32(0.5), v))
    q = np.clip(q, -127, 127).astype(np.int8)
    out = np.empty((b.shape[0], Q8_0_BLOCK_BYTES), np.uint8)
    out[:, 0:2] = d.astype(np.float16).view(np.uint8).reshape(-1, 2)
    out[:, 2:] = q.view(np.uint8)
    return out.reshape(*lead, (K // QK) * Q8_0_BLOCK_BYTES)


def quantize_q4_0(x: np.ndarray) -> np.ndarray:
    """Rows of float values -> q4_0 blocks (uint8 [..., K/32 * 18]).

    Per block: m = the element of largest magnitude (first on ties), d = m/-8,
    q = min(15, floor(x/d + 8.5)), value (q-8)*d; d stored as binary16.  Byte j
    of the 16 nibble bytes holds element j in its low and element j+16 in its
    high nibble (ggml's q4_0 packing)."""
    x = np.ascontiguousarray(x, dtype=np.float32)
    lead, K = x.shape[:-1], x.shape[-1]
    assert K % QK == 0, "q4_0 needs the row length to be a multiple of 32"
    b = x.reshape(-1, QK)
    idx = np.argmax(np.abs(b), axis=1)
    m = b[np.arange(b.shape[0]), idx]
    d = (m / np.float32(-8.0)).astype(np.float32)
    inv = np.where(d != 0, np.float32(1.0) / np.where(d != 0, d, 1), 0).astype(np.float32)
    q = np.floor(b * inv[:, None] + np.float32(8.5))
    q = np.clip(q, 0, 15).astype(np.uint8)
    out = np.empty((b.shape[0], Q4_0_BLOCK_BYTES), np.uint8)
    out[:, 0:2] = d.astype(np.float16).view(np.uint8).reshape(-1, 2)
    out[:, 2:] = q[:, :16] | (q[:, 16:] << 4)
    return out.reshape(*lead, (K // QK) * Q4_0_BLOCK_BYTES)


def _store(name: str, shape: tuple, vals: np.ndarray, wdt: str) -> Tensor:
    if wdt in ("q8_0", "q4_0") and is_retyped(name) and shape[-1] % QK == 0:
        q = quantize_q8_0(vals) if wdt == "q8_0" else quantize_q4_0(vals)
        return Tensor(name, DTYPE_IDS[wdt], shape, np.ascontiguousarray(q))
    if wdt == "f32":
        return Tensor(name, DT_F32, shape, np.ascontiguousarray(vals, np.float32))
    return Tensor(name, DT_F16, shape, np.ascontiguousarray(vals.astype(np.float16)))


def make_tensor_table(cfg: EncoderConfig, seed: Optional[int] = None,
                      std: float = 0.02) -> List[Tensor]:
    """Seeded tensor table: weights, biases, pos_embed, cls, query ~ N(0, std);
    LayerNorm gamma = 1, beta = 0 (or, with ``random_ln_affine``, gamma ~
    1 + N(0, 0.1) and beta ~ N(0, 0.02)).  Tensors are drawn in table order
    from one PCG64 stream."""
    rng = np.random.default_rng(cfg.seed if seed is None else seed)
    table = []
    for name, shape, kind in tensor_specs(cfg):
        if kind == "ln_g":
            v = (np.float32(1.0) + np.float32(0.1) * rng.standard_normal(shape, dtype=np.float32)
                 if cfg.random_ln_affine else np.ones(shape, np.float32))
        elif kind == "ln_b":
            v = (np.float32(std) * rng.standard_normal(shape, dtype=np.float32)
                 if cfg.random_ln_affine else np.zeros(shape, np.float32))
        else:
            v = np.float32(std) * rng.standard_normal(shape, dtype=np.float32)
        table.append(_store(name, shape, v, cfg.weights))
    return table


def table_dict(table: List[Tensor]) -> Dict[str, Tensor]:
    return {t.name: t for t in table}


def make_pixels(cfg: EncoderConfig, batch: Optional[int] = None,
                seed: Optional[int] = None) -> np.ndarray:
    """Seeded uint8 frames [B, T, 3, H, W] normalised per channel:
    (x/255 - mean[c]) / std[c], as float32."""
    B = cfg.batch if batch is None else batch
    rng = np.random.default_rng((cfg.seed if seed is None else seed) + 1000)
    u8 = rng.integers(0, 256, size=(B, cfg.frames, 3, cfg.img_h, cfg.img_w), dtype=np.uint8)
    mean = np.asarray(cfg.pix_mean, np.float32).reshape(1, 1, 3, 1, 1)
    sd = np.asarray(cfg.pix_std, np.float32).reshape(1, 1, 3, 1, 1)
    return np.ascontiguousarray((u8.astype(np.float32) / np.float32(255.0) - mean) / sd)


def param_count(cfg: EncoderConfig, with_pos: bool = False) -> int:
    """Number of parameters of the encoder (and head) tensors."""
    return int(sum(int(np.prod(s)) for _, s, _ in tensor_specs(cfg, with_pos=with_pos)))


def table_bytes(cfg: EncoderConfig, wdt: str, with_pos: bool = False,
                rest: str = "f32") -> int:
    """Bytes of the tensor data with the re-typed matrices stored as ``wdt``
    and every other tensor as ``rest``."""
    per = {"f32": 4, "f16": 2}
    total = 0
    for name, shape, _ in tensor_specs(cfg, with_pos=with_pos):
        n = int(np.prod(shape))
        if wdt in ("q8_0", "q4_0") and is_retyped(name):
            total += n // QK * (Q8_0_BLOCK_BYTES if wdt == "q8_0" else Q4_0_BLOCK_BYTES)
        elif wdt in per and is_retyped(name):
            total += n * per[wdt]
        else:
            total += n * per[rest]
    return total
