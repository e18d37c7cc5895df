"""B200-native JEPA ViT encoder forward.

Python binding of libjepa_b200.so (include/jepa_b200.h): argument marshalling
only.  Every step of the forward -- patch-embed, LayerNorm, the tcgen05 GEMMs,
flash attention, pooling and the attentive head -- runs in the library's
sm_100a kernels; PyTorch supplies device memory and streams.  There is no CPU
path: without the built library (or a CUDA device) the calls raise.
"""
from __future__ import annotations

import ctypes
from typing import List, Optional, Tuple

from . import _abi, synth
from ._abi import JepaError, check, load_library

POOLS = synth.POOL_IDS


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _dptr(t) -> int:
    """Device address of a CUDA tensor on the current device.  The library
    takes raw pointers; a host tensor or another device's memory handed to a
    kernel would be read as device memory, so both are refused here."""
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise ValueError("expected a CUDA tensor, got " + (str(t.device) if isinstance(t, torch.Tensor) else
                                                           type(t).__name__))
    if t.device.index != torch.cuda.current_device():
        raise ValueError(f"tensor on {t.device}, but the current device is cuda:{torch.cuda.current_device()}")
    return t.data_ptr()


def check_pixels(cfg: "synth.EncoderConfig", pixels, on_cuda: bool, device: Optional[int] = None) -> int:
    """Validate a pixel batch for encode / encode_host: float32, contiguous,
    [B, frames, 3, img_h, img_w] with B >= 1, on a CUDA device (``device``)
    or on the host.  Returns B."""
    import torch
    if not isinstance(pixels, torch.Tensor):
        raise TypeError("pixels must be a torch.Tensor")
    want = (cfg.frames, 3, cfg.img_h, cfg.img_w)
    if pixels.dim() != 5 or tuple(pixels.shape[1:]) != want or pixels.shape[0] < 1:
        raise ValueError(f"pixels must be [B, {', '.join(map(str, want))}], got {list(pixels.shape)}")
    if pixels.dtype != torch.float32:
        raise ValueError(f"pixels must be float32, got {pixels.dtype}")
    if not pixels.is_contiguous():
        raise ValueError("pixels must be contiguous")
    if pixels.is_cuda != on_cuda or (on_cuda and device is not None and pixels.device.index != device):
        raise ValueError(f"pixels on {pixels.device}; expected " + (f"cuda:{device}" if on_cuda else "the host"))
    return int(pixels.shape[0])


def check_tokens(cfg: "synth.EncoderConfig", tokens, device: Optional[int] = None, on_cuda: bool = True) -> int:
    """Validate the predictor's input, the encoder's last_hidden_state: a
    contiguous float32 tensor [B, N, dim] on a CUDA device (``device``; the
    host with on_cuda False) with B >= 1, N the encoder's tokens per clip and
    dim its width (the library reads B * N * dim values from the pointer and
    cannot see the tensor's size).  Returns B."""
    import torch
    if not isinstance(tokens, torch.Tensor) or tokens.is_cuda != on_cuda or tokens.dtype != torch.float32 \
            or not tokens.is_contiguous() or (on_cuda and device is not None and tokens.device.index != device):
        raise ValueError("tokens must be a contiguous float32 tensor on " + (f"cuda:{device}" if on_cuda else "the host"))
    want = (cfg.n_tokens, cfg.dim)
    if tokens.dim() != 3 or tuple(tokens.shape[1:]) != want or tokens.shape[0] < 1:
        raise ValueError(f"tokens must be [B, {want[0]}, {want[1]}], got {list(tokens.shape)}")
    return int(tokens.shape[0])


def check_world_model_inputs(wc: "synth.WorldModelConfig", states, actions, steps: int = 0,
                             device: Optional[int] = None, on_cuda: bool = True) -> Tuple[int, int]:
    """Validate a world-model call's inputs: contiguous float32 tensors of
    three dims on a CUDA device (``device``; the host with on_cuda False),
    states [C, T, dim] with C, T >= 1, and actions [C, A_rows, action_dim]
    with A_rows = T for a predictor call (steps 0) or T + steps - 1 for a
    rollout of steps >= 1 (the library reads exactly those rows and cannot
    see the tensors' sizes).  Returns (C, T)."""
    import torch
    for t, name in ((states, "states"), (actions, "actions")):
        if not isinstance(t, torch.Tensor) or t.is_cuda != on_cuda or t.dtype != torch.float32 \
                or not t.is_contiguous() or t.dim() != 3 or (on_cuda and device is not None and t.device.index != device):
            raise ValueError(f"{name} must be a contiguous float32 tensor of 3 dims on "
                             + (f"cuda:{device}" if on_cuda else "the host"))
    C, T = int(states.shape[0]), int(states.shape[1])
    if C < 1 or T < 1 or int(states.shape[2]) != wc.dim:
        raise ValueError(f"states must be [C, T, {wc.dim}] with C, T >= 1, got {list(states.shape)}")
    if steps < 0:
        raise ValueError(f"steps must be >= 1 for a rollout, got {steps}")
    rows = T if steps == 0 else T + steps - 1
    if tuple(actions.shape) != (C, rows, wc.action_dim):
        raise ValueError(f"actions must be [{C}, {rows}, {wc.action_dim}], got {list(actions.shape)}")
    return C, T


def check_out(out, on_cuda: bool, device: Optional[int] = None) -> None:
    """A caller-supplied output: float32, contiguous, on the same side as the
    pixels (its size is checked by the library against the pool mode)."""
    import torch
    if not isinstance(out, torch.Tensor) or out.dtype != torch.float32 or not out.is_contiguous():
        raise ValueError("out must be a contiguous float32 tensor")
    if out.is_cuda != on_cuda or (on_cuda and device is not None and out.device.index != device):
        raise ValueError(f"out on {out.device}; expected " + (f"cuda:{device}" if on_cuda else "the host"))


def make_config(cfg: "synth.EncoderConfig", quant_f16_copy: bool = False,
                predictor: Optional["synth.PredictorConfig"] = None,
                world_model: Optional["synth.WorldModelConfig"] = None) -> _abi.Config:
    pr, wm = predictor, world_model
    return _abi.Config(dim=cfg.dim, depth=cfg.depth, heads=cfg.heads, mlp=cfg.mlp, patch=cfg.patch,
                       tubelet=cfg.tubelet, img_h=cfg.img_h, img_w=cfg.img_w, frames=cfg.frames,
                       has_cls=1 if cfg.has_cls else 0, mask=synth.MASK_IDS[cfg.mask],
                       head_sa_blocks=cfg.head_sa_blocks, n_classes=cfg.n_classes, ln_eps=cfg.ln_eps,
                       rope=1 if cfg.rope else 0, quant_f16_copy=1 if quant_f16_copy else 0,
                       pred_depth=pr.depth if pr else 0, pred_dim=pr.dim if pr else 0,
                       pred_heads=pr.heads if pr else 0, pred_mlp=pr.mlp if pr else 0,
                       act_bf16=1 if cfg.act_bf16 else 0,
                       wm_depth=wm.depth if wm else 0, wm_heads=wm.heads if wm else 0, wm_mlp=wm.mlp if wm else 0,
                       wm_action_dim=wm.action_dim if wm else 0, wm_window=wm.window if wm else 0,
                       wm_proj_hidden=wm.proj_hidden if wm else 0, wm_pred_hidden=wm.pred_hidden if wm else 0)


class Model:
    """A loaded encoder on one CUDA device.  quant_f16_copy: also keep an f16
    copy of the q8_0 / q4_0 matrices for the large GEMMs (default: blocks
    only, unpacked in every GEMM's loader).  predictor: the shape of a masked
    predictor whose pred.* tensors are in the table (see predict);
    world_model: the shape of a LeWM world model whose tensors are in the
    table (see lewm_predict, lewm_rollout and the "lewm" pool)."""

    def __init__(self, cfg: "synth.EncoderConfig", table: List["synth.Tensor"], device: int = 0,
                 quant_f16_copy: bool = False, predictor: Optional["synth.PredictorConfig"] = None,
                 world_model: Optional["synth.WorldModelConfig"] = None):
        lib = load_library()
        self.cfg = cfg
        self.device = device
        self.world_model = world_model
        entries = (_abi.TensorEntry * len(table))()
        self._keep = []
        for i, t in enumerate(table):
            name = t.name.encode()
            self._keep.append(name)
            e = entries[i]
            e.name = name
            e.dtype = t.dtype
            e.ndim = len(t.shape)
            for j, s in enumerate(t.shape):
                e.shape[j] = s
            e.data = t.data.ctypes.data
            e.nbytes = t.nbytes
        self._cfg = make_config(cfg, quant_f16_copy, predictor, world_model)
        h = ctypes.c_void_p()
        check(lib.jepa_b200_load_weights(ctypes.byref(self._cfg), entries, len(table), device, ctypes.byref(h)),
              "load_weights")
        self._h = h
        self._keep = None

    # -- queries ----------------------------------------------------------
    def out_shape(self, B: int, pool: str):
        shp = (ctypes.c_int64 * 3)()
        nd = load_library().jepa_b200_out_shape(self._h, B, POOLS[pool], shp)
        if nd < 0:
            raise JepaError(nd, "out_shape")
        return tuple(int(shp[i]) for i in range(nd))

    @property
    def n_bytes(self) -> int:
        return int(load_library().jepa_b200_model_n_bytes(self._h))

    def last_ms(self) -> float:
        return float(load_library().jepa_b200_last_ms(self._h))

    def last_launch_count(self) -> int:
        return int(load_library().jepa_b200_last_launch_count(self._h))

    def set_timeout_ns(self, ns: int) -> None:
        check(load_library().jepa_b200_set_timeout_ns(self._h, ns), "set_timeout_ns")

    def set_graph(self, enable: bool) -> None:
        """Replay repeated forwards as a CUDA graph (default on)."""
        check(load_library().jepa_b200_set_graph(self._h, 1 if enable else 0), "set_graph")

    def set_profiling(self, enable: bool) -> None:
        check(load_library().jepa_b200_set_profiling(self._h, 1 if enable else 0), "set_profiling")

    def profile_read(self) -> dict:
        """{kernel class: (device ms, launches)} since the last read."""
        n = len(_abi.KERNEL_CLASSES)
        ms = (ctypes.c_double * n)()
        cnt = (ctypes.c_int * n)()
        check(load_library().jepa_b200_profile_read(self._h, ms, cnt, n), "profile_read")
        return {k: (float(ms[i]), int(cnt[i])) for i, k in enumerate(_abi.KERNEL_CLASSES)}

    def sync_status(self, stream=None) -> int:
        return int(load_library().jepa_b200_sync_status(self._h, _stream_ptr(stream)))

    # -- forward ----------------------------------------------------------
    def encode(self, pixels, pool: Optional[str] = None, out=None, stream=None):
        """pixels: CUDA float32 [B, T, 3, H, W] (contiguous).  Returns the
        output tensor (allocated if ``out`` is None).  Asynchronous."""
        import torch
        pool = self.cfg.pool if pool is None else pool
        B = check_pixels(self.cfg, pixels, True, self.device)
        if out is None:
            out = torch.empty(self.out_shape(B, pool), dtype=torch.float32, device=pixels.device)
        check_out(out, True, self.device)
        check(load_library().jepa_b200_encode(self._h, pixels.data_ptr(), B, POOLS[pool], out.data_ptr(),
                                              out.numel() * 4, _stream_ptr(stream)), "encode")
        return out

    def predict(self, tokens, ctx_idx, tgt_idx, out=None, stream=None):
        """Masked predictor: tokens CUDA float32 [B, N, dim] (the encoder's
        last_hidden_state), ctx_idx / tgt_idx sequences of token indices ->
        float32 [B, len(tgt_idx), dim].  Asynchronous."""
        import numpy as np
        import torch
        B = check_tokens(self.cfg, tokens, self.device)
        ci = np.ascontiguousarray(np.asarray(ctx_idx, dtype=np.int32))
        ti = np.ascontiguousarray(np.asarray(tgt_idx, dtype=np.int32))
        if out is None:
            out = torch.empty((B, len(ti), int(tokens.shape[2])), dtype=torch.float32, device=tokens.device)
        check_out(out, True, self.device)
        check(load_library().jepa_b200_predict(self._h, tokens.data_ptr(), B, ci.ctypes.data, len(ci), ti.ctypes.data,
                                               len(ti), out.data_ptr(), out.numel() * 4, _stream_ptr(stream)),
              "predict")
        return out

    def _wm_cfg(self):
        if self.world_model is None:
            raise JepaError(_abi.ERR_ARG, "the model was loaded without a world model")
        return self.world_model

    def lewm_predict(self, states, actions, out=None, stream=None):
        """LeWM predictor call: states CUDA float32 [C, T, dim], actions
        [C, T, action_dim] -> float32 [C, T, dim], row t the predicted state
        of frame t + 1.  Asynchronous."""
        import torch
        C, T = check_world_model_inputs(self._wm_cfg(), states, actions, 0, self.device)
        if out is None:
            out = torch.empty((C, T, int(states.shape[2])), dtype=torch.float32, device=states.device)
        check_out(out, True, self.device)
        check(load_library().jepa_b200_lewm_predict(self._h, states.data_ptr(), actions.data_ptr(), C, T,
                                                    out.data_ptr(), out.numel() * 4, _stream_ptr(stream)),
              "lewm_predict")
        return out

    def lewm_rollout(self, states, actions, steps: int, out=None, stream=None):
        """LeWM rollout: states CUDA float32 [C, T0, dim] (observed frames),
        actions [C, T0 + steps - 1, action_dim] -> float32 [C, steps, dim],
        the predicted states of frames T0 .. T0 + steps - 1.  Asynchronous."""
        import torch
        if steps < 1:
            raise ValueError(f"steps must be >= 1, got {steps}")
        C, T0 = check_world_model_inputs(self._wm_cfg(), states, actions, steps, self.device)
        if out is None:
            out = torch.empty((C, steps, int(states.shape[2])), dtype=torch.float32, device=states.device)
        check_out(out, True, self.device)
        check(load_library().jepa_b200_lewm_rollout(self._h, states.data_ptr(), T0, actions.data_ptr(), C, steps,
                                                    out.data_ptr(), out.numel() * 4, _stream_ptr(stream)),
              "lewm_rollout")
        return out

    def encode_host(self, pixels, pool: Optional[str] = None, out=None, stream=None):
        """End to end from host memory: pixels CPU float32 (pinned for
        asynchronous copies) -> result in a CPU tensor.  Synchronous."""
        import torch
        pool = self.cfg.pool if pool is None else pool
        B = check_pixels(self.cfg, pixels, False)
        if out is None:
            out = torch.empty(self.out_shape(B, pool), dtype=torch.float32, pin_memory=True)
        check_out(out, False)
        check(load_library().jepa_b200_encode_host(self._h, pixels.data_ptr(), B, POOLS[pool], out.data_ptr(),
                                                   out.numel() * 4, _stream_ptr(stream)), "encode_host")
        return out

    def debug_stage(self, pixels, layer: int, out=None, stream=None):
        """Residual stream f32 [B, N, D] after patch-embed and ``layer`` blocks."""
        import torch
        B = check_pixels(self.cfg, pixels, True, self.device)
        if out is None:
            out = torch.empty((B, self.cfg.n_tokens, self.cfg.dim), dtype=torch.float32, device=pixels.device)
        check_out(out, True, self.device)
        check(load_library().jepa_b200_debug_stage(self._h, pixels.data_ptr(), B, layer, 0, out.data_ptr(),
                                                   out.numel() * 4, _stream_ptr(stream)), "debug_stage")
        return out

    def close(self) -> None:
        if getattr(self, "_h", None):
            load_library().jepa_b200_free(self._h)
            self._h = None

    def __del__(self):
        try:
            self.close()
        except Exception:
            pass


# ---------------------------------------------------------------------------
# Single-kernel entry points (torch CUDA tensors in, asynchronous)
# ---------------------------------------------------------------------------
def _buf(t, nbytes: int, name: str) -> int:
    """Device address of an operand of a single-op call, after checking that
    it is a contiguous tensor of at least nbytes bytes: the library reads and
    writes through the plain pointer the sizes that the call's dimensions
    give, and cannot see the tensor's own."""
    import torch
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor, got {type(t).__name__}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    have = t.numel() * t.element_size()
    if have < nbytes:
        raise ValueError(f"{name} holds {have} bytes; the call's dimensions address {nbytes}")
    return _dptr(t)


def _opt(t, nbytes: int, name: str) -> Optional[int]:
    return None if t is None else _buf(t, nbytes, name)


def _weight_bytes(w_dtype: int, N: int, K: int) -> int:
    """Bytes of a weight operand of op_linear / op_gemv: f16 [N, K], or the
    repacked q8_0 codes [N, K] / q4_0 nibble bytes [N, K/2]."""
    if w_dtype == synth.DT_Q8_0:
        return N * K
    if w_dtype == synth.DT_Q4_0:
        return N * (K // 2)
    if w_dtype == synth.DT_F32:
        return N * K * 4
    return N * K * 2


def _scale_bytes(w_dtype: int, N: int, K: int) -> int:
    return N * (K // 32) * 2 if w_dtype in (synth.DT_Q8_0, synth.DT_Q4_0) else 0


def op_sync_status(stream=None) -> int:
    return int(load_library().jepa_b200_op_sync_status(_stream_ptr(stream)))


def op_set_timeout_ns(ns: int) -> None:
    load_library().jepa_b200_op_set_timeout_ns(ns)


def layernorm(x, gamma, beta, eps: float, out, in_row_stride: int = 1, rows: Optional[int] = None, stream=None):
    import torch
    D = x.shape[-1]
    rows = out.numel() // D if rows is None else rows
    dt = synth.DT_F16 if out.dtype == torch.float16 else synth.DT_F32
    x_rows = (rows - 1) * in_row_stride + 1 if rows > 0 else 0
    check(load_library().jepa_b200_op_layernorm(_buf(x, x_rows * D * 4, "x"), rows, D, in_row_stride,
                                                _buf(gamma, D * 4, "gamma"), _buf(beta, D * 4, "beta"), eps,
                                                _buf(out, rows * D * out.element_size(), "out"), dt,
                                                _stream_ptr(stream)), "layernorm")
    return out


def repack(dtype: int, blocks, N: int, K: int, qs, scales, stream=None):
    block_bytes = 34 if dtype == synth.DT_Q8_0 else 18
    check(load_library().jepa_b200_op_repack(dtype, _buf(blocks, N * (K // 32) * block_bytes, "blocks"), N, K,
                                             _buf(qs, _weight_bytes(dtype, N, K), "qs"),
                                             _buf(scales, _scale_bytes(dtype, N, K), "scales"),
                                             _stream_ptr(stream)), "repack")


def dequant_f16(dtype: int, qs, scales, N: int, K: int, out, stream=None):
    check(load_library().jepa_b200_op_dequant_f16(dtype, _buf(qs, _weight_bytes(dtype, N, K), "qs"),
                                                  _buf(scales, _scale_bytes(dtype, N, K), "scales"), N, K,
                                                  _buf(out, N * K * 2, "out"), _stream_ptr(stream)), "dequant_f16")
    return out


def linear(A, w, w_dtype: int, N: int, bias, epilogue: int, out, w_scales=None, stream=None):
    M, K = A.shape
    ldo = out.shape[-1]
    out_es = 2 if epilogue in (0, 1) else 4
    check(load_library().jepa_b200_op_linear(_buf(A, M * K * 2, "A"), M, K, _buf(w, _weight_bytes(w_dtype, N, K), "w"),
                                             _opt(w_scales, _scale_bytes(w_dtype, N, K), "w_scales"), w_dtype, N,
                                             _opt(bias, N * 4, "bias"), epilogue, _buf(out, M * ldo * out_es, "out"),
                                             ldo, _stream_ptr(stream)), "linear")
    return out


def linear_qkv(A, w, w_dtype: int, N: int, bias, ntok: int, heads: int, npad: int, first_part: int, q, k, vt,
               w_scales=None, stream=None):
    M, K = A.shape
    clips = M // ntok if ntok > 0 else 0
    qk_bytes = clips * heads * ntok * 64 * 2
    check(load_library().jepa_b200_op_linear_qkv(_buf(A, M * K * 2, "A"), M, K, _buf(w, _weight_bytes(w_dtype, N, K), "w"),
                                                 _opt(w_scales, _scale_bytes(w_dtype, N, K), "w_scales"), w_dtype, N,
                                                 _opt(bias, N * 4, "bias"), ntok, heads, npad, first_part,
                                                 _opt(q, qk_bytes, "q"), _opt(k, qk_bytes, "k"),
                                                 _opt(vt, clips * heads * 64 * npad * 2, "vt"), _stream_ptr(stream)),
          "linear_qkv")


def attention(q, k, vt, B: int, heads: int, ntok: int, npad: int, mask: int, has_cls: int, ppf: int, out,
              stream=None):
    qk_bytes = B * heads * ntok * 64 * 2
    check(load_library().jepa_b200_op_attention(_buf(q, qk_bytes, "q"), _buf(k, qk_bytes, "k"),
                                                _buf(vt, B * heads * 64 * npad * 2, "vt"), B, heads, ntok, npad, mask,
                                                has_cls, ppf, _buf(out, B * ntok * heads * 64 * 2, "out"),
                                                _stream_ptr(stream)), "attention")
    return out


def patch_embed(pixels, patch: int, tubelet: int, w_pe, D: int, bias, pos, cls, has_cls: int, x, stream=None):
    B, T, _, H, W = pixels.shape
    if patch < 1 or tubelet < 1:
        raise ValueError("patch and tubelet must be positive")
    kpad = (3 * tubelet * patch * patch + 63) // 64 * 64
    ntok = (1 if has_cls else 0) + (T // tubelet) * (H // patch) * (W // patch)
    check(load_library().jepa_b200_op_patch_embed(_buf(pixels, pixels.numel() * 4, "pixels"), B, T, H, W, patch,
                                                  tubelet, _buf(w_pe, D * kpad * 2, "w_pe"), D,
                                                  _opt(bias, D * 4, "bias"), _buf(pos, ntok * D * 4, "pos"),
                                                  _opt(cls, D * 4 if has_cls else 0, "cls"), has_cls,
                                                  _buf(x, B * ntok * D * 4, "x"), _stream_ptr(stream)), "patch_embed")
    return x


def gemv(x, w, w_dtype: int, N: int, bias, epi: int, y, resid=None, resid_row_stride: int = 0, w_scales=None,
         stream=None):
    M, K = x.shape
    resid_bytes = ((M - 1) * resid_row_stride + N) * 4 if M > 0 else 0
    check(load_library().jepa_b200_op_gemv(_buf(x, M * K * 4, "x"), M, K, _buf(w, _weight_bytes(w_dtype, N, K), "w"),
                                           _opt(w_scales, _scale_bytes(w_dtype, N, K), "w_scales"), w_dtype, N,
                                           _opt(bias, N * 4, "bias"), epi, _opt(resid, resid_bytes, "resid"),
                                           resid_row_stride, _buf(y, M * N * 4, "y"), _stream_ptr(stream)), "gemv")
    return y


def xattn_1q(q, k, vt, B: int, heads: int, ntok: int, npad: int, out, stream=None):
    check(load_library().jepa_b200_op_xattn_1q(_buf(q, heads * 64 * 4, "q"), _buf(k, B * heads * ntok * 64 * 2, "k"),
                                               _buf(vt, B * heads * 64 * npad * 2, "vt"), B, heads, ntok, npad,
                                               _buf(out, B * heads * 64 * 4, "out"), _stream_ptr(stream)), "xattn_1q")
    return out


def mean_pool(y, B: int, ntok: int, D: int, first: int, out, stream=None):
    check(load_library().jepa_b200_op_mean_pool(_buf(y, B * ntok * D * 4, "y"), B, ntok, D, first,
                                                _buf(out, B * D * 4, "out"), _stream_ptr(stream)), "mean_pool")
    return out
