"""B200-native JEPA ViT encoder forward.

Python binding of libjepa_b200.so (include/jepa_b200.h): argument marshalling
only.  Every step of the forward -- patch-embed, LayerNorm, the tcgen05 GEMMs,
flash attention, pooling and the attentive head -- runs in the library's
sm_100a kernels; PyTorch supplies device memory and streams.  There is no CPU
path: without the built library (or a CUDA device) the calls raise.
"""
from __future__ import annotations

import ctypes
from typing import List, Optional

from . import _abi, synth
from ._abi import JepaError, check, load_library

POOLS = synth.POOL_IDS


def _stream_ptr(stream) -> Optional[int]:
    import torch
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _ptr(t) -> int:
    return t.data_ptr()


def make_config(cfg: "synth.EncoderConfig") -> _abi.Config:
    return _abi.Config(dim=cfg.dim, depth=cfg.depth, heads=cfg.heads, mlp=cfg.mlp, patch=cfg.patch,
                       tubelet=cfg.tubelet, img_h=cfg.img_h, img_w=cfg.img_w, frames=cfg.frames,
                       has_cls=1 if cfg.has_cls else 0, mask=synth.MASK_IDS[cfg.mask],
                       head_sa_blocks=cfg.head_sa_blocks, n_classes=cfg.n_classes, ln_eps=cfg.ln_eps,
                       rope=1 if cfg.rope else 0)


class Model:
    """A loaded encoder on one CUDA device."""

    def __init__(self, cfg: "synth.EncoderConfig", table: List["synth.Tensor"], device: int = 0):
        lib = load_library()
        self.cfg = cfg
        self.device = device
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
        self._cfg = make_config(cfg)
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
        B = pixels.shape[0]
        if out is None:
            out = torch.empty(self.out_shape(B, pool), dtype=torch.float32, device=pixels.device)
        check(load_library().jepa_b200_encode(self._h, _ptr(pixels), B, POOLS[pool], _ptr(out),
                                              out.numel() * 4, _stream_ptr(stream)), "encode")
        return out

    def encode_host(self, pixels, pool: Optional[str] = None, out=None, stream=None):
        """End to end from host memory: pixels CPU float32 (pinned for
        asynchronous copies) -> result in a CPU tensor.  Synchronous."""
        import torch
        pool = self.cfg.pool if pool is None else pool
        B = pixels.shape[0]
        if out is None:
            out = torch.empty(self.out_shape(B, pool), dtype=torch.float32, pin_memory=True)
        check(load_library().jepa_b200_encode_host(self._h, _ptr(pixels), B, POOLS[pool], _ptr(out),
                                                   out.numel() * 4, _stream_ptr(stream)), "encode_host")
        return out

    def debug_stage(self, pixels, layer: int, out=None, stream=None):
        """Residual stream f32 [B, N, D] after patch-embed and ``layer`` blocks."""
        import torch
        B = pixels.shape[0]
        if out is None:
            out = torch.empty((B, self.cfg.n_tokens, self.cfg.dim), dtype=torch.float32, device=pixels.device)
        check(load_library().jepa_b200_debug_stage(self._h, _ptr(pixels), B, layer, 0, _ptr(out),
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
def op_sync_status(stream=None) -> int:
    return int(load_library().jepa_b200_op_sync_status(_stream_ptr(stream)))


def op_set_timeout_ns(ns: int) -> None:
    load_library().jepa_b200_op_set_timeout_ns(ns)


def layernorm(x, gamma, beta, eps: float, out, in_row_stride: int = 1, rows: Optional[int] = None, stream=None):
    import torch
    D = x.shape[-1]
    rows = out.numel() // D if rows is None else rows
    dt = synth.DT_F16 if out.dtype == torch.float16 else synth.DT_F32
    check(load_library().jepa_b200_op_layernorm(_ptr(x), rows, D, in_row_stride, _ptr(gamma), _ptr(beta), eps,
                                                _ptr(out), dt, _stream_ptr(stream)), "layernorm")
    return out


def repack(dtype: int, blocks, N: int, K: int, qs, scales, stream=None):
    check(load_library().jepa_b200_op_repack(dtype, _ptr(blocks), N, K, _ptr(qs), _ptr(scales),
                                             _stream_ptr(stream)), "repack")


def dequant_f16(dtype: int, qs, scales, N: int, K: int, out, stream=None):
    check(load_library().jepa_b200_op_dequant_f16(dtype, _ptr(qs), _ptr(scales), N, K, _ptr(out),
                                                  _stream_ptr(stream)), "dequant_f16")
    return out


def linear(A, w, w_dtype: int, N: int, bias, epilogue: int, out, w_scales=None, stream=None):
    M, K = A.shape
    check(load_library().jepa_b200_op_linear(_ptr(A), M, K, _ptr(w), _ptr(w_scales) if w_scales is not None else None,
                                             w_dtype, N, _ptr(bias) if bias is not None else None, epilogue,
                                             _ptr(out), out.shape[-1], _stream_ptr(stream)), "linear")
    return out


def linear_qkv(A, w, w_dtype: int, N: int, bias, ntok: int, heads: int, npad: int, first_part: int, q, k, vt,
               w_scales=None, stream=None):
    M, K = A.shape
    f = lambda t: _ptr(t) if t is not None else None
    check(load_library().jepa_b200_op_linear_qkv(_ptr(A), M, K, _ptr(w), f(w_scales), w_dtype, N, f(bias), ntok,
                                                 heads, npad, first_part, f(q), f(k), f(vt), _stream_ptr(stream)),
          "linear_qkv")


def attention(q, k, vt, B: int, heads: int, ntok: int, npad: int, mask: int, has_cls: int, ppf: int, out,
              stream=None):
    check(load_library().jepa_b200_op_attention(_ptr(q), _ptr(k), _ptr(vt), B, heads, ntok, npad, mask, has_cls,
                                                ppf, _ptr(out), _stream_ptr(stream)), "attention")
    return out


def patch_embed(pixels, patch: int, tubelet: int, w_pe, D: int, bias, pos, cls, has_cls: int, x, stream=None):
    B, T, _, H, W = pixels.shape
    check(load_library().jepa_b200_op_patch_embed(_ptr(pixels), B, T, H, W, patch, tubelet, _ptr(w_pe), D,
                                                  _ptr(bias) if bias is not None else None, _ptr(pos),
                                                  _ptr(cls) if cls is not None else None, has_cls, _ptr(x),
                                                  _stream_ptr(stream)), "patch_embed")
    return x


def gemv(x, w, w_dtype: int, N: int, bias, epi: int, y, resid=None, resid_row_stride: int = 0, w_scales=None,
         stream=None):
    M, K = x.shape
    f = lambda t: _ptr(t) if t is not None else None
    check(load_library().jepa_b200_op_gemv(_ptr(x), M, K, _ptr(w), f(w_scales), w_dtype, N, f(bias), epi, f(resid),
                                           resid_row_stride, _ptr(y), _stream_ptr(stream)), "gemv")
    return y


def xattn_1q(q, k, vt, B: int, heads: int, ntok: int, npad: int, out, stream=None):
    check(load_library().jepa_b200_op_xattn_1q(_ptr(q), _ptr(k), _ptr(vt), B, heads, ntok, npad, _ptr(out),
                                               _stream_ptr(stream)), "xattn_1q")
    return out


def mean_pool(y, B: int, ntok: int, D: int, first: int, out, stream=None):
    check(load_library().jepa_b200_op_mean_pool(_ptr(y), B, ntok, D, first, _ptr(out), _stream_ptr(stream)),
          "mean_pool")
    return out
