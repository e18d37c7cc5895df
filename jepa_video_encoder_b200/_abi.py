"""ctypes declarations of the C ABI in include/jepa_b200.h (argument
marshalling only; every step of the forward runs in libjepa_b200.so)."""
from __future__ import annotations

import ctypes
import os
from ctypes import (POINTER, c_char_p, c_double, c_float, c_int, c_int64, c_size_t, c_ulonglong, c_void_p)

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libjepa_b200.so")

OK, ERR_ARG, ERR_MISSING_TENSOR, ERR_SHAPE, ERR_DTYPE, ERR_CUDA, ERR_TIMEOUT, ERR_UNSUPPORTED = \
    0, -1, -2, -3, -4, -5, -6, -7
EPI_F16, EPI_GELU_F16, EPI_RESID_F32, EPI_F32 = 0, 1, 2, 3
KERNEL_CLASSES = ("patch_embed", "layernorm", "gemm_qkv", "attention", "gemm_out", "gemm_up", "gemm_down",
                  "pool_head")


class Config(ctypes.Structure):
    _fields_ = [("dim", c_int), ("depth", c_int), ("heads", c_int), ("mlp", c_int),
                ("patch", c_int), ("tubelet", c_int), ("img_h", c_int), ("img_w", c_int),
                ("frames", c_int), ("has_cls", c_int), ("mask", c_int),
                ("head_sa_blocks", c_int), ("n_classes", c_int), ("ln_eps", c_float), ("rope", c_int),
                ("quant_f16_copy", c_int), ("pred_depth", c_int), ("pred_dim", c_int), ("pred_heads", c_int),
                ("pred_mlp", c_int), ("act_bf16", c_int), ("wm_depth", c_int), ("wm_heads", c_int),
                ("wm_mlp", c_int), ("wm_action_dim", c_int), ("wm_window", c_int), ("wm_proj_hidden", c_int),
                ("wm_pred_hidden", c_int)]


class TensorEntry(ctypes.Structure):
    _fields_ = [("name", c_char_p), ("dtype", c_int), ("ndim", c_int), ("shape", c_int64 * 5),
                ("data", c_void_p), ("nbytes", c_size_t)]


# name -> (restype, argtypes); every symbol the header declares
SIGNATURES = {
    "jepa_b200_load_weights": (c_int, [POINTER(Config), POINTER(TensorEntry), c_int, c_int, POINTER(c_void_p)]),
    "jepa_b200_encode": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "jepa_b200_encode_host": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "jepa_b200_predict": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, c_void_p, c_int, c_void_p, c_size_t,
                                  c_void_p]),
    "jepa_b200_lewm_predict": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "jepa_b200_lewm_rollout": (c_int, [c_void_p, c_void_p, c_int, c_void_p, c_int, c_int, c_void_p, c_size_t,
                                       c_void_p]),
    "jepa_b200_out_shape": (c_int, [c_void_p, c_int, c_int, POINTER(c_int64)]),
    "jepa_b200_debug_stage": (c_int, [c_void_p, c_void_p, c_int, c_int, c_int, c_void_p, c_size_t, c_void_p]),
    "jepa_b200_sync_status": (c_int, [c_void_p, c_void_p]),
    "jepa_b200_last_ms": (c_double, [c_void_p]),
    "jepa_b200_model_n_bytes": (c_size_t, [c_void_p]),
    "jepa_b200_set_timeout_ns": (c_int, [c_void_p, c_ulonglong]),
    "jepa_b200_set_graph": (c_int, [c_void_p, c_int]),
    "jepa_b200_last_launch_count": (c_int, [c_void_p]),
    "jepa_b200_set_profiling": (c_int, [c_void_p, c_int]),
    "jepa_b200_profile_read": (c_int, [c_void_p, POINTER(c_double), POINTER(c_int), c_int]),
    "jepa_b200_status_str": (c_char_p, [c_int]),
    "jepa_b200_free": (None, [c_void_p]),
    "jepa_b200_op_layernorm": (c_int, [c_void_p, c_int, c_int, c_int, c_void_p, c_void_p, c_float, c_void_p,
                                       c_int, c_void_p]),
    "jepa_b200_op_repack": (c_int, [c_int, c_void_p, c_int, c_int, c_void_p, c_void_p, c_void_p]),
    "jepa_b200_op_dequant_f16": (c_int, [c_int, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "jepa_b200_op_linear": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p, c_int,
                                    c_void_p, c_int, c_void_p]),
    "jepa_b200_op_linear_qkv": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p, c_int,
                                        c_int, c_int, c_int, c_void_p, c_void_p, c_void_p, c_void_p]),
    "jepa_b200_op_attention": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_int, c_int,
                                       c_int, c_void_p, c_void_p]),
    "jepa_b200_op_patch_embed": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_int, c_int, c_void_p, c_int,
                                         c_void_p, c_void_p, c_void_p, c_int, c_void_p, c_void_p]),
    "jepa_b200_op_gemv": (c_int, [c_void_p, c_int, c_int, c_void_p, c_void_p, c_int, c_int, c_void_p, c_int,
                                  c_void_p, c_int, c_void_p, c_void_p]),
    "jepa_b200_op_xattn_1q": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_int, c_int, c_void_p,
                                      c_void_p]),
    "jepa_b200_op_mean_pool": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "jepa_b200_op_mean_pool_noalloc": (c_int, [c_void_p, c_int, c_int, c_int, c_int, c_void_p, c_void_p]),
    "jepa_b200_op_sync_status": (c_int, [c_void_p]),
    "jepa_b200_op_set_timeout_ns": (None, [c_ulonglong]),
}

_lib = None


class JepaError(RuntimeError):
    def __init__(self, status: int, what: str = ""):
        self.status = status
        msg = status_str(status) if _lib is not None else str(status)
        super().__init__(f"{what}: {msg} ({status})" if what else f"{msg} ({status})")


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libjepa_b200.so.  There is no fallback: without the library the
    package cannot compute anything and says so."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise RuntimeError(f"{path} is missing: build it with `python -m jepa_video_encoder_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def status_str(status: int) -> str:
    return load_library().jepa_b200_status_str(status).decode()


def check(status: int, what: str = "") -> None:
    if status != OK:
        raise JepaError(status, what)
