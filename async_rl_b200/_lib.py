"""ctypes loader for libbi_isloss.so (the C ABI in include/bi_isloss.h).

Loading fails loudly when the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libbi_isloss.so")

EXPORTED = ("bi_workspace_bytes", "bi_workspace_bytes_min", "bi_workspace_bytes_pstore", "bi_logprob_fwd", "bi_logprob_fwd_noalloc", "bi_is_loss_fwd_bwd", "bi_d3_stats",
            "bi_status_string", "bi_version", "bi_debug_force_timeout_once", "bi_profile_enable",
            "bi_profile_reset", "bi_profile_read", "bi_gemm_bf16", "bi_rmsnorm")

STATUS_NAMES = {0: "BI_OK", 1: "BI_ERR_INVALID_ARG", 2: "BI_ERR_UNSUPPORTED_SHAPE", 3: "BI_ERR_WORKSPACE",
                4: "BI_ERR_CUDA", 5: "BI_ERR_TIMEOUT", 6: "BI_ERR_BAD_TARGET", 7: "BI_ERR_NONFINITE",
                8: "BI_ERR_BAD_OFFSETS"}

_lib = None


class LossCfg(ctypes.Structure):
    """bi_loss_cfg"""
    _fields_ = [("variant", ctypes.c_int32), ("eps_low", ctypes.c_float), ("eps_high", ctypes.c_float),
                ("gate", ctypes.c_float), ("flags", ctypes.c_int32)]


LOSS_STORE_P = 1  # bi_loss_cfg.flags: BI_LOSS_STORE_P


LOSS_VARIANTS = {"unclipped": 0, "ppo_clip": 1, "seq_gate": 2}

_p = ctypes.c_void_p
_i32 = ctypes.c_int32
_i64 = ctypes.c_int64
_u64 = ctypes.c_uint64
_sz = ctypes.c_size_t
_f64 = ctypes.c_double


def load() -> ctypes.CDLL:
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with `python -m async_rl_b200.build` "
                           "(there is no CPU fallback)")
    lib = ctypes.CDLL(LIB_PATH)
    lib.bi_workspace_bytes.argtypes = [_i64, _i32, _i32, _i32]
    lib.bi_workspace_bytes.restype = _sz
    lib.bi_workspace_bytes_min.argtypes = [_i64, _i32, _i32, _i32]
    lib.bi_workspace_bytes_min.restype = _sz
    lib.bi_workspace_bytes_pstore.argtypes = [_i64, _i32, _i32, _i32]
    lib.bi_workspace_bytes_pstore.restype = _sz
    lib.bi_logprob_fwd.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p, _p, _p, _p, _sz, _p]
    lib.bi_logprob_fwd.restype = ctypes.c_int
    lib.bi_logprob_fwd_noalloc.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p, _p, _p, _p]
    lib.bi_logprob_fwd_noalloc.restype = ctypes.c_int
    lib.bi_is_loss_fwd_bwd.argtypes = [_p, _p, _p, _p, _p, _p, _p, _p, _i32, _i32, _f64, _p, _i64, _i32, _i32,
                                       _p, _p, _p, _p, _p, _p, _p, _p, _p, _sz, _p]
    lib.bi_is_loss_fwd_bwd.restype = ctypes.c_int
    lib.bi_d3_stats.argtypes = [_p, _p, _p, _i64, _p, _p, _p, _sz, _p]
    lib.bi_d3_stats.restype = ctypes.c_int
    lib.bi_status_string.argtypes = [ctypes.c_int]
    lib.bi_status_string.restype = ctypes.c_char_p
    lib.bi_version.argtypes = []
    lib.bi_version.restype = _i32
    lib.bi_debug_force_timeout_once.argtypes = [_u64]
    lib.bi_debug_force_timeout_once.restype = None
    lib.bi_profile_enable.argtypes = [_i32]
    lib.bi_profile_enable.restype = None
    lib.bi_profile_reset.argtypes = []
    lib.bi_profile_reset.restype = None
    lib.bi_profile_read.argtypes = [ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                                    ctypes.POINTER(ctypes.c_int64), _i32]
    lib.bi_profile_read.restype = _i32
    lib.bi_gemm_bf16.argtypes = [_p, _p, _p, _i64, _i32, _i32, _p, _p]
    lib.bi_gemm_bf16.restype = ctypes.c_int
    lib.bi_rmsnorm.argtypes = [_p, _p, ctypes.c_float, _p, _i64, _i32, _p, _p]
    lib.bi_rmsnorm.restype = ctypes.c_int
    _lib = lib
    return lib
