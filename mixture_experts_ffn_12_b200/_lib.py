"""ctypes view of libmoe.so (include/moe.h).  Loading never falls back: if the
library is missing or stale the caller gets an exception, not a CPU path."""
from __future__ import annotations

import ctypes
import os
import threading

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe.so")

MOE_OK = 0
MOE_ERR_INVALID_ARG = 1
MOE_ERR_UNSUPPORTED = 2
MOE_ERR_WORKSPACE = 3
MOE_ERR_CUDA = 4
MOE_ERR_TIMEOUT = 5
MOE_ERR_DEVICE_BOUNDS = 6

MOE_F32, MOE_BF16 = 0, 1
MOE_W_DENSE, MOE_W_MXFP4, MOE_W_MXFP4_A8 = 0, 1, 2

SIZE_INVALID = ctypes.c_size_t(-1).value
ABI_VERSION = 2


class MoeConfig(ctypes.Structure):
    _fields_ = [
        ("hidden_size", ctypes.c_int32),
        ("intermediate_size", ctypes.c_int32),
        ("num_local_experts", ctypes.c_int32),
        ("num_experts_per_tok", ctypes.c_int32),
        ("swiglu_limit", ctypes.c_float),
        ("swiglu_alpha", ctypes.c_float),
        ("dtype", ctypes.c_int32),
        ("wfmt", ctypes.c_int32),
        ("y_f32", ctypes.c_int32),
        ("h_split", ctypes.c_int32),
    ]


class MoeExpertWeights(ctypes.Structure):
    _fields_ = [(n, ctypes.c_void_p) for n in (
        "w_gate", "w_up", "w_down", "s_gate", "s_up", "s_down", "b_gate", "b_up", "b_down")]


class MoeGlmParams(ctypes.Structure):
    _fields_ = [
        ("norm_topk_prob", ctypes.c_int32),
        ("routed_scaling_factor", ctypes.c_float),
        ("e_score_correction_bias", ctypes.c_void_p),
        ("ws_gate", ctypes.c_void_p),
        ("ws_up", ctypes.c_void_p),
        ("ws_down", ctypes.c_void_p),
        ("shared_intermediate_size", ctypes.c_int32),
    ]


_P = ctypes.c_void_p
_CFG = ctypes.POINTER(MoeConfig)
_W = ctypes.POINTER(MoeExpertWeights)
_GP = ctypes.POINTER(MoeGlmParams)
_I64 = ctypes.c_int64
_ST = ctypes.c_int

SIGNATURES = {
    "moe_abi_version": (ctypes.c_int32, []),
    "moe_status_string": (ctypes.c_char_p, [_ST]),
    "moe_config_check": (_ST, [_CFG]),
    "moe_permute_workspace_size": (ctypes.c_size_t, [_CFG, _I64]),
    "moe_expert_ffn_workspace_size": (ctypes.c_size_t, [_CFG, _I64]),
    "moe_workspace_size": (ctypes.c_size_t, [_CFG, _I64]),
    "moe_router_topk": (_ST, [_CFG, _I64, _P, _P, _P, _P, _P, _P]),
    "moe_permute": (_ST, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_permute_noalloc": (_ST, [_CFG, _I64, _P, _P, _P, _P, _P, _P, _P]),
    "moe_expert_ffn": (_ST, [_CFG, _I64, _P, _P, _W, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_combine": (_ST, [_CFG, _I64, _P, _P, _P, _P, _P]),
    "moe_layer_forward": (_ST, [_CFG, _I64, _P, _P, _P, _W, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_mxfp8_scale_stride": (ctypes.c_int32, [ctypes.c_int32]),
    "moe_quantize_mxfp8": (_ST, [_I64, ctypes.c_int32, _P, _P, _P, _P]),
    "moe_last_device_error": (_ST, []),
    "moe_set_stage_events": (None, [ctypes.POINTER(ctypes.c_void_p), ctypes.POINTER(ctypes.c_void_p),
                                    ctypes.c_int32]),
    "moe_launch_count": (ctypes.c_uint64, []),
    "moe_set_expert_gemm_variant": (_ST, [ctypes.c_int32]),
    "moe_set_wait_limit_ns": (None, [ctypes.c_uint64]),
    "moe_glm_router_workspace_size": (ctypes.c_size_t, [_CFG, _I64]),
    "moe_glm_workspace_size": (ctypes.c_size_t, [_CFG, _GP, _I64]),
    "moe_glm_router_topk": (_ST, [_CFG, _GP, _I64, _P, _P, _P, _P, _P, ctypes.c_size_t, _P]),
    "moe_glm_layer_forward": (_ST, [_CFG, _GP, _I64, _P, _P, _W, _P, _P, _P, _P, ctypes.c_size_t, _P]),
}

_lock = threading.Lock()
_lib = None


def load() -> ctypes.CDLL:
    """The loaded library (built in-tree by mixture_experts_ffn_12_b200.build)."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                                   "`python -m mixture_experts_ffn_12_b200.build`")
            lib = ctypes.CDLL(LIB_PATH)
            for name, (res, args) in SIGNATURES.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            if lib.moe_abi_version() != ABI_VERSION:
                raise RuntimeError("libmoe ABI version mismatch")
            _lib = lib
        return _lib


def status_string(code: int) -> str:
    return load().moe_status_string(code).decode()
