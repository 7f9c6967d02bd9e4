"""ctypes binding of libmoe.so (include/moe.h).  Argument marshalling only."""
from __future__ import annotations

import ctypes
import os
import re

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libmoe.so")
HEADER = os.path.join(os.path.dirname(_HERE), "include", "moe.h")

MOE_OK, MOE_ERR_INVALID_ARG, MOE_ERR_UNSUPPORTED, MOE_ERR_CUDA, MOE_ERR_OOM, \
    MOE_ERR_DEVICE_CHECK = range(6)
MOE_FP32, MOE_BF16, MOE_BF16_E4M3_GATEUP, MOE_BF16_E4M3 = 0, 1, 2, 3
STATUS_NAMES = {0: "MOE_OK", 1: "MOE_ERR_INVALID_ARG", 2: "MOE_ERR_UNSUPPORTED",
                3: "MOE_ERR_CUDA", 4: "MOE_ERR_OOM", 5: "MOE_ERR_DEVICE_CHECK"}


class MoeCfg(ctypes.Structure):
    _fields_ = [("T", ctypes.c_int32), ("d", ctypes.c_int32), ("n_routed", ctypes.c_int32),
                ("n_shared", ctypes.c_int32), ("top_k", ctypes.c_int32),
                ("inter", ctypes.c_int32), ("dtype", ctypes.c_int32),
                ("alpha1", ctypes.c_float), ("centroids", ctypes.c_void_p),
                ("logit_bias", ctypes.c_void_p), ("w_gate", ctypes.c_void_p),
                ("w_up", ctypes.c_void_p), ("w_down", ctypes.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_lib = None

_P = ctypes.c_void_p
_SIGS = {
    "moe_create": (ctypes.c_int, [ctypes.POINTER(MoeCfg), ctypes.POINTER(ctypes.c_void_p)]),
    "moe_forward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward_host": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_forward_host_pipelined": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_pipeline_wait": (ctypes.c_int, [_P, _P]),
    "moe_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int32, ctypes.c_int64, _P]),
    "moe_debug_copy": (ctypes.c_int, [_P, ctypes.c_int32, _P, ctypes.c_size_t, _P, _P]),
    "moe_device_status": (ctypes.c_int, [_P, _P]),
    "moe_expert_psum": (ctypes.c_int, [_P, _P, _P]),
    "moe_balance_loss": (ctypes.c_int, [_P, _P, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                                        _P, _P]),
    "moe_timing_begin": (ctypes.c_int, [_P, ctypes.c_int32]),
    "moe_timing_end": (ctypes.c_int, [_P, ctypes.POINTER(ctypes.c_double),
                                      ctypes.POINTER(ctypes.c_int32)]),
    "moe_route_noalloc": (ctypes.c_int, [_P, _P, _P, ctypes.c_int32, ctypes.c_int32,
                                         ctypes.c_int32, ctypes.c_int32, ctypes.c_float,
                                         _P, _P, _P, _P, _P, _P]),
    "moe_ep_create": (ctypes.c_int, [ctypes.POINTER(MoeCfg), ctypes.c_int32, ctypes.c_int32,
                                     ctypes.c_int64, ctypes.POINTER(ctypes.c_void_p)]),
    "moe_ep_dispatch": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, _P, _P]),
    "moe_ep_experts": (ctypes.c_int, [_P, _P, _P, ctypes.c_int64, _P, _P]),
    "moe_ep_combine": (ctypes.c_int, [_P, _P, _P, _P, _P, _P]),
    "moe_ep_expert_psum": (ctypes.c_int, [_P, _P, _P]),
    "moe_ep_device_status": (ctypes.c_int, [_P, _P]),
    "moe_ep_recv_capacity": (ctypes.c_int64, [_P]),
    "moe_ep_destroy": (None, [_P]),
    "moe_backward_prepare": (ctypes.c_int, [_P]),
    "moe_backward": (ctypes.c_int, [_P, _P, _P, _P, _P, _P, ctypes.c_float, _P, _P, _P, _P, _P, _P,
                                    _P]),
    "moe_kernels_per_forward": (ctypes.c_int32, [_P]),
    "moe_device_bytes": (ctypes.c_size_t, [_P]),
    "moe_destroy": (None, [_P]),
    "moe_last_error": (ctypes.c_char_p, []),
    "moe_abi_version": (ctypes.c_int32, []),
}


def lib() -> ctypes.CDLL:
    """Load libmoe.so (fails loudly if it has not been built: there is no fallback)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                               "`python -m mixture_experts_layer_65_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in _SIGS.items():
            if hasattr(L, name):
                fn = getattr(L, name)
                fn.restype = res
                fn.argtypes = args
        _lib = L
    return _lib


def check(status: int) -> None:
    if status != MOE_OK:
        raise MoeError(status, lib().moe_last_error().decode(errors="replace"))


def header_symbols() -> list[str]:
    """Entry points declared in include/moe.h."""
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(moe_[a-z_0-9]+)\s*\(", text)))
