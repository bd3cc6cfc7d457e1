"""ctypes binding of the C ABI in include/msgla.h (argument marshalling only).

Every computation happens in the CUDA library; this module only converts
Python/torch arguments into the C structs and pointers the ABI expects. If the
library is missing, loading fails loudly: there is no CPU fallback.
"""
from __future__ import annotations

import ctypes
import os
from ctypes import POINTER, c_char_p, c_float, c_int, c_longlong, c_size_t, c_void_p

MAX_SCALES = 8
PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG, "libmsgla.so")

STATUS = {0: "MSGLA_OK", -1: "MSGLA_ERR_INVALID_ARG", -2: "MSGLA_ERR_UNSUPPORTED", -3: "MSGLA_ERR_CUDA",
          -4: "MSGLA_ERR_DEVICE_TIMEOUT", -5: "MSGLA_ERR_RANGE", -6: "MSGLA_ERR_WORKSPACE"}

# which-codes of msgla_workspace_tensor
# msgla_workspace_tensor views: WS_QS / WS_KS are the decay-scaled queries and keys
# (q e^{b-m}, k e^{m-b} per 128-row chunk), WS_U the gate inputs and fusion logits
# of the unpooled rows, WS_GAMMA / WS_MID the per-chunk decays
WS_POOLED, WS_QS, WS_KS, WS_V = 0, 1, 2, 3
WS_O, WS_Y, WS_FUSION, WS_U, WS_GAMMA, WS_MID = 5, 6, 7, 8, 9, 10


class Config(ctypes.Structure):
    _fields_ = [("d", c_int), ("n_scales", c_int), ("scales", c_int * MAX_SCALES),
                ("heads", c_int * MAX_SCALES), ("d_k", c_int), ("d_v", c_int), ("gate_rank", c_int),
                ("chunk", c_int), ("gate_normalizer", c_float), ("qk_scale", c_float),
                ("head_norm", c_int), ("head_norm_eps", c_float)]


class Weights(ctypes.Structure):
    _fields_ = [("Wq", c_void_p * MAX_SCALES), ("Wk", c_void_p * MAX_SCALES), ("Wv", c_void_p * MAX_SCALES),
                ("Wg1", c_void_p * MAX_SCALES), ("Wg2", c_void_p * MAX_SCALES), ("bg", c_void_p * MAX_SCALES),
                ("Wo", c_void_p * MAX_SCALES), ("Wfuse", c_void_p), ("bfuse", c_void_p),
                ("norm_w", c_void_p * MAX_SCALES)]


class MSGLAError(RuntimeError):
    def __init__(self, status: int, message: str):
        super().__init__(f"{STATUS.get(status, status)}: {message}")
        self.status = status


_SIGNATURES = {
    "msgla_create": (c_int, [POINTER(c_void_p), POINTER(Config), POINTER(Weights), c_int]),
    "msgla_destroy": (None, [c_void_p]),
    "msgla_workspace_size": (c_int, [c_void_p, c_int, c_int, POINTER(c_size_t)]),
    "msgla_forward": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "msgla_forward_masked": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                     c_void_p]),
    "msgla_forward_noalloc": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p]),
    "msgla_forward_profiled": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t,
                                       c_void_p, POINTER(c_void_p), c_int, POINTER(c_int)]),
    "msgla_workspace_size_host": (c_int, [c_void_p, c_int, c_int, POINTER(c_size_t)]),
    "msgla_forward_host": (c_int, [c_void_p, c_void_p, c_int, c_int, c_void_p, c_void_p, c_size_t, c_void_p]),
    "msgla_sync_status": (c_int, [c_void_p]),
    "msgla_workspace_tensor": (c_int, [c_void_p, c_int, c_int, c_int, c_int, POINTER(c_size_t), POINTER(c_int)]),
    "msgla_test_skip_arrival": (c_int, [c_void_p, c_int]),
    "msgla_launch_plan": (c_int, [c_void_p, c_int, c_int, c_char_p, c_size_t]),
    "msgla_cache_size": (c_int, [c_void_p, c_int, POINTER(c_size_t)]),
    "msgla_cache_reset": (c_int, [c_void_p, c_void_p, c_int, c_void_p]),
    "msgla_step_workspace_size": (c_int, [c_void_p, c_int, POINTER(c_size_t)]),
    "msgla_step": (c_int, [c_void_p, c_void_p, c_void_p, c_int, c_longlong, c_void_p, c_void_p, c_size_t,
                           c_void_p]),
    "msgla_status_string": (c_char_p, [c_int]),
    "msgla_last_error": (c_char_p, []),
}

_lib = None


def load(path: str = LIB_PATH) -> ctypes.CDLL:
    """Load libmsgla.so (raises if it has not been built)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(path):
        raise ImportError(f"{path} not found: build it with `python -m scale_gated_linear_b200.build`")
    lib = ctypes.CDLL(path)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int) -> None:
    if status != 0:
        raise MSGLAError(status, load().msgla_last_error().decode())


def status_string(status: int) -> str:
    return load().msgla_status_string(status).decode()
