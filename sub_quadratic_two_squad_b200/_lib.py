"""ctypes view of include/squad_attn.h. Loads the in-tree libsquad_attn.so and fails loudly without it."""
from __future__ import annotations

import ctypes
import os

PKG_DIR = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(PKG_DIR, "libsquad_attn.so")

SQUAD_OK, SQUAD_ERR_INVALID_ARG, SQUAD_ERR_UNSUPPORTED, SQUAD_ERR_CUDA, SQUAD_ERR_TIMEOUT = range(5)
SQUAD_BWD_TC_WHOLE, SQUAD_BWD_TC_CHUNKED, SQUAD_BWD_CUDA_CORE = 1, 2, 3
SQUAD_SP_BAND, SQUAD_SP_FRAMES, SQUAD_SP_CHUNKS = 0, 1, 2
SQUAD_BF16, SQUAD_FP32 = 0, 1
SQUAD_LOCAL_THEN_GLOBAL, SQUAD_GLOBAL_THEN_LOCAL, SQUAD_LOCAL_ONLY, SQUAD_GLOBAL_ONLY = 0, 1, 2, 3
SQUAD_NOALLOC_MAX_WORKSPACE_BYTES = 128 * 1024 * 1024

# Every symbol include/squad_attn.h declares, with (restype, argtypes).
_VP = ctypes.c_void_p


class SquadParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("h", ctypes.c_int), ("d", ctypes.c_int),
                ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("tw", ctypes.c_int), ("hw", ctypes.c_int), ("ww", ctypes.c_int),
                ("order", ctypes.c_int), ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


SQUAD_KPASS_MAX_LEVELS = 4
SQUAD_KPASS_FORWARD, SQUAD_KPASS_REVERSE = 0, 1


class SquadKpassParams(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("h", ctypes.c_int), ("d", ctypes.c_int),
                ("T", ctypes.c_int), ("H", ctypes.c_int), ("W", ctypes.c_int),
                ("k", ctypes.c_int),
                ("level_h", ctypes.c_int * SQUAD_KPASS_MAX_LEVELS), ("level_w", ctypes.c_int * SQUAD_KPASS_MAX_LEVELS),
                ("order", ctypes.c_int), ("dtype", ctypes.c_int), ("scale", ctypes.c_float)]


_PP = ctypes.POINTER(SquadParams)
_KP = ctypes.POINTER(SquadKpassParams)
SIGNATURES = {
    "squad_attn_fwd_workspace_bytes": (ctypes.c_size_t, [_PP]),
    "squad_attn_fwd": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "squad_attn_fwd_status": (ctypes.c_int, [_PP, _VP, _VP]),
    "squad_attn_bwd_workspace_bytes": (ctypes.c_size_t, [_PP]),
    "squad_attn_bwd": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "squad_attn_bwd_kernels": (ctypes.c_int, [_PP, ctypes.POINTER(ctypes.c_int)]),
    "full_attn_fwd": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "squad_attn_fwd_noalloc": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP]),
    "squad_attn_fwd_host_workspace_bytes": (ctypes.c_size_t, [_PP, ctypes.c_int]),
    "squad_attn_fwd_host": (ctypes.c_int, [_PP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, ctypes.c_int, _VP, _VP,
                                           _VP]),
    "squad_attn_flops": (ctypes.c_double, [_PP]),
    "squad_window_solve": (ctypes.c_int, [ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.POINTER(ctypes.c_int),
                                          ctypes.POINTER(ctypes.c_int), ctypes.POINTER(ctypes.c_int)]),
    "full_attn_flops": (ctypes.c_double, [_PP]),
    "squad_wait_selftest": (ctypes.c_int, [_VP, ctypes.c_ulonglong, _VP]),
    "squad_kpass_pass_params": (ctypes.c_int, [_KP, ctypes.c_int, _PP]),
    "squad_kpass_fwd_workspace_bytes": (ctypes.c_size_t, [_KP]),
    "squad_kpass_fwd": (ctypes.c_int, [_KP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "squad_kpass_bwd_workspace_bytes": (ctypes.c_size_t, [_KP]),
    "squad_kpass_bwd": (ctypes.c_int, [_KP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP, _VP]),
    "squad_kpass_status": (ctypes.c_int, [_KP, _VP, _VP]),
    "squad_kpass_flops": (ctypes.c_double, [_KP]),
    "squad_seqpar_reorder": (ctypes.c_int, [_PP, ctypes.c_int, ctypes.c_int, ctypes.c_int, _VP, _VP, _VP, _VP]),
    "squad_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "squad_attn_abi_version": (ctypes.c_int, []),
}

_lib = None


def load() -> ctypes.CDLL:
    """The loaded library (built in-tree by ``python -m sub_quadratic_two_squad_b200.build``)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sub_quadratic_two_squad_b200.build`")
        lib = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            fn = getattr(lib, name)
            fn.restype = res
            fn.argtypes = args
        _lib = lib
    return _lib
