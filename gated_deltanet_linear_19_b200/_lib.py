"""ctypes loader for libgdn.so (the C ABI declared in include/gdn.h).

The shared library is built in-tree by ``gated_deltanet_linear_19_b200.build``. There is no
fallback of any kind: if the library is missing or cannot be loaded, ``load()`` raises.
"""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdn.so")

GDN_OK = 0
GDN_EINVAL = -1
GDN_ESLOT = -2
GDN_EALIGN = -3
GDN_ECUDA = -4
GDN_ETIMEOUT = -5
GDN_EWORKSPACE = -6
GDN_EUNSUPPORTED = -7

GDN_F32 = 0
GDN_BF16 = 1
GDN_F16 = 2

GDN_PREFILL_DEFAULT = 0
GDN_PREFILL_SIMT = 1
GDN_PREFILL_RECURRENT = 4
GDN_PREFILL_OUT_GATE = 8
GDN_PREFILL_TC_HEAD_SCAN = 16
GDN_PREFILL_TC_TILE_SCAN = 32

# Every symbol include/gdn.h declares.
EXPORTS = ("gdn_conv_step", "gdn_decode_step", "gdn_layer_decode", "gdn_decode_workspace_size",
           "gdn_layer_decode_launches",
           "gdn_chunked_prefill", "gdn_layer_prefill",
           "gdn_chunked_prefill_noalloc", "gdn_prefill_workspace_size", "gdn_state_slot_copy",
           "gdn_device_status", "gdn_status_string", "gdn_abi_version", "gdn_gated_norm",
           "gdn_debug_set_wait_limit", "gdn_decode_pipe_buffer_size", "gdn_decode_pipe_create",
           "gdn_decode_pipe_step", "gdn_decode_pipe_flush", "gdn_decode_pipe_destroy",
           "gdn_decode_pipe_packed_bytes", "gdn_decode_pipe_step_packed")


GDN_LAYOUT_DEFAULT = 0
GDN_GQA_TILED = 1
GDN_GATES_MIXED_BA = 2


class GdnDims(ctypes.Structure):
    _fields_ = [("n_slots", ctypes.c_int32), ("H_k", ctypes.c_int32), ("H_v", ctypes.c_int32),
                ("d_k", ctypes.c_int32), ("d_v", ctypes.c_int32), ("d_conv", ctypes.c_int32),
                ("layout", ctypes.c_int32)]


class GdnOutGate(ctypes.Structure):
    _fields_ = [("z", ctypes.c_void_p), ("z_dtype", ctypes.c_int32),
                ("norm_w", ctypes.c_void_p), ("eps", ctypes.c_float)]


_lock = threading.Lock()
_lib = None


def load(path: str | None = None):
    """Load libgdn.so and declare argument types. Raises if it is not built."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(
                f"libgdn.so not found at {p}; build it with "
                "`python -m gated_deltanet_linear_19_b200.build` (no CPU fallback exists)")
        lib = ctypes.CDLL(p)
        P = ctypes.c_void_p
        I32 = ctypes.c_int32
        I64 = ctypes.c_int64
        F = ctypes.c_float
        S = ctypes.c_size_t
        U32 = ctypes.c_uint32
        D = ctypes.POINTER(GdnDims)
        lib.gdn_conv_step.argtypes = [D, P, I32, P, P, I32, P, P, P, I32, I64, P, P, P, P, F, F,
                                      P, P, P, I32, P, P, P]
        lib.gdn_conv_step.restype = ctypes.c_int
        lib.gdn_decode_step.argtypes = [D, P, P, P, I32, P, P, P, P, P, I32, P, I32, P]
        lib.gdn_decode_step.restype = ctypes.c_int
        G = ctypes.POINTER(GdnOutGate)
        lib.gdn_layer_decode.argtypes = [D, P, I32, P, P, I32, P, P, I32, P, P, P, P, F, F, P,
                                         P, I32, P, S, G, P]
        lib.gdn_layer_decode.restype = ctypes.c_int
        lib.gdn_decode_workspace_size.argtypes = [D, I32]
        lib.gdn_decode_workspace_size.restype = S
        lib.gdn_layer_decode_launches.argtypes = [D, I32, I32]
        lib.gdn_layer_decode_launches.restype = I32
        lib.gdn_chunked_prefill.argtypes = [D, P, P, P, I32, P, P, P, P, P, P, I32, I64, I32,
                                            P, I32, P, S, U32, P]
        lib.gdn_chunked_prefill.restype = ctypes.c_int
        lib.gdn_layer_prefill.argtypes = [D, P, I32, P, P, I32, P, P, P, I32, I64, P, P, P, P,
                                          F, F, P, I32, P, I32, P, S, U32, G, P]
        lib.gdn_gated_norm.argtypes = [D, P, I32, G, P, I32, I64, P]
        lib.gdn_gated_norm.restype = ctypes.c_int
        lib.gdn_layer_prefill.restype = ctypes.c_int
        lib.gdn_chunked_prefill_noalloc.argtypes = [D, P, P, P, I32, P, P, P, P, P, P, I32,
                                                    I64, I32, P, I32, P]
        lib.gdn_chunked_prefill_noalloc.restype = ctypes.c_int
        lib.gdn_prefill_workspace_size.argtypes = [D, I64, I32, I32, I32, U32]
        lib.gdn_prefill_workspace_size.restype = S
        lib.gdn_state_slot_copy.argtypes = [D, P, P, I32, P, P, I32, P]
        lib.gdn_state_slot_copy.restype = ctypes.c_int
        lib.gdn_device_status.argtypes = [ctypes.POINTER(ctypes.c_int32), I32, P]
        lib.gdn_device_status.restype = ctypes.c_int
        lib.gdn_status_string.argtypes = [I32]
        lib.gdn_status_string.restype = ctypes.c_char_p
        lib.gdn_debug_set_wait_limit.argtypes = [I64]
        lib.gdn_debug_set_wait_limit.restype = I32
        lib.gdn_decode_pipe_buffer_size.argtypes = [D, I32, I32, I32]
        lib.gdn_decode_pipe_buffer_size.restype = S
        lib.gdn_decode_pipe_create.argtypes = [D, I32, I32, P, P, I32, P, P, F, F, P, I32, P, S,
                                               P, ctypes.POINTER(ctypes.c_void_p)]
        lib.gdn_decode_pipe_create.restype = ctypes.c_int
        lib.gdn_decode_pipe_step.argtypes = [P, P, P, P, P, P, P]
        lib.gdn_decode_pipe_step.restype = ctypes.c_int
        lib.gdn_decode_pipe_packed_bytes.argtypes = [D, I32, I32]
        lib.gdn_decode_pipe_packed_bytes.restype = S
        lib.gdn_decode_pipe_step_packed.argtypes = [P, P, P, P]
        lib.gdn_decode_pipe_step_packed.restype = ctypes.c_int
        lib.gdn_decode_pipe_flush.argtypes = [P]
        lib.gdn_decode_pipe_flush.restype = ctypes.c_int
        lib.gdn_decode_pipe_destroy.argtypes = [P]
        lib.gdn_decode_pipe_destroy.restype = ctypes.c_int
        lib.gdn_abi_version.argtypes = []
        lib.gdn_abi_version.restype = I32
        _lib = lib
        return lib
