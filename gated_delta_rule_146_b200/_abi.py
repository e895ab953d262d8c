"""ctypes declarations of include/gdr.h and the loader of libgdr.so."""
from __future__ import annotations

import ctypes
import os
import threading

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libgdr.so")

GDR_OK, GDR_ERR_INVALID_ARG, GDR_ERR_UNSUPPORTED, GDR_ERR_ALIGNMENT = 0, 1, 2, 3
GDR_ERR_WORKSPACE, GDR_ERR_CUDA, GDR_ERR_DEVICE_CHECK, GDR_ERR_TIMEOUT = 4, 5, 6, 7
GDR_ERR_RANGE = 8
F32, BF16 = 0, 1
READ_POST, READ_PRE = 0, 1

# every symbol include/gdr.h declares
EXPORTS = ["gdr_chunk_fwd_workspace_size", "gdr_chunk_fwd", "gdr_chunk_fwd_noalloc",
           "gdr_noalloc_read_device_error",
           "gdr_chunk_bwd_workspace_size", "gdr_chunk_bwd",
           "gdr_chunk_fwd_bidir_workspace_size", "gdr_chunk_fwd_bidir",
           "gdr_chunk_fwd_path", "gdr_chunk_bwd_path",
           "gdr_decode_step", "gdr_status_string", "gdr_read_device_error", "gdr_version"]


class ChunkArgs(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("T", ctypes.c_int), ("Hk", ctypes.c_int),
                ("Hv", ctypes.c_int), ("dk", ctypes.c_int), ("dv", ctypes.c_int),
                ("n_seqs", ctypes.c_int), ("chunk", ctypes.c_int), ("io_dtype", ctypes.c_int),
                ("gate_dtype", ctypes.c_int), ("read_mode", ctypes.c_int),
                ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int),
                ("reverse", ctypes.c_int), ("o_accumulate", ctypes.c_int),
                ("gate_raw", ctypes.c_int), ("gate_A", ctypes.c_void_p),
                ("gate_dt_bias", ctypes.c_void_p), ("beta_scale", ctypes.c_float),
                ("gdn2", ctypes.c_int), ("gdn2_w", ctypes.c_void_p),
                ("status", ctypes.c_void_p)]


class DecodeArgs(ctypes.Structure):
    _fields_ = [("N", ctypes.c_int), ("Hk", ctypes.c_int), ("Hv", ctypes.c_int),
                ("dk", ctypes.c_int), ("dv", ctypes.c_int), ("io_dtype", ctypes.c_int),
                ("gate_dtype", ctypes.c_int), ("read_mode", ctypes.c_int),
                ("scale", ctypes.c_float), ("qk_l2norm", ctypes.c_int),
                ("gate_raw", ctypes.c_int), ("gate_A", ctypes.c_void_p),
                ("gate_dt_bias", ctypes.c_void_p), ("beta_scale", ctypes.c_float),
                ("out_norm", ctypes.c_int), ("norm_z", ctypes.c_void_p),
                ("norm_weight", ctypes.c_void_p), ("norm_eps", ctypes.c_float),
                ("gdn2", ctypes.c_int), ("gdn2_w", ctypes.c_void_p)]


class GdrError(RuntimeError):
    def __init__(self, status: int, msg: str = ""):
        self.status = status
        super().__init__(msg or status_string(status))


_lock = threading.Lock()
_lib = None


def _declare(lib):
    vp, sz = ctypes.c_void_p, ctypes.c_size_t
    lib.gdr_chunk_fwd_workspace_size.argtypes = [ctypes.POINTER(ChunkArgs)]
    lib.gdr_chunk_fwd_workspace_size.restype = sz
    lib.gdr_chunk_fwd.argtypes = [ctypes.POINTER(ChunkArgs)] + [vp] * 10 + [sz, vp]
    lib.gdr_chunk_fwd.restype = ctypes.c_int
    lib.gdr_chunk_fwd_noalloc.argtypes = [ctypes.POINTER(ChunkArgs)] + [vp] * 10
    lib.gdr_chunk_fwd_noalloc.restype = ctypes.c_int
    lib.gdr_noalloc_read_device_error.argtypes = [vp]
    lib.gdr_noalloc_read_device_error.restype = ctypes.c_int
    lib.gdr_chunk_fwd_bidir_workspace_size.argtypes = [ctypes.POINTER(ChunkArgs)]
    lib.gdr_chunk_fwd_bidir_workspace_size.restype = sz
    lib.gdr_chunk_fwd_bidir.argtypes = [ctypes.POINTER(ChunkArgs)] + [vp] * 10 + [sz, vp]
    lib.gdr_chunk_fwd_bidir.restype = ctypes.c_int
    lib.gdr_chunk_bwd_workspace_size.argtypes = [ctypes.POINTER(ChunkArgs)]
    lib.gdr_chunk_bwd_workspace_size.restype = sz
    lib.gdr_chunk_bwd.argtypes = [ctypes.POINTER(ChunkArgs)] + [vp] * 16 + [sz, vp]
    lib.gdr_chunk_bwd.restype = ctypes.c_int
    lib.gdr_chunk_fwd_path.argtypes = [ctypes.POINTER(ChunkArgs)]
    lib.gdr_chunk_fwd_path.restype = ctypes.c_char_p
    lib.gdr_chunk_bwd_path.argtypes = [ctypes.POINTER(ChunkArgs)]
    lib.gdr_chunk_bwd_path.restype = ctypes.c_char_p
    lib.gdr_decode_step.argtypes = [ctypes.POINTER(DecodeArgs)] + [vp] * 8
    lib.gdr_decode_step.restype = ctypes.c_int
    lib.gdr_status_string.argtypes = [ctypes.c_int]
    lib.gdr_status_string.restype = ctypes.c_char_p
    lib.gdr_read_device_error.argtypes = [ctypes.POINTER(ChunkArgs), vp, vp]
    lib.gdr_read_device_error.restype = ctypes.c_int
    lib.gdr_version.argtypes = []
    lib.gdr_version.restype = ctypes.c_char_p
    return lib


def lib():
    """Load libgdr.so once.  Raises FileNotFoundError if it has not been built: there is
    no fallback implementation."""
    global _lib
    with _lock:
        if _lib is None:
            if not os.path.exists(LIB_PATH):
                raise FileNotFoundError(
                    f"{LIB_PATH} is missing; build it with "
                    "`python -m gated_delta_rule_146_b200.build`")
            _lib = _declare(ctypes.CDLL(LIB_PATH))
    return _lib


def status_string(status: int) -> str:
    try:
        return lib().gdr_status_string(int(status)).decode()
    except FileNotFoundError:
        return f"gdr status {status}"


def check(status: int):
    if status != GDR_OK:
        raise GdrError(status)
