"""Thin ctypes binding over libcvq.so (argument marshalling only).

Every computation runs in the library's CUDA kernels; this module only turns torch
tensors into device pointers, sizes and the current CUDA stream.  There is no CPU
path: if libcvq.so is missing, importing the package raises.
"""
from __future__ import annotations

import ctypes
import os

PKG = os.path.dirname(os.path.abspath(__file__))
# CVQ_LIBRARY=debug loads the debug build (device-side range checks, libcvq_debug.so)
LIB_PATH = os.path.join(PKG, "libcvq_debug.so" if os.environ.get("CVQ_LIBRARY") == "debug"
                        else "libcvq.so")

CVQ_OK = 0
CVQ_F32 = 0
CVQ_BF16 = 1
STATUS_NAMES = {0: "CVQ_OK", 1: "CVQ_ERR_NULL", 2: "CVQ_ERR_SHAPE", 3: "CVQ_ERR_ALIGN",
                4: "CVQ_ERR_UNSUPPORTED", 5: "CVQ_ERR_WORKSPACE", 6: "CVQ_ERR_CUDA",
                7: "CVQ_ERR_STATIC_LIMIT"}


class CvqError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{msg} (status {status})")
        self.status = status


class cvq_shape(ctypes.Structure):
    _fields_ = [("batch", ctypes.c_int32), ("n_q_heads", ctypes.c_int32),
                ("n_kv_heads", ctypes.c_int32), ("head_dim", ctypes.c_int32),
                ("R", ctypes.c_int32), ("t_cap", ctypes.c_int32), ("rope_base", ctypes.c_float),
                ("group_dim", ctypes.c_int32), ("code_bits", ctypes.c_int32)]


def _load():
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{os.path.basename(LIB_PATH)} not built at {LIB_PATH}; run "
                          "`python -m compressed_attention_cvq_b200.build` (needs nvcc)")
    lib = ctypes.CDLL(LIB_PATH)
    P, I, I64, SZ = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    S = ctypes.POINTER(cvq_shape)
    sig = {
        "cvq_status_str": (ctypes.c_char_p, [I]),
        "cvq_abi_version": (I, []),
        "cvq_ptable_bytes": (SZ, [S]),
        "cvq_partials_bytes": (SZ, [S, I]),
        "cvq_split_tokens": (ctypes.c_int32, [S, I]),
        "cvq_suggest_splits": (I, [S, I]),
        "cvq_qtable": (I, [S, P, I, P, I64, P, P]),
        "cvq_decode_attn": (I, [S, P, P, P, P, P, I64, I, P, P, P, P]),
        "cvq_decode_attn_gqa": (I, [S, P, I, P, I64, P, P, P, P, I64, I, P, P, P, P]),
        "cvq_combine": (I, [S, I, P, P, P, P, P, P]),
        "cvq_attend_static": (I, [S, P, I, P, I64, P, P, P, P, I64, I, P, P, P]),
        "cvq_naive_cache_bytes": (SZ, [S]),
        "cvq_naive_dequant": (I, [S, P, I64, P, P, P, P, I64, P, P, P]),
        "cvq_naive_decode": (I, [S, P, I, P, P, P, I, P, P, P, P]),
        "cvq_encode_append": (I, [S, P, P, P, I64, P, I64, P, P, P, P]),
        "cvq_attend_workspace_bytes": (SZ, [S, I]),
        "cvq_attend": (I, [S, P, I, P, I64, P, P, P, P, I64, I, P, P, P, P]),
        "cvq_fault_status": (I, [ctypes.POINTER(ctypes.c_uint32), I]),
        "cvq_pack_codes6": (I, [S, P, P, P]),
    }
    for name, (res, args) in sig.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    return lib


class _LazyLib:
    """Loads libcvq.so on first use; raises ImportError if it was never built."""

    _lib = None

    def __getattr__(self, name):
        if _LazyLib._lib is None:
            _LazyLib._lib = _load()
        fn = getattr(_LazyLib._lib, name)
        setattr(self, name, fn)          # later lookups skip __getattr__
        return fn


lib = _LazyLib()
EXPORTED = ["cvq_status_str", "cvq_abi_version", "cvq_ptable_bytes", "cvq_partials_bytes",
            "cvq_split_tokens", "cvq_suggest_splits", "cvq_qtable", "cvq_decode_attn",
            "cvq_decode_attn_gqa", "cvq_combine", "cvq_attend_static",
            "cvq_naive_cache_bytes", "cvq_naive_dequant", "cvq_naive_decode",
            "cvq_encode_append", "cvq_attend_workspace_bytes", "cvq_attend",
            "cvq_fault_status", "cvq_pack_codes6"]
CVQ_FAULT_COPY_TIMEOUT = 1
CVQ_FAULT_BOUNDS = 2
FAULT_NAMES = {CVQ_FAULT_COPY_TIMEOUT: "copy_timeout", CVQ_FAULT_BOUNDS: "bounds"}


def fault_names(word: int) -> list:
    """Names of the bits set in a device fault word (cvq_fault_status); unknown bits as hex."""
    names = [n for bit, n in sorted(FAULT_NAMES.items()) if word & bit]
    rest = word & ~sum(FAULT_NAMES)
    return names + ([hex(rest)] if rest else [])


def status_str(st: int) -> str:
    return lib.cvq_status_str(st).decode()


def check(st: int, what: str):
    if st != CVQ_OK:
        raise CvqError(st, f"{what}: {status_str(st)}")


def make_shape(batch, n_q_heads, n_kv_heads, R, t_cap, rope_base=500000.0, head_dim=128,
               group_dim=8, code_bits=0):
    return cvq_shape(batch, n_q_heads, n_kv_heads, head_dim, R, t_cap, rope_base, group_dim,
                     code_bits)
