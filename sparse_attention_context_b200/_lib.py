"""ctypes loader of libisa.so (built in-tree by ``build.py``).

Loading fails loudly when the library is missing: there is no other
implementation of the ISA path in this package.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libisa.so")

ISA_OK = 0
STATUS = {0: "ok", 1: "invalid argument", 2: "unsupported shape", 3: "workspace too small", 4: "CUDA error",
          5: "device wait timed out"}


class IsaShape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int), ("H", ctypes.c_int), ("N_src", ctypes.c_int), ("N_ctx", ctypes.c_int),
                ("d", ctypes.c_int), ("block", ctypes.c_int), ("keep", ctypes.c_float), ("rho", ctypes.c_float),
                ("scale", ctypes.c_float)]


class IsaError(RuntimeError):
    def __init__(self, fn: str, code: int, detail: str = ""):
        super().__init__(f"{fn} failed: {STATUS.get(code, code)} ({code}){': ' + detail if detail else ''}")
        self.code = code


_P = ctypes.c_void_p
_SZ = ctypes.c_size_t
_I = ctypes.c_int
_F = ctypes.c_float
_SH = ctypes.POINTER(IsaShape)

# name -> (restype, argtypes)
SIGNATURES = {
    "isa_n_keep": (_I, [_SH]),
    "isa_n_route": (_I, [_SH]),
    "isa_n_route_blocks": (_I, [_SH]),
    "isa_workspace_size": (_SZ, [_SH]),
    "isa_preselect_ctx": (_I, [_SH, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_route_queries": (_I, [_SH, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_attn_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_route_taylor_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_full_attn_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_taylor_attn_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_full_attn_rows_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _I, _P, _P, _SZ, _P]),
    "isa_route_blocks_taylor_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_forward_blocks": (_I, [_SH, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_taylor1_workspace_size": (_SZ, [_SH]),
    "isa_taylor1_attn_fwd": (_I, [_SH, _P, _P, _P, _P, _P, _P, _P, _SZ, _P, _SZ, _P]),
    "isa_forward_taylor1": (_I, [_SH, _P, _P, _P, _P, _P, _SZ, _P, _SZ, _P]),
    "isa_forward": (_I, [_SH, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_forward_static": (_I, [_SH, _P, _P, _P, _P, _P]),
    "isa_host_staging_size": (_SZ, [_SH, _I]),
    "isa_forward_host": (_I, [_SH, _P, _P, _P, _P, _P, _SZ, _I, _P, _P, _P]),
    "isa_dense_workspace_size": (_SZ, [_I]),
    "isa_dense_attn_fwd": (_I, [_I, _I, _I, _I, _F, _P, _P, _P, _P, _P, _SZ, _P]),
    "isa_read_device_status": (_I, [_P, _P]),
    "isa_status_string": (ctypes.c_char_p, [_I]),
    "isa_last_error": (ctypes.c_char_p, []),
    "isa_selftest_umma": (_I, [_I, _I, _P, _P, _P, _P, _P, _P, _P, _P, _P]),
    "isa_selftest_ex2": (_I, [_P, _P, _P, _P, _I, _P]),
    "isa_selftest_umma_pair": (_I, [_P, _P, _P, _P, _P, _P, _P, _P]),
}

_lib = None


def lib():
    """The loaded library (loaded on first use)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"{LIB_PATH} is missing: build it with `python -m sparse_attention_context_b200.build`")
        L = ctypes.CDLL(LIB_PATH)
        for name, (res, args) in SIGNATURES.items():
            f = getattr(L, name)
            f.restype = res
            f.argtypes = args
        _lib = L
    return _lib


def check(fn: str, code: int) -> None:
    if code != ISA_OK:
        detail = lib().isa_last_error().decode() if code == 4 else ""
        raise IsaError(fn, code, detail)
