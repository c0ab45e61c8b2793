"""ctypes binding of libkascade.so: the C entry points under the same names.

Only argument marshalling lives here.  Every entry point takes raw device
pointers (ints) and sizes, exactly as declared in include/kascade.h.  Loading
fails loudly when the library has not been built: there is no fallback.
"""
from __future__ import annotations

import ctypes
import os

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libkascade.so")

KASCADE_OK = 0
STATIC_SCRATCH_BYTES = 16 * 1024 * 1024  # KASCADE_STATIC_SCRATCH_BYTES in include/kascade.h
STATUS_NAMES = {
    0: "KASCADE_OK",
    1: "KASCADE_ERR_INVALID_ARG",
    2: "KASCADE_ERR_UNSUPPORTED_SHAPE",
    3: "KASCADE_ERR_WORKSPACE_TOO_SMALL",
    4: "KASCADE_ERR_CUDA",
    5: "KASCADE_ERR_BAD_INDEX",
    6: "KASCADE_ERR_NONFINITE",
    7: "KASCADE_ERR_TIMEOUT",
}
KASCADE_ERR_TIMEOUT = 7

# Every symbol the header declares (checked by the CPU tests).
EXPORTS = (
    "kascade_k_for_len",
    "kascade_decode_anchor_workspace_bytes",
    "kascade_decode_anchor",
    "kascade_decode_anchor_static_ws",
    "kascade_topk_workspace_bytes",
    "kascade_topk",
    "kascade_decode_reuse_workspace_bytes",
    "kascade_decode_reuse",
    "kascade_prefill_anchor_workspace_bytes",
    "kascade_prefill_anchor",
    "kascade_prefill_reuse_workspace_bytes",
    "kascade_prefill_reuse",
    "kascade_decode_anchor_f16",
    "kascade_decode_reuse_f16",
    "kascade_prefill_anchor_f16",
    "kascade_prefill_reuse_f16",
    "kascade_decode_anchor_paged",
    "kascade_decode_reuse_paged",
    "kascade_decode_anchor_paged_f16",
    "kascade_decode_reuse_paged_f16",
    "kascade_similarity_rows",
    "kascade_similarity_mean_workspace_bytes",
    "kascade_similarity_mean",
    "kascade_head_remap_workspace_bytes",
    "kascade_head_remap",
    "kascade_select_anchors",
    "kascade_get_device_status",
    "kascade_status_string",
    "kascade_selftest_wait_timeout",
)


class Shape(ctypes.Structure):
    _fields_ = [("B", ctypes.c_int32), ("Hq", ctypes.c_int32), ("Hkv", ctypes.c_int32),
                ("d", ctypes.c_int32)]


class KascadeError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS_NAMES.get(status, status)}")


_P = ctypes.c_void_p
_I32 = ctypes.c_int32
_I64 = ctypes.c_int64
_SZ = ctypes.c_size_t
_F = ctypes.c_float

_SIGNATURES = {
    "kascade_k_for_len": (_I32, [_I32]),
    "kascade_decode_anchor_workspace_bytes": (_SZ, [Shape, _I32]),
    "kascade_decode_anchor": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _I32, _F, _P, _P, _P, _I64,
                                             _P, _SZ, _P]),
    "kascade_decode_anchor_static_ws": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _I32, _F, _P, _P,
                                                       _P, _I64, _P]),
    "kascade_topk_workspace_bytes": (_SZ, [_I32, _I64]),
    "kascade_topk": (ctypes.c_int, [_P, _I32, _I64, _P, _P, _I32, _P, _P, _SZ, _P]),
    "kascade_decode_reuse_workspace_bytes": (_SZ, [Shape, _I32]),
    "kascade_decode_reuse": (ctypes.c_int, [Shape, _P, _P, _P, _P, _P, _P, _P, _I32, _P, _F, _P,
                                            _P, _P, _SZ, _P]),
    "kascade_prefill_anchor_workspace_bytes": (_SZ, [Shape, _I32]),
    "kascade_prefill_anchor": (ctypes.c_int, [Shape, _I32, _P, _P, _P, _F, _P, _P, _P, _P, _SZ,
                                              _P]),
    "kascade_prefill_reuse_workspace_bytes": (_SZ, [Shape, _I32, _I32]),
    "kascade_prefill_reuse": (ctypes.c_int, [Shape, _I32, _P, _P, _P, _P, _P, _I32, _P, _F, _P, _P,
                                             _P, _SZ, _P]),
    "kascade_decode_anchor_paged": (ctypes.c_int, [Shape, _P, _P, _P, _I32, _P, _I32, _I32, _P, _I32,
                                                   _F, _P, _P, _P, _I64, _P, _SZ, _P]),
    "kascade_decode_reuse_paged": (ctypes.c_int, [Shape, _P, _P, _P, _I32, _P, _I32, _I32, _P, _P,
                                                  _P, _I32, _P, _F, _P, _P, _P, _SZ, _P]),
    "kascade_similarity_rows": (ctypes.c_int, [_P, _I32, _I64, _P, _P, _P, _P, _I32, _I32, _P, _P,
                                               _P, _P]),
    "kascade_similarity_mean_workspace_bytes": (_SZ, [_I32]),
    "kascade_similarity_mean": (ctypes.c_int, [_P, _I32, _I64, _P, _P, _P, _P, _I32, _P, _P, _SZ,
                                               _P]),
    "kascade_head_remap_workspace_bytes": (_SZ, [_I32, _I32]),
    "kascade_head_remap": (ctypes.c_int, [_P, _I32, _I32, _I64, _P, _P, _P, _P, _I32, _P, _P, _P,
                                          _SZ, _P]),
    "kascade_select_anchors": (ctypes.c_int, [_P, _I32, _I32, _P, _P]),
    "kascade_get_device_status": (ctypes.c_int, [_P]),
    "kascade_status_string": (ctypes.c_char_p, [ctypes.c_int]),
    "kascade_selftest_wait_timeout": (ctypes.c_int, [ctypes.c_int32, _P]),
}
# fp16 variants take the same arguments as their bfloat16 counterparts
for _name in ("kascade_decode_anchor", "kascade_decode_reuse", "kascade_prefill_anchor",
              "kascade_prefill_reuse", "kascade_decode_anchor_paged", "kascade_decode_reuse_paged"):
    _SIGNATURES[_name + "_f16"] = _SIGNATURES[_name]

_lib = None


def load() -> ctypes.CDLL:
    """Load libkascade.so (built in-tree) and declare every signature."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(
            f"{LIB_PATH} is missing: build it with `python -m long_context_emitting_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    for name, (res, args) in _SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    _lib = lib
    return lib


def check(status: int, where: str) -> None:
    if status != KASCADE_OK:
        raise KascadeError(status, where)
