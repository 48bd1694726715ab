"""ctypes declarations of the C ABI in include/moe.h (argument marshalling only).

The shared library is built in-tree (``build.py``) and loaded from next to
this file.  There is no fallback: if the library is missing or cannot be
loaded, importing the API raises.
"""
from __future__ import annotations

import ctypes as C
import os

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libmoe_b200.so")

MOE_STAGE_EVENTS = 8
ACT_FP8, ACT_NVFP4 = 0, 1  # moe_weights.act
MOE_TRACE_EVENTS = 8
MOE_TRACE_STAGES = 1024

STATUS = {
    0: "MOE_OK", 1: "MOE_ERR_ARG", 2: "MOE_ERR_ALIGN", 3: "MOE_ERR_SHAPE", 4: "MOE_ERR_WORKSPACE",
    5: "MOE_ERR_FORMAT", 6: "MOE_ERR_CUDA", 7: "MOE_ERR_TIMEOUT", 8: "MOE_ERR_UNSUPPORTED_DEVICE",
    9: "MOE_ERR_RANGE",
}

EXPORTS = ("moe_pack", "moe_layer_forward", "moe_layer_forward_noalloc")
NOALLOC_SCRATCH_BYTES = 32 << 20


class MoeWeights(C.Structure):
    _fields_ = [("E", C.c_int32), ("H", C.c_int32), ("F", C.c_int32), ("fmt", C.c_void_p),
                ("packed", C.c_void_p), ("packed_bytes", C.c_uint64), ("act", C.c_int32)]


class MoeDebug(C.Structure):
    _fields_ = [("topk_idx", C.c_void_p), ("topk_w", C.c_void_p), ("perm", C.c_void_p),
                ("inv", C.c_void_p), ("counts", C.c_void_p), ("xq", C.c_void_p), ("sx", C.c_void_p),
                ("hq", C.c_void_p), ("sh", C.c_void_p), ("status", C.c_void_p),
                ("stage_events", C.c_void_p), ("trace", C.c_void_p),
                ("test_withhold", C.c_uint32), ("wait_cycles", C.c_uint32), ("xsb", C.c_void_p),
                ("hsb", C.c_void_p)]


class MoeError(RuntimeError):
    def __init__(self, call: str, code: int):
        super().__init__(f"{call} failed: {STATUS.get(code, code)}")
        self.code = code
        self.name = STATUS.get(code, str(code))


_lib = None


def load() -> C.CDLL:
    """Load libmoe_b200.so; raises if it is missing (build it with build.py)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise ImportError(f"CUDA library not built: {LIB_PATH} is missing "
                              "(run python mixed_precision_quantized_fp32_b200/build.py)")
        L = C.CDLL(LIB_PATH)
        P, i32, u64 = C.c_void_p, C.c_int32, C.c_uint64
        L.moe_pack.restype = C.c_int
        L.moe_pack.argtypes = [P, i32, i32, i32, i32, i32, P, P, u64, P, P, P, P]
        L.moe_layer_forward.restype = C.c_int
        L.moe_layer_forward.argtypes = [P, i32, P, P, C.POINTER(MoeWeights), i32, P, P, u64, P,
                                        C.POINTER(MoeDebug), P]
        L.moe_layer_forward_noalloc.restype = C.c_int
        L.moe_layer_forward_noalloc.argtypes = [P, i32, P, P, C.POINTER(MoeWeights), i32, P,
                                                C.POINTER(MoeDebug), P]
        _lib = L
    return _lib


def check(call: str, rc: int) -> None:
    if rc != 0:
        raise MoeError(call, rc)
