"""CPU oracle for the quantized MoE FFN layer forward and its weight packing.

TEST INFRASTRUCTURE.  Only ``tests/``, ``__graft_entry__.smoke()`` and the
benchmark's CPU-baseline leg (``bench.py``) may import this package.  The
product library (``mixed_precision_quantized_fp32_b200``) never imports,
links or calls it, and the oracle shares no code with the CUDA path.

The arithmetic lives in ``oracle/moe_oracle.c`` (plain C, double precision
where the method leaves precision open, fp32 where a float decides a code);
this module only marshals numpy arrays through ctypes.  Each function names
the definition it follows in its C counterpart.

Parity status of each function (its pins are the ``-m "not gpu"`` tests in
``tests/test_oracle_*.py``): every function here is pinned; see the test
module docstrings for which property pins which function.  ``outliers.py``
(outlier isolation) and ``nvfp4_act.py`` (NVFP4 activations), numpy on top
of these functions, are pinned by ``tests/test_oracle_outliers.py`` and
``tests/test_oracle_nvfp4_act.py``.
"""
from __future__ import annotations

import ctypes as C
import os

import numpy as np

from . import build as _build

FMT_INT1, FMT_INT2, FMT_INT3, FMT_INT4, FMT_NVFP4 = 1, 2, 3, 4, 16
HDR_BYTES = 16384

_lib = None


def lib() -> C.CDLL:
    global _lib
    if _lib is None:
        path = _build.build()
        L = C.CDLL(path)
        P = C.c_void_p
        i32, u64, f32, f64 = C.c_int, C.c_uint64, C.c_float, C.c_double
        sig = {
            "orc_f64_to_f16": (C.c_uint16, [f64]),
            "orc_f16_to_f64": (f64, [C.c_uint16]),
            "orc_f64_to_bf16": (C.c_uint16, [f64]),
            "orc_bf16_to_f64": (f64, [C.c_uint16]),
            "orc_f64_to_e4m3_sat": (C.c_uint8, [f64]),
            "orc_e4m3_to_f64": (f64, [C.c_uint8]),
            "orc_f64_to_e2m1_sat": (C.c_uint8, [f64]),
            "orc_e2m1_to_f64": (f64, [C.c_uint8]),
            "orc_quant_int": (None, [P, i32, i32, i32, P, P]),
            "orc_quant_nvfp4": (None, [P, i32, i32, P, P, P]),
            "orc_code_bytes": (u64, [i32, i32, i32]),
            "orc_scale_bytes": (u64, [i32, i32, i32]),
            "orc_pack_int": (None, [P, P, i32, i32, i32, P, P]),
            "orc_unpack_int": (None, [P, P, i32, i32, i32, P, P]),
            "orc_pack_nvfp4": (None, [P, P, i32, i32, P, P]),
            "orc_unpack_nvfp4": (None, [P, P, i32, i32, P, P]),
            "orc_decode_row": (None, [P, P, i32, i32, i32, f32, i32, P]),
            "orc_layer_layout": (i32, [i32, i32, i32, P, P, P, P]),
            "orc_pack_layer": (i32, [P, i32, i32, i32, i32, i32, P, P]),
            "orc_layer_decode_row": (None, [P, i32, i32, i32, P]),
            "orc_router": (None, [P, i32, i32, P, P, i32, P]),
            "orc_topk_softmax": (None, [P, i32, i32, i32, P, P]),
            "orc_permute": (None, [P, i32, i32, i32, P, P, P, P]),
            "orc_act_quant_e4m3": (None, [P, i32, i32, P, P]),
            "orc_gateup": (None, [P, i32, P, P, i32, P]),
            "orc_down": (None, [P, i32, P, P, i32, P]),
            "orc_combine": (None, [P, P, P, i32, i32, i32, P]),
            "orc_moe_forward": (i32, [P, P, i32, P, P, i32, P, P, P, P, P, P, P, P, P]),
        }
        for name, (res, args) in sig.items():
            fn = getattr(L, name)
            fn.restype = res
            fn.argtypes = args
        _lib = L
    return _lib


def _p(a):
    if a is None:
        return None
    assert a.flags["C_CONTIGUOUS"], "oracle arrays must be C-contiguous"
    return a.ctypes.data_as(C.c_void_p)


def _c(a, dtype):
    return np.ascontiguousarray(a, dtype=dtype)


# ---------------------------------------------------------------- scalar codecs
def f16_bits(v: float) -> int:
    return int(lib().orc_f64_to_f16(float(v)))


def f16_value(b: int) -> float:
    return float(lib().orc_f16_to_f64(int(b)))


def bf16_bits(v: float) -> int:
    return int(lib().orc_f64_to_bf16(float(v)))


def bf16_value(b: int) -> float:
    return float(lib().orc_bf16_to_f64(int(b)))


def e4m3_code(v: float) -> int:
    return int(lib().orc_f64_to_e4m3_sat(float(v)))


def e4m3_value(c: int) -> float:
    return float(lib().orc_e4m3_to_f64(int(c)))


def e2m1_code(v: float) -> int:
    return int(lib().orc_f64_to_e2m1_sat(float(v)))


def e2m1_value(c: int) -> float:
    return float(lib().orc_e2m1_to_f64(int(c)))


E4M3_TABLE = None


def e4m3_table() -> np.ndarray:
    """Values of all 256 e4m3 codes (NaN for the two NaN codes)."""
    global E4M3_TABLE
    if E4M3_TABLE is None:
        E4M3_TABLE = np.array([e4m3_value(c) for c in range(256)], dtype=np.float64)
    return E4M3_TABLE


# ---------------------------------------------------------------- matrices
def quant_int(W: np.ndarray, bits: int):
    W = _c(W, np.float32)
    N, K = W.shape
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 32), np.uint16)
    lib().orc_quant_int(_p(W), N, K, bits, _p(q), _p(s))
    return q, s


def quant_nvfp4(W: np.ndarray):
    W = _c(W, np.float32)
    N, K = W.shape
    v = np.empty((N, K), np.uint8)
    sb = np.empty((N, K // 16), np.uint8)
    sT = np.zeros(1, np.float32)
    lib().orc_quant_nvfp4(_p(W), N, K, _p(v), _p(sb), _p(sT))
    return v, sb, float(sT[0])


def code_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().orc_code_bytes(fmt, N, K))


def scale_bytes(fmt: int, N: int, K: int) -> int:
    return int(lib().orc_scale_bytes(fmt, N, K))


def pack_int(q, s, bits):
    q = _c(q, np.int8)
    s = _c(s, np.uint16)
    N, K = q.shape
    codes = np.empty(code_bytes(bits, N, K), np.uint8)
    scales = np.empty(scale_bytes(bits, N, K), np.uint8)
    lib().orc_pack_int(_p(q), _p(s), N, K, bits, _p(codes), _p(scales))
    return codes, scales


def unpack_int(codes, scales, N, K, bits):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    q = np.empty((N, K), np.int8)
    s = np.empty((N, K // 32), np.uint16)
    lib().orc_unpack_int(_p(codes), _p(scales), N, K, bits, _p(q), _p(s))
    return q, s


def pack_nvfp4(v, sb):
    v = _c(v, np.uint8)
    sb = _c(sb, np.uint8)
    N, K = v.shape
    codes = np.empty(code_bytes(FMT_NVFP4, N, K), np.uint8)
    scales = np.empty(scale_bytes(FMT_NVFP4, N, K), np.uint8)
    lib().orc_pack_nvfp4(_p(v), _p(sb), N, K, _p(codes), _p(scales))
    return codes, scales


def unpack_nvfp4(codes, scales, N, K):
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    v = np.empty((N, K), np.uint8)
    sb = np.empty((N, K // 16), np.uint8)
    lib().orc_unpack_nvfp4(_p(codes), _p(scales), N, K, _p(v), _p(sb))
    return v, sb


def decode_matrix(codes, scales, fmt, N, K, tscale=0.0) -> np.ndarray:
    codes = _c(codes, np.uint8)
    scales = _c(scales, np.uint8)
    out = np.empty((N, K), np.float64)
    L = lib()
    for n in range(N):
        L.orc_decode_row(_p(codes), _p(scales), fmt, N, K, float(tscale), n,
                         out[n].ctypes.data_as(C.c_void_p))
    return out


# ---------------------------------------------------------------- layer buffer
def layer_layout(E, H, F, fmt):
    fmt = _c(fmt, np.uint8).reshape(-1)
    co = np.zeros(E * 3, np.uint64)
    so = np.zeros(E * 3, np.uint64)
    tot = np.zeros(1, np.uint64)
    rc = lib().orc_layer_layout(E, H, F, _p(fmt), _p(co), _p(so), _p(tot))
    if rc:
        raise ValueError("bad layer layout arguments")
    return co, so, int(tot[0])


def pack_layer(W, e0, E, H, F, fmt, out=None):
    """Pack experts [e0, e0+len(W)) (W fp32 [ne][3][N*K]) into a layer buffer."""
    W = _c(W, np.float32)
    ne = W.shape[0]
    fmt = _c(fmt, np.uint8).reshape(-1)
    _, _, total = layer_layout(E, H, F, fmt)
    if out is None:
        out = np.zeros(total, np.uint8)
    rc = lib().orc_pack_layer(_p(W), e0, ne, E, H, F, _p(fmt), _p(out))
    if rc:
        raise ValueError("orc_pack_layer failed")
    return out


def layer_decode_matrix(layer, e, p) -> np.ndarray:
    """Dequantized (double) matrix of projection p of expert e."""
    H = int(np.frombuffer(layer[12:16].tobytes(), np.int32)[0])
    F = int(np.frombuffer(layer[16:20].tobytes(), np.int32)[0])
    N, K = (F, H) if p < 2 else (H, F)
    out = np.empty((N, K), np.float64)
    L = lib()
    for n in range(N):
        L.orc_layer_decode_row(_p(layer), e, p, n, out[n].ctypes.data_as(C.c_void_p))
    return out


# ---------------------------------------------------------------- forward stages
def router(x_bf16, Wr, b=None):
    x = _c(x_bf16, np.uint16)
    Wr = _c(Wr, np.float32)
    T, H = x.shape
    E = Wr.shape[0]
    bb = None if b is None else _c(b, np.float32)
    out = np.empty((T, E), np.float32)
    lib().orc_router(_p(x), T, H, _p(Wr), _p(bb), E, _p(out))
    return out


def topk_softmax(logits, k):
    logits = _c(logits, np.float32)
    T, E = logits.shape
    idx = np.empty((T, k), np.int32)
    w = np.empty((T, k), np.float32)
    lib().orc_topk_softmax(_p(logits), T, E, k, _p(idx), _p(w))
    return idx, w


def permute(idx, E):
    idx = _c(idx, np.int32)
    T, k = idx.shape
    counts = np.empty(E, np.int32)
    offsets = np.empty(E + 1, np.int32)
    perm = np.empty(T * k, np.int32)
    inv = np.empty(T * k, np.int32)
    lib().orc_permute(_p(idx), T, k, E, _p(counts), _p(offsets), _p(perm), _p(inv))
    return counts, offsets, perm, inv


def act_quant_e4m3(a):
    a = _c(a, np.float32)
    R, Cc = a.shape
    q = np.empty((R, Cc), np.uint8)
    s = np.empty(R, np.float32)
    lib().orc_act_quant_e4m3(_p(a), R, Cc, _p(q), _p(s))
    return q, s


def gateup(layer, e, a, a_scale=None):
    a = _c(a, np.float64)
    R = a.shape[0]
    F = int(np.frombuffer(layer[16:20].tobytes(), np.int32)[0])
    h = np.empty((R, F), np.float64)
    if R:
        lib().orc_gateup(_p(layer), e, _p(a), _p(None if a_scale is None else _c(a_scale, np.float64)),
                         R, _p(h))
    return h


def down(layer, e, h, h_scale=None):
    h = _c(h, np.float64)
    R = h.shape[0]
    H = int(np.frombuffer(layer[12:16].tobytes(), np.int32)[0])
    o = np.empty((R, H), np.float64)
    if R:
        lib().orc_down(_p(layer), e, _p(h), _p(None if h_scale is None else _c(h_scale, np.float64)),
                       R, _p(o))
    return o


def combine(o, w, inv):
    o = _c(o, np.float64)
    w = _c(w, np.float32)
    inv = _c(inv, np.int32)
    T, k = w.shape
    H = o.shape[1]
    y = np.empty((T, H), np.uint16)
    lib().orc_combine(_p(o), _p(w), _p(inv), T, k, H, _p(y))
    return y


def moe_forward(layer, x_bf16, Wr, b, k, want_debug=False):
    """Whole layer; returns y (bf16 bits [T,H]) or (y, debug dict)."""
    layer = _c(layer, np.uint8)
    x = _c(x_bf16, np.uint16)
    Wr = _c(Wr, np.float32)
    T, H = x.shape
    E = int(np.frombuffer(layer[8:12].tobytes(), np.int32)[0])
    F = int(np.frombuffer(layer[16:20].tobytes(), np.int32)[0])
    bb = None if b is None else _c(b, np.float32)
    y = np.empty((T, H), np.uint16)
    dbg = dict(idx=np.empty((T, k), np.int32), w=np.empty((T, k), np.float32),
               counts=np.empty(E, np.int32), perm=np.empty(T * k, np.int32),
               xq=np.zeros((T, H), np.uint8), sx=np.zeros(T, np.float32),
               hq=np.zeros((T * k, F), np.uint8), sh=np.zeros(T * k, np.float32))
    d = dbg if want_debug else {key: None for key in dbg}
    rc = lib().orc_moe_forward(_p(layer), _p(x), T, _p(Wr), _p(bb), k, _p(y), _p(d["idx"]), _p(d["w"]),
                               _p(d["counts"]), _p(d["perm"]), _p(d["xq"]), _p(d["sx"]), _p(d["hq"]),
                               _p(d["sh"]))
    if rc:
        raise ValueError("oracle forward refused the layer (mixed NVFP4 and integer formats)")
    return (y, dbg) if want_debug else y


def layer_fmt(layer) -> np.ndarray:
    E = int(np.frombuffer(layer[8:12].tobytes(), np.int32)[0])
    return np.array(layer[32:32 + 3 * E], np.uint8).reshape(E, 3)


def num_threads() -> int:
    return int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
