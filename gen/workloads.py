"""The synthetic workloads: shapes, per-expert formats and input recipes of the
five MoE layers (tiny, Mixtral-like, hot/cold tiered, NVFP4, large-expert).

Input recipe (seed 0): x = bf16 of N(0,1) values (tensor id 1, element t*H+h);
router weights fp32 N(0, 0.02) (id 2, element e*H+h); expert (e, p) weights
fp32 N(0, 0.02) (id 16+3e+p, row-major N x K).  The hot/cold layer adds the
calibrated router bias of tests/golden/hotcold_bias.json and puts its 64 hot
experts at 4 bits, the other 192 at 2 bits.  The graded layer is the same
layer with precision falling with hotness: the 64 hot experts at 4 bits, the
next 64 by router bias (ties to the lower index) at 2 bits, the last 128 at
1 bit (sign code).  No public dataset is involved.

This module only builds inputs; it holds none of the layer's arithmetic.
"""
from __future__ import annotations

import ctypes as C
import json
import os
from dataclasses import dataclass, field

import numpy as np

from . import TID_ROUTER_W, TID_X, fill_f32, f32_to_bf16_bits, tid_expert

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
HOTCOLD_JSON = os.path.join(ROOT, "tests", "golden", "hotcold_bias.json")
SEED = 0


@dataclass
class Layer:
    name: str
    H: int
    F: int
    E: int
    k: int
    fmt: np.ndarray                    # uint8 [E, 3] (gate, up, down)
    decode_T: tuple = ()
    prefill_T: tuple = ()
    bias: np.ndarray | None = None     # fp32 [E] router bias
    notes: dict = field(default_factory=dict)

    @property
    def fp4(self) -> bool:
        return bool(np.all(self.fmt == 16))


def _hotcold() -> Layer:
    d = json.load(open(HOTCOLD_JSON))
    E = 256
    fmt = np.full((E, 3), 2, np.uint8)
    fmt[d["hot_experts"]] = 4
    return Layer("hotcold", 2048, 512, E, 8, fmt, (32,), (4096,), np.array(d["bias"], np.float32),
                 {"hot_experts": d["hot_experts"], "top32_share": d["top32_share"], "gini": d["gini"]})


def _graded() -> Layer:
    L = _hotcold()
    hot = set(L.notes["hot_experts"])
    rest = sorted((e for e in range(L.E) if e not in hot), key=lambda e: (-float(L.bias[e]), e))
    fmt = np.full((L.E, 3), 1, np.uint8)
    fmt[sorted(hot)] = 4
    fmt[rest[:64]] = 2
    return Layer("graded", L.H, L.F, L.E, L.k, fmt, L.decode_T, L.prefill_T, L.bias,
                 dict(L.notes, warm_experts=sorted(rest[:64])))


def layer(name: str) -> Layer:
    if name == "tiny":
        return Layer("tiny", 256, 512, 8, 2, np.full((8, 3), 4, np.uint8), (16,), ())
    if name == "mixtral":
        return Layer("mixtral", 4096, 14336, 8, 2, np.tile(np.array([3, 2, 4], np.uint8), (8, 1)),
                     (1, 8, 64), (2048,))
    if name == "hotcold":
        return _hotcold()
    if name == "graded":
        return _graded()
    if name == "nvfp4":
        return Layer("nvfp4", 2048, 768, 256, 6, np.full((256, 3), 16, np.uint8), (16,), (8192,))
    if name == "large":
        return Layer("large", 12288, 14336, 128, 2, np.tile(np.array([4, 4, 2], np.uint8), (128, 1)),
                     (64,), (8192,))
    raise KeyError(name)


NAMES = ("tiny", "mixtral", "hotcold", "nvfp4", "large", "graded")


# ------------------------------------------------------------------ host inputs
def x_bf16_bits(T: int, H: int, seed: int = SEED) -> np.ndarray:
    return f32_to_bf16_bits(fill_f32(seed, TID_X, T * H, 1.0)).reshape(T, H)


def router_w(E: int, H: int, seed: int = SEED) -> np.ndarray:
    return fill_f32(seed, TID_ROUTER_W, E * H, 0.02).reshape(E, H)


def expert_w(e: int, H: int, F: int, seed: int = SEED) -> np.ndarray:
    """fp32 [3, H*F] weights of expert e (gate [F,H], up [F,H], down [H,F])."""
    out = np.empty((3, H * F), np.float32)
    for p in range(3):
        fill_f32(seed, tid_expert(e, p), H * F, 0.02, out=out[p])
    return out


# ------------------------------------------------------------------ device inputs
_dev = None


def _dev_lib():
    global _dev
    if _dev is None:
        path = os.path.join(HERE, "libmoegen.so")
        if not os.path.exists(path):
            raise ImportError(f"{path} missing: build with python mixed_precision_quantized_fp32_b200/build.py")
        L = C.CDLL(path)
        for fn in (L.moegen_fill_f32, L.moegen_fill_bf16):
            fn.restype = C.c_int
            fn.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_uint64, C.c_float, C.c_void_p]
        _dev = L
    return _dev


def fill_device_f32(t, seed: int, tid: int, sigma: float, start: int = 0, stream=None) -> None:
    """Fill a contiguous cuda float32 tensor with generator values (elements start..)."""
    import torch
    s = (stream or torch.cuda.current_stream()).cuda_stream
    rc = _dev_lib().moegen_fill_f32(t.data_ptr(), seed, tid, start, t.numel(), sigma, s)
    if rc:
        raise RuntimeError(f"moegen_fill_f32 failed ({rc})")


def fill_device_bf16(t, seed: int, tid: int, sigma: float, start: int = 0, stream=None) -> None:
    import torch
    s = (stream or torch.cuda.current_stream()).cuda_stream
    rc = _dev_lib().moegen_fill_bf16(t.data_ptr(), seed, tid, start, t.numel(), sigma, s)
    if rc:
        raise RuntimeError(f"moegen_fill_bf16 failed ({rc})")


def device_x(T: int, H: int, seed: int = SEED):
    import torch
    x = torch.empty((T, H), dtype=torch.bfloat16, device="cuda")
    fill_device_bf16(x, seed, TID_X, 1.0)
    return x


def device_router(L: Layer, seed: int = SEED):
    import torch
    w = torch.empty((L.E, L.H), dtype=torch.float32, device="cuda")
    fill_device_f32(w, seed, TID_ROUTER_W, 0.02)
    b = None if L.bias is None else torch.from_numpy(L.bias).cuda()
    return w, b


def device_expert_weights(L: Layer, e0: int, ne: int, out=None, seed: int = SEED):
    """cuda fp32 [ne, 3, H*F] weights of experts e0..e0+ne-1."""
    import torch
    if out is None:
        out = torch.empty((ne, 3, L.H * L.F), dtype=torch.float32, device="cuda")
    for i in range(ne):
        for p in range(3):
            fill_device_f32(out[i, p], seed, tid_expert(e0 + i, p), 0.02)
    return out
