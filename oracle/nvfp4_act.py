"""NVFP4 activations: the layer of the NVFP4 model with its expert inputs x (per
token) and SwiGLU outputs h (per row) quantized to NVFP4 instead of FP8, the
form a block-scaled FP4 tensor-core product consumes on both operands
("quantized MoE LLM inference", the NVFP4 remarks, for the weight format;
"MoE混合精度量化实战" (MoE mixed-precision quantization in practice), sec. 2.1, for
per-token dynamic activation scales).

TEST INFRASTRUCTURE, like the rest of ``oracle/``: numpy composition of the
oracle's pinned functions.

Readings:
  * a row of activations takes the weights' NVFP4 rule with the row as the
    "tensor": s = amax(row) / (448*6) in fp32 (1 for an all-zero row); per block
    of 16 inputs sb = e4m3(blockmax / (6*s)) (nearest even, saturating at 448;
    never negative, so it reads the same as an unsigned e4m3 scale);
    v = e2m1(a / (sb*s)) (nearest even, saturating at 6; 0 where sb = 0);
  * the products run on the block values e2m1(v)*sb of both operands, and the
    per-row scale s and the weights' tensor scale multiply the sums;
  * h is quantized from its fp32 rounding, as in the FP8 form of the layer.
"""
from __future__ import annotations

import numpy as np

from . import (combine, down, e2m1_value, e4m3_value, gateup, permute, quant_nvfp4, router,
               topk_softmax)


def quant_rows(a: np.ndarray):
    """Per-row NVFP4 codes of a float32 [R, K] array: (v [R, K] e2m1 codes,
    sb [R, K/16] e4m3 codes, s [R] fp32 row scales)."""
    a = np.ascontiguousarray(a, np.float32)
    R, K = a.shape
    v = np.empty((R, K), np.uint8)
    sb = np.empty((R, K // 16), np.uint8)
    s = np.empty(R, np.float32)
    for r in range(R):
        vr, sbr, sr = quant_nvfp4(a[r:r + 1])
        v[r], sb[r], s[r] = vr[0], sbr[0], sr
    return v, sb, s


def block_values(v: np.ndarray, sb: np.ndarray) -> np.ndarray:
    """float64 e2m1(v) * e4m3(sb), without the row scale."""
    e2 = np.array([e2m1_value(c) for c in range(16)])
    e4 = np.array([e4m3_value(c) for c in range(256)])
    return e2[v] * np.repeat(e4[sb], 16, axis=1)


def moe_forward(layer: np.ndarray, x_bf16: np.ndarray, Wr: np.ndarray, b, k: int):
    """Whole layer with NVFP4 activations; returns y (bf16 bits [T, H])."""
    x_bits = np.ascontiguousarray(x_bf16, np.uint16)
    T, H = x_bits.shape
    E = int(np.frombuffer(layer[8:12].tobytes(), np.int32)[0])
    idx, w = topk_softmax(router(x_bits, Wr, b), k)
    counts, offsets, perm, inv = permute(idx, E)
    x = (x_bits.astype(np.uint32) << 16).view(np.float32)
    xv, xsb, xs = quant_rows(x)
    xa = block_values(xv, xsb)
    o = np.zeros((T * k, H), np.float64)
    for e in range(E):
        rows = np.arange(offsets[e], offsets[e + 1])
        if len(rows) == 0:
            continue
        tok = perm[rows] // k
        h = gateup(layer, e, xa[tok], xs[tok].astype(np.float64))
        hv, hsb, hs = quant_rows(h.astype(np.float32))
        o[rows] = down(layer, e, block_values(hv, hsb), hs.astype(np.float64))
    return combine(o, w, inv)
