"""Independent numpy/torch restatement of the layer, used only to pin the oracle.

It is written from the same definitions as the oracle but with different
machinery: numpy's float16 cast, torch's float8_e4m3fn cast, dense float64
matrix products and sort-based top-k.  A mistake in the oracle's loops,
layouts or codecs shows up as a disagreement with this module.
"""
from __future__ import annotations

import numpy as np
import torch

E2M1_MAGS = np.array([0.0, 0.5, 1.0, 1.5, 2.0, 3.0, 4.0, 6.0])


def quant_int(W, bits):
    qmax = (1 << (bits - 1)) - 1
    N, K = W.shape
    G = W.reshape(N, K // 32, 32)
    if bits == 1:  # sign code, scale = fp16(sum|w| / 32) with the fp32 sum taken in input order
        acc = np.zeros((N, K // 32), np.float32)
        for i in range(32):
            acc = (acc + np.abs(G[:, :, i])).astype(np.float32)
        with np.errstate(over="ignore"):
            s16 = (acc / np.float32(32)).astype(np.float32).astype(np.float16)
        s16[np.isinf(s16)] = np.float16(65504.0)
        return np.where(G >= 0, 1, -1).reshape(N, K).astype(np.int8), s16.view(np.uint16)
    amax = np.abs(G).max(axis=2)
    ratio = (amax / np.float32(qmax)).astype(np.float32)
    with np.errstate(over="ignore"):
        s16 = ratio.astype(np.float16)
    s16[np.isinf(s16)] = np.float16(65504.0)
    s = s16.astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        q = np.rint(G / s[:, :, None])
    q = np.where(s[:, :, None] == 0, 0, np.clip(q, -qmax, qmax))
    return q.reshape(N, K).astype(np.int8), s16.view(np.uint16)


def dequant_int(q, s16):
    s = s16.view(np.float16).astype(np.float64)
    N, K = q.shape
    return (q.reshape(N, K // 32, 32).astype(np.float64) * s[:, :, None]).reshape(N, K)


def e2m1_nearest_even(x):
    a = np.abs(x.astype(np.float64))
    d = np.abs(a[..., None] - E2M1_MAGS)
    best = d.min(axis=-1, keepdims=True)
    cand = d == best
    even = cand & (np.arange(8) % 2 == 0)
    pick = np.where(even.any(axis=-1), even.argmax(axis=-1), cand.argmax(axis=-1))
    return (pick | np.where(np.signbit(x), 8, 0)).astype(np.uint8)


def e4m3_codes(a_f32):
    a = np.clip(np.asarray(a_f32, np.float32), -448.0, 448.0)
    return torch.from_numpy(np.ascontiguousarray(a)).to(torch.float8_e4m3fn).view(torch.uint8).numpy()


def e4m3_values(codes):
    return torch.from_numpy(np.ascontiguousarray(codes, np.uint8)).view(torch.float8_e4m3fn).double().numpy()


def quant_nvfp4(W):
    N, K = W.shape
    amax = np.float32(np.abs(W).max())
    sT = np.float32(1.0) if amax == 0 else np.float32(amax / np.float32(2688.0))
    B = W.reshape(N, K // 16, 16)
    bmax = np.abs(B).max(axis=2)
    ratio = (bmax / (np.float32(6.0) * sT)).astype(np.float32)
    sb = e4m3_codes(ratio)
    sbv = e4m3_values(sb).astype(np.float32)
    denom = (sbv * sT).astype(np.float32)
    with np.errstate(divide="ignore", invalid="ignore"):
        r = (B / denom[:, :, None]).astype(np.float32)
    v = np.where(sbv[:, :, None] == 0, 0, e2m1_nearest_even(np.nan_to_num(r)))
    return v.reshape(N, K).astype(np.uint8), sb, float(sT)


def dequant_nvfp4(v, sb, sT):
    vals = np.where(v & 8, -1.0, 1.0) * E2M1_MAGS[v & 7]
    return vals * np.repeat(e4m3_values(sb), 16, axis=1) * float(sT)


def dense_layer(W, fmt, H, F):
    """Dequantized float64 matrices mats[e][p] from fp32 weights W [E][3][N*K]."""
    mats = []
    for e in range(W.shape[0]):
        row = []
        for p in range(3):
            N, K = (F, H) if p < 2 else (H, F)
            w = W[e, p].reshape(N, K)
            f = int(fmt[e][p])
            if f == 16:
                row.append(dequant_nvfp4(*quant_nvfp4(w)))
            else:
                row.append(dequant_int(*quant_int(w, f)))
        mats.append(row)
    return mats


def bf16_to_f64(bits):
    return (np.asarray(bits, np.uint16).astype(np.uint32) << 16).view(np.float32).astype(np.float64)


def topk_sorted(logits, k):
    T, E = logits.shape
    idx = np.empty((T, k), np.int64)
    for t in range(T):
        order = sorted(range(E), key=lambda e: (-float(logits[t, e]), e))
        idx[t] = order[:k]
    return idx


def forward(x_bits, Wr, b, k, mats, fp4):
    """Returns (y float64 [T,H] before bf16 rounding, idx, w)."""
    x = bf16_to_f64(x_bits)
    T, H = x.shape
    logits = (x @ Wr.astype(np.float64).T + (0 if b is None else b.astype(np.float64))).astype(np.float32)
    idx = topk_sorted(logits, k)
    sel = np.take_along_axis(logits, idx, axis=1).astype(np.float64)
    ex = np.exp(sel - sel[:, :1])
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)
    if fp4:
        xf = x.astype(np.float32)
        amax = np.abs(xf).max(axis=1)
        sx = np.where(amax == 0, np.float32(1), amax / np.float32(448)).astype(np.float32)
        xa = e4m3_values(e4m3_codes(xf / sx[:, None]))
    else:
        sx = np.ones(T, np.float32)
        xa = x
    y = np.zeros((T, H))
    for t in range(T):
        for j in range(k):
            Wg, Wu, Wd = mats[idx[t, j]]
            g = float(sx[t]) * (Wg @ xa[t])
            u = float(sx[t]) * (Wu @ xa[t])
            h = g / (1 + np.exp(-g)) * u
            if fp4:
                hf = h.astype(np.float32)
                am = np.abs(hf).max()
                sh = np.float32(1) if am == 0 else np.float32(am / np.float32(448))
                h = e4m3_values(e4m3_codes(hf / sh)) * float(sh)
            y[t] += float(w[t, j]) * (Wd @ h)
    return y, idx, w
