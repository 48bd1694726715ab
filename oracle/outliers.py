"""Outlier isolation of one expert matrix: the largest weights by magnitude leave
the quantization grid and are kept in fp16 beside it ("MoE混合精度量化实战"
(MoE mixed-precision quantization in practice), sec. 4.2, tip 2: take each
expert's top 0.05% of weights by |w| out, store them in FP16, quantize the
other 99.95%).

TEST INFRASTRUCTURE, like the rest of ``oracle/``; plain numpy on top of the
oracle's own quantize / pack / decode functions.

Readings (the page gives the fraction and the idea only):
  * per matrix (one expert, one projection) n_out = floor(frac * N * K),
    frac = 5 / 10000, in integer arithmetic;
  * the outliers are the n_out entries of largest |w|, ties going to the lower
    row-major index;
  * they are set to 0 before the group quantization, so they do not inflate
    the group scales (nor the NVFP4 tensor scale);
  * the side list keeps, per outlier, r = fp16(w - dequant(w)) with w the
    original weight and dequant the dense part at that position (0 for every
    format that represents 0; the 1-bit sign code dequantizes a zero to +s),
    sorted by (row, column);
  * the matrix the layer uses is dequant(codes) plus r at the outlier positions.
"""
from __future__ import annotations

import numpy as np

from . import (FMT_NVFP4, decode_matrix, f16_bits, f16_value, pack_int, pack_nvfp4, quant_int,
               quant_nvfp4)

FRAC_NUM, FRAC_DEN = 5, 10000  # 0.05 %


def count(N: int, K: int) -> int:
    """Outliers of an N x K matrix."""
    return (N * K * FRAC_NUM) // FRAC_DEN


def select(W: np.ndarray, n_out: int | None = None):
    """(rows, cols) of the n_out largest |w|, ties to the lower row-major index,
    returned in (row, column) order."""
    N, K = W.shape
    if n_out is None:
        n_out = count(N, K)
    mag = np.abs(W.astype(np.float64)).ravel()
    order = np.argsort(-mag, kind="stable")  # descending |w|; stable keeps equal |w| in index order
    flat = np.sort(order[:n_out])
    return flat // K, flat % K


def isolate(W: np.ndarray, fmt: int, n_out: int | None = None) -> dict:
    """Dense codes of W with its outliers zeroed, plus the fp16 residual side list."""
    W = np.ascontiguousarray(W, np.float32)
    N, K = W.shape
    rows, cols = select(W, n_out)
    Wd = W.copy()
    Wd[rows, cols] = 0.0
    tscale = 0.0
    if fmt == FMT_NVFP4:
        v, sb, tscale = quant_nvfp4(Wd)
        codes, scales = pack_nvfp4(v, sb)
    else:
        q, s = quant_int(Wd, fmt)
        codes, scales = pack_int(q, s, fmt)
    dense = decode_matrix(codes, scales, fmt, N, K, tscale)
    resid = np.array([f16_bits(float(W[n, k]) - dense[n, k]) for n, k in zip(rows, cols)], np.uint16)
    return dict(codes=codes, scales=scales, tscale=tscale, rows=rows.astype(np.int32),
                cols=cols.astype(np.int32), resid=resid)


def dequant(iso: dict, fmt: int, N: int, K: int) -> np.ndarray:
    """float64 matrix: the dense part plus the residuals at the outlier positions."""
    W = decode_matrix(iso["codes"], iso["scales"], fmt, N, K, iso["tscale"])
    for n, k, r in zip(iso["rows"], iso["cols"], iso["resid"]):
        W[n, k] += f16_value(int(r))
    return W
