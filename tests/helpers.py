"""Shared test plumbing: pack layers on the GPU through the C ABI, build the
oracle's own packed copy from host-generated weights, run the oracle forward
stage by stage (with optional re-feed of the GPU's top-k choice) and compare.
"""
from __future__ import annotations

import numpy as np

import gen
import gen.workloads as W
import oracle as orc

TOL = 2e-2  # max |y_gpu - y_oracle| <= TOL * max |y_oracle| (bf16 outputs)
TIE_GAP = 1e-5  # top-k sets may differ where the oracle's k-th vs (k+1)-th logit gap is below this


_cache: dict = {}


def gpu_pack_cached(L: W.Layer):
    """gpu_pack of one of the named layers, kept for the rest of the session."""
    if L.name not in _cache:
        _cache.clear()  # at most one large layer resident at a time
        _cache[L.name] = gpu_pack(L)
    return _cache[L.name]


def gpu_pack(L: W.Layer, experts_per_call: int | None = None):
    """Pack the whole layer on the GPU, a few experts at a time; returns a PackedLayer."""
    import torch

    import mixed_precision_quantized_fp32_b200 as moe
    fmt = np.ascontiguousarray(L.fmt.reshape(-1))
    total = moe.pack_layout(L.E, L.H, L.F, fmt)[0]
    packed = moe.alloc_packed(total)
    per = experts_per_call or max(1, min(L.E, (1 << 31) // (3 * L.H * L.F * 4)))
    stage = torch.empty((per, 3, L.H * L.F), dtype=torch.float32, device="cuda")
    for e0 in range(0, L.E, per):
        ne = min(per, L.E - e0)
        w = W.device_expert_weights(L, e0, ne, out=stage[:ne])
        moe.moe_pack(w, e0, L.E, L.H, L.F, fmt, packed)
    torch.cuda.synchronize()
    del stage
    return moe.PackedLayer(L.E, L.H, L.F, fmt, packed)


def oracle_pack(L: W.Layer, experts) -> np.ndarray:
    """The oracle's packed buffer with the sections of `experts` filled (others zero)."""
    buf = None
    for e in sorted(set(int(e) for e in experts)):
        w = W.expert_w(e, L.H, L.F)[None]
        buf = orc.pack_layer(w, e, L.E, L.H, L.F, L.fmt.reshape(-1), out=buf)
    if buf is None:
        buf = orc.pack_layer(np.zeros((0, 3, L.H * L.F), np.float32), 0, L.E, L.H, L.F, L.fmt.reshape(-1))
    return buf


def sections(L: W.Layer, e: int):
    co, so, _ = orc.layer_layout(L.E, L.H, L.F, L.fmt.reshape(-1))
    out = []
    for p in range(3):
        N, K = (L.F, L.H) if p < 2 else (L.H, L.F)
        f = int(L.fmt[e, p])
        out.append((int(co[e * 3 + p]), orc.code_bytes(f, N, K)))
        out.append((int(so[e * 3 + p]), orc.scale_bytes(f, N, K)))
    return out


def oracle_route(x_bits, Wr, b, k):
    logits = orc.router(x_bits, Wr, b)
    idx, w = orc.topk_softmax(logits, k)
    return logits, idx, w


def near_tie_tokens(logits, k, idx_gpu, idx_orc):
    """Tokens whose chosen set differs; asserts every one is a near-tie. Returns their list."""
    bad = []
    for t in range(idx_orc.shape[0]):
        if set(idx_gpu[t].tolist()) != set(idx_orc[t].tolist()):
            srt = np.sort(logits[t].astype(np.float64))[::-1]
            gap = srt[k - 1] - srt[k] if k < logits.shape[1] else np.inf
            assert gap < TIE_GAP, f"token {t}: top-k sets differ with gap {gap}"
            bad.append(t)
    return bad


def oracle_forward_rows(layer_buf, x_bits, Wr, b, k, tokens=None, idx_override=None, fp4=False,
                        hq_override=None):
    """Oracle output for the given tokens (default all), from the oracle's stages.

    idx_override: [T, k] expert choice to use instead of the oracle's own (re-feed of
    the GPU's choice at near-ties; weights are still the oracle's softmax of the
    oracle logits of those experts).  hq_override: dict row -> (codes [F], scale)
    to re-feed the GPU's quantized SwiGLU output (NVFP4 down stage)."""
    T = x_bits.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    xt = x_bits[tokens]
    logits = orc.router(xt, Wr, b)
    idx, w = orc.topk_softmax(logits, k)
    if idx_override is not None:
        idx = np.ascontiguousarray(idx_override[tokens], np.int32)
        sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
        ex = np.exp(sel - sel.max(1, keepdims=True))
        w = (ex / ex.sum(1, keepdims=True)).astype(np.float32)
        order = np.argsort(-sel, axis=1, kind="stable")
        idx = np.take_along_axis(idx, order, 1)
        w = np.take_along_axis(w, order, 1)
    xf = gen.bf16_bits_to_f32(xt)
    if fp4:
        xq, sx = orc.act_quant_e4m3(xf)
        a = orc.e4m3_table()[xq]
        a_scale = sx.astype(np.float64)
    else:
        a = xf.astype(np.float64)
        a_scale = None
    H = x_bits.shape[1]
    y = np.zeros((len(tokens), H))
    for e in np.unique(idx):
        ts, js = np.nonzero(idx == e)
        h = orc.gateup(layer_buf, int(e), a[ts], None if a_scale is None else a_scale[ts])
        hs = None
        if fp4:
            hq, sh = orc.act_quant_e4m3(h.astype(np.float32))
            h = orc.e4m3_table()[hq]
            hs = sh.astype(np.float64)
        o = orc.down(layer_buf, int(e), h, hs)
        for r, (t, j) in enumerate(zip(ts, js)):
            y[t] += float(w[t, j]) * o[r]
    return y, idx, w


def oracle_forward_rows_act4(layer_buf, x_bits, Wr, b, k, tokens=None, idx_override=None):
    """As oracle_forward_rows for an NVFP4 layer with NVFP4 activations (the oracle's
    NVFP4-activation mode, oracle/nvfp4_act.py): x per token and h per row quantized to
    e2m1 codes with e4m3 block scales, products on the block values, the row and
    tensor scales applied to the sums."""
    from oracle import nvfp4_act as na
    T = x_bits.shape[0]
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    xt = x_bits[tokens]
    logits = orc.router(xt, Wr, b)
    idx, w = orc.topk_softmax(logits, k)
    if idx_override is not None:
        idx = np.ascontiguousarray(idx_override[tokens], np.int32)
        sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
        ex = np.exp(sel - sel.max(1, keepdims=True))
        w = (ex / ex.sum(1, keepdims=True)).astype(np.float32)
        order = np.argsort(-sel, axis=1, kind="stable")
        idx = np.take_along_axis(idx, order, 1)
        w = np.take_along_axis(w, order, 1)
    xv, xsb, xs = na.quant_rows(gen.bf16_bits_to_f32(xt))
    a = na.block_values(xv, xsb)
    H = x_bits.shape[1]
    y = np.zeros((len(tokens), H))
    for e in np.unique(idx):
        ts, js = np.nonzero(idx == e)
        h = orc.gateup(layer_buf, int(e), a[ts], xs[ts].astype(np.float64))
        hv, hsb, hs = na.quant_rows(h.astype(np.float32))
        o = orc.down(layer_buf, int(e), na.block_values(hv, hsb), hs.astype(np.float64))
        for r, (t, j) in enumerate(zip(ts, js)):
            y[t] += float(w[t, j]) * o[r]
    return y, idx, w


def oracle_forward_rows_dense(mats, x_bits, Wr, b, k, fp4=False, idx_override=None):
    """The oracle's stages (router, top-k, FP8 activation quantization of NVFP4
    layers) with the expert products taken on given float64 matrices: mats(e) ->
    (W_gate [F,H], W_up [F,H], W_down [H,F]).  Used for layers whose matrices are
    more than their packed dense part (outlier side lists): g = s_x * W_gate a,
    u = s_x * W_up a, h = silu(g) * u, o = s_h * W_down h, y = sum_j w_j o_j."""
    T = x_bits.shape[0]
    logits = orc.router(x_bits, Wr, b)
    idx, w = orc.topk_softmax(logits, k)
    if idx_override is not None:
        idx = np.ascontiguousarray(idx_override, np.int32)
        sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
        ex = np.exp(sel - sel.max(1, keepdims=True))
        w = (ex / ex.sum(1, keepdims=True)).astype(np.float32)
    xf = gen.bf16_bits_to_f32(x_bits)
    if fp4:
        xq, sx = orc.act_quant_e4m3(xf)
        a, a_scale = orc.e4m3_table()[xq], sx.astype(np.float64)
    else:
        a, a_scale = xf.astype(np.float64), np.ones(T)
    y = np.zeros((T, x_bits.shape[1]))
    for e in np.unique(idx):
        ts, js = np.nonzero(idx == e)
        Wg, Wu, Wd = mats(int(e))
        g = (a[ts] @ Wg.T) * a_scale[ts, None]
        u = (a[ts] @ Wu.T) * a_scale[ts, None]
        h = g / (1.0 + np.exp(-g)) * u
        h_scale = np.ones(len(ts))
        if fp4:
            hq, sh = orc.act_quant_e4m3(h.astype(np.float32))
            h, h_scale = orc.e4m3_table()[hq], sh.astype(np.float64)
        o = (h @ Wd.T) * h_scale[:, None]
        y[ts] += w[ts, js].astype(np.float64)[:, None] * o
    return y


def check_output(y_gpu_bf16, y_ref):
    """|y_gpu - y_ref| <= TOL * max|y_ref|; returns the error ratio."""
    import torch
    yg = y_gpu_bf16.float().cpu().numpy().astype(np.float64) if isinstance(y_gpu_bf16, torch.Tensor) \
        else np.asarray(y_gpu_bf16, np.float64)
    scale = np.abs(y_ref).max()
    err = np.abs(yg - y_ref).max()
    assert np.all(np.isfinite(yg))
    assert err <= TOL * scale, f"max err {err:.4g} > {TOL} * {scale:.4g}"
    return err / scale
