"""Pins for the oracle's NVFP4-activation mode (oracle/nvfp4_act.py):

  * per-row codes, block scales and row scales equal an independent numpy /
    torch restatement of the NVFP4 rule applied row by row;
  * the hand-worked weight block of tests/golden/nvfp4_group_example.json,
    read as one token, quantizes to its worked codes, and the same token halved
    keeps the codes with half the row scale;
  * an all-zero token has row scale 1, zero codes and a zero output;
  * the whole layer equals a dense float64 restatement (dequantized weights,
    NVFP4-rounded x and h, softmax over the chosen k) before the bf16 rounding.
"""
import json
import os

import numpy as np

import gen
import oracle as orc
from oracle import nvfp4_act as na
from tests import npref

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def test_rows_match_numpy_restatement():
    a = gen.normal_f32(0, 951, 0, 37 * 256, 1.0).reshape(37, 256)
    a[5] = 0.0
    a[9, :16] *= np.float32(1e-6)  # a tiny block beside normal ones
    v, sb, s = na.quant_rows(a)
    for r in range(a.shape[0]):
        vn, sbn, sn = npref.quant_nvfp4(a[r:r + 1])
        np.testing.assert_array_equal(v[r], vn[0])
        np.testing.assert_array_equal(sb[r], sbn[0])
        assert s[r] == np.float32(sn)


def test_hand_worked_token():
    ex = json.load(open(os.path.join(GOLD, "nvfp4_group_example.json")))
    a = np.zeros((2, 32), np.float32)
    a[0, :8] = np.asarray(ex["w_block0"], np.float32)
    a[1] = a[0] * np.float32(0.5)
    v, sb, s = na.quant_rows(a)
    assert s[0] == ex["tensor_scale"] and s[1] == ex["tensor_scale"] / 2
    assert v[0, :8].tolist() == ex["codes_first8"] and v[1, :8].tolist() == ex["codes_first8"]
    assert sb[0, 0] == ex["block0_scale_code"] and sb[1, 0] == ex["block0_scale_code"]
    assert np.all(sb[:, 1] == 0) and np.all(v[:, 8:] == 0)
    vals = na.block_values(v, sb) * s[:, None].astype(np.float64)
    np.testing.assert_array_equal(vals[0, :8], np.asarray(ex["dequant_first8"]))
    np.testing.assert_array_equal(vals[1, :8], np.asarray(ex["dequant_first8"]) / 2)


def test_zero_token():
    v, sb, s = na.quant_rows(np.zeros((1, 64), np.float32))
    assert s[0] == 1.0 and not v.any() and not sb.any()


def test_layer_matches_dense_restatement():
    T, H, F, E, k = 9, 256, 256, 6, 2
    W = gen.expert_weights_f32(0, 0, E, H, F)
    fmt = np.full((E, 3), 16, np.uint8)
    layer = orc.pack_layer(W, 0, E, H, F, fmt)
    x = gen.normal_bf16_bits(0, 1, 0, T * H, 1.0).reshape(T, H)
    x[4] = 0  # an all-zero token
    Wr = gen.normal_f32(0, 2, 0, E * H, 0.02).reshape(E, H)
    y = na.moe_forward(layer, x, Wr, None, k)

    mats = npref.dense_layer(W, fmt, H, F)
    xf = npref.bf16_to_f64(x).astype(np.float32)
    logits = (xf.astype(np.float64) @ Wr.astype(np.float64).T).astype(np.float32)
    idx = npref.topk_sorted(logits, k)
    sel = np.take_along_axis(logits, idx, axis=1).astype(np.float64)
    ex = np.exp(sel - sel[:, :1])
    w = (ex / ex.sum(axis=1, keepdims=True)).astype(np.float32)

    def nv(rowvec):
        v, sb, s = npref.quant_nvfp4(rowvec.astype(np.float32)[None, :])
        return npref.dequant_nvfp4(v, sb, s)[0]

    want = np.zeros((T, H))
    for t in range(T):
        xa = nv(xf[t])
        for j in range(k):
            g_w, u_w, d_w = mats[idx[t, j]]
            g, u = g_w @ xa, u_w @ xa
            h = g / (1 + np.exp(-g)) * u
            want[t] += float(w[t, j]) * (d_w @ nv(h))
    got = npref.bf16_to_f64(y)
    np.testing.assert_allclose(got, want, rtol=2 ** -8, atol=1e-30)
    assert not got[4].any()
