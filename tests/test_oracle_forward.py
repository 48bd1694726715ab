"""Pins for the oracle's forward stages and whole layer.

  * router logits against a numpy float64 matrix product;
  * top-k against sort-based brute force on inputs full of ties (lower index
    wins); softmax weights sum to 1 and equal 1/E for k = E with equal logits;
  * permutation against numpy's stable argsort and bincount, plus invariants;
  * per-row FP8 activation codes against torch's float8_e4m3fn cast;
  * expert FFN and the whole layer against the dense float64 restatement in
    tests/npref.py (its own quantizer, dequantizer, top-k and combine);
  * closed forms: an all-zero expert contributes exactly 0; k = E with equal
    logits gives the mean of the experts; k = 1 gives that expert's output;
    a constant weight matrix gives g = s*qmax*sum(x) for every output.
"""
import numpy as np
import pytest

import gen
from tests import npref


def _inputs(T, H, E, seed=0):
    x = gen.normal_bf16_bits(seed, gen.TID_X, 0, T * H).reshape(T, H)
    Wr = gen.normal_f32(seed, gen.TID_ROUTER_W, 0, E * H, 0.02).reshape(E, H)
    return x, Wr


def test_router_against_numpy(orc):
    T, H, E = 33, 384, 24
    x, Wr = _inputs(T, H, E)
    b = gen.normal_f32(0, 77, 0, E, 0.5)
    got = orc.router(x, Wr, b)
    want = npref.bf16_to_f64(x) @ Wr.astype(np.float64).T + b.astype(np.float64)
    np.testing.assert_allclose(got, want, rtol=2e-7, atol=1e-7)
    assert np.abs(got - orc.router(x, Wr, None) - b).max() < 1e-6


def test_topk_brute_force_with_ties(orc):
    rng = np.random.default_rng(5)
    for E, k in [(8, 2), (16, 6), (256, 8), (5, 5), (7, 1)]:
        logits = rng.integers(-3, 4, size=(64, E)).astype(np.float32)  # many ties
        idx, w = orc.topk_softmax(logits, k)
        np.testing.assert_array_equal(idx, npref.topk_sorted(logits, k))
        np.testing.assert_allclose(w.sum(axis=1), 1.0, atol=1e-6)
        sel = np.take_along_axis(logits, idx, 1).astype(np.float64)
        ex = np.exp(sel - sel.max(axis=1, keepdims=True))
        np.testing.assert_allclose(w, ex / ex.sum(1, keepdims=True), rtol=1e-6)
    # k = E, equal logits: all experts in index order, weight 1/E each
    idx, w = orc.topk_softmax(np.zeros((3, 8), np.float32), 8)
    np.testing.assert_array_equal(idx, np.tile(np.arange(8), (3, 1)))
    np.testing.assert_allclose(w, 1 / 8, rtol=1e-7)
    # k = 1 is argmax (first maximum)
    logits = rng.standard_normal((50, 9)).astype(np.float32)
    idx, w = orc.topk_softmax(logits, 1)
    np.testing.assert_array_equal(idx[:, 0], logits.argmax(1))
    assert np.all(w == 1.0)


def test_permute_against_stable_sort(orc):
    rng = np.random.default_rng(6)
    for T, k, E in [(1, 1, 1), (37, 2, 8), (300, 8, 256), (64, 6, 256)]:
        idx = np.stack([rng.permutation(E)[:k] for _ in range(T)]).astype(np.int32)
        counts, offsets, perm, inv = orc.permute(idx, E)
        np.testing.assert_array_equal(counts, np.bincount(idx.ravel(), minlength=E))
        np.testing.assert_array_equal(offsets, np.concatenate([[0], np.cumsum(counts)]))
        np.testing.assert_array_equal(perm, np.argsort(idx.ravel(), kind="stable"))
        np.testing.assert_array_equal(inv[perm], np.arange(T * k))
        assert sorted(perm) == list(range(T * k))


def test_act_quant_against_torch(orc):
    a = gen.normal_f32(0, 9, 0, 40 * 256, 1.0).reshape(40, 256)
    a[3] = 0.0
    a[4] *= np.float32(1e-30)
    q, s = orc.act_quant_e4m3(a)
    amax = np.abs(a).max(1)
    s_want = np.where(amax == 0, np.float32(1), amax / np.float32(448)).astype(np.float32)
    np.testing.assert_array_equal(s, s_want)
    np.testing.assert_array_equal(q, npref.e4m3_codes(a / s_want[:, None]))
    assert np.all(q[3] == 0)
    # the element of largest magnitude in a non-zero row maps onto +-448
    big = np.abs(npref.e4m3_values(q[5:])).max(1)
    assert np.all(big == 448.0)


@pytest.mark.parametrize("fmt_kind", ["int4", "mixed", "graded", "nvfp4"])
def test_forward_against_dense_restatement(orc, fmt_kind):
    if fmt_kind == "graded":  # precision falling with hotness: 4-, 2- and 1-bit experts
        T, H, F, E, k = 12, 256, 384, 6, 2
        fmt = np.array([[4, 4, 4], [2, 2, 2], [1, 1, 1], [4, 2, 1], [1, 2, 4], [2, 1, 2]], np.uint8)
    elif fmt_kind == "nvfp4":
        T, H, F, E, k = 8, 256, 256, 16, 6
        fmt = np.full((E, 3), 16, np.uint8)
    elif fmt_kind == "mixed":
        T, H, F, E, k = 12, 256, 384, 6, 2
        fmt = np.array([[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 4, 2], [3, 3, 3], [2, 4, 3]], np.uint8)
    else:
        T, H, F, E, k = 16, 256, 512, 8, 2  # the tiny layer
        fmt = np.full((E, 3), 4, np.uint8)
    W = gen.expert_weights_f32(0, 0, E, H, F)
    layer = orc.pack_layer(W, 0, E, H, F, fmt)
    x, Wr = _inputs(T, H, E)
    y, dbg = orc.moe_forward(layer, x, Wr, None, k, want_debug=True)
    mats = npref.dense_layer(W, fmt, H, F)
    y_ref, idx_ref, w_ref = npref.forward(x, Wr, None, k, mats, fmt_kind == "nvfp4")
    np.testing.assert_array_equal(dbg["idx"], idx_ref)
    np.testing.assert_allclose(dbg["w"], w_ref, rtol=1e-6)
    yo = npref.bf16_to_f64(y)
    # both round a float64 sum to bf16: at most one bf16 ulp apart
    assert np.all(np.abs(yo - y_ref) <= np.abs(y_ref) * 2.0 ** -8 + 1e-30)
    if fmt_kind == "nvfp4":
        xf = npref.bf16_to_f64(x).astype(np.float32)
        np.testing.assert_array_equal(dbg["xq"], npref.e4m3_codes(xf / dbg["sx"][:, None]))


def test_zero_expert_contributes_nothing(orc):
    T, H, F, E, k = 10, 128, 256, 4, 2
    fmt = np.full((E, 3), 4, np.uint8)
    W = gen.expert_weights_f32(0, 0, E, H, F)
    W[2] = 0.0
    layer = orc.pack_layer(W, 0, E, H, F, fmt)
    x, _ = _inputs(T, H, E)
    a = npref.bf16_to_f64(x)
    h = orc.gateup(layer, 2, a)
    assert np.all(h == 0.0)
    assert np.all(orc.down(layer, 2, np.ones((3, F))) == 0.0)
    # route everything to experts {1, 2} with k = 2: y equals w1 * expert1 only
    b = np.array([-100, 100, 99, -100], np.float32)
    Wr = np.zeros((E, H), np.float32)
    y, dbg = orc.moe_forward(layer, x, Wr, b, k, want_debug=True)
    assert np.all(dbg["idx"] == np.array([1, 2]))
    o1 = orc.down(layer, 1, orc.gateup(layer, 1, a))
    want = dbg["w"][:, :1].astype(np.float64) * o1
    assert np.all(np.abs(npref.bf16_to_f64(y) - want) <= np.abs(want) * 2.0 ** -8)


def test_k_equals_E_equal_logits_is_mean(orc):
    T, H, F, E = 6, 128, 128, 4
    fmt = np.array([[4, 4, 4], [2, 2, 2], [3, 2, 4], [4, 4, 2]], np.uint8)
    W = gen.expert_weights_f32(1, 0, E, H, F)
    layer = orc.pack_layer(W, 0, E, H, F, fmt)
    x, _ = _inputs(T, H, E, seed=1)
    y = orc.moe_forward(layer, x, np.zeros((E, H), np.float32), np.zeros(E, np.float32), E)
    a = npref.bf16_to_f64(x)
    mean = sum(orc.down(layer, e, orc.gateup(layer, e, a)) for e in range(E)) / E
    assert np.all(np.abs(npref.bf16_to_f64(y) - mean) <= np.abs(mean) * 2.0 ** -8 + 1e-12)


def test_k1_is_single_expert(orc):
    T, H, F, E = 5, 128, 256, 3
    fmt = np.full((E, 3), 3, np.uint8)
    W = gen.expert_weights_f32(2, 0, E, H, F)
    layer = orc.pack_layer(W, 0, E, H, F, fmt)
    x, _ = _inputs(T, H, E, seed=2)
    b = np.array([0, 5, 0], np.float32)
    y = orc.moe_forward(layer, x, np.zeros((E, H), np.float32), b, 1)
    o = orc.down(layer, 1, orc.gateup(layer, 1, npref.bf16_to_f64(x)))
    np.testing.assert_array_equal(y, np.array([[orc.bf16_bits(v) for v in row] for row in o], np.uint16))


def test_constant_weights_closed_form_sign_code(orc):
    # every weight = c (few significant bits, so the fp32 sum of 32 of them is exact):
    # s = fp16(32c/32) = c and every code is +1, so g_n = u_n = c*sum_k x_k.
    T, H, F, E = 4, 256, 128, 1
    c = np.float32(0.025390625)  # 1.625 * 2^-6
    W = np.full((E, 3, H * F), c, np.float32)
    layer = orc.pack_layer(W, 0, E, H, F, np.full((E, 3), 1, np.uint8))
    x, _ = _inputs(T, H, E, seed=3)
    a = npref.bf16_to_f64(x)
    g = float(c) * a.sum(1)
    h = orc.gateup(layer, 0, a)
    want = g / (1 + np.exp(-g)) * g
    np.testing.assert_allclose(h, np.repeat(want[:, None], F, 1), rtol=1e-12)


def test_constant_weights_closed_form(orc):
    # every weight = c: each group's scale is s = fp16(c/qmax), every code is qmax,
    # so g_n = u_n = s*qmax*sum_k x_k for every output n.
    T, H, F, E = 4, 256, 128, 1
    for bits in (2, 3, 4):
        qmax = (1 << (bits - 1)) - 1
        c = np.float32(0.013)
        W = np.full((E, 3, H * F), c, np.float32)
        layer = orc.pack_layer(W, 0, E, H, F, np.full((E, 3), bits, np.uint8))
        x, _ = _inputs(T, H, E, seed=3)
        a = npref.bf16_to_f64(x)
        s = float(np.float16(np.float32(c) / np.float32(qmax)))
        g = s * qmax * a.sum(1)
        h = orc.gateup(layer, 0, a)
        want = g / (1 + np.exp(-g)) * g
        np.testing.assert_allclose(h, np.repeat(want[:, None], F, 1), rtol=1e-12)
