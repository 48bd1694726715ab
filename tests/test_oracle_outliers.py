"""Pins for the oracle's outlier isolation (oracle/outliers.py):

  * the count is floor(0.05% of N*K);
  * the selection equals a brute-force one (repeated arg-max with masking, ties
    to the lower index), with planted ties;
  * no kept weight is larger in magnitude than the smallest outlier;
  * at outlier positions the matrix is the weight rounded once to fp16; elsewhere
    it is the plain quantization of the matrix with its outliers zeroed;
  * planted large outliers no longer inflate their groups' scales, and the
    reconstruction error drops;
  * the 1-bit sign code keeps the residual w - (+s) of a zeroed weight;
  * zero outliers reproduce plain quantization bit for bit.
"""
import numpy as np
import pytest

import gen
from oracle import outliers as ol


def _brute_select(W, n_out):
    mag = np.abs(W.astype(np.float64)).ravel().copy()
    picked = []
    for _ in range(n_out):
        best = int(np.argmax(mag))  # first index among equal maxima
        picked.append(best)
        mag[best] = -1.0
    picked.sort()
    return np.array(picked) // W.shape[1], np.array(picked) % W.shape[1]


def _weights(N, K, seed):
    return gen.normal_f32(0, seed, 0, N * K, 0.02).reshape(N, K)


def test_count_is_the_floor_of_five_per_ten_thousand():
    assert ol.count(256, 256) == 32        # 65536 * 0.0005 = 32.768
    assert ol.count(128, 128) == 8         # 8.192
    assert ol.count(14336, 4096) == 29360  # 29360.128


def test_selection_matches_brute_force_with_ties():
    W = _weights(128, 256, 901)
    W[3, 7] = W[100, 2] = np.float32(0.5)     # a tie among the largest
    W[50, 50] = np.float32(-0.5)              # same magnitude, negative
    W[9, 9] = np.float32(0.75)
    for n_out in (1, 2, 3, 4, ol.count(128, 256)):
        r, c = ol.select(W, n_out)
        br, bc = _brute_select(W, n_out)
        np.testing.assert_array_equal(r, br)
        np.testing.assert_array_equal(c, bc)
    r, c = ol.select(W, 3)  # 0.75 and the first two of the three 0.5 ties in index order
    assert list(zip(r, c)) == [(3, 7), (9, 9), (50, 50)]


@pytest.mark.parametrize("fmt", [1, 2, 3, 4, 16])
def test_isolation_reconstructs_outliers_and_keeps_the_rest(fmt):
    N, K = 128, 256
    W = _weights(N, K, 902 + fmt)
    iso = ol.isolate(W, fmt)
    r, c = iso["rows"], iso["cols"]
    assert len(r) == ol.count(N, K)
    keep = np.ones((N, K), bool)
    keep[r, c] = False
    assert np.abs(W[keep]).max() <= np.abs(W[r, c]).min()
    Wh = ol.dequant(iso, fmt, N, K)
    if fmt != 1:  # every other format represents 0: the outlier is fp16(w) itself
        np.testing.assert_array_equal(Wh[r, c], W[r, c].astype(np.float16).astype(np.float64))
    # the kept weights are exactly the plain quantization of the zeroed matrix
    Wz = W.copy()
    Wz[r, c] = 0.0
    plain = ol.isolate(Wz, fmt, n_out=0)
    np.testing.assert_array_equal(plain["codes"], iso["codes"])
    np.testing.assert_array_equal(plain["scales"], iso["scales"])
    np.testing.assert_array_equal(ol.dequant(plain, fmt, N, K)[keep], Wh[keep])


def test_sign_code_residual_is_w_minus_plus_s():
    N, K = 128, 256
    W = _weights(N, K, 911)
    iso = ol.isolate(W, 1)
    s = iso["scales"].view(np.float16).astype(np.float64)  # [N/128][K/32][128] order
    for n, k, res in zip(iso["rows"], iso["cols"], iso["resid"]):
        sv = s[((n // 128) * (K // 32) + k // 32) * 128 + n % 128]
        want = np.float16(np.float64(W[n, k]) - sv)  # the zeroed weight decodes to +s
        assert np.uint16(res) == want.view(np.uint16)


def test_planted_outliers_stop_inflating_scales():
    N, K = 128, 256
    W = _weights(N, K, 921)
    rng = np.random.default_rng(3)
    flat = rng.choice(N * K, ol.count(N, K), replace=False)
    # +-0.5 is far above every N(0, 0.02) weight, so the planted outliers are exactly the top set
    W.ravel()[flat] = np.where(W.ravel()[flat] >= 0, np.float32(0.5), np.float32(-0.5))
    iso = ol.isolate(W, 4)
    np.testing.assert_array_equal(np.sort(iso["rows"] * K + iso["cols"]), np.sort(flat))
    plain = ol.isolate(W, 4, n_out=0)
    # the other weights of the groups that held an outlier: with the outlier taken out their
    # group scale shrinks from 0.5/7 to about max|w|/7, so their error drops several-fold
    rows, cols = flat // K, flat % K
    mask = np.zeros((N, K), bool)
    for n, k in zip(rows, cols):
        mask[n, (k // 32) * 32:(k // 32) * 32 + 32] = True
    mask[rows, cols] = False
    err_iso = np.abs(ol.dequant(iso, 4, N, K) - W)[mask].sum()
    err_plain = np.abs(ol.dequant(plain, 4, N, K) - W)[mask].sum()
    assert err_iso < 0.25 * err_plain
    assert iso["scales"].view(np.float16).max() < plain["scales"].view(np.float16).max()


def test_zero_outliers_is_plain_quantization():
    import oracle as orc
    W = _weights(128, 128, 931)
    iso = ol.isolate(W, 3, n_out=0)
    q, s = orc.quant_int(W, 3)
    codes, scales = orc.pack_int(q, s, 3)
    np.testing.assert_array_equal(iso["codes"], codes)
    np.testing.assert_array_equal(iso["scales"], scales)
    assert len(iso["rows"]) == 0
