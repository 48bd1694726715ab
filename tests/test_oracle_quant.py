"""Pins for the oracle's weight quantization, packing and layer layout.

  * hand-worked groups (tests/golden/int_group_examples.json, 1- to 4-bit): scale bits,
    codes (round-half-even ties) and packed words;
  * a hand-worked NVFP4 block (tests/golden/nvfp4_group_example.json): tensor
    scale, e4m3 block scale, e2m1 codes with ties to even, packed word and
    the dequantized values;
  * hand-computed word / byte positions of single codes in multi-tile
    matrices for every format (the 128x128 tile layout);
  * an independent numpy implementation of the quantization rule built on
    numpy's float16 cast and torch's e4m3 cast (library routines);
  * invariants: pack/unpack round trip, re-quantizing the dequantized matrix
    reproduces the codes bit-exactly, |w - w'| <= s/2 for unclamped values,
    codes in range;
  * layer layout: sections on 256-byte boundaries, disjoint, inside the buffer.
"""
import json
import os

import numpy as np
import torch

import gen
from tests import npref

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _word(buf: np.ndarray, byte_off: int) -> int:
    return int(np.frombuffer(buf[byte_off:byte_off + 4].tobytes(), "<u4")[0])


def test_hand_worked_groups(orc):
    ex = json.load(open(os.path.join(GOLD, "int_group_examples.json")))["examples"]
    for e in ex:
        W = np.zeros((128, 128), np.float32)
        for k, v in e["w_nonzero"].items():
            W[0, int(k)] = np.float32(v)
        q, s = orc.quant_int(W, e["bits"])
        assert int(s[0, 0]) == e["scale_bits"]
        assert list(q[0, :8]) == e["codes_first8"]
        assert np.all(s[1:] == 0) and np.all(s[0, 1:] == 0)
        codes, scales = orc.pack_int(q, s, e["bits"])
        for w_i, hexw in enumerate(e["words"]):
            assert _word(codes, 512 * w_i) == int(hexw, 16), (e["bits"], w_i)
        assert int(np.frombuffer(scales[:2].tobytes(), "<u2")[0]) == e["scale_bits"]


def test_hand_worked_nvfp4_group(orc):
    ex = json.load(open(os.path.join(GOLD, "nvfp4_group_example.json")))
    N = K = 128
    W = np.zeros((N, K), np.float32)
    W[0, :8] = np.asarray(ex["w_block0"], np.float32)
    v, sb, sT = orc.quant_nvfp4(W)
    assert sT == ex["tensor_scale"]
    assert int(sb[0, 0]) == ex["block0_scale_code"]
    assert np.count_nonzero(sb) == 1
    assert v[0, :8].tolist() == ex["codes_first8"]
    assert np.count_nonzero(v) == np.count_nonzero(ex["codes_first8"])
    codes, scales = orc.pack_nvfp4(v, sb)
    assert _word(codes, 0) == int(ex["word0"], 16)
    assert np.count_nonzero(codes) == 4  # the nonzero nibbles of word 0 fill four bytes
    assert scales[0] == ex["block0_scale_code"] and np.count_nonzero(scales) == 1
    deq = orc.decode_matrix(codes, scales, orc.FMT_NVFP4, N, K, sT)
    np.testing.assert_array_equal(deq[0, :8], np.asarray(ex["dequant_first8"]))
    assert np.count_nonzero(deq) == 7


def test_layout_positions_hand_computed(orc):
    # element (n=130, k=200) of a 256x256 matrix: n-block 1, k-block 1, group 2
    # inside the tile, position 8 inside the group (an even code: 4-bit nibble 0 of
    # word 1; 2-bit field 4 of word 0; 3-bit field 4 of word 0 and, pair m=4 being
    # c=1, j=0, bit 8*0 + 1 + 0 = 1 of word 2).
    # 1-bit: code 8 of the group at bit 0*16 + 8/2 = 4 of word (((1*2+1)*4+2)*1)*128+2 = 1794.
    N = K = 256
    cases = {
        # bits: (code, [(byte offset, expected word), ...], base word); other codes 0 (1-bit: +1)
        1: (-1, [(7176, 0xFFFFFFEF)], 0xFFFFFFFF),
        4: (5, [(29192, 0x8888888D)], 0x88888888),
        2: (-1, [(14344, 0xAAAAA9AA)], 0xAAAAAAAA),
        3: (-3, [(21512, 0x00000100), (22536, 0xFFFFFFFD)], None),
    }
    for bits, (code, checks, base) in cases.items():
        q = np.full((N, K), 1 if bits == 1 else 0, np.int8)
        q[130, 200] = code
        s = np.zeros((N, K // 32), np.uint16)
        s[130, 6] = 0x1234
        codes, scales = orc.pack_int(q, s, bits)
        for off, want in checks:
            assert _word(codes, off) == want, (bits, off)
        words = np.frombuffer(codes.tobytes(), "<u4").copy()
        if base is not None:
            words[[off // 4 for off, _ in checks]] = base
            assert np.all(words == base)
        # scale of (n=130, group 6) at index (1*8 + 6)*128 + 2 = 1794
        sc = np.frombuffer(scales.tobytes(), "<u2")
        assert sc[1794] == 0x1234 and np.count_nonzero(sc) == 1
    # NVFP4: same element, e2m1 code 0xB in nibble 0 of word (((1*2+1)*4+2)*4+1)*128+2
    v = np.zeros((N, K), np.uint8)
    v[130, 200] = 0xB
    sb = np.zeros((N, K // 16), np.uint8)
    sb[130, 12] = 0x38
    codes, scales = orc.pack_nvfp4(v, sb)
    assert _word(codes, 29192) == 0x0000000B
    assert np.count_nonzero(codes) == 1
    # block scale (n=130, block 12) at (1*16 + 12)*128 + 2 = 3586
    assert scales[3586] == 0x38 and np.count_nonzero(scales) == 1


def test_quant_int_matches_numpy(orc):
    for bits in (1, 2, 3, 4):
        W = gen.normal_f32(0, 99 + bits, 0, 256 * 512, 0.02).reshape(256, 512)
        W[3, 64:96] = 0.0  # an all-zero group
        W[5, :32] *= np.float32(1e-6)  # tiny scales (fp16 subnormal)
        q, s = orc.quant_int(W, bits)
        qn, sn = npref.quant_int(W, bits)
        np.testing.assert_array_equal(s, sn)
        np.testing.assert_array_equal(q, qn)
        if bits == 1:
            assert set(np.unique(q)) <= {-1, 1}
            assert np.all(q[3, 64:96] == 1) and s[3, 2] == 0
            continue
        qmax = (1 << (bits - 1)) - 1
        assert q.min() >= -qmax and q.max() <= qmax
        assert np.all(q[3, 64:96] == 0) and s[3, 2] == 0


def test_sign_code_scale_is_least_squares(orc):
    # for a sign code q, sum (w - s q)^2 = sum w^2 - 2 s sum|w| + 32 s^2 is minimized at
    # s = mean|w|, so the fp16 value nearest to it beats both fp16 neighbours
    W = gen.normal_f32(0, 321, 0, 64 * 256, 0.02).reshape(64, 256)
    q, s = orc.quant_int(W, 1)
    G = W.reshape(64, 8, 32).astype(np.float64)
    Q = q.reshape(64, 8, 32).astype(np.float64)
    assert np.all(Q == np.where(G >= 0, 1.0, -1.0))
    s16 = s.view(np.float16)
    def err(sv):
        return ((G - sv.astype(np.float64)[:, :, None] * Q) ** 2).sum(axis=2)
    e0 = err(s16)
    assert np.all(e0 <= err(np.nextafter(s16, np.float16(np.inf))))
    assert np.all(e0 <= err(np.nextafter(s16, np.float16(0))))


def test_int_roundtrip_and_requant(orc):
    for bits in (1, 2, 3, 4):
        W = gen.normal_f32(0, 200 + bits, 0, 384 * 256, 0.02).reshape(384, 256)
        q, s = orc.quant_int(W, bits)
        codes, scales = orc.pack_int(q, s, bits)
        q2, s2 = orc.unpack_int(codes, scales, 384, 256, bits)
        np.testing.assert_array_equal(q, q2)
        np.testing.assert_array_equal(s, s2)
        Wd = npref.dequant_int(q, s)
        # dequantized values are exact in fp32; re-quantizing reproduces the codes
        q3, s3 = orc.quant_int(Wd.astype(np.float32), bits)
        np.testing.assert_array_equal(q, q3)
        np.testing.assert_array_equal(s, s3)
        # decode_row through the packed layout equals s*q
        np.testing.assert_array_equal(orc.decode_matrix(codes, scales, bits, 384, 256), Wd)
        if bits == 1:  # the sign code has its own pin (least-squares scale)
            continue
        # error bound for values that were not clamped
        qmax = (1 << (bits - 1)) - 1
        sf = np.repeat(s.view(np.float16).astype(np.float64), 32, axis=1)
        inner = np.abs(W.astype(np.float64) / np.where(sf == 0, 1, sf)) <= qmax
        err = np.abs(W.astype(np.float64) - Wd)
        assert np.all(err[inner] <= sf[inner] / 2 * (1 + 1e-6))


def test_nvfp4_matches_numpy_and_roundtrip(orc):
    W = gen.normal_f32(0, 300, 0, 256 * 512, 0.02).reshape(256, 512)
    W[7, 16:32] = 0.0
    v, sb, sT = orc.quant_nvfp4(W)
    vn, sbn, sTn = npref.quant_nvfp4(W)
    assert sT == sTn
    np.testing.assert_array_equal(sb, sbn)
    np.testing.assert_array_equal(v, vn)
    assert np.all(v[7, 16:32] == 0)
    codes, scales = orc.pack_nvfp4(v, sb)
    v2, sb2 = orc.unpack_nvfp4(codes, scales, 256, 512)
    np.testing.assert_array_equal(v, v2)
    np.testing.assert_array_equal(sb, sb2)
    Wd = orc.decode_matrix(codes, scales, orc.FMT_NVFP4, 256, 512, sT)
    want = npref.dequant_nvfp4(v, sb, sT)
    np.testing.assert_array_equal(Wd, want)
    # constant matrix: sT = c/2688, every block scale 448, every code +6 -> w' ~ c
    c = np.float32(0.03)
    v, sb, sT = orc.quant_nvfp4(np.full((128, 128), c, np.float32))
    assert np.all(sb == 0x7E) and np.all(v == 7)


def test_layer_layout(orc):
    E, H, F = 5, 256, 384
    fmt = np.array([[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 4, 2], [16, 16, 16]], np.uint8)
    co, so, total = orc.layer_layout(E, H, F, fmt)
    spans = []
    for e in range(E):
        for p in range(3):
            N, K = (F, H) if p < 2 else (H, F)
            f = int(fmt[e, p])
            assert co[e * 3 + p] % 256 == 0 and so[e * 3 + p] % 256 == 0
            spans.append((int(co[e * 3 + p]), int(co[e * 3 + p]) + orc.code_bytes(f, N, K)))
            spans.append((int(so[e * 3 + p]), int(so[e * 3 + p]) + orc.scale_bytes(f, N, K)))
    spans.sort()
    assert spans[0][0] >= orc.HDR_BYTES
    for (a0, a1), (b0, _) in zip(spans[:-1], spans[1:]):
        assert a1 <= b0
    assert spans[-1][1] <= total
    # bytes: int b-bit codes = N*K*b/8, scales = N*K/32*2; NVFP4 codes N*K/2, scales N*K/16
    assert orc.code_bytes(3, F, H) == F * H * 3 // 8
    assert orc.scale_bytes(4, F, H) == F * H // 16
    assert orc.code_bytes(16, F, H) == F * H // 2
    assert orc.scale_bytes(16, F, H) == F * H // 16


def test_pack_layer_partial_equals_full(orc):
    E, H, F = 3, 256, 256
    fmt = np.array([[4, 4, 4], [3, 2, 4], [2, 2, 2]], np.uint8)
    W = gen.expert_weights_f32(0, 0, E, H, F)
    full = orc.pack_layer(W, 0, E, H, F, fmt)
    part = orc.pack_layer(W[:1], 0, E, H, F, fmt)
    part = orc.pack_layer(W[1:], 1, E, H, F, fmt, out=part)
    np.testing.assert_array_equal(full, part)
    hdr = np.frombuffer(full[:20].tobytes(), "<u4")
    assert hdr[0] == 0x51454F4D and hdr[1] == 1 and hdr[2] == E and hdr[3] == H and hdr[4] == F
    np.testing.assert_array_equal(orc.layer_fmt(full), fmt)
