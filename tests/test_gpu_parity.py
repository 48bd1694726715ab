"""GPU parity: the CUDA library (through the C ABI) against the CPU oracle.

Bars (per layer):
  * packed codes, scales and header bytes: bit-exact;
  * permutation rows and per-expert counts: bit-exact;
  * top-k sets: exact except where the oracle's k-th vs (k+1)-th logit gap is
    below 1e-5 (counted; the oracle is then re-fed the GPU's choice);
  * top-k weights: within 1e-6;
  * NVFP4 layers: FP8 codes and scales of x bit-exact;
  * outputs: max |y_gpu - y_oracle| <= 2e-2 * max |y_oracle|.
"""
import numpy as np
import pytest

import gen
import gen.workloads as W
import oracle as orc
from tests import helpers as hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import mixed_precision_quantized_fp32_b200 as moe  # noqa: E402
from mixed_precision_quantized_fp32_b200 import _lib  # noqa: E402


def custom(name, T, H, F, E, k, fmt, bias=None):
    # a named configuration's packed buffer is cached by name, so custom layers use other names
    assert name not in W.NAMES, name
    L = W.Layer(name, H, F, E, k, np.asarray(fmt, np.uint8).reshape(E, 3), (T,), (), bias)
    return L


def run_gpu(L, layer, T, x=None, Wr=None, b=None, k=None, act=0):
    k = k or L.k
    x = W.device_x(T, L.H) if x is None else x
    if Wr is None:
        Wr, b = W.device_router(L)
    R = T * k
    dbg = dict(topk_idx=torch.empty(R, dtype=torch.int32, device="cuda"),
               topk_w=torch.empty(R, dtype=torch.float32, device="cuda"),
               perm=torch.empty(R, dtype=torch.int32, device="cuda"),
               inv=torch.empty(R, dtype=torch.int32, device="cuda"),
               counts=torch.empty(L.E, dtype=torch.int32, device="cuda"),
               status=torch.zeros(1, dtype=torch.int32, device="cuda"))
    if L.fp4:
        dbg.update(xq=torch.empty(T * L.H, dtype=torch.uint8, device="cuda"),
                   sx=torch.empty(T, dtype=torch.float32, device="cuda"),
                   hq=torch.empty(R * L.F, dtype=torch.uint8, device="cuda"),
                   sh=torch.empty(R, dtype=torch.float32, device="cuda"))
    if act:
        dbg.update(xsb=torch.empty(T * L.H // 16, dtype=torch.uint8, device="cuda"),
                   hsb=torch.empty(R * L.F // 16, dtype=torch.uint8, device="cuda"))
    # y inside a guard band: 4 KiB of a sentinel (exact in bf16) on each side must survive the call
    G, SENTINEL = 2048, -12288.0
    buf = torch.full((T * L.H + 2 * G,), SENTINEL, dtype=torch.bfloat16, device="cuda")
    y = buf[G:G + T * L.H].view(T, L.H)
    moe.moe_layer_forward(x, Wr, b, layer, k, y=y, debug=dbg)
    torch.cuda.synchronize()
    guard = torch.cat([buf[:G], buf[G + T * L.H:]])
    assert bool((guard == SENTINEL).all()), "output guard band overwritten"
    out = {n: t.cpu().numpy() for n, t in dbg.items()}
    out["y"] = y
    assert out["status"][0] == 0
    return out


def check_layer(L, T, tokens=None, bias=None, router_zero=False, max_ties=None, act=0):
    """Full parity of one layer / batch.  tokens: the subset whose outputs are
    compared against the oracle (default all).  act: the activation format of an
    NVFP4 layer (moe.ACT_NVFP4: the oracle's NVFP4-activation mode)."""
    k = L.k
    layer = hp.gpu_pack_cached(L) if L.name in W.NAMES else hp.gpu_pack(L)
    if act:
        layer = moe.PackedLayer(layer.E, layer.H, layer.F, layer.fmt, layer.packed, act)
    x_bits = W.x_bf16_bits(T, L.H)
    Wr_h = np.zeros((L.E, L.H), np.float32) if router_zero else W.router_w(L.E, L.H)
    b_h = bias if bias is not None else L.bias
    Wr = torch.from_numpy(Wr_h).cuda()
    b = None if b_h is None else torch.from_numpy(np.asarray(b_h, np.float32)).cuda()
    g = run_gpu(L, layer, T, Wr=Wr, b=b, act=act)

    logits, idx_o, w_o = hp.oracle_route(x_bits, Wr_h, b_h, k)
    idx_g = g["topk_idx"].reshape(T, k)
    ties = hp.near_tie_tokens(logits, k, idx_g, idx_o)
    if max_ties is not None:
        assert len(ties) <= max_ties
    same = np.setdiff1d(np.arange(T), ties)
    np.testing.assert_array_equal(idx_g[same], idx_o[same])
    np.testing.assert_allclose(g["topk_w"].reshape(T, k)[same], w_o[same], rtol=0, atol=1e-6)
    # permutation of the GPU's own choice: bit-exact against the oracle's permutation step
    counts, offsets, perm, inv = orc.permute(idx_g.astype(np.int32), L.E)
    np.testing.assert_array_equal(g["counts"], counts)
    np.testing.assert_array_equal(g["perm"], perm)
    np.testing.assert_array_equal(g["inv"], inv)
    if L.fp4 and act:
        from oracle import nvfp4_act as na
        xv, xsb, xs = na.quant_rows(gen.bf16_bits_to_f32(x_bits))
        np.testing.assert_array_equal(g["xq"].reshape(T, L.H), xv)
        np.testing.assert_array_equal(g["xsb"].reshape(T, L.H // 16), xsb)
        np.testing.assert_array_equal(g["sx"], xs)
    elif L.fp4:
        xq, sx = orc.act_quant_e4m3(gen.bf16_bits_to_f32(x_bits))
        np.testing.assert_array_equal(g["xq"].reshape(T, L.H), xq)
        np.testing.assert_array_equal(g["sx"], sx)

    if callable(tokens):
        tokens = tokens(g["perm"], g["counts"], k)
    tokens = np.arange(T) if tokens is None else np.asarray(tokens)
    experts = np.unique(np.concatenate([idx_o[tokens].ravel(), idx_g[tokens].ravel()]))
    buf = hp.oracle_pack(L, experts)
    if act:
        y_ref, _, _ = hp.oracle_forward_rows_act4(buf, x_bits, Wr_h, b_h, k, tokens=tokens,
                                                  idx_override=idx_g if ties else None)
    else:
        y_ref, _, _ = hp.oracle_forward_rows(buf, x_bits, Wr_h, b_h, k, tokens=tokens,
                                             idx_override=idx_g if ties else None, fp4=L.fp4)
    ratio = hp.check_output(g["y"][torch.from_numpy(tokens).cuda()], y_ref)
    return dict(ties=len(ties), err_ratio=ratio, counts=g["counts"], n_tokens=len(tokens))


# ------------------------------------------------------------------ generator / packing
def test_device_generator_matches_host():
    for tid, sigma, n in [(1, 1.0, 100_003), (gen.tid_expert(3, 2), 0.02, 65_536)]:
        t = torch.empty(n, dtype=torch.float32, device="cuda")
        W.fill_device_f32(t, 0, tid, sigma, start=77)
        np.testing.assert_array_equal(t.cpu().numpy(), gen.normal_f32(0, tid, 77, n, sigma))
        b = torch.empty(n, dtype=torch.bfloat16, device="cuda")
        W.fill_device_bf16(b, 0, tid, sigma)
        np.testing.assert_array_equal(b.view(torch.int16).cpu().numpy().view(np.uint16),
                                      gen.normal_bf16_bits(0, tid, 0, n, sigma))


PACK_CASES = [
    ("int4", 384, 256, 3, [[4, 4, 4]] * 3),
    ("mixed", 256, 640, 6, [[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 4, 2], [3, 3, 3], [2, 4, 3]]),
    ("nvfp4_small", 256, 384, 4, [[16, 16, 16]] * 4),
    ("graded_mix", 256, 384, 6, [[4, 4, 4], [2, 2, 2], [1, 1, 1], [4, 2, 1], [1, 2, 4], [2, 1, 2]]),
]


@pytest.mark.parametrize("name,H,F,E,fmt", PACK_CASES)
def test_pack_bit_exact(name, H, F, E, fmt):
    L = custom(name, 1, H, F, E, 1, fmt)
    layer = hp.gpu_pack(L, experts_per_call=2)
    got = layer.packed.cpu().numpy()
    want = hp.oracle_pack(L, range(E))
    np.testing.assert_array_equal(got, want)


def test_pack_edge_values_bit_exact():
    # all-zero expert, tiny values (fp16-subnormal scales), a large-magnitude group
    L = custom("edge", 1, 256, 256, 3, 1, [[4, 3, 2], [16, 16, 16], [2, 4, 3]])
    fmt = L.fmt.reshape(-1)
    Wh = np.stack([W.expert_w(e, 256, 256) for e in range(3)])
    Wh[0, 1] = 0.0
    Wh[1, 0, :4096] *= np.float32(1e-7)
    Wh[2, 2, :64] *= np.float32(3000.0)
    total = moe.pack_layout(3, 256, 256, fmt)[0]
    packed = moe.alloc_packed(total)
    moe.moe_pack(torch.from_numpy(Wh).cuda(), 0, 3, 256, 256, fmt, packed)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy(), orc.pack_layer(Wh, 0, 3, 256, 256, fmt))


def test_pack_edge_values_sign_code():
    # 1-bit sign code: an all-zero matrix (scale 0, every code +1), signed zeros, tiny
    # values (fp16-subnormal scale), and a group whose mean |w| overflows fp16 (scale
    # saturated to 65504)
    L = custom("edge1", 1, 256, 256, 2, 1, [[1, 1, 1], [1, 1, 1]])
    fmt = L.fmt.reshape(-1)
    Wh = np.stack([W.expert_w(e, 256, 256) for e in range(2)])
    Wh[0, 0] = 0.0
    Wh[0, 1, :4096] *= np.float32(1e-7)
    Wh[0, 2, :32] = np.float32(70000.0)
    Wh[1, 0, ::7] = np.float32(-0.0)
    total = moe.pack_layout(2, 256, 256, fmt)[0]
    packed = moe.alloc_packed(total)
    moe.moe_pack(torch.from_numpy(Wh).cuda(), 0, 2, 256, 256, fmt, packed)
    torch.cuda.synchronize()
    np.testing.assert_array_equal(packed.cpu().numpy(), orc.pack_layer(Wh, 0, 2, 256, 256, fmt))


@pytest.mark.parametrize("T", [37, 600])
def test_forward_graded_tiers(T):
    # precision falling with hotness, down to the 1-bit sign code; T=37 runs the GEMV,
    # T=600 the tcgen05 GEMMs on CTA pairs (F/128 = 2, H/128 = 4)
    L = custom("graded_small", T, 512, 256, 6, 2, [[4, 4, 4], [2, 2, 2], [1, 1, 1], [4, 2, 1], [1, 2, 4], [2, 1, 2]])
    check_layer(L, T)


@pytest.mark.parametrize("name", ["tiny", "mixtral", "hotcold", "nvfp4", "large", "graded"])
def test_pack_bit_exact_configs(name):
    L = W.layer(name)
    layer = hp.gpu_pack_cached(L)
    if name == "tiny":
        sample = range(L.E)
    elif name == "hotcold":
        hot = L.notes["hot_experts"]
        sample = [hot[0], next(e for e in range(L.E) if e not in hot), L.E - 1]
    elif name == "graded":  # one expert of each tier: 4-, 2- and 1-bit
        tiers = [int(np.flatnonzero(L.fmt[:, 0] == b)[0]) for b in (4, 2, 1)]
        sample = sorted(tiers)
    else:
        sample = [0, L.E - 1]
    want = hp.oracle_pack(L, sample)
    got_hdr = layer.packed[:orc.HDR_BYTES].cpu().numpy()
    # header: identical except tensor scales of experts the oracle did not pack
    ts_g = got_hdr[13088:13088 + 3072].view(np.float32).copy()
    ts_w = want[13088:13088 + 3072].view(np.float32).copy()
    for e in range(L.E):
        if e not in sample:
            ts_g[3 * e:3 * e + 3] = 0
    np.testing.assert_array_equal(ts_g, ts_w)
    gh = got_hdr.copy()
    gh[13088:13088 + 3072] = 0
    wh = want[:orc.HDR_BYTES].copy()
    wh[13088:13088 + 3072] = 0
    np.testing.assert_array_equal(gh, wh)
    for e in sample:
        for off, n in hp.sections(L, e):
            np.testing.assert_array_equal(layer.packed[off:off + n].cpu().numpy(), want[off:off + n],
                                          err_msg=f"{name} expert {e} section @{off}")


# ------------------------------------------------------------------ forward, small shapes
def test_forward_tiny_layer():
    r = check_layer(W.layer("tiny"), 16)
    assert r["ties"] == 0


def test_forward_ragged_mixed_formats():
    # several 128-row tiles, a ragged token count, every integer format
    L = custom("ragged", 37, 384, 640, 12, 3,
               [[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 4, 2], [3, 3, 3], [2, 4, 3]] * 2)
    check_layer(L, 37)


@pytest.mark.parametrize("fmt,act", [
    ([[3, 2, 4], [1, 1, 1], [4, 1, 2], [2, 3, 3], [4, 4, 4], [2, 2, 1]], 0),
    ([[16, 16, 16]] * 6, 0),
    ([[16, 16, 16]] * 6, 1),
], ids=["int", "nvfp4", "nvfp4-act4"])
def test_forward_gemv_several_chunks_per_expert(fmt, act):
    # 100 expert rows over 6 experts (about 17 each, below the tcgen05 threshold): the GEMV walks
    # each expert's rows as two or three 8-row chunks over the same weight tiles, the last ragged
    L = custom("gemvchunks" + str(fmt[0][0]) + str(fmt[1][0]) + str(act), 50, 384, 640, 6, 2, fmt)
    r = check_layer(L, 50, act=act)
    assert r["counts"].max() > 16  # some expert takes three chunks


def test_forward_prefill_chunks_and_tails():
    # more than 16 rows per expert: 64-row chunks, several per expert, ragged tails
    L = custom("chunks", 300, 256, 384, 4, 2, [[4, 4, 4], [3, 2, 4], [2, 2, 2], [4, 3, 2]])
    check_layer(L, 300)


def test_forward_cta_pairs_ragged_chunks():
    # tcgen05 path on CTA pairs for both GEMMs: gate/up F/128 = 2 weight tiles, down H/128 = 4 (two
    # pairs of tiles).  12 experts share 600 rows, a few dozen each, so every chunk's token count N
    # (rounded up to 16) splits over the two CTAs at N/2 rows, well short of a full 128-row half.
    L = custom("pairs", 300, 512, 256, 12, 2, [[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 3, 2]] * 3)
    check_layer(L, 300)


def _sweep_case(i):
    """Seeded random shape: H, F in 128*{1..8}, E in {1..16}, k in {1..min(E, 8)}, T in {1..300};
    every fourth case NVFP4, the rest a random integer width (1 to 4 bits) per expert and projection.  Cases
    i % 5 == 2 push two experts' router bias to -1e4 (experts with no tokens), cases i % 5 == 4
    push one expert's bias to +1e4 (every token picks it)."""
    rng = np.random.default_rng(7000 + i)
    H, F = 128 * int(rng.integers(1, 9)), 128 * int(rng.integers(1, 9))
    E = int(rng.integers(1, 17))
    k = int(rng.integers(1, min(E, 8) + 1))
    T = int(rng.integers(1, 301))
    fmt = [[16, 16, 16]] * E if i % 4 == 3 else rng.choice([1, 2, 3, 4], size=(E, 3)).tolist()
    bias = None
    if i % 5 == 2 and E - 2 >= k:
        bias = np.zeros(E, np.float32)
        bias[rng.choice(E, 2, replace=False)] = -1e4
    elif i % 5 == 4:
        bias = np.zeros(E, np.float32)
        bias[int(rng.integers(0, E))] = 1e4
    tokens = np.sort(rng.choice(T, min(T, 48), replace=False))
    return custom(f"sweep{i}", T, H, F, E, k, fmt), T, bias, tokens


@pytest.mark.parametrize("i", range(16))
def test_forward_random_shape_sweep(i):
    L, T, bias, tokens = _sweep_case(i)
    r = check_layer(L, T, tokens=tokens, bias=bias)
    if bias is not None and bias.min() < 0:
        assert np.all(r["counts"][bias < 0] == 0)      # the pushed-down experts got no rows
    if bias is not None and bias.max() > 0:
        assert r["counts"][int(np.argmax(bias))] == T  # every token chose the pushed-up expert


@pytest.mark.parametrize("T", [8, 600])
def test_bounded_wait_timeout_keeps_context_usable(T):
    # Test hook: the expert GEMMs' copy warps withhold every load and the pipeline waits get a
    # budget of 200k cycles (~0.1 ms).  The consumers give up, every role leaves its loop, the
    # call reports MOE_ERR_TIMEOUT in the status word, and an ordinary call on the same context
    # afterwards is still exact.  T=8 runs the decode GEMV, T=600 the tcgen05 GEMMs on CTA pairs.
    L = custom("timeout", T, 512, 256, 4, 2, [[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 3, 2]])
    layer = hp.gpu_pack(L)
    x = W.device_x(T, L.H)
    Wr, b = W.device_router(L)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(x, Wr, b, layer, L.k,
                          debug={"status": st, "test_withhold": 1, "wait_cycles": 200_000})
    torch.cuda.synchronize()
    assert _lib.STATUS[int(st.item())] == "MOE_ERR_TIMEOUT"
    check_layer(L, T)


@pytest.mark.parametrize("T", [9, 300])
def test_forward_single_tile_dims(T):
    # H = F = 128: one 128-input tile per row block (no split-K), a gather row of 16
    # chunks; decode (GEMV) and prefill (tcgen05) batch sizes
    L = custom("tile1", T, 128, 128, 5, 2, [[3, 2, 4], [4, 4, 4], [2, 2, 2], [4, 3, 2], [2, 4, 3]])
    check_layer(L, T)


def test_forward_single_tile_dims_nvfp4():
    L = custom("tile1fp4", 11, 128, 128, 4, 2, [[16, 16, 16]] * 4)
    check_layer(L, 11)


def test_forward_router_gemm_ragged_experts_bias():
    # 72 experts (the last 64-expert tile ragged), split-K router planes, a bias
    E = 72
    L = custom("rgemm", 300, 1024, 256, E, 4, [[4, 2, 3]] * E)
    bias = (np.random.default_rng(5).standard_normal(E) * 0.05).astype(np.float32)
    check_layer(L, 300, bias=bias)


def test_forward_permutation_block_edges():
    # T*k = 1024 (the one-block permutation at its limit) and 1028 (the three-pass path)
    L = custom("perm1k", 256, 256, 256, 16, 4, [[4, 4, 4], [2, 2, 2], [3, 2, 4], [4, 3, 2]] * 4)
    check_layer(L, 256)
    check_layer(L, 257)


def test_forward_nvfp4_small():
    L = custom("fp4small", 23, 256, 384, 16, 6, [[16, 16, 16]] * 16)
    check_layer(L, 23)


def test_forward_nvfp4_prefill_chunks():
    L = custom("fp4chunks", 200, 256, 256, 8, 2, [[16, 16, 16]] * 8)
    check_layer(L, 200)


def test_nvfp4_down_stage_refeed():
    # feed the GPU's e4m3 codes of h into the oracle's down stage: output parity of the
    # down GEMM + combine alone (h codes depend on summation order and are not required
    # to match bit for bit).
    L = custom("fp4refeed", 9, 256, 256, 8, 2, [[16, 16, 16]] * 8)
    T, k = 9, 2
    layer = hp.gpu_pack(L)
    g = run_gpu(L, layer, T)
    x_bits = W.x_bf16_bits(T, L.H)
    buf = hp.oracle_pack(L, range(L.E))
    idx = g["topk_idx"].reshape(T, k)
    counts, offsets, perm, inv = orc.permute(idx.astype(np.int32), L.E)
    hq = g["hq"].reshape(T * k, L.F)
    sh = g["sh"]
    o = np.zeros((T * k, L.H))
    for e in range(L.E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            o[r0:r1] = orc.down(buf, e, orc.e4m3_table()[hq[r0:r1]], sh[r0:r1].astype(np.float64))
    y_ref = np.zeros((T, L.H))
    w = g["topk_w"].reshape(T, k)
    for t in range(T):
        for j in range(k):
            y_ref[t] += float(w[t, j]) * o[inv[t * k + j]]
    hp.check_output(g["y"], y_ref)
    # and the h codes themselves: count disagreements with the oracle's own h codes
    a = orc.e4m3_table()[orc.act_quant_e4m3(gen.bf16_bits_to_f32(x_bits))[0]]
    sx = orc.act_quant_e4m3(gen.bf16_bits_to_f32(x_bits))[1]
    n_diff = 0
    for e in range(L.E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            ts = perm[r0:r1] // k
            h = orc.gateup(buf, e, a[ts], sx[ts].astype(np.float64))
            hq_o, _ = orc.act_quant_e4m3(h.astype(np.float32))
            n_diff += int(np.count_nonzero(hq_o != hq[r0:r1]))
    assert n_diff <= 0.01 * hq.size, f"{n_diff} of {hq.size} h codes differ"


def test_forward_single_token():
    L = custom("one", 1, 256, 256, 8, 2, [[4, 2, 3]] * 8)
    check_layer(L, 1)


def test_forward_all_tokens_one_expert():
    # bias sends every token to expert 3 (k = 1): one expert, 200 rows, 4 chunks
    L = custom("onehot", 200, 256, 256, 8, 1, [[4, 4, 4]] * 8)
    b = np.zeros(8, np.float32)
    b[3] = 100.0
    r = check_layer(L, 200, bias=b)
    assert r["counts"][3] == 200 and r["counts"].sum() == 200


def test_forward_k_equals_E_equal_logits_is_mean():
    L = custom("mean", 5, 256, 256, 8, 8, [[4, 3, 2]] * 8)
    r = check_layer(L, 5, bias=np.zeros(8, np.float32), router_zero=True)
    assert np.all(r["counts"] == 5)


def test_forward_zero_expert():
    L = custom("zero", 12, 256, 256, 4, 2, [[4, 4, 4]] * 4)
    layer = hp.gpu_pack(L)
    # overwrite expert 1 with zero weights through the ABI
    zeros = torch.zeros((1, 3, L.H * L.F), dtype=torch.float32, device="cuda")
    moe.moe_pack(zeros, 1, L.E, L.H, L.F, L.fmt.reshape(-1), layer.packed)
    b = np.array([0, 50, 49, -50], np.float32)  # every token -> experts {1, 2}
    Wr = torch.zeros((L.E, L.H), dtype=torch.float32, device="cuda")
    g = run_gpu(L, layer, 12, Wr=Wr, b=torch.from_numpy(b).cuda())
    assert np.all(np.sort(g["topk_idx"].reshape(12, 2), 1) == [1, 2])
    Wh = np.stack([W.expert_w(e, L.H, L.F) for e in range(L.E)])
    Wh[1] = 0
    buf = orc.pack_layer(Wh, 0, L.E, L.H, L.F, L.fmt.reshape(-1))
    y_ref, _, _ = hp.oracle_forward_rows(buf, W.x_bf16_bits(12, L.H), np.zeros((L.E, L.H), np.float32), b, 2)
    hp.check_output(g["y"], y_ref)


def _x_device(bits):
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).cuda().view(torch.bfloat16)


@pytest.mark.parametrize("T", [9, 600])
def test_forward_x_beyond_fp16_range(T):
    # bf16 x reaches far beyond fp16.  Planted |x| of 1e5, 3e6 and 131008 in column 17 of three
    # tokens: those tokens' rows are prescaled by a power of two before the fp16 conversion and
    # rescaled after the gate/up sums.  Inputs 0..31 (the quantization group of column 17) of
    # every gate, up and router row are zero, so the group scales are 0 (the 1-bit sign code has
    # no zero code) and the SwiGLU outputs and routing stay ordinary.  1-bit matrices are
    # included (their decode path once doubled the activations).  T=9 runs the decode GEMV,
    # T=600 the tcgen05 GEMMs.
    E, H, F, k = 6, 256, 256, 2
    fmt = np.array([[4, 4, 4], [2, 2, 2], [1, 1, 1], [4, 2, 1], [1, 2, 4], [3, 3, 3]], np.uint8)
    Wh = np.stack([W.expert_w(e, H, F) for e in range(E)])
    Wh[:, 0].reshape(E, F, H)[:, :, :32] = 0.0
    Wh[:, 1].reshape(E, F, H)[:, :, :32] = 0.0
    layer_fmt = fmt.reshape(-1)
    packed = moe.alloc_packed(moe.pack_layout(E, H, F, layer_fmt)[0])
    moe.moe_pack(torch.from_numpy(Wh).cuda(), 0, E, H, F, layer_fmt, packed)
    layer = moe.PackedLayer(E, H, F, layer_fmt, packed)
    Wr_h = W.router_w(E, H)
    Wr_h[:, :32] = 0.0
    x_bits = W.x_bf16_bits(T, H).copy()
    big = {0: 1e5, 3: -3e6, T - 1: 65504.0 * 2}
    for t, v in big.items():
        x_bits[t, 17] = gen.f32_to_bf16_bits(np.array([v], np.float32))[0]
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    y = moe.moe_layer_forward(_x_device(x_bits), torch.from_numpy(Wr_h).cuda(), None, layer, k,
                              debug={"status": st})
    torch.cuda.synchronize()
    assert int(st.item()) == 0
    buf = orc.pack_layer(Wh, 0, E, H, F, layer_fmt)
    y_ref, _, _ = hp.oracle_forward_rows(buf, x_bits, Wr_h, None, k)
    hp.check_output(y, y_ref)


@pytest.mark.parametrize("T", [9, 600])
def test_swiglu_overflow_reports_range(T):
    # x at 3000 sigma: h = silu(g) * u lands far beyond fp16 in an integer layer, which stores h
    # in fp16.  The call must write MOE_ERR_RANGE to the status word, and the next ordinary call
    # on the same context must be clean and exact.
    L = custom("hrange", T, 256, 256, 4, 2, [[4, 4, 4], [3, 2, 4], [2, 2, 2], [4, 3, 1]])
    layer = hp.gpu_pack(L)
    x = W.device_x(T, L.H) * 3000.0
    Wr, b = W.device_router(L)
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    moe.moe_layer_forward(x, Wr, b, layer, L.k, debug={"status": st})
    torch.cuda.synchronize()
    assert _lib.STATUS[int(st.item())] == "MOE_ERR_RANGE"
    check_layer(L, T)


def test_forward_deterministic_and_empty_batch():
    L = W.layer("tiny")
    layer = hp.gpu_pack(L)
    x = W.device_x(40, L.H)
    Wr, b = W.device_router(L)
    y1 = moe.moe_layer_forward(x, Wr, b, layer, L.k)
    y2 = moe.moe_layer_forward(x, Wr, b, layer, L.k)
    torch.cuda.synchronize()
    assert torch.equal(y1.view(torch.int16), y2.view(torch.int16))
    y0 = moe.moe_layer_forward(x[:0], Wr, b, layer, L.k)
    assert y0.shape == (0, L.H)


@pytest.mark.parametrize("name,T", [("mixtral", 1), ("mixtral", 8), ("tiny", 512)])
def test_forward_replays_from_cuda_graph(name, T):
    """The forward captures into a CUDA graph (no host sync or allocation inside)
    and every replay gives the eager result bit for bit: split-K decode (Mixtral
    T=1, 8) and the tcgen05 path (T=512 of the small layer)."""
    L = W.layer(name)
    layer = hp.gpu_pack_cached(L) if name != "tiny" else hp.gpu_pack(L)
    x = W.device_x(T, L.H)
    Wr, b = W.device_router(L)
    ws = moe.alloc_packed(moe.workspace_bytes(layer, T, L.k))
    y_eager = moe.moe_layer_forward(x, Wr, b, layer, L.k, ws=ws).clone()
    y = torch.empty_like(x)
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        moe.moe_layer_forward(x, Wr, b, layer, L.k, y=y, ws=ws)
    for _ in range(3):
        y.zero_()
        g.replay()
        torch.cuda.synchronize()
        assert torch.equal(y.view(torch.int16), y_eager.view(torch.int16))
    del g


def test_stage_events_record():
    L = W.layer("tiny")
    layer = hp.gpu_pack(L)
    x = W.device_x(16, L.H)
    Wr, b = W.device_router(L)
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(moe.MOE_STAGE_EVENTS)]
    for e in ev:
        e.record()
    moe.moe_layer_forward(x, Wr, b, layer, L.k, stage_events=ev)
    torch.cuda.synchronize()
    times = [ev[i].elapsed_time(ev[i + 1]) for i in range(len(ev) - 1)]
    assert all(t >= 0 for t in times) and ev[0].elapsed_time(ev[-1]) > 0


# ------------------------------------------------------------------ NVFP4 activations (block-scaled FP4 MMA)
@pytest.mark.parametrize("T", [9, 300])
def test_nvfp4_activations_small(T):
    # x and h quantized to NVFP4 (e2m1 + e4m3 per 16 + fp32 row scale): x codes, block scales
    # and row scales bit-exact, outputs within the bound.  T=9 runs the decode GEMV on fp16
    # block values, T=300 the block-scaled FP4 tcgen05 GEMM (chunks of up to 128 rows).
    L = custom("act4", T, 256, 384, 6, 2, [[16, 16, 16]] * 6)
    check_layer(L, T, act=moe.ACT_NVFP4)


@pytest.mark.parametrize("T", [7, 260])
def test_nvfp4_activations_half_stages_odd_tiles(T):
    # H = 384 and F = 640: the FP4 GEMM's last 256-input stage holds one 128-input tile
    # (K % 256 = 128) for both GEMMs, and the down projection has three 128-row tiles (the
    # last item holds one tile).
    L = custom("act4odd", T, 384, 640, 5, 2, [[16, 16, 16]] * 5)
    check_layer(L, T, act=moe.ACT_NVFP4)


def test_nvfp4_activations_down_stage_refeed():
    # the GPU's NVFP4 codes of h (row scale, block scales, codes) fed into the oracle's down
    # stage: output parity of the down GEMM + combine alone; the h codes themselves depend on
    # summation order and are counted (at most 1% may differ)
    from oracle import nvfp4_act as na
    T, k = 300, 2
    L = custom("act4refeed", T, 256, 256, 4, k, [[16, 16, 16]] * 4)
    layer = hp.gpu_pack(L)
    layer = moe.PackedLayer(layer.E, layer.H, layer.F, layer.fmt, layer.packed, moe.ACT_NVFP4)
    g = run_gpu(L, layer, T, act=moe.ACT_NVFP4)
    x_bits = W.x_bf16_bits(T, L.H)
    buf = hp.oracle_pack(L, range(L.E))
    idx = g["topk_idx"].reshape(T, k)
    counts, offsets, perm, inv = orc.permute(idx.astype(np.int32), L.E)
    hq = g["hq"].reshape(T * k, L.F)
    hsb = g["hsb"].reshape(T * k, L.F // 16)
    sh = g["sh"]
    o = np.zeros((T * k, L.H))
    for e in range(L.E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            o[r0:r1] = orc.down(buf, e, na.block_values(hq[r0:r1], hsb[r0:r1]), sh[r0:r1].astype(np.float64))
    w = g["topk_w"].reshape(T, k)
    y_ref = np.zeros((T, L.H))
    for t in range(T):
        for j in range(k):
            y_ref[t] += float(w[t, j]) * o[inv[t * k + j]]
    hp.check_output(g["y"], y_ref)
    xv, xsb, xs = na.quant_rows(gen.bf16_bits_to_f32(x_bits))
    a = na.block_values(xv, xsb)
    n_diff = 0
    for e in range(L.E):
        r0, r1 = offsets[e], offsets[e + 1]
        if r1 > r0:
            ts = perm[r0:r1] // k
            h = orc.gateup(buf, e, a[ts], xs[ts].astype(np.float64))
            hv, _, _ = na.quant_rows(h.astype(np.float32))
            n_diff += int(np.count_nonzero(hv != hq[r0:r1]))
    assert n_diff <= 0.01 * hq.size, f"{n_diff} of {hq.size} h codes differ"


@pytest.mark.parametrize("T", [16, 8192])
def test_forward_nvfp4_layer_nvfp4_activations(T):
    # the 256-expert top-6 NVFP4 layer with NVFP4 activations: decode T=16 (all tokens) and
    # prefill T=8192 (every expert's first and last rows plus 256 seeded tokens)
    L = W.layer("nvfp4")
    r = check_layer(L, T, tokens=strata(halves=False, extra=256) if T > 64 else None, act=moe.ACT_NVFP4)
    print(f"nvfp4 act4 T={T}: near-ties {r['ties']}, err/max {r['err_ratio']:.3g}, tokens compared {r['n_tokens']}")


# ------------------------------------------------------------------ forward, the five layers
def strata(halves=True, extra=0, seed=0):
    """Token sample for a full-size batch, taken from the GPU's own permutation: for every
    expert, every 256-row chunk the tcgen05 GEMM walks, and (halves) each half of a chunk's
    rows (the two CTAs of a pair), the tokens of the first and last row; plus `extra` seeded
    random tokens.  Every expert with rows is compared, at the chunk and CTA-half edges where
    offset or ragged-tail mistakes would show."""
    def pick(perm, counts, k):
        T = len(perm) // k
        rows, off = [], 0
        for c in counts:
            c = int(c)
            for c0 in range(0, c, 256):
                n = min(256, c - c0)
                nmma = min(256, (n + 15) // 16 * 16)
                parts = [(0, min(n, nmma // 2)), (nmma // 2, n)] if halves else [(0, n)]
                for a, b in parts:
                    if b > a:
                        rows += [off + c0 + a, off + c0 + b - 1]
            off += c
        tok = set(int(perm[r]) // k for r in rows)
        if extra:
            tok |= set(np.random.default_rng(seed).choice(T, min(T, extra), replace=False).tolist())
        return np.array(sorted(tok))
    return pick


CONFIG_RUNS = [
    ("mixtral", 1, None), ("mixtral", 8, None), ("mixtral", 64, None),
    ("hotcold", 32, None), ("nvfp4", 16, None), ("large", 64, None),
    ("mixtral", 2048, strata(extra=200)), ("hotcold", 4096, strata(extra=256)),
    ("nvfp4", 8192, strata(extra=256)), ("large", 8192, strata(halves=False, extra=16)),
    ("graded", 32, None), ("graded", 4096, strata(extra=128)),
]


@pytest.mark.parametrize("name,T,tokens", CONFIG_RUNS, ids=[f"{n}-T{t}" for n, t, _ in CONFIG_RUNS])
def test_forward_config(name, T, tokens):
    L = W.layer(name)
    r = check_layer(L, T, tokens=tokens)
    print(f"{name} T={T}: near-ties {r['ties']}, err/max {r['err_ratio']:.3g}, tokens compared {r['n_tokens']}")
