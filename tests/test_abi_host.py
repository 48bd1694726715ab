"""Host-side checks of the C ABI (no GPU needed): the library loads, exports
every entry point declared in include/moe.h, sizes its buffers like the
oracle's independent layout, and rejects bad arguments before launching.
Pointers passed here are fake device addresses: validation must return
before anything touches them."""
import ctypes as C
import os
import re

import numpy as np
import pytest

import gen.workloads as W
import mixed_precision_quantized_fp32_b200 as moe
from mixed_precision_quantized_fp32_b200 import _lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
ST = {v: k for k, v in _lib.STATUS.items()}
FAKE = 0x7F0000000000  # 256-byte aligned, never dereferenced


def declared_symbols():
    names = set()
    for fn in os.listdir(os.path.join(ROOT, "include")):
        if fn.endswith(".h"):
            src = open(os.path.join(ROOT, "include", fn)).read()
            names |= set(re.findall(r"MOE_API\s+\w+\s+(\w+)\s*\(", src))
    return names


def test_exports_every_declared_symbol():
    L = _lib.load()
    names = declared_symbols()
    assert {"moe_pack", "moe_layer_forward"} <= names
    for n in names:
        assert hasattr(L, n), n


def test_layout_matches_oracle(orc):
    for name in W.NAMES:
        L = W.layer(name)
        total, co, so = moe.pack_layout(L.E, L.H, L.F, L.fmt)
        oco, oso, ototal = orc.layer_layout(L.E, L.H, L.F, L.fmt)
        assert total == ototal
        np.testing.assert_array_equal(co, oco)
        np.testing.assert_array_equal(so, oso)


def _pack(W_ptr, e0, ne, E, H, F, fmt, out, out_bytes, want_total=True):
    total = C.c_uint64(0)
    f = None if fmt is None else np.ascontiguousarray(fmt, np.uint8).ravel()
    rc = _lib.load().moe_pack(W_ptr, e0, ne, E, H, F, None if f is None else f.ctypes.data, out, out_bytes,
                              C.byref(total) if want_total else None, None, None, None)
    return _lib.STATUS[rc], total.value


def test_pack_argument_errors():
    fmt = np.full((4, 3), 4, np.uint8)
    total = moe.pack_layout(4, 256, 256, fmt)[0]
    assert _pack(None, 0, 0, 4, 256, 256, fmt, None, 0)[0] == "MOE_OK"
    assert _pack(None, 0, 0, 4, 256, 256, None, None, 0)[0] == "MOE_ERR_ARG"
    assert _pack(None, 0, 0, 4, 200, 256, fmt, None, 0)[0] == "MOE_ERR_SHAPE"
    assert _pack(None, 0, 0, 4, 256, 0, fmt, None, 0)[0] == "MOE_ERR_SHAPE"
    assert _pack(None, 0, 0, 257, 256, 256, np.full((257, 3), 4), None, 0)[0] == "MOE_ERR_SHAPE"
    bad = fmt.copy()
    bad[2, 1] = 5
    assert _pack(None, 0, 0, 4, 256, 256, bad, None, 0)[0] == "MOE_ERR_FORMAT"
    bad[2, 1] = 0
    assert _pack(None, 0, 0, 4, 256, 256, bad, None, 0)[0] == "MOE_ERR_FORMAT"
    one = fmt.copy()
    one[1] = 1                                            # 1-bit codes: N*K/8 bytes, fp16 scales
    st, t1 = _pack(None, 0, 0, 4, 256, 256, one, None, 0)[:2]
    assert st == "MOE_OK" and t1 == moe.pack_layout(4, 256, 256, one)[0] < total
    assert _pack(None, 0, 0, 4, 256, 256, fmt, None, 0, want_total=False)[0] == "MOE_ERR_ARG"
    assert _pack(None, 0, 1, 4, 256, 256, fmt, FAKE, total)[0] == "MOE_ERR_ARG"   # W null
    assert _pack(FAKE, 3, 2, 4, 256, 256, fmt, FAKE, total)[0] == "MOE_ERR_ARG"   # e0+ne > E
    assert _pack(FAKE, -1, 1, 4, 256, 256, fmt, FAKE, total)[0] == "MOE_ERR_ARG"
    assert _pack(FAKE, 0, 1, 4, 256, 256, fmt, FAKE + 16, total)[0] == "MOE_ERR_ALIGN"
    assert _pack(FAKE + 4, 0, 1, 4, 256, 256, fmt, FAKE, total)[0] == "MOE_ERR_ALIGN"
    assert _pack(FAKE, 0, 1, 4, 256, 256, fmt, FAKE, total - 1)[0] == "MOE_ERR_WORKSPACE"


def _fwd(T, k, E=8, H=256, F=512, fmt=None, x=FAKE, rw=FAKE, y=FAKE, packed=FAKE, packed_bytes=None,
         ws=FAKE, ws_bytes=1 << 40, query=False):
    fmt = np.full((E, 3), 4, np.uint8) if fmt is None else np.asarray(fmt, np.uint8)
    f = np.ascontiguousarray(fmt).ravel()
    if packed_bytes is None:
        packed_bytes = moe.pack_layout(E, H, F, f)[0] if (E <= 256 and H % 128 == 0 and F % 128 == 0
                                                          and set(f) <= {1, 2, 3, 4, 16}) else 1 << 40
    w = _lib.MoeWeights(E, H, F, f.ctypes.data, packed, packed_bytes)
    need = C.c_uint64(0)
    rc = _lib.load().moe_layer_forward(x, T, rw, None, C.byref(w), k, y, None if query else ws, ws_bytes,
                                       C.byref(need), None, None)
    return _lib.STATUS[rc], need.value


def test_forward_argument_errors():
    st, need = _fwd(16, 2, query=True)
    assert st == "MOE_OK" and need > 0
    st, need64 = _fwd(64, 2, query=True)
    assert need64 > need
    assert _fwd(16, 0)[0] == "MOE_ERR_SHAPE"
    assert _fwd(16, 9, E=16)[0] == "MOE_ERR_SHAPE"
    assert _fwd(16, 5, E=4)[0] == "MOE_ERR_SHAPE"
    assert _fwd(-1, 2)[0] == "MOE_ERR_SHAPE"
    assert _fwd(16, 2, H=200)[0] == "MOE_ERR_SHAPE"
    mixed = np.full((8, 3), 16, np.uint8)
    mixed[3, 2] = 4
    assert _fwd(16, 2, fmt=mixed)[0] == "MOE_ERR_FORMAT"
    assert _fwd(16, 2, fmt=np.full((8, 3), 7))[0] == "MOE_ERR_FORMAT"
    mixed1 = np.full((8, 3), 16, np.uint8)
    mixed1[5, 0] = 1                                      # the 1-bit code is an integer format too
    assert _fwd(16, 2, fmt=mixed1)[0] == "MOE_ERR_FORMAT"
    graded = np.tile(np.array([[4, 2, 1], [1, 1, 1]], np.uint8), (4, 1))
    st, need_g = _fwd(16, 2, fmt=graded, query=True)       # 1-bit matrices are accepted
    assert st == "MOE_OK" and need_g > 0
    assert _fwd(0, 2)[0] == "MOE_OK"                      # empty batch: nothing to do
    assert _fwd(16, 2, x=None)[0] == "MOE_ERR_ARG"
    assert _fwd(16, 2, y=None)[0] == "MOE_ERR_ARG"
    assert _fwd(16, 2, rw=None)[0] == "MOE_ERR_ARG"
    assert _fwd(16, 2, packed=None)[0] == "MOE_ERR_ARG"
    assert _fwd(16, 2, x=FAKE + 8)[0] == "MOE_ERR_ALIGN"
    assert _fwd(16, 2, packed=FAKE + 128)[0] == "MOE_ERR_ALIGN"
    assert _fwd(16, 2, ws=FAKE + 64)[0] == "MOE_ERR_ALIGN"
    assert _fwd(16, 2, ws_bytes=need - 1)[0] == "MOE_ERR_WORKSPACE"
    total = moe.pack_layout(8, 256, 512, np.full((8, 3), 4))[0]
    assert _fwd(16, 2, packed_bytes=total - 1)[0] == "MOE_ERR_WORKSPACE"


def test_valid_call_without_gpu_fails_cleanly():
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st, _ = _fwd(16, 2)
    assert st in ("MOE_ERR_CUDA", "MOE_ERR_UNSUPPORTED_DEVICE")


def test_generator_libraries_load_and_export():
    import ctypes
    import gen
    from gen import workloads
    L = workloads._dev_lib()
    for name in ("moegen_fill_f32", "moegen_fill_bf16"):
        assert hasattr(L, name)
    assert hasattr(gen._host_lib(), "moegen_host_fill_f32")
    assert isinstance(L, ctypes.CDLL)


def test_ctypes_structs_match_the_header(tmp_path):
    # compile a probe against include/moe.h and compare every struct the binding mirrors:
    # size and the offset of each field
    structs = {"moe_debug": _lib.MoeDebug, "moe_weights": _lib.MoeWeights}
    lines = ["#include <stdio.h>", "#include <stddef.h>", '#include "moe.h"', "int main(void) {"]
    for cname, py in structs.items():
        lines.append(f'  printf("{cname} size %zu\\n", sizeof({cname}));')
        for fname, _ in py._fields_:
            lines.append(f'  printf("{cname} {fname} %zu\\n", offsetof({cname}, {fname}));')
    lines += ["  return 0;", "}"]
    src = tmp_path / "probe.c"
    src.write_text("\n".join(lines) + "\n")
    exe = tmp_path / "probe"
    cuda_inc = os.environ.get("CUDA_HOME", "/usr/local/cuda") + "/include"
    import subprocess
    subprocess.run(["gcc", "-I", os.path.join(ROOT, "include"), "-I", cuda_inc, str(src), "-o", str(exe)], check=True)
    got = {}
    for line in subprocess.run([str(exe)], check=True, capture_output=True, text=True).stdout.splitlines():
        cname, field, value = line.split()
        got[(cname, field)] = int(value)
    for cname, py in structs.items():
        assert got[(cname, "size")] == C.sizeof(py), cname
        for fname, _ in py._fields_:
            assert got[(cname, fname)] == getattr(py, fname).offset, (cname, fname)


def test_outlier_flag_layout_and_errors():
    # MOE_FMT_OUTLIERS adds a section after the expert sections: 256-aligned start,
    # a 3*256-entry u64 table and 4*(64+65536) bytes of scratch, then one side list
    # (u32 row_ptr[N+1] + u32 entry[floor(N*K*5/10000)]) per flagged matrix, 256-aligned
    E, H, F = 4, 256, 384
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    base = np.array([[4, 3, 2], [1, 2, 4], [3, 4, 1], [2, 1, 3]], np.uint8)
    flagged = base.copy()
    flagged[0, :] |= moe.FMT_OUTLIERS
    flagged[2, 2] |= moe.FMT_OUTLIERS
    t_base, co, so = moe.pack_layout(E, H, F, base)
    t_out, co2, so2 = moe.pack_layout(E, H, F, flagged)
    np.testing.assert_array_equal(co, co2)  # expert sections do not move
    np.testing.assert_array_equal(so, so2)
    pos = up(up(t_base) + 8 * 768 + 4 * (64 + 65536))
    for N, K in [(F, H), (F, H), (H, F), (H, F)]:  # gate, up, down of expert 0; down of expert 2
        pos = up(pos + 4 * (N + 1 + N * K * 5 // 10000))
    assert t_out == pos
    for bad_flag in (0x40, 0x20):
        bad = base.copy()
        bad[1, 1] |= bad_flag
        assert _pack(None, 0, 0, E, H, F, bad, None, 0)[0] == "MOE_ERR_FORMAT"
    # a buffer sized for the unflagged layout is too small for the flagged one
    assert _fwd(16, 2, E=E, H=H, F=F, fmt=flagged, packed_bytes=t_base)[0] == "MOE_ERR_WORKSPACE"
    st, need = _fwd(16, 2, E=E, H=H, F=F, fmt=flagged, query=True)
    assert st == "MOE_OK" and need > 0
    # side lists are read with FP8 activations only: NVFP4 activations are rejected
    fp4 = np.full((E, 3), 16, np.uint8)
    fp4[1, 0] |= moe.FMT_OUTLIERS
    f = np.ascontiguousarray(fp4).ravel()
    for act, want in ((moe.ACT_FP8, "MOE_OK"), (moe.ACT_NVFP4, "MOE_ERR_FORMAT")):
        w = _lib.MoeWeights(E, H, F, f.ctypes.data, FAKE, moe.pack_layout(E, H, F, f)[0], act)
        need = C.c_uint64(0)
        rc = _lib.load().moe_layer_forward(FAKE, 16, FAKE, None, C.byref(w), 2, FAKE, None, 0, C.byref(need),
                                           None, None)
        assert _lib.STATUS[rc] == want


def test_outlier_layout_random_shapes():
    # the outlier section's size for seeded random shapes and flag patterns, against the
    # layout rule restated here (section after the expert sections, 256-byte aligned;
    # 768-entry u64 table + 4*(64+65536) bytes of scratch; per flagged matrix, in
    # (expert, projection) order, 4*(N+1+floor(N*K*5/10000)) bytes, 256-byte aligned)
    rng = np.random.default_rng(11)
    up = lambda v: (v + 255) // 256 * 256  # noqa: E731
    for _ in range(25):
        E = int(rng.integers(1, 33))
        H, F = 128 * int(rng.integers(1, 17)), 128 * int(rng.integers(1, 17))
        base = rng.choice([1, 2, 3, 4], size=(E, 3)).astype(np.uint8) if rng.random() < 0.7 \
            else np.full((E, 3), 16, np.uint8)
        flags = (rng.random((E, 3)) < 0.4).astype(np.uint8) * moe.FMT_OUTLIERS
        fmt = (base | flags).astype(np.uint8)
        t_base = moe.pack_layout(E, H, F, base)[0]
        t_out = moe.pack_layout(E, H, F, fmt)[0]
        if not flags.any():
            assert t_out == t_base
            continue
        pos = up(up(t_base) + 8 * 768 + 4 * (64 + 65536))
        for e in range(E):
            for p in range(3):
                if flags[e, p]:
                    N, K = (F, H) if p < 2 else (H, F)
                    pos = up(pos + 4 * (N + 1 + N * K * 5 // 10000))
        assert t_out == pos, (E, H, F)
