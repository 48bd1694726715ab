"""Seeded, counter-based synthetic input generator shared by the tests, the bench
and the oracle's callers.

This module holds no arithmetic of the MoE method itself: it only turns
(seed, tensor id, element index) into numbers.  The same definition is
implemented for the GPU in ``gen/gen_device.cu`` (built into
``gen/libmoegen.so``); the two are bit-identical, which a GPU test checks.

Definition (element ``i`` of tensor ``tid``, seed ``seed``):

* ``key = splitmix64(seed XOR (tid << 40))``
* ``r0 = splitmix64(key XOR 2i)``, ``r1 = splitmix64(key XOR (2i+1))``.
  splitmix64 is the published mixer of Steele, Lea and Flood,
  "Fast splittable pseudorandom number generators" (OOPSLA 2014), in the
  constant set popularised by Vigna's SplitMix64.
* Twelve 10-bit uniforms: bits [10j, 10j+10) of r0 and of r1 for j = 0..5.
* ``S`` = their sum; ``z = (S - 6138) / 1024`` (Irwin-Hall, mean 0, std ~1;
  exact in fp32 because ``|S - 6138| < 2**13``).
* fp32 values: ``float32(z) * float32(sigma)`` (one IEEE multiply).
* bf16 values: bf16 round-to-nearest-even of ``float32(z) * float32(sigma)``.

Tensor ids used by the workloads: activations x = 1, router weights = 2,
hot/cold permutation keys = 4, expert ``e`` projection ``p`` (gate 0, up 1,
down 2) = 16 + 3e + p.
"""
from __future__ import annotations

import numpy as np

TID_X = 1
TID_ROUTER_W = 2
TID_PERM = 4


def tid_expert(e: int, p: int) -> int:
    """Tensor id of projection p (0 gate, 1 up, 2 down) of expert e."""
    return 16 + 3 * e + p


_C0 = np.uint64(0x9E3779B97F4A7C15)
_C1 = np.uint64(0xBF58476D1CE4E5B9)
_C2 = np.uint64(0x94D049BB133111EB)


def splitmix64(x: np.ndarray) -> np.ndarray:
    """splitmix64 finaliser on a uint64 array (wrapping arithmetic)."""
    with np.errstate(over="ignore"):
        z = x + _C0
        z = (z ^ (z >> np.uint64(30))) * _C1
        z = (z ^ (z >> np.uint64(27))) * _C2
        return z ^ (z >> np.uint64(31))


def raw128(seed: int, tid: int, idx: np.ndarray) -> tuple[np.ndarray, np.ndarray]:
    idx = np.asarray(idx, dtype=np.uint64)
    base = splitmix64(np.array([np.uint64(seed) ^ (np.uint64(tid) << np.uint64(40))], np.uint64))[0]
    two = np.uint64(2)
    return splitmix64(base ^ (two * idx)), splitmix64(base ^ (two * idx + np.uint64(1)))


def irwin_hall_sum(seed: int, tid: int, idx: np.ndarray) -> np.ndarray:
    """Integer sum S of the twelve 10-bit uniforms (int64)."""
    r0, r1 = raw128(seed, tid, idx)
    m = np.uint64(1023)
    s = np.zeros(r0.shape, dtype=np.uint64)
    for j in range(6):
        sh = np.uint64(10 * j)
        s += (r0 >> sh) & m
        s += (r1 >> sh) & m
    return s.astype(np.int64)


def normal_f32(seed: int, tid: int, start: int, count: int, sigma: float = 1.0,
               idx: np.ndarray | None = None) -> np.ndarray:
    """fp32 values float32(z) * float32(sigma) for elements [start, start+count)
    (or for the explicit element indices ``idx``)."""
    if idx is None:
        idx = np.arange(start, start + count, dtype=np.uint64)
    z = (irwin_hall_sum(seed, tid, idx) - 6138).astype(np.float32) / np.float32(1024.0)
    return z * np.float32(sigma)


def f32_to_bf16_bits(a: np.ndarray) -> np.ndarray:
    """bf16 round-to-nearest-even of finite fp32 values, as uint16 bit patterns."""
    u = np.ascontiguousarray(a, dtype=np.float32).view(np.uint32).astype(np.uint64)
    bias = np.uint64(0x7FFF) + ((u >> np.uint64(16)) & np.uint64(1))
    return ((u + bias) >> np.uint64(16)).astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.asarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


def normal_bf16_bits(seed: int, tid: int, start: int, count: int, sigma: float = 1.0,
                     idx: np.ndarray | None = None) -> np.ndarray:
    return f32_to_bf16_bits(normal_f32(seed, tid, start, count, sigma, idx))


_host = None


def _host_lib():
    """ctypes handle of gen/libmoegen_host.so (built on first use)."""
    global _host
    if _host is None:
        import ctypes as C
        import os
        import subprocess
        here = os.path.dirname(os.path.abspath(__file__))
        lib = os.path.join(here, "libmoegen_host.so")
        src = os.path.join(here, "gen_host.c")
        if not os.path.exists(lib) or os.path.getmtime(lib) < os.path.getmtime(src):
            subprocess.run(["gcc", "-std=c11", "-O2", "-fopenmp", "-fPIC", "-shared", "-ffp-contract=off",
                            "-fvisibility=hidden", src, "-o", lib + ".tmp"], check=True)
            os.replace(lib + ".tmp", lib)
        L = C.CDLL(lib)
        L.moegen_host_fill_f32.restype = None
        L.moegen_host_fill_f32.argtypes = [C.c_void_p, C.c_uint64, C.c_uint64, C.c_uint64, C.c_uint64,
                                           C.c_float]
        _host = L
    return _host


def fill_f32(seed: int, tid: int, count: int, sigma: float = 1.0, start: int = 0,
             out: np.ndarray | None = None) -> np.ndarray:
    """Same values as normal_f32, filled by the multi-threaded C twin."""
    import ctypes as C
    if out is None:
        out = np.empty(count, np.float32)
    assert out.dtype == np.float32 and out.flags["C_CONTIGUOUS"] and out.size >= count
    _host_lib().moegen_host_fill_f32(out.ctypes.data_as(C.c_void_p), seed, tid, start, count, sigma)
    return out


def expert_weights_f32(seed: int, e0: int, ne: int, H: int, F: int,
                       sigma: float = 0.02) -> np.ndarray:
    """fp32 expert weights [ne][3][N*K] in the order gate [F,H], up [F,H], down [H,F]
    (row-major, N output rows by K inputs)."""
    out = np.empty((ne, 3, H * F), dtype=np.float32)
    for i in range(ne):
        for p in range(3):
            fill_f32(seed, tid_expert(e0 + i, p), H * F, sigma, out=out[i, p])
    return out


def permutation(seed: int, tid: int, n: int) -> np.ndarray:
    """Seeded permutation of range(n): argsort of splitmix64 keys (stable on ties)."""
    key = splitmix64(np.array([np.uint64(seed) ^ (np.uint64(tid) << np.uint64(40))], np.uint64))[0]
    keys = splitmix64(key ^ np.arange(n, dtype=np.uint64))
    return np.argsort(keys, kind="stable").astype(np.int64)
