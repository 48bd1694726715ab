"""Python binding of the C ABI: marshals torch tensors (device memory, streams)
into ``moe_pack`` / ``moe_layer_forward``.  Every step of the layer runs in the
CUDA library; nothing here computes.
"""
from __future__ import annotations

import ctypes as C
from dataclasses import dataclass

import numpy as np
import torch

from . import _lib
from ._lib import MoeDebug, MoeError, MoeWeights, check

FMT_INT1, FMT_INT2, FMT_INT3, FMT_INT4, FMT_NVFP4 = 1, 2, 3, 4, 16
FMT_OUTLIERS = 0x80  # or-ed into a format code: the matrix keeps its top 0.05% |w| in an fp16 side list


def _ptr(t: torch.Tensor | None) -> int | None:
    if t is None:
        return None
    return t.data_ptr()


def _stream(stream: torch.cuda.Stream | None) -> int | None:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _fmt_array(fmt, E: int) -> np.ndarray:
    a = np.ascontiguousarray(np.asarray(fmt, dtype=np.uint8).reshape(-1))
    if a.size != 3 * E:
        raise ValueError(f"fmt must have E*3 = {3 * E} entries, got {a.size}")
    return a


def pack_layout(E: int, H: int, F: int, fmt) -> tuple[int, np.ndarray, np.ndarray]:
    """Size of the packed layer buffer and the section offsets (host-only query)."""
    f = _fmt_array(fmt, E)
    total = C.c_uint64(0)
    co = np.zeros(3 * E, np.uint64)
    so = np.zeros(3 * E, np.uint64)
    rc = _lib.load().moe_pack(None, 0, 0, E, H, F, f.ctypes.data, None, 0, C.byref(total),
                              co.ctypes.data, so.ctypes.data, None)
    check("moe_pack(size query)", rc)
    return int(total.value), co, so


def moe_pack(W: torch.Tensor, e0: int, E: int, H: int, F: int, fmt, out: torch.Tensor,
             stream: torch.cuda.Stream | None = None) -> None:
    """Quantize experts [e0, e0+W.shape[0]) (W: cuda fp32 [ne, 3, H*F]) into ``out``
    (cuda uint8, the whole layer buffer)."""
    f = _fmt_array(fmt, E)
    if W.dtype != torch.float32 or not W.is_cuda or not W.is_contiguous():
        raise ValueError("W must be a contiguous cuda float32 tensor [ne, 3, H*F]")
    if out.dtype != torch.uint8 or not out.is_cuda:
        raise ValueError("out must be a cuda uint8 tensor")
    total = C.c_uint64(0)
    rc = _lib.load().moe_pack(_ptr(W), e0, W.shape[0], E, H, F, f.ctypes.data, _ptr(out), out.numel(),
                              C.byref(total), None, None, _stream(stream))
    check("moe_pack", rc)


def alloc_packed(nbytes: int, device=None) -> torch.Tensor:
    """A device byte buffer whose start is 256-byte aligned."""
    buf = torch.empty(nbytes + 256, dtype=torch.uint8, device=device or "cuda")
    off = (-buf.data_ptr()) % 256
    return buf[off:off + nbytes]


@dataclass
class PackedLayer:
    E: int
    H: int
    F: int
    fmt: np.ndarray       # host uint8 [E*3]
    packed: torch.Tensor  # cuda uint8, 256-byte aligned
    act: int = 0          # NVFP4 layers: activation format (ACT_FP8 or ACT_NVFP4)

    def weights_struct(self) -> MoeWeights:
        return MoeWeights(self.E, self.H, self.F, self.fmt.ctypes.data, self.packed.data_ptr(),
                          self.packed.numel(), self.act)


def workspace_bytes(layer: PackedLayer, T: int, k: int) -> int:
    w = layer.weights_struct()
    need = C.c_uint64(0)
    rc = _lib.load().moe_layer_forward(None, T, None, None, C.byref(w), k, None, None, 0, C.byref(need),
                                       None, None)
    check("moe_layer_forward(workspace query)", rc)
    return int(need.value)


DEBUG_FIELDS = ("topk_idx", "topk_w", "perm", "inv", "counts", "xq", "sx", "hq", "sh", "status", "trace", "xsb",
                "hsb")
DEBUG_INTS = ("test_withhold", "wait_cycles")  # plain integers, see moe_debug in moe.h


def moe_layer_forward(x: torch.Tensor, router_w: torch.Tensor, router_b: torch.Tensor | None,
                      layer: PackedLayer, k: int, y: torch.Tensor | None = None,
                      ws: torch.Tensor | None = None, debug: dict | None = None,
                      stage_events: list | None = None,
                      stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """y = MoE(x) for x cuda bf16 [T, H].  ``debug`` maps names in DEBUG_FIELDS to
    preallocated cuda tensors; ``stage_events`` is a list of MOE_STAGE_EVENTS
    torch.cuda.Event objects recorded between the stages."""
    T = x.shape[0]
    if y is None:
        y = torch.empty_like(x)
    w = layer.weights_struct()
    if ws is None:
        ws = alloc_packed(max(workspace_bytes(layer, T, k), 256), x.device)
    dbg = None
    ev_arr = None
    if debug or stage_events:
        dbg = MoeDebug()
        for name, t in (debug or {}).items():
            if name in DEBUG_INTS:
                setattr(dbg, name, int(t))
                continue
            if name not in DEBUG_FIELDS:
                raise KeyError(name)
            setattr(dbg, name, _ptr(t))
        if stage_events:
            if len(stage_events) != _lib.MOE_STAGE_EVENTS:
                raise ValueError("need MOE_STAGE_EVENTS events")
            ev_arr = (C.c_void_p * _lib.MOE_STAGE_EVENTS)(*[e.cuda_event for e in stage_events])
            dbg.stage_events = C.cast(ev_arr, C.c_void_p)
    rc = _lib.load().moe_layer_forward(_ptr(x), T, _ptr(router_w), _ptr(router_b), C.byref(w), k, _ptr(y),
                                       _ptr(ws), ws.numel(), None,
                                       C.byref(dbg) if dbg is not None else None, _stream(stream))
    check("moe_layer_forward", rc)
    return y


def moe_layer_forward_noalloc(x: torch.Tensor, router_w: torch.Tensor, router_b: torch.Tensor | None,
                              layer: PackedLayer, k: int, y: torch.Tensor,
                              stream: torch.cuda.Stream | None = None) -> torch.Tensor:
    """y = MoE(x) with the workspace in the library's fixed device array (for callers
    that cannot allocate device memory; batches whose workspace exceeds the array
    raise MoeError MOE_ERR_WORKSPACE).  y must be preallocated: this call makes no
    allocation of its own.  Calls that overlap on the GPU share the array and race."""
    w = layer.weights_struct()
    rc = _lib.load().moe_layer_forward_noalloc(_ptr(x), x.shape[0], _ptr(router_w), _ptr(router_b), C.byref(w), k,
                                               _ptr(y), None, _stream(stream))
    check("moe_layer_forward_noalloc", rc)
    return y


__all__ = ["FMT_INT2", "FMT_INT3", "FMT_INT4", "FMT_NVFP4", "MoeError", "PackedLayer", "alloc_packed",
           "moe_layer_forward", "moe_layer_forward_noalloc", "moe_pack", "pack_layout", "workspace_bytes"]
