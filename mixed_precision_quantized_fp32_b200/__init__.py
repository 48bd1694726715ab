"""B200 (sm_100a) quantized Mixture-of-Experts FFN layer.

The layer runs in the CUDA library ``libmoe_b200.so`` (C ABI in
``include/moe.h``); this package is its thin Python binding.  Importing it
fails loudly if the library has not been built.
"""
from ._lib import ACT_FP8, ACT_NVFP4, MOE_STAGE_EVENTS, MoeError, load as _load
from .api import (FMT_INT1, FMT_INT2, FMT_INT3, FMT_INT4, FMT_NVFP4, FMT_OUTLIERS, DEBUG_FIELDS, PackedLayer, alloc_packed,
                  moe_layer_forward, moe_layer_forward_noalloc, moe_pack, pack_layout, workspace_bytes)

_load()

__all__ = ["ACT_FP8", "ACT_NVFP4", "FMT_INT1", "FMT_INT2", "FMT_INT3", "FMT_INT4", "FMT_NVFP4", "FMT_OUTLIERS",
           "DEBUG_FIELDS", "MOE_STAGE_EVENTS", "MoeError",
           "PackedLayer", "alloc_packed", "moe_layer_forward", "moe_layer_forward_noalloc", "moe_pack", "pack_layout", "workspace_bytes"]
