"""The allocation-free forward (moe_layer_forward_noalloc) against the regular
moe_layer_forward on the same inputs.

Some callers cannot allocate device memory (code inside a captured CUDA graph or
an allocator callback, embedded runtimes without cudaMalloc, pools that must
not grow); they use the variant whose workspace is a fixed 32 MiB array inside
the library.  This file is collected last on purpose so that a run stopping at
its first failure has already run every other test; it passes both alone and
after the others.
"""
import numpy as np
import pytest

import gen.workloads as W
from tests import helpers as hp

pytestmark = pytest.mark.gpu

torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("no CUDA device", allow_module_level=True)

import mixed_precision_quantized_fp32_b200 as moe  # noqa: E402


def _same_bits(a, b):
    return torch.equal(a.view(torch.int16), b.view(torch.int16))


@pytest.mark.parametrize("name,T", [("tiny", 16), ("mixtral", 8), ("nvfp4", 16)])
def test_noalloc_matches_regular_forward_twice(name, T):
    # Same kernels on the same inputs: the result must be identical bit for bit (which is
    # also within the output tolerance of the other tests).  A second, smaller batch then
    # runs on an array still holding the larger call's contents.
    L = W.layer(name)
    layer = hp.gpu_pack(L)
    Wr, b = W.device_router(L)
    for TT in (T, T, max(1, T // 2 - 1)):
        x = W.device_x(TT, L.H)
        y_ref = moe.moe_layer_forward(x, Wr, b, layer, L.k)
        torch.cuda.synchronize()
        ref = y_ref.float().cpu().numpy()
        y = torch.full_like(x, float("nan"))
        moe.moe_layer_forward_noalloc(x, Wr, b, layer, L.k, y)
        torch.cuda.synchronize()
        got = y.float().cpu().numpy()
        assert np.all(np.isfinite(got))
        assert np.abs(got - ref).max() <= hp.TOL * np.abs(ref).max()
        assert _same_bits(y, y_ref), f"{name} T={TT}: noalloc output differs from the regular forward"


def test_noalloc_rejects_batches_beyond_the_array():
    L = W.layer("tiny")
    layer = hp.gpu_pack(L)
    T = 8192  # workspace of ~37 MiB > 32 MiB
    assert moe.workspace_bytes(layer, T, L.k) > (32 << 20)
    x = W.device_x(T, L.H)
    Wr, b = W.device_router(L)
    y = torch.zeros_like(x)
    with pytest.raises(moe.MoeError) as ei:
        moe.moe_layer_forward_noalloc(x, Wr, b, layer, L.k, y)
    assert ei.value.name == "MOE_ERR_WORKSPACE"
    torch.cuda.synchronize()
    assert torch.count_nonzero(y) == 0  # nothing ran
