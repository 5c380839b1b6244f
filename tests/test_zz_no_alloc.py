"""The allocation-free layer entry point, moe_layer_forward_noalloc.

Some callers cannot allocate device memory themselves (a plugin inside a host
application that already owns the GPU's memory through its own pool, or code
that must avoid cudaMalloc/cudaFree because they can synchronise the device).
For them the library keeps a fixed 4 MiB scratch array and this entry point
uses it instead of a caller-provided workspace.  These tests call it through
the C ABI twice in a row and compare each result with moe_layer_forward on the
same inputs: the same kernels run on the same inputs, so the bits must be
equal.  The device check word of that scratch is read back through
moe_noalloc_device_status.  This file is collected last on purpose.
"""

import pytest

import gpu_cases as gc
import moe_inputs as mi
import quantized_expert_ffn_moe_b200 as q

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    torch = pytest.importorskip("torch")
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from quantized_expert_ffn_moe_b200 import build
    from moe_inputs import build as ibuild
    build.build()
    ibuild.build()
    q.load_library()


@pytest.mark.parametrize("shape,T", [(mi.FULL4, 16), (mi.FULL2, 23), (mi.TINY, 40)], ids=["full4", "full2", "tiny"])
def test_noalloc_matches_workspace_entry_point_twice(shape, T):
    torch = gc.torch()
    cfg = gc.cfg_of(shape)
    w = gc.device_layer(shape, 0, 0)
    ws = gc.workspace(cfg, T)
    for batch in (11, 12):                       # two calls in a row, different tokens
        x = gc.to_dev_bits(mi.hidden_states_bf16(T, shape.hidden, 0, batch))
        ref = torch.empty_like(x)
        got = torch.full_like(x, 0x7FC0)         # poison: every element must be rewritten
        q.moe_layer_forward(cfg, w, x, ref, ws)
        q.moe_layer_forward_noalloc(cfg, w, x, got)
        torch.cuda.synchronize()
        assert q.moe_noalloc_device_status() == 0
        assert torch.equal(got, ref)


def test_noalloc_rejects_sizes_beyond_its_scratch():
    torch = gc.torch()
    shape = mi.FULL4
    cfg = gc.cfg_of(shape)
    assert q.moe_workspace_bytes(cfg, 23) <= q.NOALLOC_SCRATCH_BYTES < q.moe_workspace_bytes(cfg, 24)
    w = gc.device_layer(shape, 0, 1)
    x = gc.to_dev_bits(mi.hidden_states_bf16(24, shape.hidden, 0, 3))
    y = torch.full_like(x, 5)
    assert q.moe_layer_forward_noalloc(cfg, w, x, y, check=False) == -3      # MOE_ERR_WORKSPACE
    torch.cuda.synchronize()
    assert bool((y == 5).all())                  # nothing was launched
