"""moe_layer_static_ws, the entry point for callers that cannot allocate.

Callers whose device memory belongs to another allocator, latency-critical
decode loops that cannot afford cudaMalloc/cudaFree, and deployments that forbid
allocation after start-up call the layer without handing it a workspace; the
library then uses the scratch array it carries. This checks, through the C ABI,
that calls in a row give bit for bit what moe_layer gives with a caller
workspace (the same kernels run on the same inputs) — including a sequence
whose batch shrinks on the one array, so that what an earlier, larger call left
there is never read — and that a call too large for the array is refused before
anything is launched. The file sorts last so a run that stops at the first
failure has already run every other test; it builds its own inputs, so it also
passes on its own.
"""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)

import routed_expert_ffn_05_b200 as M  # noqa: E402
from harness import Case  # noqa: E402


def _both(c, x, T):
    d = c.cfg.d
    ref = torch.empty((T, d), dtype=torch.float32, device="cuda")
    got = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    M.moe_layer(c.dims, c.weights, x, c.tok_d, ref, c.ws)
    M.moe_layer_static_ws(c.dims, c.weights, x, c.tok_d, got)
    torch.cuda.synchronize()
    assert M.moe_get_device_error() == 0
    r, g = ref.cpu().numpy(), got.cpu().numpy()
    assert np.all(np.isfinite(g))
    np.testing.assert_array_equal(g.view(np.uint32), r.view(np.uint32))


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode", 8)])
def test_static_ws_matches_moe_layer(name, T):
    c = Case(synth.CONFIGS[name].with_T(T))
    other = torch.from_numpy(synth.make_x(c.cfg, 0, 1).astype(np.int16)).cuda()
    for x in (c.x_d, other):  # two calls in a row, different inputs
        _both(c, x, T)


def test_static_ws_shrinking_batches():
    """Decode T = 8, then 2, then 1 on the one array: each smaller call finds
    the larger call's leftovers in the array and must not read them."""
    for T in (8, 2, 1):
        c = Case(synth.CONFIGS["decode"].with_T(T))
        _both(c, c.x_d, T)


def test_static_ws_w4a8():
    """MXFP8 activations at the decode dims (the tensor-core path) from the
    built-in array, after the decode calls above left their contents there."""
    c = Case(synth.CONFIGS["prefill"].with_T(24))
    _both(c, c.x_d, 24)


def test_static_ws_refuses_oversized_calls():
    dims = M.make_dims(4096, 4096, 2048, 256, 8, d_ff_shared=2048)
    assert M.moe_workspace_size(dims) > M.MOE_STATIC_WS_BYTES
    w = M.make_weights(0x100, 0x100, 0x100, 0x100, 0x100, 0x100, 0x100)
    with pytest.raises(M.MoeError) as ei:
        M.moe_layer_static_ws(dims, w, 0x100, None, 0x100)
    assert ei.value.status == M.MOE_ERR_INVALID_ARG
