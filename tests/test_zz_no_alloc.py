"""moe_layer_static_ws, the entry point for callers that cannot allocate.

Callers whose device memory belongs to another allocator, latency-critical
decode loops that cannot afford cudaMalloc/cudaFree, and deployments that forbid
allocation after start-up call the layer without handing it a workspace; the
library then uses the scratch array it carries. This checks, through the C ABI,
that two calls in a row give what moe_layer gives with a caller workspace, and
that a call too large for the array is refused before anything is launched.
The file sorts last so a run that stops at the first failure has already run
every other test; it builds its own inputs, so it also passes on its own.
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


@pytest.mark.parametrize("name,T", [("tiny", 4), ("decode", 8)])
def test_static_ws_matches_moe_layer(name, T):
    c = Case(synth.CONFIGS[name].with_T(T))
    d = c.cfg.d
    other = torch.from_numpy(synth.make_x(c.cfg, 0, 1).astype(np.int16)).cuda()
    for x in (c.x_d, other):  # two calls in a row, different inputs
        ref = torch.empty((T, d), dtype=torch.float32, device="cuda")
        got = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        M.moe_layer(c.dims, c.weights, x, c.tok_d, ref, c.ws)
        M.moe_layer_static_ws(c.dims, c.weights, x, c.tok_d, got)
        torch.cuda.synchronize()
        assert M.moe_get_device_error() == 0
        r, g = ref.cpu().numpy(), got.cpu().numpy()
        assert np.all(np.isfinite(g))
        assert np.abs(g - r).max() <= 2e-3 * np.abs(r).max()


def test_static_ws_refuses_oversized_calls():
    dims = M.make_dims(4096, 4096, 2048, 256, 8, d_ff_shared=2048)
    assert M.moe_workspace_size(dims) > M.MOE_STATIC_WS_BYTES
    w = M.make_weights(0x100, 0x100, 0x100, 0x100, 0x100, 0x100, 0x100)
    with pytest.raises(M.MoeError) as ei:
        M.moe_layer_static_ws(dims, w, 0x100, None, 0x100)
    assert ei.value.status == M.MOE_ERR_INVALID_ARG
