"""The device copy of the seeded generator reproduces the host stream."""
import numpy as np
import pytest

import synth

pytestmark = pytest.mark.gpu
torch = pytest.importorskip("torch")
if not torch.cuda.is_available():
    pytest.skip("needs a CUDA device", allow_module_level=True)


def test_device_normals_match_host():
    for first, n in ((0, 1 << 20), (3, 1001), (12345, 77)):
        h = synth.normal_f32(0, synth.W2, 5, n, 0.0, 0.02, first=first)
        d = synth.normal_f32_device(0, synth.W2, 5, n, 0.0, 0.02, first=first).cpu().numpy()
        same = np.mean(h == d)
        assert same > 0.9999, same
        ulp = np.abs(h.view(np.int32).astype(np.int64) - d.view(np.int32).astype(np.int64))
        assert ulp.max() <= 1
