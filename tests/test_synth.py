"""The seeded input generator: determinism, stream independence, distributions."""
import numpy as np


def test_normals_deterministic_and_distributed(syn):
    a = syn.normal_f32(0, syn.W1, 3, 200000, 0.0, 0.02)
    b = syn.normal_f32(0, syn.W1, 3, 200000, 0.0, 0.02)
    np.testing.assert_array_equal(a, b)
    assert abs(a.mean()) < 3 * 0.02 / np.sqrt(len(a))
    assert abs(a.std() - 0.02) < 0.02 * 0.01
    # an offset window reproduces the same values
    np.testing.assert_array_equal(syn.normal_f32(0, syn.W1, 3, 1000, 0.0, 0.02, first=5000), a[5000:6000])
    # other tensor / sub / seed -> unrelated values
    c = syn.normal_f32(0, syn.W3, 3, 200000, 0.0, 0.02)
    d = syn.normal_f32(0, syn.W1, 4, 200000, 0.0, 0.02)
    e = syn.normal_f32(1, syn.W1, 3, 200000, 0.0, 0.02)
    for o in (c, d, e):
        assert abs(np.corrcoef(a, o)[0, 1]) < 0.01


def test_bf16_is_rounded_normal(syn):
    import torch
    f = syn.normal_f32(7, syn.X, 0, 10000)
    b = syn.normal_bf16(7, syn.X, 0, 10000)
    ref = torch.from_numpy(f).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(b, ref)


def test_ints_permutation_zipf(syn):
    t = syn.uniform_int(0, syn.TOK, 0, 100000, 0, 129280)
    assert t.min() >= 0 and t.max() < 129280
    assert abs(t.mean() - 129280 / 2) < 129280 * 0.01
    p = syn.permutation(0, syn.ZIPF, 0, 256)
    assert sorted(p) == list(range(256))
    cfg = syn.CONFIGS["prefill"]
    bias = syn.make_bias(cfg)
    assert bias.shape == (256,) and bias.max() == 0.0
    r = 1 + p
    np.testing.assert_allclose(bias, -0.02 * 64 * 1.1 * np.log(r), rtol=1e-6)
