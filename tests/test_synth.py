"""The seeded input generator: determinism and bf16 rounding (CPU only)."""
import numpy as np
import torch

from binary_weight_gemm_b200 import synth


def test_bf16_round_matches_torch_rne():
    rng = np.random.default_rng(0)
    x = np.concatenate([rng.standard_normal(10000).astype(np.float32) * 37,
                        np.array([0.0, -0.0, 1.0, -1.0, 1e-40, 3.0e38], dtype=np.float32)])
    bits, vals = synth.bf16_round(x)
    t = torch.from_numpy(x).to(torch.bfloat16)
    assert np.array_equal(bits, t.view(torch.int16).numpy().view(np.uint16))
    assert np.array_equal(vals, t.float().numpy())


def test_generators_are_deterministic():
    a1 = synth.activations(1, 4, 64, outliers=True)[0]
    a2 = synth.activations(1, 4, 64, outliers=True)[0]
    assert np.array_equal(a1, a2)
    assert np.array_equal(synth.weights(2, 8, 32), synth.weights(2, 8, 32))
    assert not np.array_equal(synth.weights(2, 8, 32), synth.weights(3, 8, 32))


def test_outlier_channels_scaled():
    K = 4096
    ch = synth.outlier_channels(K)
    assert len(ch) == 6 and len(set(ch.tolist())) == 6
    _, x = synth.activations(4, 64, K, outliers=True)
    _, x0 = synth.activations(4, 64, K, outliers=False)
    ratio = np.abs(x[:, ch]).mean() / np.abs(x0[:, ch]).mean()
    assert 55 < ratio < 65


def test_weight_statistics():
    W = synth.weights(1, 512, 512)
    assert abs(W.std() - 0.02) < 5e-4
    f = synth.dbf_factors(3, 64, 32, 96)
    assert set(np.unique(f["S_A"]).tolist()) == {-1, 1}
    assert (f["m"] > 1e-3 - 1e-9).all()
