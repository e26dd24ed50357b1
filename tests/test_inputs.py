"""The seeded input generator: determinism, block independence, recipe shape."""
import numpy as np
import torch

from linear_rnn_sequence_wkv7_b200 import inputs


def test_bf16_rounding_matches_torch():
    x = np.random.default_rng(0).standard_normal(100000).astype(np.float32) * 3.0
    x[:4] = [1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0]   # ties
    ours = inputs.f32_to_bf16_bits(x)
    ref = torch.from_numpy(x).to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)
    np.testing.assert_array_equal(ours, ref)
    back = inputs.bf16_bits_to_f32(ours)
    np.testing.assert_array_equal(back, torch.from_numpy(x).to(torch.bfloat16).float().numpy())


def test_deterministic_and_thread_independent():
    a = inputs.gen_sequence(2, 300, 3, 64, seed=5, dtype="bf16", s0_std=0.1, threads=1)
    b = inputs.gen_sequence(2, 300, 3, 64, seed=5, dtype="bf16", s0_std=0.1, threads=4)
    for n in inputs.INPUT_NAMES + ("s0",):
        np.testing.assert_array_equal(a[n], b[n])
    c = inputs.gen_sequence(2, 300, 3, 64, seed=6, dtype="bf16")
    assert not np.array_equal(a["r"], c["r"])


def test_recipe_ranges():
    d = inputs.gen_sequence(1, 2048, 4, 64, seed=1, dtype="f32", s0_std=0.1)
    w = d["w"].astype(np.float64)
    assert w.min() >= np.exp(-0.6065) - 1e-6 and w.max() <= 1.0
    a, b = d["a"].astype(np.float64), d["b"].astype(np.float64)
    np.testing.assert_allclose(np.linalg.norm(a, axis=-1), 1.0, rtol=1e-5)
    nz = a != 0.0                       # float32 normal draws can be exactly 0
    lr = b[nz] / (-a[nz])
    assert lr.min() > 0.0 and lr.max() < 1.0
    for n in ("r", "k", "v"):
        x = d[n].astype(np.float64)
        assert abs(x.mean()) < 0.01 and abs(x.std() - 1.0) < 0.01
    assert abs(d["s0"].std() - 0.1) < 0.002
    long = inputs.gen_sequence(1, 256, 4, 64, seed=3, dtype="f32", x_mean=-2.0)
    assert long["w"].mean() > w.mean()


def test_steps_layout_matches_flat_vectors():
    s = inputs.gen_steps(3, 4, 2, 64, seed=2)
    v = inputs.gen_vectors(3 * 4 * 2, 64, seed=2)
    np.testing.assert_array_equal(s["k"].reshape(-1, 64), v["k"])
