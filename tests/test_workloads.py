"""The seeded input generator: deterministic, sliceable by counter, and the
distributions it states (normal moments, outlier channel count, bf16 X)."""

import math

import torch

from workloads import CONFIGS, LayerSpec, channel_scales, gen_activations, gen_weights, normals


def test_normals_deterministic_and_counter_based():
    a = normals(0, 2, 1000, 5000)
    b = normals(0, 2, 0, 6000)[1000:]
    assert torch.equal(a, b)
    assert not torch.equal(normals(0, 2, 0, 100), normals(0, 3, 0, 100))
    assert not torch.equal(normals(0, 2, 0, 100), normals(1, 2, 0, 100))


def test_normal_moments():
    z = normals(7, 9, 0, 1 << 20)
    assert abs(z.mean().item()) < 4 / math.sqrt(1 << 20)
    assert abs(z.std().item() - 1.0) < 5e-3
    assert abs((z ** 4).mean().item() - 3.0) < 0.05          # Gaussian kurtosis


def test_outlier_channels_and_scales():
    spec = CONFIGS["llama7b_down"][0]
    s = channel_scales(spec)
    assert s.shape == (spec.d_in,)
    m = int(math.floor(spec.p_out * spec.d_in + 0.5))
    base = torch.exp(spec.sigma * normals(spec.seed, 3, 0, spec.d_in))
    ratio = s / base
    assert int((ratio > 1.5).sum()) == m                       # exactly m channels scaled
    assert torch.allclose(ratio[ratio > 1.5], torch.full((m,), spec.f_out, dtype=torch.float64))


def test_activation_and_weight_slices():
    spec = LayerSpec("t", d_in=64, d_out=48, n_tok=300, seed=3)
    X = gen_activations(spec)
    assert X.dtype == torch.bfloat16 and X.shape == (300, 64)
    assert torch.equal(gen_activations(spec, t0=123, count=77), X[123:200])
    W = gen_weights(spec)
    assert W.dtype == torch.float32 and W.shape == (48, 64)
    assert torch.equal(gen_weights(spec, rows=[5, 40]), W[[5, 40]])
    assert abs(W.std().item() * math.sqrt(64) - 1.0) < 0.1
    # distinct inputs and weights of one block draw distinct streams
    blk = CONFIGS["qwen3_32b_block"]
    assert len({s.x_key for s in blk}) == 4 and len({s.w_key for s in blk}) == 7
