"""Pins of the multi-layer driver's oracle (oracle/mlp_block_ref.py) to facts
that do not come from the oracle itself: hand-derived bf16 roundings and
torch's own float32 -> bfloat16 conversion, identities of silu, a block whose
output is known in closed form, and the relations between the sequential and
the layer-parallel modes."""

import math

import numpy as np
import pytest
import torch

from oracle import mlp_block_ref as mb


def test_bf16_round_hand_cases():
    cases = [
        (1.0, 1.0),
        (1 + 2 ** -8, 1.0),                      # tie: the even neighbour 1.0
        (1 + 3 * 2 ** -8, 1 + 2 ** -6),          # tie: 1 + 2^-6 has the even last bit
        (1 + 2 ** -8 + 2 ** -20, 1 + 2 ** -7),   # just above the tie
        (-3.0, -3.0),
        (0.1, 205 / 256 * 2 ** -3),              # 0.1 = 0.8 * 2^-3; 0.8 * 256 = 204.8 -> 205
        (300.5, 300.0),                          # 300.5 = 0.5869 * 2^9; 150.25 -> 150
    ]
    for x, want in cases:
        assert mb.bf16_round(x) == want, x


def test_bf16_round_matches_torch_on_float32_inputs():
    rng = np.random.default_rng(0)
    x = (rng.standard_normal(100000) * np.exp(rng.uniform(-10, 10, 100000))).astype(np.float32)
    want = torch.from_numpy(x).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(mb.bf16_round(x.astype(np.float64)), want)


def test_silu_identities():
    x = np.linspace(-20, 20, 4001)
    assert mb.silu(0.0) == 0.0
    assert np.allclose(mb.silu(x) - mb.silu(-x), x, rtol=0, atol=1e-12)
    assert np.allclose(mb.silu(x[x > 15]), x[x > 15], rtol=1e-6)


def test_block_forward_closed_form():
    """W_gate = I, W_up = 2 I, W_down = I: z = bf16(silu(x) * 2x) and
    x' = bf16(x + z), channel by channel."""
    d = 32
    rng = np.random.default_rng(1)
    X = mb.bf16_round(rng.standard_normal((16, d)))
    I = np.eye(d)
    Z = mb.down_input(X, I, 2 * I)
    assert np.array_equal(Z, mb.bf16_round(X / (1 + np.exp(-X)) * 2 * X))
    Xn = mb.block_output(X, Z, I)
    assert np.array_equal(Xn, mb.bf16_round(X + Z))


def _block(rng, h=64, f=128, n=512):
    X = mb.bf16_round(rng.standard_normal((n, h)) * np.exp(rng.standard_normal(h)))
    Wg = rng.standard_normal((f, h)).astype(np.float32) / math.sqrt(h)
    Wu = rng.standard_normal((f, h)).astype(np.float32) / math.sqrt(h)
    Wd = rng.standard_normal((h, f)).astype(np.float32) / math.sqrt(f)
    return X, Wg, Wu, Wd


def test_modes_agree_when_nothing_is_pruned():
    X, Wg, Wu, Wd = _block(np.random.default_rng(2))
    a = mb.prune_mlp_block(X, Wg, Wu, Wd, "unstructured:0.0", mode="sequential", blocksize=64)
    b = mb.prune_mlp_block(X, Wg, Wu, Wd, "unstructured:0.0", mode="parallel", blocksize=64)
    for name, W in (("gate", Wg), ("up", Wu), ("down", Wd)):
        assert np.array_equal(a[name]["W"], W.astype(np.float64))     # no error, nothing moves
        assert a[name]["mask"].all()
        assert np.array_equal(a[name]["W"], b[name]["W"])
    assert np.array_equal(a["Z"], b["Z"]) and np.array_equal(a["X_next"], b["X_next"])


def test_sequential_down_sees_the_pruned_activations():
    """[SGPT] 九: after the earlier layers are pruned, the later layer is
    pruned on the pruned model's activations; the parallel mode uses the dense
    ones ([V])."""
    X, Wg, Wu, Wd = _block(np.random.default_rng(3))
    a = mb.prune_mlp_block(X, Wg, Wu, Wd, "2:4", mode="sequential", blocksize=64)
    b = mb.prune_mlp_block(X, Wg, Wu, Wd, "2:4", mode="parallel", blocksize=64)
    assert np.array_equal(a["gate"]["W"], b["gate"]["W"]) and np.array_equal(a["up"]["W"], b["up"]["W"])
    assert np.array_equal(b["Z"], mb.down_input(X, Wg, Wu))
    assert np.array_equal(a["Z"], mb.down_input(X, a["gate"]["W"], a["up"]["W"]))
    assert not np.array_equal(a["Z"], b["Z"])
    assert not np.array_equal(a["down"]["W"], b["down"]["W"])
    assert np.array_equal(b["X_next"], mb.block_output(X, b["Z"], Wd))       # the dense block's output
    assert np.array_equal(a["X_next"], mb.block_output(X, a["Z"], a["down"]["W"]))
