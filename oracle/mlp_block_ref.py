"""Double-precision CPU oracle of the multi-layer driver on a synthetic MLP block.

TEST INFRASTRUCTURE ONLY: used by the tests alone; the CUDA path never calls
it and shares no code with it.

Sources (web pages; cited by title and section):
* [SGPT] review of "SparseGPT: Massive Language Models Can Be Accurately
  Pruned in One-Shot" (devpress.csdn.net), section 九: layers are processed one
  after the other: collect the current layer's input activations, form its
  Hessian, prune with error compensation, pass the pruned layer's output on to
  the next layer; later layers see the activations of the pruned model, not
  of the dense one. Section 十一, steps three to six: the same per layer.
* [V] V-SparseGPT press release (voc.com.cn): layer-parallel sparsification
  records the inputs of every layer of the original (dense) model first, so
  several layers can be sparsified side by side.

Readings (listed in the design notes): the pages name no model, so the block
is the MLP part of a decoder block, x -> x + W_down (silu(W_gate x) * (W_up
x)); the activations x, z and x' are bf16 (rounded to nearest even from the
exact float64 value), each product uses the bf16 rounding of the fp32
weights, and silu(g) = g / (1 + e^-g).
"""

from __future__ import annotations

import numpy as np

from . import sparsegpt_ref as sg


def bf16_round(x) -> np.ndarray:
    """x (float64) rounded once to the nearest bfloat16 (8 significant bits),
    ties to even, returned as float64. Normal-range values only (the block's
    activations and weights are far from under- and overflow)."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def silu(g):
    g = np.asarray(g, dtype=np.float64)
    return g / (1.0 + np.exp(-g))


def linear(X, W):
    """X [n, d_in] (bf16 values) times the bf16 rounding of W [d_out, d_in],
    transposed: [n, d_out] in float64."""
    return np.asarray(X, dtype=np.float64) @ bf16_round(np.asarray(W, dtype=np.float32).astype(np.float64)).T


def down_input(X, W_gate, W_up):
    """z = bf16(silu(x Wg^T) * (x Wu^T))."""
    return bf16_round(silu(linear(X, W_gate)) * linear(X, W_up))


def block_output(X, Z, W_down):
    """x' = bf16(x + z Wd^T)."""
    return bf16_round(np.asarray(X, dtype=np.float64) + linear(Z, W_down))


def prune_mlp_block(X, W_gate, W_up, W_down, pattern="2:4", mode="sequential", blocksize=128,
                    damp_ratio=0.01, qbits=None):
    """One block of the driver. Returns the pruned weights and masks of the
    three layers, the down projection's input z and the block output x'.

    sequential ([SGPT] 九): gate and up from x, z from the PRUNED gate and up,
    down from that z, x' from the pruned block.
    parallel ([V]): z and x' from the DENSE block, every layer pruned from
    the recorded dense input.
    """
    X = np.asarray(X, dtype=np.float64)
    out = {}
    if mode == "parallel":
        Z = down_input(X, W_gate, W_up)
        X_next = block_output(X, Z, W_down)
    H = sg.hessian(X)
    Hd, _ = sg.damp(H, damp_ratio)
    U = sg.inverse_cholesky_upper(Hd)
    for name, W in (("gate", W_gate), ("up", W_up)):
        r = sg.sweep(np.asarray(W, dtype=np.float64), U, pattern, blocksize, qbits=qbits)
        out[name] = r
    if mode == "sequential":
        Z = down_input(X, out["gate"]["W"], out["up"]["W"])
    Hz = sg.hessian(Z)
    Hzd, _ = sg.damp(Hz, damp_ratio)
    Uz = sg.inverse_cholesky_upper(Hzd)
    out["down"] = sg.sweep(np.asarray(W_down, dtype=np.float64), Uz, pattern, blocksize, qbits=qbits)
    if mode == "sequential":
        X_next = block_output(X, Z, out["down"]["W"])
    out.update(Z=Z, X_next=X_next, H_x=H, U_x=U, H_z=Hz, U_z=Uz)
    return out
