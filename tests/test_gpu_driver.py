"""The multi-layer driver (sgpt_prune_mlp_block) against the float64 oracle.

Each layer is checked on the very inputs the GPU used: gate and up against
the oracle's prune of the block input, the down projection's input z against
the oracle's forward pass of the GPU's pruned (sequential) or dense
(parallel) gate and up, down against the oracle's prune of the GPU's z, and
the block output likewise. bf16 activations may differ from the oracle's by
one unit in the last place where fp32 and float64 sums fall on either side of
a rounding tie.
"""

import math

import numpy as np
import pytest
import torch

import oracle
import post_pruning_b200 as pp
from oracle import mlp_block_ref as mb
from workloads import LayerSpec, bf16_bits_to_f64, gen_activations, gen_weights

from parity import assert_parity, compare

pytestmark = pytest.mark.gpu

ULP_FRACTION = 0.01        # share of bf16 activations allowed one ulp apart


def _f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().cpu().to(torch.float64).numpy()


def _bf16_close(gpu: np.ndarray, ref: np.ndarray, err_bound: np.ndarray):
    """Each value within one bf16 ulp of the oracle's plus the error bound of
    the fp32 sums it came from (fp32 accumulation of exact bf16 products,
    1e-5 of the sum of |products|, carried through the elementwise step);
    at most ULP_FRACTION of the values differ at all."""
    diff = gpu != ref
    mag = np.maximum(np.abs(gpu), np.abs(ref))
    ulp = np.ldexp(1.0, np.frexp(mag)[1] - 8)
    excess = np.abs(gpu - ref) - (ulp * 1.0001 + err_bound)
    assert np.all(excess <= 0), float(excess.max())
    assert diff.mean() <= ULP_FRACTION, diff.mean()
    return float(diff.mean())


def _z_bound(Xf, Wg, Wu):
    """Error bound of z = silu(g) u from the fp32 sums of g and u: |d silu/dg|
    <= 1.1 everywhere."""
    g, u = mb.linear(Xf, Wg), mb.linear(Xf, Wu)
    absX = np.abs(Xf)
    bg = 1e-5 * (absX @ np.abs(mb.bf16_round(np.asarray(Wg, dtype=np.float32).astype(np.float64))).T)
    bu = 1e-5 * (absX @ np.abs(mb.bf16_round(np.asarray(Wu, dtype=np.float32).astype(np.float64))).T)
    return 1.1 * np.abs(u) * bg + np.abs(mb.silu(g)) * bu + bg * bu


def _x_bound(Z, Wd):
    return 1e-5 * (np.abs(Z) @ np.abs(mb.bf16_round(np.asarray(Wd, dtype=np.float32).astype(np.float64))).T)


def test_linear_bf16_matches_float64():
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(0)
    n, d_in, d_out = 1000, 320, 224              # ragged tiles in M, N and K
    X = (torch.randn(n, d_in, generator=g) * 3).to(torch.bfloat16)
    Wb = torch.randn(d_out, d_in, generator=g).to(torch.bfloat16)
    Y = torch.empty(n, d_out, device=dev)
    info = pp.new_info()
    pp.linear_bf16(X.to(dev), Wb.to(dev), Y, info)
    pp.raise_on_info(info)
    Xf, Wf = _f64(X), _f64(Wb)
    ref = Xf @ Wf.T
    bound = np.abs(Xf) @ np.abs(Wf).T
    assert np.all(np.abs(Y.cpu().numpy() - ref) <= 1e-5 * bound + 1e-30)


def test_to_bf16_is_round_to_nearest_even():
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(1)
    W = torch.randn(96, 64, generator=g) * torch.exp(torch.randn(96, 64, generator=g) * 4)
    Wb = torch.empty(96, 64, dtype=torch.bfloat16, device=dev)
    info = pp.new_info()
    pp.to_bf16(W.to(dev), Wb, info)
    pp.raise_on_info(info)
    assert np.array_equal(_f64(Wb), mb.bf16_round(W.numpy().astype(np.float64)))


def _block_inputs(h, f, n, seed):
    spec = LayerSpec("blk", d_in=h, d_out=f, n_tok=n, sigma=1.0, seed=seed)
    X = gen_activations(spec)
    Wg = gen_weights(spec.with_(w_key=1))
    Wu = gen_weights(spec.with_(w_key=2))
    Wd = gen_weights(LayerSpec("down", d_in=f, d_out=h, n_tok=n, seed=seed, w_key=3))
    return X, Wg, Wu, Wd


def _run_block(X, Wg, Wu, Wd, p, mode):
    dev = torch.device("cuda")
    f, h = Wg.shape
    n = X.shape[0]
    W = [w.to(dev).contiguous() for w in (Wg, Wu, Wd)]
    masks = (torch.empty(f, h // 32, dtype=torch.int32, device=dev),
             torch.empty(f, h // 32, dtype=torch.int32, device=dev),
             torch.empty(h, f // 32, dtype=torch.int32, device=dev))
    X_next = torch.empty(n, h, dtype=torch.bfloat16, device=dev)
    Z = torch.empty(n, f, dtype=torch.bfloat16, device=dev)
    ws = pp.mlp_block_workspace(h, f, n)
    info = pp.new_info()
    pp.prune_mlp_block(*W, masks, X.to(dev), p, X_next, ws, info, mode=mode, Z=Z)
    assert pp.sync_status(info) == 0
    out = {}
    for name, w, m_, d in (("gate", W[0], masks[0], h), ("up", W[1], masks[1], h), ("down", W[2], masks[2], f)):
        out[name] = {"W": w.cpu().numpy(), "mask": oracle.bits_to_mask(m_.cpu().numpy().view(np.uint32), d)}
    out["Z"] = Z
    out["X_next"] = X_next
    return out


def _layer_parity(gpu_layer, W0, Xin, p):
    H = oracle.hessian(Xin)
    Hd, _ = oracle.damp(H, 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    m = compare(dict(gpu_layer), W0.numpy().astype(np.float64), H, U, p)
    assert_parity(m, p)
    return m


def _check_block(X, Wg, Wu, Wd, p, mode):
    gpu = _run_block(X, Wg, Wu, Wd, p, mode)
    Xf = bf16_bits_to_f64(X).numpy()
    # gate and up: pruned from the block input
    for name, W0 in (("gate", Wg), ("up", Wu)):
        _layer_parity(gpu[name], W0, Xf, p)
    # the down projection's input: the oracle's forward of the GPU's pruned
    # (sequential) or the dense (parallel) gate and up
    Zg = _f64(gpu["Z"])
    if mode == pp.DRIVER_SEQUENTIAL:
        Wg_used, Wu_used = gpu["gate"]["W"], gpu["up"]["W"]
    else:
        Wg_used, Wu_used = Wg.numpy(), Wu.numpy()
    Zo = mb.down_input(Xf, Wg_used, Wu_used)
    z_frac = _bf16_close(Zg, Zo, _z_bound(Xf, Wg_used, Wu_used))
    # down: pruned from the GPU's z
    _layer_parity(gpu["down"], Wd, Zg, p)
    # the block output
    Wd_used = gpu["down"]["W"] if mode == pp.DRIVER_SEQUENTIAL else Wd.numpy()
    x_frac = _bf16_close(_f64(gpu["X_next"]), mb.block_output(Xf, Zg, Wd_used), _x_bound(Zg, Wd_used))
    print(f"mode {mode} {p.pattern}: z ulp-flips {z_frac:.2e}, x' ulp-flips {x_frac:.2e}")
    return gpu


@pytest.mark.parametrize("mode", [pp.DRIVER_SEQUENTIAL, pp.DRIVER_PARALLEL], ids=["sequential", "parallel"])
@pytest.mark.parametrize("p", [pp.Params("2:4"), pp.Params("unstructured:0.5"), pp.Params("16:64")],
                         ids=lambda p: p.pattern)
def test_mlp_block_layer_by_layer(mode, p):
    X, Wg, Wu, Wd = _block_inputs(256, 512, 3000, seed=5)
    _check_block(X, Wg, Wu, Wd, p, mode)


def test_two_block_stack_sequential():
    """Block 2 is pruned on block 1's pruned output."""
    p = pp.Params("2:4")
    X, Wg, Wu, Wd = _block_inputs(256, 384, 2048, seed=6)
    first = _check_block(X, Wg, Wu, Wd, p, pp.DRIVER_SEQUENTIAL)
    X2 = first["X_next"].cpu()
    _, Wg2, Wu2, Wd2 = _block_inputs(256, 384, 2048, seed=7)
    _check_block(X2, Wg2, Wu2, Wd2, p, pp.DRIVER_SEQUENTIAL)
