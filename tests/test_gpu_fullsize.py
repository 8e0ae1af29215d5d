"""Full-size parity of the Llama-7B-shaped layers against the float64 oracle.

The oracle computes H from the very bf16 activations the GPU consumed (in
float64, token chunk by token chunk), factors it and runs the whole sweep on
all rows; the GPU runs the whole layer from X through the C ABI. Slow: the
oracle's Hessian alone is 4e13 float64 flops on the host.
"""

import numpy as np
import pytest
import torch

import oracle
import post_pruning_b200 as pp
from workloads import CONFIGS, bf16_bits_to_f64, gen_activations, gen_weights

from parity import assert_parity, compare, gpu_prune_layer, sample_rows

pytestmark = [pytest.mark.gpu, pytest.mark.slow]

def _oracle_h(X: torch.Tensor) -> np.ndarray:
    n, d = X.shape
    H = np.zeros((d, d))
    for t0 in range(0, n, 8192):
        Xc = bf16_bits_to_f64(X[t0:t0 + 8192].cpu()).numpy()
        H += Xc.T @ Xc
    return H * (2.0 / n)


@pytest.mark.parametrize("name", ["llama7b_q", "llama7b_down"])
def test_full_size_layer_from_X(name):
    spec = CONFIGS[name][0]
    X = gen_activations(spec, device="cuda")
    W = gen_weights(spec)
    H = _oracle_h(X)
    Hd, _ = oracle.damp(H, 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    W0 = W.numpy().astype(np.float64)
    for run in spec.runs:
        p = pp.Params(run)
        gpu = gpu_prune_layer(W, X, p)
        m = compare(gpu, W0, H, U, p)
        print(name, run, {k: v for k, v in m.items() if not isinstance(v, bool)})
        assert_parity(m, p)


def _oracle_h_sym(X: torch.Tensor) -> np.ndarray:
    """Same H, accumulated with a symmetric rank-k update (half the flops)."""
    import scipy.linalg.blas as blas
    n, d = X.shape
    H = np.zeros((d, d), order="F")
    for t0 in range(0, n, 4096):
        Xc = np.asfortranarray(bf16_bits_to_f64(X[t0:t0 + 4096].cpu()).numpy())
        H = blas.dsyrk(1.0, Xc, beta=1.0, c=H, trans=1, lower=0, overwrite_c=1)
    H = np.triu(H) + np.triu(H, 1).T
    return H * (2.0 / n)


def _check_h_and_u(Hg_sum: torch.Tensor, Ug: torch.Tensor, H: np.ndarray, U: np.ndarray, n: int):
    """Every element of the GPU's H (the fp32 sum X^T X, scaled here by 2/n)
    against the float64 one, within 1e-5 of sqrt(H_ii H_jj) (by
    Cauchy-Schwarz at least the sum of |products|, so a bound on fp32
    accumulation error); every row of the GPU's U within 1e-4 relative of
    the oracle's. Row chunks bound the host memory."""
    d = H.shape[0]
    dg = np.sqrt(np.diag(H))
    worst_h = worst_u = 0.0
    for r0 in range(0, d, 2048):
        r1 = min(d, r0 + 2048)
        hg = Hg_sum[r0:r1].cpu().numpy().astype(np.float64) * (2.0 / n)
        err = np.abs(hg - H[r0:r1]) / np.outer(dg[r0:r1], dg)
        worst_h = max(worst_h, float(err.max()))
        ug = Ug[r0:r1].cpu().numpy().astype(np.float64)
        rel = np.linalg.norm(ug - U[r0:r1], axis=1) / np.linalg.norm(U[r0:r1], axis=1)
        worst_u = max(worst_u, float(rel.max()))
        below = np.tril(np.ones((r1 - r0, d), dtype=bool), r0 - 1)
        assert np.all(ug[below] == 0.0)
    print(f"H max err / sqrt(Hii Hjj) = {worst_h:.3g}, U max row rel err = {worst_u:.3g}")
    assert worst_h <= 1e-5
    assert worst_u < 1e-4


def _qwen_group(x_key):
    """One input of the Qwen3-32B-shaped block: the GPU computes H and U once
    and sweeps every matrix that reads the input. The oracle computes H and U
    in full and checks them element by element; it sweeps a 256-row sample
    of each matrix (2:4 rows are independent, so the sample's result is
    exactly those rows of the full result) and the GPU's rows are compared
    on the same sample."""
    specs = [s for s in CONFIGS["qwen3_32b_block"] if s.x_key == x_key]
    X = gen_activations(specs[0], device="cuda")
    H = _oracle_h_sym(X)
    Hd, _ = oracle.damp(H, 0.01)
    U = oracle.inverse_cholesky_upper(Hd)
    dev = torch.device("cuda")
    # the GPU path: one Hessian and factor per input, a sweep per matrix
    first = None
    for sp in specs:
        W = gen_weights(sp)
        p = pp.Params("2:4")
        if first is None:
            first = pp.LayerBuffers.allocate(sp.d_out, sp.d_in, sp.n_tok, dev)
            b = first
            Wd = W.to(dev)
            b.run(Wd, X, p)
            assert pp.sync_status(b.info) == 0
            _check_h_and_u(b.H, b.U, H, U, sp.n_tok)
        else:
            b = pp.LayerBuffers.sharing(first, sp.d_out, dev)
            Wd = W.to(dev)
            pp.info_clear(b.info)
            b.row_loss.zero_()
            pp.prune(Wd, b.U, p, b.mask, b.ws, b.info, row_loss=b.row_loss)
            pp.pack24(Wd, b.mask, b.values, b.meta, b.info)
        assert pp.sync_status(b.info) == 0
        gpu = {"W": Wd.cpu().numpy(),
               "mask": oracle.bits_to_mask(b.mask.cpu().numpy().view(np.uint32), sp.d_in),
               "row_loss": b.row_loss.cpu().numpy().astype(np.float64),
               "values": b.values.cpu().numpy(), "meta": b.meta.cpu().numpy().view(np.uint32)}
        rows = sample_rows(sp.d_out)
        m = compare(gpu, W.numpy().astype(np.float64), H, U, p, rows=rows)
        print(sp.name, f"{len(rows)} sampled rows", {k: v for k, v in m.items() if not isinstance(v, bool)})
        assert_parity(m, p)
        # the rows outside the sample: the 2:4 invariants hold everywhere
        groups = gpu["mask"].reshape(sp.d_out, -1, 4).sum(axis=2)
        assert np.all(groups == 2) and np.all(gpu["W"][~gpu["mask"]] == 0.0)


@pytest.mark.parametrize("x_key", [0, 1, 2], ids=["qkv", "o", "gate_up"])
def test_qwen3_block_shared_hessian(x_key):
    """q/k/v share one H and U, o has its own, gate/up share one."""
    _qwen_group(x_key)


def test_qwen3_block_down_proj():
    """d_in = 25,600: H and U in full on the host (~1e14 float64 flops), the
    sweep on a row sample."""
    _qwen_group(3)
