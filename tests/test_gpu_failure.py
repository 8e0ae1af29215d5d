"""Failure paths on the GPU without faulting it: every device-side wait on
other threads or CTAs is bounded, and a wait that runs out records
SGPT_INFO_TIMEOUT, lets its kernel drain its own copies and tensor-core
operations and return, and leaves the context usable.

Each test lowers the wait limit to one cycle (sgpt_set_wait_limit), so the
first wait that does not succeed at once gives up, runs one kernel family
(the Hessian's tensor-core pipeline, the FP32-accurate GEMM of the
factorisation, the unstructured selection's grid barrier), checks that the
call reports TIMEOUT and wrote nothing it should not have, then restores the
default limit and checks that the same call now succeeds with the same
result as before.
"""

import numpy as np
import pytest
import torch

import post_pruning_b200 as pp
from workloads import LayerSpec, gen_activations, gen_weights

pytestmark = pytest.mark.gpu

TIMEOUT = 4


@pytest.fixture
def tiny_wait_limit():
    def lower():
        pp.set_wait_limit(1)
    yield lower
    pp.set_wait_limit(0)


def _spec(d_in, d_out, n_tok):
    return LayerSpec(f"fail_{d_in}", d_in=d_in, d_out=d_out, n_tok=n_tok, seed=21)


def test_hessian_wait_times_out(tiny_wait_limit):
    spec = _spec(768, 64, 65536)
    dev = torch.device("cuda")
    X = gen_activations(spec, device=dev)
    ws = pp.workspace(spec.d_out, spec.d_in, spec.n_tok)
    info = pp.new_info()
    H_ok = torch.empty(spec.d_in, spec.d_in, device=dev)
    pp.hessian_compute(H_ok, X, ws, info)
    assert pp.sync_status(info) == 0

    tiny_wait_limit()
    H = torch.full_like(H_ok, 7.0)
    pp.info_clear(info)
    pp.hessian_compute(H, X, ws, info)
    assert pp.sync_status(info) == TIMEOUT
    pp.set_wait_limit(0)

    pp.info_clear(info)
    pp.hessian_compute(H, X, ws, info)
    assert pp.sync_status(info) == 0
    assert torch.equal(H, H_ok)


def test_gemm_wait_times_out(tiny_wait_limit):
    """The factorisation's tensor-core products (d = 1024: eight block
    columns, panels and rank-128 updates on the 3xTF32 GEMM)."""
    spec = _spec(1024, 64, 8192)
    dev = torch.device("cuda")
    X = gen_activations(spec, device=dev)
    ws = pp.workspace(spec.d_out, spec.d_in, spec.n_tok)
    info = pp.new_info()
    H = torch.empty(spec.d_in, spec.d_in, device=dev)
    pp.hessian_compute(H, X, ws, info)
    U_ok = torch.empty_like(H)
    pp.factor(H, spec.n_tok, 0.01, U_ok, ws, info)
    assert pp.sync_status(info) == 0

    tiny_wait_limit()
    U = torch.empty_like(H)
    pp.factor(H, spec.n_tok, 0.01, U, ws, info)
    assert pp.sync_status(info) == TIMEOUT
    pp.set_wait_limit(0)

    pp.info_clear(info)
    pp.factor(H, spec.n_tok, 0.01, U, ws, info)
    assert pp.sync_status(info) == 0
    assert torch.equal(U, U_ok)


def test_selection_grid_barrier_times_out(tiny_wait_limit):
    """One 128-column block (no trailing product), 4096 rows: the
    cooperative selection meets its grid barrier once per digit pass."""
    spec = _spec(128, 4096, 4096)
    dev = torch.device("cuda")
    X = gen_activations(spec, device=dev)
    W0 = gen_weights(spec, device=dev)
    ws = pp.workspace(spec.d_out, spec.d_in, spec.n_tok)
    info = pp.new_info()
    H = torch.empty(spec.d_in, spec.d_in, device=dev)
    U = torch.empty_like(H)
    pp.hessian_compute(H, X, ws, info)
    pp.factor(H, spec.n_tok, 0.01, U, ws, info)
    assert pp.sync_status(info) == 0
    p = pp.Params("unstructured:0.5")
    mask = torch.zeros(spec.d_out, spec.d_in // 32, dtype=torch.int32, device=dev)
    W_ok = W0.clone()
    pp.prune(W_ok, U, p, mask, ws, info)
    assert pp.sync_status(info) == 0
    mask_ok = mask.clone()

    tiny_wait_limit()
    W = W0.clone()
    mask.zero_()
    pp.prune(W, U, p, mask, ws, info)
    assert pp.sync_status(info) == TIMEOUT
    # the sweep saw the recorded timeout and left W and the mask alone
    assert torch.equal(W, W0)
    assert int(mask.abs().sum()) == 0
    pp.set_wait_limit(0)

    pp.info_clear(info)
    pp.prune(W, U, p, mask, ws, info)
    assert pp.sync_status(info) == 0
    assert torch.equal(W, W_ok) and torch.equal(mask, mask_ok)
    kept = np.unpackbits(mask.cpu().numpy().view(np.uint8), bitorder="little").sum()
    assert spec.d_out * spec.d_in - kept == spec.d_out * spec.d_in // 2
