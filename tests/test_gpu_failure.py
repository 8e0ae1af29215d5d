"""Failure paths on the GPU without faulting it: every device-side wait on
other threads or CTAs is bounded, and a wait that runs out records
SGPT_INFO_TIMEOUT, lets its kernel drain its own copies and tensor-core
operations and return, and leaves the context usable.

Each test lowers the wait limit to one cycle (sgpt_set_wait_limit), so the
first wait that does not succeed at once gives up, runs one kernel family
(the Hessian's tensor-core pipeline, the FP32-accurate GEMM of the
factorisation, the unstructured selection's grid barrier, the bf16 product
on wide tiles, the 2:4 sparse product), checks that the
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


def test_wide_bf16_gemm_wait_times_out(tiny_wait_limit):
    """The bf16 product on 128 x 256 tiles (the driver's forward pass)."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(3)
    n, d_in, d_out = 2048, 512, 768
    X = torch.randn(n, d_in, device=dev, generator=g).to(torch.bfloat16)
    Wb = torch.randn(d_out, d_in, device=dev, generator=g).to(torch.bfloat16)
    info = pp.new_info()
    Y_ok = torch.empty(n, d_out, device=dev)
    pp.linear_bf16(X, Wb, Y_ok, info)
    assert pp.sync_status(info) == 0

    tiny_wait_limit()
    Y = torch.empty_like(Y_ok)
    pp.info_clear(info)
    pp.linear_bf16(X, Wb, Y, info)
    assert pp.sync_status(info) == TIMEOUT
    pp.set_wait_limit(0)

    pp.info_clear(info)
    pp.linear_bf16(X, Wb, Y, info)
    assert pp.sync_status(info) == 0
    assert torch.equal(Y, Y_ok)


def test_sparse24_consumer_wait_times_out(tiny_wait_limit):
    """The persistent 2:4 sparse product (TMA ring, metadata copied into
    TMEM, register epilogue)."""
    dev = torch.device("cuda")
    g = torch.Generator(device=dev).manual_seed(4)
    n, d_in, d_out = 1024, 512, 512
    W = torch.randn(d_out, d_in, device=dev, generator=g)
    keep = torch.zeros(d_out, d_in // 4, 4, dtype=torch.bool, device=dev)
    keep.scatter_(2, torch.rand(d_out, d_in // 4, 4, device=dev, generator=g).topk(2, dim=2).indices, True)
    keep = keep.reshape(d_out, d_in)
    W = torch.where(keep, W, torch.zeros_like(W))
    bits = (keep.reshape(d_out, d_in // 32, 32).to(torch.int64) << torch.arange(32, device=dev)).sum(2)
    mask = torch.where(bits >= 2 ** 31, bits - 2 ** 32, bits).to(torch.int32)
    info = pp.new_info()
    vals = torch.empty(d_out, d_in // 2, device=dev)
    meta = torch.empty(d_out, d_in // 32, dtype=torch.int32, device=dev)
    pp.pack24(W, mask, vals, meta, info)
    vb = torch.empty(d_out, d_in // 2, dtype=torch.bfloat16, device=dev)
    pp.to_bf16(vals, vb, info)
    tiles = pp.sparse24_meta_tiles(meta, d_in)
    X = torch.randn(n, d_in, device=dev, generator=g).to(torch.bfloat16)
    Y_ok = torch.empty(n, d_out, device=dev)
    pp.sparse24_linear(vb, tiles, X, Y_ok, info)
    assert pp.sync_status(info) == 0

    tiny_wait_limit()
    Y = torch.empty_like(Y_ok)
    pp.info_clear(info)
    pp.sparse24_linear(vb, tiles, X, Y, info)
    assert pp.sync_status(info) == TIMEOUT
    pp.set_wait_limit(0)

    pp.info_clear(info)
    pp.sparse24_linear(vb, tiles, X, Y, info)
    assert pp.sync_status(info) == 0
    assert torch.equal(Y, Y_ok)
