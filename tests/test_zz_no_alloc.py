"""The allocation-free prune entry point against the workspace one.

sgpt_prune_noalloc is for callers that cannot hand the library device memory
at the call site (for example a plugin whose execution path forbids
allocation): it keeps its scratch in a fixed array inside the library. This
test calls it through the C ABI twice in a row, with different patterns and
shapes so that the second call starts from the first call's leftovers, and
checks each result against sgpt_prune on the same inputs with the tolerances
the parity tests use. It also checks that a too-large d_out is refused.
"""

import ctypes

import numpy as np
import pytest
import torch

import oracle
import post_pruning_b200 as pp
from post_pruning_b200 import sgpt as S
from workloads import LayerSpec, gen_activations, gen_weights

pytestmark = pytest.mark.gpu

MASK_AGREEMENT = 0.999
WEIGHT_REL_L2 = 1e-3


def _layer(spec):
    dev = torch.device("cuda")
    X = gen_activations(spec, device=dev)
    W = gen_weights(spec, device=dev)
    H = torch.zeros(spec.d_in, spec.d_in, device=dev)
    U = torch.empty_like(H)
    ws = pp.workspace(spec.d_out, spec.d_in, spec.n_tok)
    info = pp.new_info()
    pp.hessian_accumulate(H, X, ws, info)
    pp.factor(H, spec.n_tok, 0.01, U, ws, info)
    pp.raise_on_info(info)
    return W, U, ws


def _run(entry, W0, U, params, ws=None):
    r, d = W0.shape
    W = W0.clone()
    mask = torch.zeros(r, d // 32, dtype=torch.int32, device=W.device)
    loss = torch.zeros(r, device=W.device)
    info = pp.new_info()
    if entry == "noalloc":
        pp.prune_noalloc(W, U, params, mask, info, row_loss=loss)
    else:
        pp.prune(W, U, params, mask, ws, info, row_loss=loss)
    assert pp.sync_status(info) == 0
    return W.cpu().numpy(), oracle.bits_to_mask(mask.cpu().numpy().view(np.uint32), d), loss.cpu().numpy()


def _close(a, b):
    Wa, Ma, La = a
    Wb, Mb, Lb = b
    assert np.mean(Ma == Mb) >= MASK_AGREEMENT
    assert np.linalg.norm(Wa - Wb) <= WEIGHT_REL_L2 * np.linalg.norm(Wb)
    assert np.allclose(La, Lb, rtol=1e-3, atol=1e-12)


def test_noalloc_matches_workspace_entry_twice_in_a_row():
    first = LayerSpec("noalloc_a", d_in=384, d_out=512, n_tok=4096, seed=7)
    second = LayerSpec("noalloc_b", d_in=256, d_out=1000, n_tok=3000, sigma=1.5, seed=8)
    W1, U1, ws1 = _layer(first)
    W2, U2, ws2 = _layer(second)
    p1 = pp.Params("2:4")
    p2 = pp.Params("unstructured:0.5", blocksize=64)
    a1 = _run("noalloc", W1, U1, p1)
    a2 = _run("noalloc", W2, U2, p2)
    _close(a1, _run("workspace", W1, U1, p1, ws1))
    _close(a2, _run("workspace", W2, U2, p2, ws2))
    # and once more on the first layer, after the second call's leftovers
    _close(_run("noalloc", W1, U1, p1), a1)


def test_noalloc_refuses_rows_beyond_its_scratch():
    L = pp.lib()
    p = S.Params("2:4").to_c()
    fake = 1 << 20                                  # never dereferenced
    st = L.sgpt_prune_noalloc(fake, S.NOALLOC_MAX_ROWS + 1, 256, 256, fake, ctypes.byref(p), fake,
                              None, fake, None)
    assert st == 1                                  # SGPT_ERR_INVALID_ARG, before any launch
