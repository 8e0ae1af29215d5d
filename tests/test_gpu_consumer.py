"""The 2:4 consumer (sgpt_sparse24_linear) against the float64 oracle: Y =
X W^T computed on the sparse tensor cores from W's packed form only (the
kept values and sgpt_pack24's metadata words) must equal the dense product
of the oracle's unpacking of that same packed form. A wrong metadata layout,
bit order or value order gives a wrong product, so this checks the packing
semantically (2:4 production guide, section on the 2:4 mechanism)."""

import numpy as np
import pytest
import torch

import oracle
import post_pruning_b200 as pp
from oracle import mlp_block_ref as mb

pytestmark = pytest.mark.gpu


def _f64(t):
    return t.detach().cpu().to(torch.float64).numpy()


# ragged in every dimension: rows past a 256-row tile, K past a 128-K stage
# (d_in = 320, 96), tokens past a 128-token tile; one tile; many tiles per CTA
@pytest.mark.parametrize("d_out,d_in,n", [(256, 256, 384), (224, 320, 1000), (384, 1024, 130), (128, 128, 1),
                                          (520, 96, 300), (1024, 512, 40000)])
def test_sparse24_linear_matches_unpacked_product(d_out, d_in, n):
    dev = torch.device("cuda")
    g = torch.Generator().manual_seed(d_out + d_in + n)
    W = torch.randn(d_out, d_in, generator=g)
    # a 2:4 mask: two random positions of every four
    scores = torch.rand(d_out, d_in // 4, 4, generator=g)
    keep = torch.zeros_like(scores, dtype=torch.bool)
    keep.scatter_(2, scores.topk(2, dim=2).indices, True)
    keep = keep.reshape(d_out, d_in)
    W = torch.where(keep, W, torch.zeros_like(W))
    mask = torch.from_numpy(oracle.mask_bits(keep.numpy()).view(np.int32)).to(dev)
    Wd = W.to(dev)
    vals = torch.empty(d_out, d_in // 2, device=dev)
    meta = torch.empty(d_out, d_in // 32, dtype=torch.int32, device=dev)
    info = pp.new_info()
    pp.pack24(Wd, mask, vals, meta, info)
    vb = torch.empty(d_out, d_in // 2, dtype=torch.bfloat16, device=dev)
    pp.to_bf16(vals, vb, info)
    X = (torch.randn(n, d_in, generator=g) * 2).to(torch.bfloat16)
    Y = torch.full((n, d_out), float("nan"), device=dev)
    tiles = pp.sparse24_meta_tiles(meta, d_in)
    pp.sparse24_linear(vb, tiles, X.to(dev), Y, info)
    pp.raise_on_info(info)
    # the oracle's reading of the packed form, then the dense product
    W_hat = oracle.unpack24(_f64(vb), meta.cpu().numpy().view(np.uint32), d_in)
    assert np.array_equal(W_hat, mb.bf16_round(W.numpy().astype(np.float64)))
    Xf = _f64(X)
    ref = Xf @ W_hat.T
    bound = np.abs(Xf) @ np.abs(W_hat).T
    err = np.abs(Y.cpu().numpy() - ref)
    assert np.all(err <= 1e-5 * bound + 1e-30), float((err / (bound + 1e-30)).max())
    # and the dense tensor-core product of the same weights agrees (its
    # entry point takes output widths that are multiples of 32)
    if d_out % 32:
        return
    Wb = torch.from_numpy(W_hat).to(torch.bfloat16).to(dev)
    Yd = torch.empty(n, d_out, device=dev)
    pp.linear_bf16(X.to(dev), Wb, Yd, info)
    pp.raise_on_info(info)
    assert torch.allclose(Y, Yd, rtol=1e-5, atol=1e-4)
