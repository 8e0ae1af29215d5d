"""Shared helpers of the GPU parity tests: run the CUDA path through the
C ABI and the float64 oracle on the same seeded bytes, and measure the
agreement the way the solver's acceptance criteria state it:

* mask agreement >= 99.9%, every disagreement a near-tie (competing saliencies
  within 1e-5 relative at the moment the decision was made);
* surviving weights within 1e-3 relative L2 of the oracle run on the GPU's
  mask (forced-mask mode, so a near-tie flip does not cascade);
* 2:4 values and metadata bit-exact given identical masks;
* relative layer reconstruction error within 1% of the oracle's.
"""

from __future__ import annotations

import math

import numpy as np
import torch

import oracle
import post_pruning_b200 as pp

MASK_AGREEMENT = 0.999
NEAR_TIE = 1e-5
WEIGHT_REL_L2 = 1e-3
RECON_REL = 0.01
CODE_NEAR_TIE = 1e-3     # code units from the rounding boundary


def f32(x) -> float:
    """The float32 value the C ABI receives for a float parameter."""
    return float(np.float32(x))


def pattern_of(p: pp.Params) -> str:
    return p.pattern if p.is_nm else f"unstructured:{f32(p.sparsity)!r}"


def gpu_prune_layer(W: torch.Tensor, X: torch.Tensor | None, p: pp.Params,
                    H_sum: torch.Tensor | None = None, n_tok: int | None = None,
                    forced_mask: np.ndarray | None = None, check=True) -> dict:
    """W (cpu fp32), X (bf16, cpu or cuda) -> host results of the CUDA path."""
    dev = torch.device("cuda")
    r, d = W.shape
    n = X.shape[0] if X is not None else n_tok
    bufs = pp.LayerBuffers.allocate(r, d, n, dev, nm=p.nm if p.is_nm else (2, 4))
    Wd = W.to(dev).contiguous()
    Xd = X.to(dev).contiguous() if X is not None else None
    if H_sum is not None:
        bufs.H.copy_(H_sum.to(dev))
    if forced_mask is not None:
        bufs.mask.copy_(torch.from_numpy(oracle.mask_bits(forced_mask).view(np.int32)))
    bufs.run(Wd, Xd, p)
    status = pp.sync_status(bufs.info)
    if check:
        assert status == 0, f"device status {status}"
    out = {
        "status": status,
        "W": Wd.cpu().numpy(),
        "mask": oracle.bits_to_mask(bufs.mask.cpu().numpy().view(np.uint32), d),
        "row_loss": bufs.row_loss.cpu().numpy().astype(np.float64),
        "U": bufs.U.cpu().numpy(),
        "H": bufs.H.cpu().numpy(),
    }
    if p.is_nm:
        out["values"] = bufs.values.cpu().numpy()
        out["meta"] = bufs.meta.cpu().numpy().view(np.uint32)
    return out


def nm_decisions_disagree(mask_gpu: np.ndarray, S_dec: np.ndarray, n_keep=2, m=4):
    """Groups where the GPU's kept set differs from the top-n of S_dec, and
    the relative gap between the n-th and (n+1)-th saliency of each group."""
    r, d = mask_gpu.shape
    S = S_dec.reshape(r, d // m, m)
    order = np.argsort(-S, axis=2, kind="stable")
    want = np.zeros_like(S, dtype=bool)
    np.put_along_axis(want, order[:, :, :n_keep], True, axis=2)
    got = mask_gpu.reshape(r, d // m, m)
    differ = np.any(want != got, axis=2)
    s_sorted = -np.sort(-S, axis=2)
    a, b = s_sorted[:, :, n_keep - 1], s_sorted[:, :, n_keep]
    gap = (a - b) / np.maximum(np.abs(a), 1e-300)
    return differ, gap


def unstructured_disagree(mask_gpu: np.ndarray, S_dec: np.ndarray, sparsity: float, blocksize: int):
    """Per block: entries where the GPU's decision differs from the k smallest
    S_dec, and their relative distance to the block's k-th smallest S."""
    r, d = mask_gpu.shape
    differ = np.zeros_like(mask_gpu)
    dist = np.full(mask_gpu.shape, np.inf)
    for i1 in range(0, d, blocksize):
        i2 = min(d, i1 + blocksize)
        S = S_dec[:, i1:i2]
        k = int(math.floor(sparsity * r * (i2 - i1)))
        flat = S.ravel()
        if k == 0:
            continue
        thr = np.partition(flat, k - 1)[k - 1]
        want_pruned = np.zeros(flat.shape, dtype=bool)
        want_pruned[np.lexsort((np.arange(flat.size), flat))[:k]] = True
        got_pruned = ~mask_gpu[:, i1:i2].ravel()
        dd = (want_pruned != got_pruned).reshape(S.shape)
        differ[:, i1:i2] = dd
        dist[:, i1:i2] = np.abs(S - thr) / max(abs(thr), 1e-300)
    return differ, dist


def sample_rows(d_out: int, count: int = 256) -> np.ndarray:
    """Evenly spaced rows across the matrix (every 128-row tile is met once
    the count allows) plus the last row, for checks on a row sample."""
    step = max(1, d_out // count)
    return np.unique(np.r_[np.arange(0, d_out, step), d_out - 1])


def restrict(gpu: dict, rows: np.ndarray) -> dict:
    """The per-row outputs of a GPU run on a subset of rows."""
    keys = ("W", "mask", "row_loss", "values", "meta")
    return {k: (v[rows] if k in keys else v) for k, v in gpu.items()}


def compare(gpu: dict, W0: np.ndarray, H: np.ndarray, U: np.ndarray, p: pp.Params,
            rows: np.ndarray | None = None) -> dict:
    """All parity metrics of one GPU run against the oracle (given H, U).

    With ``rows`` the oracle sweeps only those rows of W0 and the GPU's
    outputs are compared on the same rows. N:M decisions and compensation
    stay inside a row, so the oracle's result on a row subset equals those
    rows of its full result (row independence); unstructured selection is
    coupled across rows and is always compared on every row."""
    if rows is not None:
        assert p.is_nm, "a row sample is exact only for N:M patterns"
        gpu = restrict(gpu, rows)
        W0 = W0[rows]
    pat = pattern_of(p)
    qb = p.qbits or None
    free = oracle.sweep(W0, U, pat, p.blocksize, qbits=qb)
    # the oracle along the GPU's decisions: its mask and, with quantization,
    # the grid values it chose for the kept weights
    forced = oracle.sweep(W0, U, pat, p.blocksize, forced_mask=gpu["mask"], qbits=qb,
                          forced_values=gpu["W"].astype(np.float64) if qb else None)
    m = {}
    m["mask_agree_free"] = float(np.mean(gpu["mask"] == free["mask"]))
    if p.is_nm:
        differ, gap = nm_decisions_disagree(gpu["mask"], forced["S_dec"], *p.nm)
        m["decisions"] = differ.size
        m["decision_flips"] = int(differ.sum())
        m["flip_max_gap"] = float(gap[differ].max()) if differ.any() else 0.0
        m["decision_agree"] = 1.0 - differ.mean()
    else:
        differ, dist = unstructured_disagree(gpu["mask"], forced["S_dec"], f32(p.sparsity), p.blocksize)
        m["decisions"] = differ.size
        m["decision_flips"] = int(differ.sum())
        m["flip_max_gap"] = float(dist[differ].max()) if differ.any() else 0.0
        m["decision_agree"] = 1.0 - differ.mean()
    ref = forced["W"]
    if qb:
        # integer codes of the kept weights: the GPU's against the code the
        # oracle would pick for the weight its column had along the GPU's
        # trajectory; a differing code must be a rounding near-tie (the
        # weight within 1e-3 of a code step of the boundary)
        scale, zero = oracle.quant_grid(W0, qb)
        sc = scale[:, None].astype(np.float64)
        kept = gpu["mask"]
        cg = np.rint(gpu["W"].astype(np.float64) / sc)
        t = forced["W_dec"] / sc
        lo, hi = -zero[:, None].astype(np.float64), (2 ** qb - 1) - zero[:, None].astype(np.float64)
        co = np.clip(np.rint(t), lo, hi)
        diff = kept & (cg != co)
        m["code_agree"] = float(1.0 - diff.sum() / max(kept.sum(), 1))
        m["code_flip_max_gap"] = float(np.max(np.abs(np.abs(t - np.floor(t)) - 0.5)[diff])) if diff.any() else 0.0
        m["on_grid"] = bool(np.all(np.abs(gpu["W"] / scale[:, None] - cg) < 1e-3))
        # the weights themselves: the oracle along the GPU's mask alone
        # (its own codes), as for unquantized runs
        ref = oracle.sweep(W0, U, pat, p.blocksize, forced_mask=gpu["mask"], qbits=qb)["W"]
    m["weight_rel_l2"] = float(np.linalg.norm(gpu["W"] - ref) / max(np.linalg.norm(ref), 1e-300))
    num_g, den = oracle.recon_error(W0, gpu["W"], H)
    num_o, _ = oracle.recon_error(W0, free["W"], H)
    m["recon_gpu"] = num_g / den
    m["recon_oracle"] = num_o / den
    m["recon_rel_diff"] = abs(num_g - num_o) / max(num_o, 1e-300)
    if "row_loss" in gpu:
        m["loss_rel"] = float(np.abs(gpu["row_loss"].sum() - forced["loss"].sum()) /
                              max(forced["loss"].sum(), 1e-300))
    m["pruned_zero"] = bool(np.all(gpu["W"][~gpu["mask"]] == 0.0))
    if p.is_nm:
        n_keep, m_grp = p.nm
        groups = gpu["mask"].reshape(gpu["mask"].shape[0], -1, m_grp).sum(axis=2)
        m["exact_nm"] = bool(np.all(groups == n_keep))
        vals, meta = oracle.pack_nm(gpu["W"].astype(np.float64), gpu["mask"], n_keep, m_grp)
        if "values" in gpu:
            m["pack_exact"] = bool(np.array_equal(vals.astype(np.float32), gpu["values"])
                               and np.array_equal(meta, gpu["meta"]))
    else:
        r, d = gpu["mask"].shape
        counts = []
        for i1 in range(0, d, p.blocksize):
            i2 = min(d, i1 + p.blocksize)
            counts.append(int((~gpu["mask"][:, i1:i2]).sum()) == math.floor(f32(p.sparsity) * r * (i2 - i1)))
        m["exact_count"] = all(counts)
    return m


def assert_parity(m: dict, p: pp.Params):
    assert m["pruned_zero"]
    if p.is_nm:
        assert m["exact_nm"]
        assert m.get("pack_exact", True)
    else:
        assert m["exact_count"]
    # the literal criterion: the GPU's mask against the oracle's own run ...
    assert m["mask_agree_free"] >= MASK_AGREEMENT, m
    # ... and every decision the GPU took against the oracle re-run along the
    # GPU's mask trajectory, each differing one a near-tie
    assert m["decision_agree"] >= MASK_AGREEMENT, m
    assert m["flip_max_gap"] < NEAR_TIE, m
    if "code_agree" in m:
        assert m["on_grid"], m
        assert m["code_agree"] >= MASK_AGREEMENT, m
        assert m["code_flip_max_gap"] < CODE_NEAR_TIE, m
        # along the GPU's own decisions the per-row losses agree closely
        assert m.get("loss_rel", 0.0) <= 1e-4, m
    else:
        assert m["weight_rel_l2"] <= WEIGHT_REL_L2, m
    assert m["recon_rel_diff"] <= RECON_REL, m
