"""Pins of the double-precision oracle to facts the pages and mathematics fix.

Each check is independent of the oracle's own routines: brute-force least
squares on the activations X (numpy lstsq, no Cholesky), sub-matrix solves,
closed forms, hand-computed fixtures from the pages, and invariants. The last
test plants plausible mistakes in a copy of the oracle and checks that these
pins catch every one.
"""

import inspect
import itertools
import json
import math
import os

import numpy as np
import pytest

import oracle
from oracle import sparsegpt_ref as ref

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


def _layer(rng, r=6, d=16, n=64, scale_spread=1.0):
    s = np.exp(scale_spread * rng.standard_normal(d))
    X = rng.standard_normal((n, d)) * s
    W = rng.standard_normal((r, d)) / math.sqrt(d)
    return W, X


def _factor(X, damp_ratio=0.01):
    H = oracle.hessian(X)
    Hd, _ = oracle.damp(H, damp_ratio)
    return H, Hd, oracle.inverse_cholesky_upper(Hd)


# ---------------------------------------------------------------- references

def frozen_prefix_sweep(W, Hd, pattern="2:4", forced_mask=None, blocksize=None, qbits=None):
    """Sequential OBS written as explicit least-squares re-fits.

    For each column q in order: decide the mask if the pattern decides here
    (N:M at the first column of each group of M, per row; unstructured at the
    first column of each block of ``blocksize``, over every row of the block
    at once: exactly floor(s * rows * width) pruned, smallest saliency first,
    ties by row then column), with the saliency w_c^2 / [(H_d[c:, c:])^-1]_00
    taken on the current (already re-fitted) weights; set a pruned weight to
    zero, then re-fit every column right of q to minimise
    (w - w^) H_d (w - w^)^T with the columns <= q frozen. Uses general linear
    solves only: no Cholesky, no U, no lazy batching. With ``qbits`` a kept
    weight is set to its grid value (the grid of the input rows) instead and
    the later columns are re-fitted the same way.
    """
    kind, n_keep, m_grp, sparsity = ref.parse_pattern(pattern)
    assert kind == "nm" or forced_mask is not None or blocksize
    r, d = W.shape
    sal_den = np.array([np.linalg.inv(Hd[c:, c:])[0, 0] for c in range(d)])
    w0 = np.array(W, dtype=np.float64)
    cur = w0.copy()
    if qbits:
        qs, qz = oracle.quant_grid(W, qbits)
    mask = np.ones((r, d), dtype=bool) if forced_mask is None else forced_mask.copy()
    for q in range(d):
        if forced_mask is None and kind == "nm" and q % m_grp == 0:
            for row in range(r):
                S = cur[row, q:q + m_grp] ** 2 / sal_den[q:q + m_grp]
                order = sorted(range(m_grp), key=lambda j: (-S[j], j))
                mask[row, q:q + m_grp] = False
                mask[row, [q + j for j in order[:n_keep]]] = True
        if forced_mask is None and kind == "unstructured" and q % blocksize == 0:
            width = min(blocksize, d - q)
            k = int(math.floor(sparsity * r * width))
            keys = sorted((cur[row, q + j] ** 2 / sal_den[q + j], row, j)
                          for row in range(r) for j in range(width))
            mask[:, q:q + width] = True
            for _, row, j in keys[:k]:
                mask[row, q + j] = False
        for row in range(r):
            if not mask[row, q] or qbits:
                if mask[row, q]:
                    cur[row, q] = oracle.quantize(cur[row, q], qs[row], qz[row], qbits)
                else:
                    cur[row, q] = 0.0
                if q + 1 < d:
                    D_fixed = w0[row, :q + 1] - cur[row, :q + 1]
                    rhs = Hd[q + 1:, :q + 1] @ D_fixed
                    D_free = -np.linalg.solve(Hd[q + 1:, q + 1:], rhs)
                    cur[row, q + 1:] = w0[row, q + 1:] - D_free
    return cur, mask


def lstsq_fixed(X, w, fixed_idx, fixed_val):
    """argmin over the free weights of ||X (w - w^)||^2 with some fixed."""
    d = X.shape[1]
    free = [j for j in range(d) if j not in set(fixed_idx)]
    y = X @ w - X[:, fixed_idx] @ np.asarray(fixed_val, dtype=np.float64)
    sol = np.linalg.lstsq(X[:, free], y, rcond=None)[0]
    wh = np.zeros(d)
    wh[fixed_idx] = fixed_val
    wh[free] = sol
    return wh


# ---------------------------------------------------------------- the pins

def test_hessian_hand_example():
    g = _golden("hessian_2x2.json")
    H = oracle.hessian(np.array(g["X_tokens_by_channels"]))
    assert np.array_equal(H, np.array(g["H"]))


def test_hessian_quadratic_form(rng):
    X = rng.standard_normal((37, 9)) * np.exp(rng.standard_normal(9))
    H = oracle.hessian(X, chunk=5)          # chunking must not matter
    v = rng.standard_normal(9)
    assert np.allclose(v @ H @ v, 2.0 / 37 * np.sum((X @ v) ** 2), rtol=1e-12)
    assert np.array_equal(H, H.T)


def test_damping_closed_form():
    d = 10
    H = np.diag(np.arange(1.0, d + 1))
    Hd, lam = oracle.damp(H, 0.01)
    assert lam == pytest.approx(0.01 * (d + 1) / 2, rel=1e-15)
    assert np.allclose(np.diag(Hd), np.arange(1.0, d + 1) + lam, rtol=1e-15)


def test_inverse_cholesky_is_the_unique_factor(rng):
    _, X = _layer(rng, d=12, n=40)
    _, Hd, U = _factor(X)
    assert np.all(np.tril(U, -1) == 0)
    assert np.all(np.diag(U) > 0)
    assert np.allclose(U.T @ U @ Hd, np.eye(12), atol=1e-10)
    # saliency denominator: U_cc^2 = [(H_d[c:, c:])^-1]_00
    for c in range(12):
        assert U[c, c] ** 2 == pytest.approx(np.linalg.inv(Hd[c:, c:])[0, 0], rel=1e-10)


def test_not_positive_definite_raises():
    with pytest.raises(oracle.NotPositiveDefinite):
        oracle.prune_layer(np.ones((2, 4)), H=np.zeros((4, 4)))
    H = np.eye(4)
    H[2, 2] = -50.0
    with pytest.raises(oracle.NotPositiveDefinite):
        oracle.prune_layer(np.ones((2, 4)), H=H)


def test_worked_example_24():
    """Diagonal H: no compensation, 2:4 keeps the two largest |w|."""
    g = _golden("worked_example_24.json")
    W = np.array([g["dense"]])
    out = oracle.prune_layer(W, H=3.0 * np.eye(4), pattern="2:4", blocksize=4)
    assert np.array_equal(out["W"][0], np.array(g["sparse_24"]))
    assert np.flatnonzero(out["mask"][0]).tolist() == g["kept_positions"]
    assert out["meta"][0, 0] == 0 | (3 << 2)
    assert np.array_equal(out["values"][0], np.array([0.42, 0.31]))


def test_single_weight_obs_equals_least_squares(rng):
    """Removing one weight = re-fit of the later weights on X ([SGPT] 八)."""
    W, X = _layer(rng, r=3, d=8, n=50)
    _, Hd, U = _factor(X, damp_ratio=0.0)
    for q in range(8):
        forced = np.ones_like(W, dtype=bool)
        forced[:, q] = False
        out = oracle.sweep(W, U, "2:4", blocksize=4, forced_mask=forced)
        for row in range(3):
            fixed = list(range(q + 1))
            vals = list(W[row, :q]) + [0.0]
            wh = lstsq_fixed(X, W[row], fixed, vals)
            assert np.allclose(out["W"][row], wh, atol=1e-10), (q, row)
    # q = 0 is textbook OBS: delta = -(w_q / [H^-1]_qq) H^-1 e_q
    Hinv = np.linalg.inv(Hd)
    forced = np.ones_like(W, dtype=bool)
    forced[:, 0] = False
    out = oracle.sweep(W, U, "2:4", blocksize=8, forced_mask=forced)
    for row in range(3):
        obs = W[row] - W[row, 0] / Hinv[0, 0] * Hinv[:, 0]
        assert np.allclose(out["W"][row], obs, atol=1e-12)


@pytest.mark.parametrize("blocksize", [4, 8, 16])
def test_sweep_equals_frozen_prefix_least_squares(rng, blocksize):
    W, X = _layer(rng, r=5, d=16, n=60, scale_spread=1.5)
    _, Hd, U = _factor(X)
    out = oracle.sweep(W, U, "2:4", blocksize=blocksize)
    ref_W, ref_mask = frozen_prefix_sweep(W, Hd, "2:4")
    assert np.array_equal(out["mask"], ref_mask)
    assert np.allclose(out["W"], ref_W, atol=1e-11)
    # forced, arbitrary (non-2:4) mask
    forced = rng.random(W.shape) < 0.6
    out = oracle.sweep(W, U, "2:4", blocksize=blocksize, forced_mask=forced)
    ref_W, _ = frozen_prefix_sweep(W, Hd, "2:4", forced_mask=forced)
    assert np.allclose(out["W"], ref_W, atol=1e-11)


@pytest.mark.parametrize("blocksize,sparsity", [(4, 0.5), (8, 0.7), (8, 0.5), (16, 0.8)])
def test_unstructured_sweep_equals_frozen_prefix_least_squares(rng, blocksize, sparsity):
    """Unstructured selection across blocks ([SGPT] 八 and 十一 step four):
    every block after the first is scored on weights that earlier blocks
    compensated, over all rows at once; non-diagonal H, 3 to 6 blocks."""
    W, X = _layer(rng, r=6, d=24, n=70, scale_spread=1.5)
    _, Hd, U = _factor(X)
    pat = f"unstructured:{sparsity}"
    out = oracle.sweep(W, U, pat, blocksize=blocksize)
    ref_W, ref_mask = frozen_prefix_sweep(W, Hd, pat, blocksize=blocksize)
    assert np.array_equal(out["mask"], ref_mask)
    assert np.allclose(out["W"], ref_W, atol=1e-11)
    for b0 in range(0, 24, blocksize):
        width = min(blocksize, 24 - b0)
        assert (~ref_mask[:, b0:b0 + width]).sum() == math.floor(sparsity * 6 * width)


def test_diagonal_hessian_is_wanda_and_magnitude(rng):
    """H diagonal: U diagonal, no compensation, keep the largest w^2 H_ii."""
    r, d, n = 7, 16, 64
    # tokens that each excite one channel give an exactly diagonal X^T X
    X = np.zeros((n, d))
    X[np.arange(n), np.arange(n) % d] = rng.standard_normal(n) * 3
    W = rng.standard_normal((r, d))
    out = oracle.prune_layer(W, X=X, pattern="2:4", damp_ratio=0.0, blocksize=8)
    kept = out["mask"]
    assert np.array_equal(out["W"][kept], W[kept])           # bit-unchanged
    assert np.all(out["W"][~kept] == 0.0)
    wanda = np.abs(W) * np.linalg.norm(X, axis=0)            # [SGPT] 十八
    for g in range(d // 4):
        top2 = np.argsort(-wanda[:, 4 * g:4 * g + 4], axis=1, kind="stable")[:, :2]
        for row in range(r):
            assert set(np.flatnonzero(kept[row, 4 * g:4 * g + 4])) == set(top2[row])
    # H = c I: plain magnitude pruning ([SGPT] 五)
    out = oracle.prune_layer(W, H=2.5 * np.eye(d), pattern="2:4")
    for g in range(d // 4):
        top2 = np.argsort(-np.abs(W[:, 4 * g:4 * g + 4]), axis=1, kind="stable")[:, :2]
        for row in range(r):
            assert set(np.flatnonzero(out["mask"][row, 4 * g:4 * g + 4])) == set(top2[row])


def test_never_below_brute_force_optimum(rng):
    """d_in = 8: compare with all C(4,2)^2 = 36 masks, each optimally re-fit."""
    W, X = _layer(rng, r=4, d=8, n=40, scale_spread=1.0)
    out = oracle.prune_layer(W, X=X, pattern="2:4", blocksize=8)
    pairs = list(itertools.combinations(range(4), 2))
    for row in range(4):
        err_sgpt = np.sum((X @ (W[row] - out["W"][row])) ** 2)
        best = math.inf
        own = None
        for a, b in itertools.product(pairs, pairs):
            keep = list(a) + [4 + j for j in b]
            pruned = [j for j in range(8) if j not in keep]
            wh = np.zeros(8)
            wh[keep] = np.linalg.lstsq(X[:, keep], X @ W[row], rcond=None)[0]
            err = np.sum((X @ (W[row] - wh)) ** 2)
            best = min(best, err)
            if not out["mask"][row, pruned].any():
                own = err
        assert err_sgpt >= best * (1 - 1e-12)
        assert err_sgpt >= own * (1 - 1e-12)


def test_exact_counts_and_compression_table(rng):
    W, X = _layer(rng, r=12, d=32, n=80)
    _, _, U = _factor(X)
    out = oracle.sweep(W, U, "2:4", blocksize=16)
    groups = out["mask"].reshape(12, 8, 4).sum(axis=2)
    assert np.all(groups == 2)
    assert np.all(out["W"][~out["mask"]] == 0.0)
    for ratio, approx in _golden("compression_table.json")["rows"]:
        s = 1.0 - 1.0 / ratio
        assert abs(s - approx) < 0.005
        out = oracle.sweep(W, U, f"unstructured:{s}", blocksize=16)
        for b0 in range(0, 32, 16):
            pruned = (~out["mask"][:, b0:b0 + 16]).sum()
            assert pruned == math.floor(s * 12 * 16)
        assert np.all(out["W"][~out["mask"]] == 0.0)


def test_unstructured_picks_smallest_saliency_with_tiebreak():
    # U = I: saliency = w^2; equal magnitudes tie and break by (row, col)
    W = np.array([[1.0, -1.0, 3.0, 1.0],
                  [2.0, 1.0, -1.0, 5.0]])
    out = oracle.sweep(W, np.eye(4), "unstructured:0.5", blocksize=4)
    # k = 4 pruned: the five |w| = 1 entries in (row, col) order, first four
    expect = np.ones_like(W, dtype=bool)
    for rc in [(0, 0), (0, 1), (0, 3), (1, 1)]:
        expect[rc] = False
    assert np.array_equal(out["mask"], expect)
    # all pruned saliencies <= all kept ones on a random tile
    rng = np.random.default_rng(3)
    W = rng.standard_normal((9, 8))
    U = np.diag(rng.uniform(0.5, 2.0, 8))
    out = oracle.sweep(W, U, "unstructured:0.7", blocksize=8)
    S = (W / np.diag(U)) ** 2
    assert S[~out["mask"]].max() <= S[out["mask"]].min()
    assert (~out["mask"]).sum() == math.floor(0.7 * 72)


def test_telescoping_loss(rng):
    W, X = _layer(rng, r=6, d=24, n=70)
    _, Hd, U = _factor(X)
    for pat in ["2:4", "unstructured:0.6"]:
        out = oracle.sweep(W, U, pat, blocksize=8)
        dW = W - out["W"]
        assert out["loss"].sum() == pytest.approx(np.trace(dW @ Hd @ dW.T), rel=1e-10)
        assert np.allclose(out["loss"], np.einsum("ij,jk,ik->i", dW, Hd, dW), rtol=1e-10)


def test_scale_invariance(rng):
    W, X = _layer(rng, r=5, d=16, n=50)
    a = oracle.prune_layer(W, X=X, pattern="2:4", blocksize=8)
    b = oracle.prune_layer(W, X=3.0 * X, pattern="2:4", blocksize=8)
    assert np.array_equal(a["mask"], b["mask"])
    assert np.allclose(a["W"], b["W"], rtol=1e-10, atol=1e-13)
    c = oracle.prune_layer(W * np.array([[2.0], [1], [0.5], [4], [1]]), X=X,
                           pattern="2:4", blocksize=8)
    assert np.array_equal(a["mask"], c["mask"])
    assert np.allclose(c["W"][0], 2.0 * a["W"][0], rtol=1e-12, atol=1e-14)


def test_blocksize_and_row_independence(rng):
    W, X = _layer(rng, r=6, d=32, n=90, scale_spread=1.2)
    _, _, U = _factor(X)
    outs = [oracle.sweep(W, U, "2:4", blocksize=b) for b in (4, 8, 16, 32)]
    for o in outs[1:]:
        assert np.array_equal(o["mask"], outs[0]["mask"])
        assert np.allclose(o["W"], outs[0]["W"], atol=1e-12)
    sub = oracle.sweep(W[[1, 4]], U, "2:4", blocksize=16)
    assert np.array_equal(sub["mask"], outs[2]["mask"][[1, 4]])
    assert np.allclose(sub["W"], outs[2]["W"][[1, 4]], atol=1e-14)


def test_pack_roundtrip_and_bits(rng):
    W, X = _layer(rng, r=5, d=64, n=100)
    out = oracle.prune_layer(W, X=X, pattern="2:4", blocksize=32)
    back = oracle.unpack24(out["values"], out["meta"], 64)
    assert np.array_equal(back, out["W"])
    words = oracle.mask_bits(out["mask"])
    assert words.shape == (5, 2) and words.dtype == np.uint32
    assert np.array_equal(oracle.bits_to_mask(words, 64), out["mask"])
    bad = out["mask"].copy()
    bad[0, :4] = True
    with pytest.raises(ValueError):
        oracle.pack24(out["W"], bad)


def test_pack_and_mask_word_layout_beyond_the_first_word():
    """Hand-derived words for groups 8..15 and columns 32..63 of two rows
    (golden file, [2:4] section on the 2:4 mechanism): pins the word index
    and the shift of both the metadata and the mask bits, in both
    directions."""
    g = _golden("pack24_layout_64.json")
    d = g["d_in"]
    rows = len(g["kept_pairs"])
    W = np.array([[1000.0 * (r + 1) + c for c in range(d)] for r in range(rows)])
    mask = np.zeros((rows, d), dtype=bool)
    for r, pairs in enumerate(g["kept_pairs"]):
        for grp, (a, b) in enumerate(pairs):
            mask[r, 4 * grp + a] = mask[r, 4 * grp + b] = True
    Wm = np.where(mask, W, 0.0)
    meta_want = np.array([[int(h, 16) for h in row] for row in g["meta_words_hex"]], dtype=np.uint32)
    mask_want = np.array([[int(h, 16) for h in row] for row in g["mask_words_hex"]], dtype=np.uint32)
    values, meta = oracle.pack24(Wm, mask)
    assert np.array_equal(meta, meta_want)
    assert np.array_equal(values[:, 16:32], np.array(g["values_groups_8_to_15"], dtype=np.float64))
    assert np.array_equal(oracle.mask_bits(mask), mask_want)
    # and back: the golden words alone decode to the same matrices
    assert np.array_equal(oracle.bits_to_mask(mask_want, d), mask)
    assert np.array_equal(oracle.unpack24(values, meta_want, d), Wm)


def test_pack_nm_hand_derived_words():
    """General N:M layout (golden file): 3-bit positions of a 4:8 row, and
    5-bit positions of a 16:32 row that run across word boundaries."""
    g = _golden("pack_nm_layout.json")
    for case in g["cases"]:
        n, m = (int(x) for x in case["pattern"].split(":"))
        d = case["d_in"]
        W = np.array([[100.0 + c for c in range(d)]])
        mask = np.zeros((1, d), dtype=bool)
        for grp, kept in enumerate(case["kept"]):
            mask[0, [m * grp + j for j in kept]] = True
        Wm = np.where(mask, W, 0.0)
        values, meta = oracle.pack_nm(Wm, mask, n, m)
        want = np.array([[int(h, 16) for h in case["meta_words_hex"]]], dtype=np.uint32)
        assert np.array_equal(meta, want), case["pattern"]
        assert np.array_equal(values[0], np.array(case["values"], dtype=np.float64))
        assert np.array_equal(oracle.unpack_nm(values, want, d, n, m), Wm)


def test_pack_nm_reduces_to_pack24_and_round_trips(rng):
    W, X = _layer(rng, r=5, d=128, n=200)
    out = oracle.prune_layer(W, X=X, pattern="2:4", blocksize=64)
    v24, m24 = oracle.pack24(out["W"], out["mask"])
    v, m = oracle.pack_nm(out["W"], out["mask"], 2, 4)
    assert np.array_equal(v, v24) and np.array_equal(m, m24)
    for pat in ["1:4", "3:4", "4:8", "16:32", "16:64", "16:128", "8:16"]:
        n, mm = (int(x) for x in pat.split(":"))
        o = oracle.prune_layer(W, X=X, pattern=pat, blocksize=128)
        groups = o["mask"].reshape(5, -1, mm).sum(axis=2)
        assert np.all(groups == n), pat
        assert np.array_equal(oracle.unpack_nm(o["values"], o["meta"], 128, n, mm), o["W"]), pat
        b = mm.bit_length() - 1
        assert o["meta"].shape == (5, (128 // mm * n * b + 31) // 32)
    with pytest.raises(ValueError):
        oracle.pack_nm(out["W"], np.ones_like(out["mask"]), 4, 8)


@pytest.mark.parametrize("pattern", ["1:4", "3:4", "4:8", "8:16"])
def test_nm_sweep_equals_frozen_prefix_least_squares(rng, pattern):
    """N of M on the compensated weights at each group start ([SGPT] 十四
    14.4), against the general-solve reference, across several blocks."""
    W, X = _layer(rng, r=5, d=32, n=80, scale_spread=1.5)
    _, Hd, U = _factor(X)
    out = oracle.sweep(W, U, pattern, blocksize=16)
    ref_W, ref_mask = frozen_prefix_sweep(W, Hd, pattern)
    assert np.array_equal(out["mask"], ref_mask)
    assert np.allclose(out["W"], ref_W, atol=1e-11)


def test_quant_grid_hand_examples():
    g = _golden("quant_grid.json")
    for case in g["cases"]:
        bits = case["bits"]
        scale, zero = oracle.quant_grid(np.array([case["row"]]), bits)
        want_scale = (np.float32(case["scale_fraction"][0]) / np.float32(case["scale_fraction"][1])
                      if "scale_fraction" in case else np.float32(case["scale"]))
        assert scale[0] == np.float32(want_scale) and zero[0] == case["zero"]
        q = oracle.quantize(np.array(case["x"]), scale[0], zero[0], bits)
        if "q" in case:
            assert np.array_equal(q, np.array(case["q"]))
        else:
            assert np.array_equal(q, np.float64(scale[0]) * np.array(case["q_codes"], dtype=np.float64))


def test_quantized_sweep_diagonal_hessian_is_rounding(rng):
    """Diagonal H: no compensation, so every survivor is exactly its grid
    value and the mask is the one the unquantized sweep takes."""
    r, d, n = 6, 32, 64
    X = np.zeros((n, d))
    X[np.arange(n), np.arange(n) % d] = rng.standard_normal(n) * 3
    W = rng.standard_normal((r, d)).astype(np.float32).astype(np.float64)
    for bits in (3, 4, 8):
        a = oracle.prune_layer(W, X=X, pattern="2:4", damp_ratio=0.0, blocksize=16, qbits=bits)
        b = oracle.prune_layer(W, X=X, pattern="2:4", damp_ratio=0.0, blocksize=16)
        assert np.array_equal(a["mask"], b["mask"])
        s_, z_ = oracle.quant_grid(W, bits)
        want = np.where(a["mask"], oracle.quantize(W, s_[:, None], z_[:, None], bits), 0.0)
        assert np.array_equal(a["W"], want)


@pytest.mark.parametrize("pattern,bits", [("2:4", 4), ("4:8", 3), ("unstructured:0.5", 4), ("unstructured:0.0", 3)])
def test_quantized_sweep_equals_frozen_prefix_least_squares(rng, pattern, bits):
    """Joint pruning and quantization ([SGPT] 十五, 十七) against the
    general-solve reference: every pruned or quantized weight is frozen and
    the later columns re-fitted."""
    W, X = _layer(rng, r=5, d=24, n=70, scale_spread=1.5)
    _, Hd, U = _factor(X)
    out = oracle.sweep(W, U, pattern, blocksize=8, qbits=bits)
    ref_W, ref_mask = frozen_prefix_sweep(W, Hd, pattern, blocksize=8, qbits=bits)
    assert np.array_equal(out["mask"], ref_mask)
    assert np.allclose(out["W"], ref_W, atol=1e-11)
    s_, z_ = oracle.quant_grid(W, bits)
    on_grid = np.where(out["mask"], oracle.quantize(out["W"], s_[:, None], z_[:, None], bits), 0.0)
    assert np.allclose(out["W"], on_grid, atol=1e-12)      # every survivor sits on its row's grid
    dW = W - out["W"]
    assert out["loss"].sum() == pytest.approx(np.trace(dW @ Hd @ dW.T), rel=1e-10)


# ---------------------------------------------------------------- mutations

_MUTATIONS = [
    # (name, [(old, new), ...], pattern, blocksize)
    ("wrong sign of the compensation", [("W1[:, q:] -= np.outer(e, U[c, c:i2])",
                                         "W1[:, q:] += np.outer(e, U[c, c:i2])")], "2:4", 8),
    ("dropped lazy trailing update", [("W[:, i2:] -= E1 @ U[i1:i2, i2:]", "pass")], "2:4", 8),
    ("transposed U in the trailing update", [("W[:, i2:] -= E1 @ U[i1:i2, i2:]",
                                              "W[:, i2:] -= E1 @ U.T[i1:i2, i2:]")], "2:4", 8),
    ("error not divided by U_qq", [("e = (w - p) / U[c, c]", "e = (w - p)")], "2:4", 8),
    ("saliency on the starting weights",
     [("S = (W1[:, q:q + m_grp] / diagU[c:c + m_grp]) ** 2",
       "S = (W[:, c:c + m_grp] / diagU[c:c + m_grp]) ** 2")], "2:4", 8),
    ("saliency without U", [("S = (W1[:, q:q + m_grp] / diagU[c:c + m_grp]) ** 2",
                             "S = (W1[:, q:q + m_grp]) ** 2")], "2:4", 8),
    ("off-by-one in the rank-1 update", [("W1[:, q:] -= np.outer(e, U[c, c:i2])",
                                          "W1[:, q + 1:] -= np.outer(e, U[c, c:i2 - 1])")], "2:4", 8),
    # the unstructured branch scored on the weights as they were before any
    # earlier block compensated them
    ("unstructured saliency on the starting weights",
     [("W = np.array(W, dtype=np.float64, copy=True)",
       "W_start = np.array(W, dtype=np.float64, copy=True); W = W_start.copy()"),
      ("S = (W1 / diagU[i1:i2]) ** 2", "S = (W_start[:, i1:i2] / diagU[i1:i2]) ** 2")],
     "unstructured:0.5", 4),
    ("unstructured saliency without U", [("S = (W1 / diagU[i1:i2]) ** 2", "S = W1 ** 2")],
     "unstructured:0.5", 4),
    ("unstructured count rounded up",
     [("k = int(math.floor(sparsity * r * width))", "k = int(math.ceil(sparsity * r * width))")],
     "unstructured:0.53", 4),
    # joint quantization: the grid error left uncompensated, and the grid
    # value taken of the weight before this block's updates
    ("quantization error not compensated",
     [("e = (w - p) / U[c, c]", "e = (w - np.where(mask[:, c], w, 0.0)) / U[c, c]")], ("2:4", 4), 8),
    ("quantized before the in-block updates",
     [("kept = quantize(w, qscale, qzero, qbits) if qbits else w",
       "kept = quantize(W[:, c], qscale, qzero, qbits) if qbits else w")], ("2:4", 4), 8),
]


@pytest.mark.parametrize("name,edits,pattern,blocksize", _MUTATIONS, ids=[m[0] for m in _MUTATIONS])
def test_pins_catch_planted_mistakes(name, edits, pattern, blocksize):
    src = inspect.getsource(ref.sweep)
    for old, new in edits:
        assert old in src, name
        src = src.replace(old, new)
    ns = dict(vars(ref))
    exec(src, ns)
    mutated = ns["sweep"]
    # own seed: the verdict must not depend on which tests ran before
    W, X = _layer(np.random.default_rng(2024), r=16, d=32, n=80, scale_spread=1.5)
    _, Hd, U = _factor(X)
    qbits = None
    if isinstance(pattern, tuple):          # (pattern, bits): the quantized sweep
        pattern, qbits = pattern
    got = mutated(W, U, pattern, blocksize=blocksize, qbits=qbits)
    ref_W, ref_mask = frozen_prefix_sweep(W, Hd, pattern, blocksize=blocksize, qbits=qbits)
    same = np.array_equal(got["mask"], ref_mask) and np.allclose(got["W"], ref_W, atol=1e-9)
    assert not same, f"pins did not catch: {name}"
