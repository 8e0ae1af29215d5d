"""Double-precision CPU oracle of SparseGPT's layer-wise one-shot pruning solver.

TEST INFRASTRUCTURE ONLY. Only the tests, ``__graft_entry__.smoke()`` and the
CPU-baseline leg of ``bench.py`` may import this module. The CUDA path never
calls it, and it shares no code with the CUDA path.

It is deliberately plain: float64 numpy, the algorithm's steps in the order the
pages state them, library primitives (matrix product, Cholesky, triangular
solve, sort) used as single steps, no blocking or fusion beyond what the
algorithm itself prescribes.

Sources (web pages; cited by title and section):
* [SGPT] review of "SparseGPT: Massive Language Models Can Be Accurately Pruned
  in One-Shot" (Frantar & Alistarh, ICML 2023), devpress.csdn.net:
  section 六 (the layer objective: find a sparse W^ with W^X close to WX),
  section 七 (the Hessian proxy H = X X^T), section 八 (Optimal Brain Surgeon:
  remove one weight, update the remaining weights of the same row to
  compensate, using the inverse Hessian), section 十一 (the six-step pipeline;
  step four processes the weight columns block by block), section 十四 14.4
  (N:M semi-structured sparsity such as 2:4).
* [2:4] "LLM 2:4 structured sparsity production guide" (oh-bug.com), section
  "2:4 结构化稀疏的核心机制与生产状态分类": keep 2 of every 4 consecutive
  weights and record the kept positions in 2-bit metadata; worked example
  [0.42, -0.18, 0.07, 0.31] -> [0.42, 0, 0, 0.31].
* [FT] review of "Sparse Fine-tuning for Inference Acceleration of Large
  Language Models" (tqpw.cn), section 八 8.4: the GPU formats 2:4, 16:32,
  16:64 and 16:128 (keep N of every M consecutive weights), the kept
  positions recorded alongside the values.

Readings where the pages are silent (each is listed in the design notes):
* scale 2/n on H with n the number of token rows (a scalar; results do not
  depend on it because damping is relative);
* damping lambda = damp * mean(diag H), added once to the diagonal; a matrix
  that is still not positive definite is an error, never retried;
* the upper Cholesky factor U of H_d^-1 (H_d^-1 = U^T U) is formed by
  Cholesky of H_d, triangular inverse, Cholesky of the inverse;
* blocks of ``blocksize`` consecutive columns; the error of each column is
  e = (w_q - p_q) / U_qq, applied to the rest of the block by a rank-1 update
  and to the columns right of the block by one product after the block;
* N:M masks are decided at the first column of each group of M, on the weights
  as updated so far, keeping the N largest saliencies w_c^2 / U_cc^2 (equal
  saliency: the lower column wins);
* unstructured masks are decided at the start of each block over the whole
  d_out x block tile: exactly floor(s * d_out * width) weights are pruned, the
  smallest saliencies first, ties broken by row, then column;
* the packed 2:4 form keeps the two survivors of each group in index order and
  a 4-bit code a | b << 2 per group (a < b the kept positions), eight codes per
  32-bit word, least significant first;
* the packed N:M form generalises it: the N survivors of each group of M in
  index order, and each survivor's in-group position in log2(M) bits, packed
  along the row least significant bit first (2:4 gives the same words);
* joint sparsification and quantization: one uniform asymmetric grid of
  2**bits levels per output row over the dense row's range widened to 0
  (fp32 scale and zero point); each kept weight becomes its grid value when
  its column is reached and the difference is compensated like a pruning
  error; the integer code is decided in fp32.
"""

from __future__ import annotations

import math

import numpy as np
import scipy.linalg


class NotPositiveDefinite(ValueError):
    """The damped Hessian has a non-positive pivot."""


# --------------------------------------------------------------------------
# Hessian and damping  ([SGPT] section 七, H = X X^T)
# --------------------------------------------------------------------------

def hessian(X, chunk: int = 16384) -> np.ndarray:
    """H = (2/n) * sum_t x_t x_t^T over the n token rows x_t of X [n, d].

    X is any array-like whose values are the exact bf16 inputs (widened to
    float64 here). Rows are summed in chunks only to bound memory.
    """
    X = np.asarray(X)
    n, d = X.shape
    H = np.zeros((d, d), dtype=np.float64)
    for t0 in range(0, n, chunk):
        Xc = np.asarray(X[t0:t0 + chunk], dtype=np.float64)
        H += Xc.T @ Xc
    return H * (2.0 / n)


def damp(H: np.ndarray, damp_ratio: float = 0.01):
    """H_d = H + lambda I with lambda = damp_ratio * mean(diag H)."""
    lam = damp_ratio * float(np.mean(np.diag(H)))
    return H + lam * np.eye(H.shape[0]), lam


def inverse_cholesky_upper(Hd: np.ndarray) -> np.ndarray:
    """Upper-triangular U with positive diagonal and H_d^-1 = U^T U.

    Route: H_d = L L^T (Cholesky), H_d^-1 = L^-T L^-1, then the Cholesky
    factor of H_d^-1, transposed to upper form.
    """
    d = Hd.shape[0]
    try:
        L = np.linalg.cholesky(Hd)
    except np.linalg.LinAlgError as exc:
        raise NotPositiveDefinite(str(exc)) from None
    Linv = scipy.linalg.solve_triangular(L, np.eye(d), lower=True)
    Hinv = Linv.T @ Linv
    Hinv = 0.5 * (Hinv + Hinv.T)
    return np.linalg.cholesky(Hinv).T


# --------------------------------------------------------------------------
# The blocked OBS sweep  ([SGPT] sections 八 and 十一)
# --------------------------------------------------------------------------

def quant_grid(W, bits: int):
    """Per-row uniform asymmetric grid of 2**bits levels ([SGPT] sections 十五
    and 十七: survivors quantized to low-bit values, GPTQ-style).

    The range of each row of the dense input weights, widened to include 0
    (so a pruned weight stays exactly 0 on the grid); a row of zeros takes
    [-1, 1]. scale = (max - min) / (2**bits - 1) and zero = rint(-min /
    scale), both in fp32, the arithmetic the grid is stored in. Returns
    (scale, zero) as float32 arrays [d_out].
    """
    W32 = np.asarray(W, dtype=np.float32)
    maxq = np.float32(2 ** bits - 1)
    lo = np.minimum(W32.min(axis=1), np.float32(0))
    hi = np.maximum(W32.max(axis=1), np.float32(0))
    flat = lo == hi
    lo = np.where(flat, np.float32(-1), lo)
    hi = np.where(flat, np.float32(1), hi)
    scale = ((hi - lo) / maxq).astype(np.float32)
    zero = np.rint(-lo / scale).astype(np.float32)
    return scale, zero


def quantize(x, scale, zero, bits: int):
    """The grid value nearest x: scale * (clip(rint(x / scale) + zero, 0,
    2**bits - 1) - zero). The integer code is decided in fp32 (x rounded to
    fp32, fp32 division, ties to even), the precision the grid is stored in;
    the value is formed in float64."""
    x32 = np.asarray(x, dtype=np.float32)
    code = np.clip(np.rint(x32 / scale) + zero, np.float32(0), np.float32(2 ** bits - 1))
    return np.asarray(scale, dtype=np.float64) * (code.astype(np.float64) - np.asarray(zero, dtype=np.float64))


def parse_pattern(pattern):
    """'2:4' -> ('nm', 2, 4, None); 'unstructured:0.5' -> ('unstructured', .., 0.5)."""
    if isinstance(pattern, tuple):
        return pattern
    if pattern.startswith("unstructured"):
        return ("unstructured", 0, 0, float(pattern.split(":")[1]))
    n, m = pattern.split(":")
    return ("nm", int(n), int(m), None)


def sweep(W, U, pattern="2:4", blocksize: int = 128, forced_mask=None, qbits=None, qgrid=None,
          forced_values=None):
    """Prune W [d_out, d_in] column by column with OBS compensation.

    With ``qbits`` the sweep also quantizes ([SGPT] sections 十五 and 十七,
    pruning and GPTQ-style quantization in the same second-order pass): a
    kept weight is replaced by its value on the row's grid (``qgrid``, or
    quant_grid of the input W), and the difference is compensated in the
    later columns exactly like a pruning error.

    Returns a dict with
      W      the pruned, compensated weights (float64)
      mask   bool [d_out, d_in], True = kept
      loss   per-row sum of e^2 (float64 [d_out])
      S_dec  the saliency each weight had when its mask was decided
      Err    the per-column errors e (float64 [d_out, d_in])
    With ``forced_mask`` the mask is taken as given and no selection is made
    (S_dec is still recorded at the moment the pattern would decide). With
    ``forced_values`` as well, a kept weight takes the given value instead of
    its grid value (W_dec records the weight each column had just before it
    was replaced), so the sweep follows another run's decisions exactly.
    """
    kind, n_keep, m_grp, sparsity = parse_pattern(pattern)
    W = np.array(W, dtype=np.float64, copy=True)
    r, d = W.shape
    if kind == "nm" and (d % m_grp or blocksize % m_grp):
        raise ValueError("d_in and blocksize must be multiples of M")
    diagU = np.diag(U).copy()
    mask = np.ones((r, d), dtype=bool)
    if forced_mask is not None:
        mask[:] = np.asarray(forced_mask, dtype=bool)
    S_dec = np.zeros((r, d))
    W_dec = np.zeros((r, d))
    Err = np.zeros((r, d))
    loss = np.zeros(r)
    rows = np.arange(r)
    if qbits:
        qscale, qzero = quant_grid(W, qbits) if qgrid is None else qgrid

    for i1 in range(0, d, blocksize):
        i2 = min(i1 + blocksize, d)
        width = i2 - i1
        W1 = W[:, i1:i2].copy()
        E1 = np.zeros((r, width))

        if kind == "unstructured":
            # Saliency of every weight of the tile, on the weights as they
            # stand at the start of the block.
            S = (W1 / diagU[i1:i2]) ** 2
            S_dec[:, i1:i2] = S
            if forced_mask is None:
                k = int(math.floor(sparsity * r * width))
                cols = np.broadcast_to(np.arange(width), (r, width))
                rr = np.broadcast_to(rows[:, None], (r, width))
                order = np.lexsort((cols.ravel(), rr.ravel(), S.ravel()))
                blk = np.ones(r * width, dtype=bool)
                blk[order[:k]] = False
                mask[:, i1:i2] = blk.reshape(r, width)

        for q in range(width):
            c = i1 + q
            if kind == "nm" and q % m_grp == 0:
                # N of M, decided on the current (already compensated) weights.
                S = (W1[:, q:q + m_grp] / diagU[c:c + m_grp]) ** 2
                S_dec[:, c:c + m_grp] = S
                if forced_mask is None:
                    order = np.argsort(-S, axis=1, kind="stable")
                    keep = np.zeros_like(S, dtype=bool)
                    np.put_along_axis(keep, order[:, :n_keep], True, axis=1)
                    mask[:, c:c + m_grp] = keep
            w = W1[:, q]
            W_dec[:, c] = w
            if forced_values is not None:
                kept = np.asarray(forced_values[:, c], dtype=np.float64)
            else:
                kept = quantize(w, qscale, qzero, qbits) if qbits else w
            p = np.where(mask[:, c], kept, 0.0)
            e = (w - p) / U[c, c]
            W1[:, q:] -= np.outer(e, U[c, c:i2])
            W1[:, q] = p
            E1[:, q] = e
            loss += e * e

        W[:, i1:i2] = W1
        Err[:, i1:i2] = E1
        # Lazy update of every column to the right of the block.
        W[:, i2:] -= E1 @ U[i1:i2, i2:]

    return {"W": W, "mask": mask, "loss": loss, "S_dec": S_dec, "W_dec": W_dec, "Err": Err}


# --------------------------------------------------------------------------
# 2:4 packing  ([2:4] "2-bit metadata records the kept positions")
# --------------------------------------------------------------------------

def pack24(W_hat, mask):
    """values [d_out, d_in/2] and meta uint32 [d_out, ceil(d_in/32)].

    Group g of row r holds columns 4g..4g+3 with kept positions a < b:
    values[r, 2g] = W^[r, 4g+a], values[r, 2g+1] = W^[r, 4g+b], and bits
    [4(g%8), 4(g%8)+4) of meta word g//8 hold a | (b << 2).
    """
    W_hat = np.asarray(W_hat)
    mask = np.asarray(mask, dtype=bool)
    r, d = W_hat.shape
    if d % 4:
        raise ValueError("d_in must be a multiple of 4")
    values = np.zeros((r, d // 2), dtype=W_hat.dtype)
    meta = np.zeros((r, (d + 31) // 32), dtype=np.uint64)
    for g in range(d // 4):
        grp = mask[:, 4 * g:4 * g + 4]
        if not np.all(grp.sum(axis=1) == 2):
            raise ValueError(f"group {g} does not keep exactly 2 of 4")
        idx = np.argsort(~grp, axis=1, kind="stable")[:, :2]   # kept, ascending
        a, b = idx[:, 0], idx[:, 1]
        values[:, 2 * g] = W_hat[np.arange(r), 4 * g + a]
        values[:, 2 * g + 1] = W_hat[np.arange(r), 4 * g + b]
        meta[:, g // 8] |= ((a | (b << 2)).astype(np.uint64) << np.uint64(4 * (g % 8)))
    return values, meta.astype(np.uint32)


def unpack24(values, meta, d_in: int):
    """Inverse of pack24: the dense [d_out, d_in] matrix with zeros."""
    values = np.asarray(values)
    meta = np.asarray(meta, dtype=np.uint64)
    r = values.shape[0]
    out = np.zeros((r, d_in), dtype=values.dtype)
    for g in range(d_in // 4):
        code = (meta[:, g // 8] >> np.uint64(4 * (g % 8))) & np.uint64(15)
        a = (code & np.uint64(3)).astype(np.int64)
        b = (code >> np.uint64(2)).astype(np.int64)
        out[np.arange(r), 4 * g + a] = values[:, 2 * g]
        out[np.arange(r), 4 * g + b] = values[:, 2 * g + 1]
    return out


def pack_nm(W_hat, mask, n_keep: int, m_grp: int):
    """General N:M packing: values [d_out, d_in*N/M] and meta uint32 words.

    Group g of a row (columns M*g .. M*g+M-1) must keep exactly N weights;
    they are stored in column order as values N*g .. N*g+N-1 of the row. The
    in-group position of kept value k of the row (k = N*g + j) takes
    b = log2(M) bits at bit offset k*b of the row's metadata bit string,
    which fills uint32 words least significant bit first (a position may
    continue into the next word); a row has ceil(d_in*N/M*b / 32) words.
    For 2:4 this is pack24's layout: a | b << 2 per group, eight groups a
    word.
    """
    W_hat = np.asarray(W_hat)
    mask = np.asarray(mask, dtype=bool)
    r, d = W_hat.shape
    b = int(m_grp).bit_length() - 1
    if m_grp != 1 << b or d % m_grp or not 1 <= n_keep <= m_grp:
        raise ValueError("M must be a power of two dividing d_in, 1 <= N <= M")
    groups = d // m_grp
    nvals = groups * n_keep
    words = (nvals * b + 31) // 32
    values = np.zeros((r, nvals), dtype=W_hat.dtype)
    bitstr = np.zeros((r, words * 32), dtype=np.uint8)
    for g in range(groups):
        grp = mask[:, m_grp * g:m_grp * g + m_grp]
        if not np.all(grp.sum(axis=1) == n_keep):
            raise ValueError(f"group {g} does not keep exactly {n_keep} of {m_grp}")
        idx = np.argsort(~grp, axis=1, kind="stable")[:, :n_keep]      # kept, ascending
        for j in range(n_keep):
            k = n_keep * g + j
            values[:, k] = W_hat[np.arange(r), m_grp * g + idx[:, j]]
            for bit in range(b):
                bitstr[:, k * b + bit] = (idx[:, j] >> bit) & 1
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    meta = (bitstr.reshape(r, words, 32).astype(np.uint64) * weights).sum(axis=2)
    return values, meta.astype(np.uint32)


def unpack_nm(values, meta, d_in: int, n_keep: int, m_grp: int):
    """Inverse of pack_nm: the dense [d_out, d_in] matrix with zeros."""
    values = np.asarray(values)
    meta = np.asarray(meta, dtype=np.uint64)
    r = values.shape[0]
    b = int(m_grp).bit_length() - 1
    bits = ((meta[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).reshape(r, -1)
    out = np.zeros((r, d_in), dtype=values.dtype)
    for k in range(d_in // m_grp * n_keep):
        pos = np.zeros(r, dtype=np.int64)
        for bit in range(b):
            pos |= bits[:, k * b + bit].astype(np.int64) << bit
        out[np.arange(r), m_grp * (k // n_keep) + pos] = values[:, k]
    return out


def mask_bits(mask) -> np.ndarray:
    """Bool mask [d_out, d_in] -> uint32 words, bit c%32 of word c//32."""
    mask = np.asarray(mask, dtype=bool)
    r, d = mask.shape
    nw = (d + 31) // 32
    padded = np.zeros((r, nw * 32), dtype=np.uint64)
    padded[:, :d] = mask
    weights = np.uint64(1) << np.arange(32, dtype=np.uint64)
    return (padded.reshape(r, nw, 32) * weights).sum(axis=2).astype(np.uint32)


def bits_to_mask(words, d_in: int) -> np.ndarray:
    words = np.asarray(words, dtype=np.uint64)
    r, nw = words.shape
    bits = (words[:, :, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)
    return bits.reshape(r, nw * 32)[:, :d_in].astype(bool)


# --------------------------------------------------------------------------
# Reconstruction error  ([SGPT] section 六, the layer objective)
# --------------------------------------------------------------------------

def recon_error(W0, W_hat, H):
    """(tr(dW H dW^T), tr(W0 H W0^T)) with dW = W0 - W^ and H undamped."""
    W0 = np.asarray(W0, dtype=np.float64)
    dW = W0 - np.asarray(W_hat, dtype=np.float64)
    num = float(np.einsum("ij,ij->", dW @ H, dW))
    den = float(np.einsum("ij,ij->", W0 @ H, W0))
    return num, den


# --------------------------------------------------------------------------
# Whole layer  ([SGPT] section 十一 steps three to five, one linear layer)
# --------------------------------------------------------------------------

def prune_layer(W, X=None, H=None, pattern="2:4", blocksize: int = 128,
                damp_ratio: float = 0.01, forced_mask=None, qbits=None):
    """Hessian (from X, or H given), damping, factor, sweep (optionally with
    quantization of the survivors), and N:M pack."""
    if H is None:
        H = hessian(X)
    Hd, lam = damp(H, damp_ratio)
    U = inverse_cholesky_upper(Hd)
    out = sweep(W, U, pattern, blocksize, forced_mask, qbits=qbits)
    out.update(H=H, Hd=Hd, lam=lam, U=U)
    kind, n_keep, m_grp, _ = parse_pattern(pattern)
    if kind == "nm" and (n_keep, m_grp) == (2, 4):
        out["values"], out["meta"] = pack24(out["W"], out["mask"])
    elif kind == "nm":
        out["values"], out["meta"] = pack_nm(out["W"], out["mask"], n_keep, m_grp)
    return out
