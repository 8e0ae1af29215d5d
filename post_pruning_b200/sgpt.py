"""Python binding of libsgpt (the C ABI declared in include/sgpt.h).

Argument marshalling only: every function here checks tensor dtypes, devices
and shapes, passes raw device pointers and the current CUDA stream to the
C entry point of the same name, and turns a non-OK status into SgptError.
All arithmetic of the solver runs in the library's CUDA kernels; PyTorch only
provides device memory and streams. There is no fallback: if the library is
missing, every call raises.
"""

from __future__ import annotations

import ctypes
import os
from dataclasses import dataclass, field

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsgpt.so")

SGPT_OK = 0
STATUS_NAMES = {
    0: "OK", 1: "INVALID_ARG", 2: "NOT_PD", 3: "NONFINITE", 4: "TIMEOUT",
    5: "CUDA", 6: "UNSUPPORTED", 7: "BAD_MASK", 8: "WORKSPACE",
}
PATTERN_UNSTRUCTURED = 0
PATTERN_NM = 1

EXPORTS = (
    "sgpt_status_string", "sgpt_abi_version", "sgpt_kernel_launches", "sgpt_set_wait_limit",
    "sgpt_workspace_bytes",
    "sgpt_info_clear", "sgpt_sync_status", "sgpt_hessian_zero",
    "sgpt_hessian_accumulate", "sgpt_hessian_compute", "sgpt_factor", "sgpt_prune", "sgpt_prune_noalloc", "sgpt_pack24",
    "sgpt_pack_nm", "sgpt_pack_nm_meta_words", "sgpt_quant_grid", "sgpt_recon_error", "sgpt_prune_layer",
    "sgpt_mlp_block_workspace_bytes", "sgpt_prune_mlp_block", "sgpt_linear_bf16", "sgpt_to_bf16",
    "sgpt_sparse24_linear", "sgpt_sparse24_meta_tiles_bytes", "sgpt_sparse24_tile_meta",
)
DRIVER_SEQUENTIAL = 0
DRIVER_PARALLEL = 1


class SgptError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        self.name = STATUS_NAMES.get(status, str(status))
        super().__init__(f"{where}: SGPT_{'ERR_' if status else ''}{self.name} ({status})")


class _Params(ctypes.Structure):
    _fields_ = [("pattern", ctypes.c_int), ("n", ctypes.c_int), ("m", ctypes.c_int),
                ("sparsity", ctypes.c_float), ("blocksize", ctypes.c_int),
                ("damp", ctypes.c_float), ("forced", ctypes.c_int),
                ("qbits", ctypes.c_int), ("qgrid", ctypes.c_void_p)]


@dataclass(frozen=True)
class Params:
    """Sparsity pattern and solver knobs (mirrors sgpt_params)."""
    pattern: str = "2:4"        # "N:M" (e.g. "2:4", "16:64") or "unstructured:<fraction>"
    blocksize: int = 128
    damp: float = 0.01
    forced: bool = False
    qbits: int = 0              # >0: quantize the kept weights to 2**qbits levels per row
    qgrid: object = field(default=None, compare=False)   # [d_out, 2] fp32 CUDA tensor or None

    @property
    def is_nm(self) -> bool:
        return not self.pattern.startswith("unstructured")

    @property
    def nm(self) -> tuple[int, int]:
        """(N, M) of an N:M pattern."""
        n, m = (int(x) for x in self.pattern.split(":"))
        return n, m

    @property
    def sparsity(self) -> float:
        return 0.0 if self.is_nm else float(self.pattern.split(":")[1])

    def to_c(self) -> _Params:
        grid = None
        if self.qgrid is not None:
            _dev(self.qgrid, torch.float32, "qgrid")
            grid = self.qgrid.data_ptr()
        if self.is_nm:
            n, m = (int(x) for x in self.pattern.split(":"))
            return _Params(PATTERN_NM, n, m, 0.0, self.blocksize, self.damp, int(self.forced),
                           int(self.qbits), grid)
        return _Params(PATTERN_UNSTRUCTURED, 0, 0, self.sparsity, self.blocksize, self.damp,
                       int(self.forced), int(self.qbits), grid)


class _MlpBlock(ctypes.Structure):
    _fields_ = [(name, ctypes.c_void_p) for name in
                ("W_gate", "W_up", "W_down", "mask_gate", "mask_up", "mask_down")]


_lib = None


def lib() -> ctypes.CDLL:
    """Load libsgpt.so once; raise loudly if it is not built."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing: build it with "
                           "`python -m post_pruning_b200.build` (needs nvcc)")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, sz = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t
    pp = ctypes.POINTER(_Params)
    sig = {
        "sgpt_status_string": (ctypes.c_char_p, [i32]),
        "sgpt_abi_version": (i32, []),
        "sgpt_kernel_launches": (ctypes.c_uint64, []),
        "sgpt_set_wait_limit": (i64, [i64]),
        "sgpt_workspace_bytes": (sz, [i32, i32, i64, pp]),
        "sgpt_info_clear": (i32, [vp, vp]),
        "sgpt_sync_status": (i32, [vp, vp]),
        "sgpt_hessian_zero": (i32, [vp, i32, vp]),
        "sgpt_hessian_accumulate": (i32, [vp, vp, i64, i32, vp, sz, vp, vp]),
        "sgpt_hessian_compute": (i32, [vp, vp, i64, i32, vp, sz, vp, vp]),
        "sgpt_factor": (i32, [vp, i64, i32, ctypes.c_float, vp, vp, sz, vp, vp]),
        "sgpt_prune": (i32, [vp, i32, i32, i32, vp, pp, vp, vp, vp, sz, vp, vp]),
        "sgpt_prune_noalloc": (i32, [vp, i32, i32, i32, vp, pp, vp, vp, vp, vp]),
        "sgpt_pack24": (i32, [vp, i32, i32, i32, vp, vp, vp, vp, vp]),
        "sgpt_pack_nm": (i32, [vp, i32, i32, i32, vp, i32, i32, vp, vp, vp, vp]),
        "sgpt_pack_nm_meta_words": (i32, [i32, i32, i32]),
        "sgpt_quant_grid": (i32, [vp, i32, i32, i32, i32, vp, vp]),
        "sgpt_mlp_block_workspace_bytes": (sz, [i32, i32, i64]),
        "sgpt_prune_mlp_block": (i32, [ctypes.POINTER(_MlpBlock), i32, i32, vp, i64, i32, pp, vp, vp, vp, sz,
                                       vp, vp]),
        "sgpt_linear_bf16": (i32, [vp, vp, i64, i32, i32, vp, vp, vp]),
        "sgpt_to_bf16": (i32, [vp, i32, i32, i32, vp, vp, vp]),
        "sgpt_sparse24_linear": (i32, [vp, vp, i32, i32, vp, i64, vp, vp, vp]),
        "sgpt_sparse24_meta_tiles_bytes": (sz, [i32, i32]),
        "sgpt_sparse24_tile_meta": (i32, [vp, i32, i32, vp, vp]),
        "sgpt_recon_error": (i32, [vp, vp, i32, i32, i32, vp, vp, vp, sz, vp]),
        "sgpt_prune_layer": (i32, [vp, i32, i32, i32, vp, i64, vp, vp, pp, vp, vp, vp, vp,
                                   vp, sz, vp, vp]),
    }
    for name, (res, args) in sig.items():
        f = getattr(L, name)
        f.restype = res
        f.argtypes = args
    _lib = L
    return L


# ------------------------------------------------------------------ helpers

def _stream(stream=None) -> int:
    s = stream if stream is not None else torch.cuda.current_stream()
    return s.cuda_stream


def _ptr(t) -> int | None:
    return None if t is None else t.data_ptr()


def _dev(t: torch.Tensor, dtype, name: str):
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")


def _rowmajor(t: torch.Tensor, name: str) -> int:
    """Leading dimension of a 2-D tensor with unit column stride."""
    if t.dim() != 2 or t.stride(1) != 1:
        raise ValueError(f"{name} must be 2-D with contiguous rows")
    return t.stride(0)


def _check(status: int, where: str):
    if status != SGPT_OK:
        raise SgptError(status, where)


def kernel_launches() -> int:
    """Kernels libsgpt has enqueued since it was loaded."""
    return int(lib().sgpt_kernel_launches())


def set_wait_limit(cycles: int) -> int:
    """Cycles a device-side wait polls before it records TIMEOUT (<= 0: the
    default). Returns the previous value. For testing failure paths."""
    return int(lib().sgpt_set_wait_limit(int(cycles)))


def workspace_bytes(d_out: int, d_in: int, n_tok: int = 0, params: Params | None = None) -> int:
    p = (params or Params()).to_c()
    return int(lib().sgpt_workspace_bytes(d_out, d_in, n_tok, ctypes.byref(p)))


def workspace(d_out: int, d_in: int, n_tok: int = 0, params: Params | None = None,
              device="cuda") -> torch.Tensor:
    """A byte tensor large enough for every call at these sizes."""
    return torch.empty(workspace_bytes(d_out, d_in, n_tok, params), dtype=torch.uint8, device=device)


def new_info(device="cuda") -> torch.Tensor:
    return torch.zeros(1, dtype=torch.int32, device=device)


# ------------------------------------------------------------- entry points

def info_clear(dev_info: torch.Tensor, stream=None):
    _check(lib().sgpt_info_clear(_ptr(dev_info), _stream(stream)), "sgpt_info_clear")


def sync_status(dev_info: torch.Tensor, stream=None) -> int:
    """Blocking; returns the status code (0 = OK) without raising."""
    return int(lib().sgpt_sync_status(_ptr(dev_info), _stream(stream)))


def raise_on_info(dev_info: torch.Tensor, stream=None, where="device"):
    _check(sync_status(dev_info, stream), where)


def hessian_zero(H: torch.Tensor, stream=None):
    _dev(H, torch.float32, "H")
    _check(lib().sgpt_hessian_zero(_ptr(H), H.shape[0], _stream(stream)), "sgpt_hessian_zero")


def hessian_accumulate(H: torch.Tensor, X: torch.Tensor, ws: torch.Tensor, dev_info: torch.Tensor,
                       stream=None):
    _dev(H, torch.float32, "H")
    _dev(X, torch.bfloat16, "X")
    d = H.shape[0]
    if H.shape != (d, d) or not H.is_contiguous() or X.dim() != 2 or X.shape[1] != d or not X.is_contiguous():
        raise ValueError("H must be [d, d] and X [n, d], both contiguous")
    _check(lib().sgpt_hessian_accumulate(_ptr(H), _ptr(X), X.shape[0], d, _ptr(ws), ws.numel(),
                                         _ptr(dev_info), _stream(stream)), "sgpt_hessian_accumulate")


def hessian_compute(H: torch.Tensor, X: torch.Tensor, ws: torch.Tensor, dev_info: torch.Tensor, stream=None):
    """H = X^T X (sgpt_hessian_compute): like hessian_zero + hessian_accumulate
    without reading H."""
    _dev(H, torch.float32, "H")
    _dev(X, torch.bfloat16, "X")
    d = H.shape[0]
    if H.shape != (d, d) or not H.is_contiguous() or X.dim() != 2 or X.shape[1] != d or not X.is_contiguous():
        raise ValueError("H must be [d, d] and X [n, d], both contiguous")
    _check(lib().sgpt_hessian_compute(_ptr(H), _ptr(X), X.shape[0], d, _ptr(ws), ws.numel(),
                                      _ptr(dev_info), _stream(stream)), "sgpt_hessian_compute")


def factor(H: torch.Tensor, n_total: int, damp: float, U: torch.Tensor, ws: torch.Tensor,
           dev_info: torch.Tensor, stream=None):
    _dev(H, torch.float32, "H")
    _dev(U, torch.float32, "U")
    d = H.shape[0]
    if H.shape != (d, d) or U.shape != (d, d) or not H.is_contiguous() or not U.is_contiguous():
        raise ValueError("H and U must be contiguous [d, d]")
    _check(lib().sgpt_factor(_ptr(H), n_total, d, damp, _ptr(U), _ptr(ws), ws.numel(), _ptr(dev_info),
                             _stream(stream)), "sgpt_factor")


def prune(W: torch.Tensor, U: torch.Tensor, params: Params, mask: torch.Tensor, ws: torch.Tensor,
          dev_info: torch.Tensor, row_loss: torch.Tensor | None = None, stream=None):
    _dev(W, torch.float32, "W")
    _dev(U, torch.float32, "U")
    _dev(mask, torch.int32, "mask")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    if mask.shape != (r, d // 32) or not mask.is_contiguous():
        raise ValueError("mask must be contiguous int32 [d_out, d_in/32]")
    if row_loss is not None:
        _dev(row_loss, torch.float32, "row_loss")
    p = params.to_c()
    _check(lib().sgpt_prune(_ptr(W), r, d, ldw, _ptr(U), ctypes.byref(p), _ptr(mask), _ptr(row_loss),
                            _ptr(ws), ws.numel(), _ptr(dev_info), _stream(stream)), "sgpt_prune")


NOALLOC_MAX_ROWS = 8192


def prune_noalloc(W: torch.Tensor, U: torch.Tensor, params: Params, mask: torch.Tensor,
                  dev_info: torch.Tensor, row_loss: torch.Tensor | None = None, stream=None):
    """sgpt_prune without a workspace, for callers that cannot allocate device
    memory where they call it: the scratch is a fixed array inside the library
    (d_out <= NOALLOC_MAX_ROWS). Calls that overlap on the GPU race on it."""
    _dev(W, torch.float32, "W")
    _dev(U, torch.float32, "U")
    _dev(mask, torch.int32, "mask")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    if mask.shape != (r, d // 32) or not mask.is_contiguous():
        raise ValueError("mask must be contiguous int32 [d_out, d_in/32]")
    if row_loss is not None:
        _dev(row_loss, torch.float32, "row_loss")
    p = params.to_c()
    _check(lib().sgpt_prune_noalloc(_ptr(W), r, d, ldw, _ptr(U), ctypes.byref(p), _ptr(mask),
                                    _ptr(row_loss), _ptr(dev_info), _stream(stream)),
           "sgpt_prune_noalloc")


def pack24(W: torch.Tensor, mask: torch.Tensor, values: torch.Tensor, meta: torch.Tensor,
           dev_info: torch.Tensor, stream=None):
    _dev(W, torch.float32, "W")
    _dev(values, torch.float32, "values")
    _dev(mask, torch.int32, "mask")
    _dev(meta, torch.int32, "meta")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    if values.shape != (r, d // 2) or meta.shape != (r, d // 32):
        raise ValueError("values must be [d_out, d_in/2] and meta [d_out, d_in/32]")
    _check(lib().sgpt_pack24(_ptr(W), r, d, ldw, _ptr(mask), _ptr(values), _ptr(meta), _ptr(dev_info),
                             _stream(stream)), "sgpt_pack24")


def quant_grid(W: torch.Tensor, qbits: int, grid: torch.Tensor, stream=None):
    """Per-row quantization grid of the dense W (sgpt_quant_grid): grid
    [d_out, 2] fp32 = (scale, zero point)."""
    _dev(W, torch.float32, "W")
    _dev(grid, torch.float32, "grid")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    if grid.shape != (r, 2) or not grid.is_contiguous():
        raise ValueError("grid must be contiguous [d_out, 2]")
    _check(lib().sgpt_quant_grid(_ptr(W), r, d, ldw, qbits, _ptr(grid), _stream(stream)), "sgpt_quant_grid")


def to_bf16(W: torch.Tensor, Wb: torch.Tensor, dev_info: torch.Tensor, stream=None):
    """Wb = W rounded to bf16 (sgpt_to_bf16)."""
    _dev(W, torch.float32, "W")
    _dev(Wb, torch.bfloat16, "Wb")
    ldw = _rowmajor(W, "W")
    if Wb.shape != W.shape or not Wb.is_contiguous():
        raise ValueError("Wb must be contiguous with W's shape")
    _check(lib().sgpt_to_bf16(_ptr(W), W.shape[0], W.shape[1], ldw, _ptr(Wb), _ptr(dev_info), _stream(stream)),
           "sgpt_to_bf16")


def linear_bf16(X: torch.Tensor, Wb: torch.Tensor, Y: torch.Tensor, dev_info: torch.Tensor, stream=None):
    """Y = X Wb^T on the tensor cores (sgpt_linear_bf16): X [n, d_in] and Wb
    [d_out, d_in] bf16, Y [n, d_out] fp32."""
    _dev(X, torch.bfloat16, "X")
    _dev(Wb, torch.bfloat16, "Wb")
    _dev(Y, torch.float32, "Y")
    n, d_in = X.shape
    d_out = Wb.shape[0]
    if Wb.shape[1] != d_in or Y.shape != (n, d_out) or not (X.is_contiguous() and Wb.is_contiguous()
                                                             and Y.is_contiguous()):
        raise ValueError("X [n, d_in], Wb [d_out, d_in], Y [n, d_out], all contiguous")
    _check(lib().sgpt_linear_bf16(_ptr(X), _ptr(Wb), n, d_in, d_out, _ptr(Y), _ptr(dev_info), _stream(stream)),
           "sgpt_linear_bf16")


def sparse24_meta_tiles(meta: torch.Tensor, d_in: int, out: torch.Tensor | None = None,
                        stream=None) -> torch.Tensor:
    """sgpt_pack24's metadata words meta [d_out, d_in/32] int32 re-arranged
    for sparse24_linear (sgpt_sparse24_tile_meta); done once per weight
    matrix. Returns (or fills) an int32 buffer of
    sgpt_sparse24_meta_tiles_bytes(d_out, d_in) bytes."""
    _dev(meta, torch.int32, "meta")
    d_out = meta.shape[0]
    if meta.shape != (d_out, d_in // 32) or not meta.is_contiguous():
        raise ValueError("meta [d_out, d_in/32], contiguous")
    nbytes = lib().sgpt_sparse24_meta_tiles_bytes(d_out, d_in)
    if nbytes == 0:
        raise ValueError(f"unsupported sizes d_out={d_out} d_in={d_in}")
    if out is None:
        out = torch.empty(nbytes // 4, dtype=torch.int32, device=meta.device)
    _dev(out, torch.int32, "out")
    if out.numel() * 4 < nbytes or not out.is_contiguous():
        raise ValueError(f"out needs {nbytes} contiguous bytes")
    _check(lib().sgpt_sparse24_tile_meta(_ptr(meta), d_out, d_in, _ptr(out), _stream(stream)),
           "sgpt_sparse24_tile_meta")
    return out


def sparse24_linear(values: torch.Tensor, meta_tiles: torch.Tensor, X: torch.Tensor, Y: torch.Tensor,
                    dev_info: torch.Tensor, stream=None):
    """Y = X W^T from W's packed 2:4 form on the sparse tensor cores
    (sgpt_sparse24_linear): values [d_out, d_in/2] bf16, meta_tiles from
    sparse24_meta_tiles, X [n, d_in] bf16, Y [n, d_out] fp32."""
    _dev(values, torch.bfloat16, "values")
    _dev(meta_tiles, torch.int32, "meta_tiles")
    _dev(X, torch.bfloat16, "X")
    _dev(Y, torch.float32, "Y")
    d_out, half = values.shape
    n, d_in = X.shape
    if half * 2 != d_in or Y.shape != (n, d_out):
        raise ValueError("values [d_out, d_in/2], X [n, d_in], Y [n, d_out]")
    if meta_tiles.numel() * 4 < lib().sgpt_sparse24_meta_tiles_bytes(d_out, d_in):
        raise ValueError("meta_tiles too small for these sizes")
    if not (values.is_contiguous() and meta_tiles.is_contiguous() and X.is_contiguous() and Y.is_contiguous()):
        raise ValueError("all operands must be contiguous")
    _check(lib().sgpt_sparse24_linear(_ptr(values), _ptr(meta_tiles), d_out, d_in, _ptr(X), n, _ptr(Y),
                                      _ptr(dev_info), _stream(stream)), "sgpt_sparse24_linear")


def mlp_block_workspace(hidden: int, inter: int, n_tok: int, device="cuda") -> torch.Tensor:
    b = int(lib().sgpt_mlp_block_workspace_bytes(hidden, inter, n_tok))
    if b == 0:
        raise ValueError("unsupported block sizes")
    return torch.empty(b, dtype=torch.uint8, device=device)


def prune_mlp_block(W_gate: torch.Tensor, W_up: torch.Tensor, W_down: torch.Tensor, masks, X: torch.Tensor,
                    params: Params, X_next: torch.Tensor, ws: torch.Tensor, dev_info: torch.Tensor,
                    mode: int = DRIVER_SEQUENTIAL, Z: torch.Tensor | None = None, stream=None):
    """One synthetic MLP block pruned layer by layer (sgpt_prune_mlp_block).
    masks: (gate, up, down) int32 mask-bit tensors."""
    for t, name in ((W_gate, "W_gate"), (W_up, "W_up"), (W_down, "W_down")):
        _dev(t, torch.float32, name)
        if not t.is_contiguous():
            raise ValueError(f"{name} must be contiguous")
    _dev(X, torch.bfloat16, "X")
    _dev(X_next, torch.bfloat16, "X_next")
    inter, hidden = W_gate.shape
    if W_up.shape != (inter, hidden) or W_down.shape != (hidden, inter):
        raise ValueError("W_gate, W_up [inter, hidden] and W_down [hidden, inter]")
    n = X.shape[0]
    if X.shape != (n, hidden) or X_next.shape != (n, hidden):
        raise ValueError("X and X_next must be [n_tok, hidden]")
    if Z is not None:
        _dev(Z, torch.bfloat16, "Z")
        if Z.shape != (n, inter) or not Z.is_contiguous():
            raise ValueError("Z must be contiguous [n_tok, inter]")
    mg, mu, md = masks
    for m_, shape in ((mg, (inter, hidden // 32)), (mu, (inter, hidden // 32)), (md, (hidden, inter // 32))):
        _dev(m_, torch.int32, "mask")
        if m_.shape != shape or not m_.is_contiguous():
            raise ValueError(f"mask must be contiguous {shape}")
    blk = _MlpBlock(_ptr(W_gate), _ptr(W_up), _ptr(W_down), _ptr(mg), _ptr(mu), _ptr(md))
    p = params.to_c()
    _check(lib().sgpt_prune_mlp_block(ctypes.byref(blk), hidden, inter, _ptr(X), n, mode, ctypes.byref(p),
                                      _ptr(X_next), _ptr(Z), _ptr(ws), ws.numel(), _ptr(dev_info),
                                      _stream(stream)), "sgpt_prune_mlp_block")


def pack_nm_meta_words(d_in: int, n: int, m: int) -> int:
    """uint32 metadata words per row of an N:M pack (-1 if unsupported)."""
    return int(lib().sgpt_pack_nm_meta_words(d_in, n, m))


def pack_nm(W: torch.Tensor, mask: torch.Tensor, n: int, m: int, values: torch.Tensor, meta: torch.Tensor,
            dev_info: torch.Tensor, stream=None):
    """N:M packing (sgpt_pack_nm): values [d_out, d_in*n/m] fp32, meta
    [d_out, pack_nm_meta_words(d_in, n, m)] int32."""
    _dev(W, torch.float32, "W")
    _dev(values, torch.float32, "values")
    _dev(mask, torch.int32, "mask")
    _dev(meta, torch.int32, "meta")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    words = pack_nm_meta_words(d, n, m)
    if words < 0:
        raise ValueError(f"unsupported N:M {n}:{m} for d_in {d}")
    if values.shape != (r, d * n // m) or meta.shape != (r, words) or not values.is_contiguous() \
            or not meta.is_contiguous():
        raise ValueError(f"values must be [d_out, {d * n // m}] and meta [d_out, {words}], contiguous")
    _check(lib().sgpt_pack_nm(_ptr(W), r, d, ldw, _ptr(mask), n, m, _ptr(values), _ptr(meta), _ptr(dev_info),
                              _stream(stream)), "sgpt_pack_nm")


def recon_error(W0: torch.Tensor, W: torch.Tensor, H: torch.Tensor, num_den: torch.Tensor,
                ws: torch.Tensor | None = None, stream=None):
    """num_den (float64 [2], device) = (tr(dW H dW^T), tr(W0 H W0^T)).
    ws: a workspace for these sizes (one is allocated when None)."""
    _dev(W0, torch.float32, "W0")
    _dev(W, torch.float32, "W")
    _dev(H, torch.float32, "H")
    _dev(num_den, torch.float64, "num_den")
    ldw = _rowmajor(W, "W")
    if _rowmajor(W0, "W0") != ldw or W0.shape != W.shape:
        raise ValueError("W0 and W must share shape and leading dimension")
    r, d = W.shape
    if ws is None:
        ws = workspace(r, d, device=W.device)
    _check(lib().sgpt_recon_error(_ptr(W0), _ptr(W), r, d, ldw, _ptr(H), _ptr(num_den), _ptr(ws), ws.numel(),
                                  _stream(stream)), "sgpt_recon_error")


def prune_layer(W: torch.Tensor, H: torch.Tensor, U: torch.Tensor, params: Params,
                mask: torch.Tensor, ws: torch.Tensor, dev_info: torch.Tensor,
                X: torch.Tensor | None = None, n_tok: int | None = None,
                values: torch.Tensor | None = None, meta: torch.Tensor | None = None,
                row_loss: torch.Tensor | None = None, stream=None):
    """One layer end to end (sgpt_prune_layer); X None means H holds X^T X."""
    _dev(W, torch.float32, "W")
    _dev(H, torch.float32, "H")
    _dev(U, torch.float32, "U")
    _dev(mask, torch.int32, "mask")
    ldw = _rowmajor(W, "W")
    r, d = W.shape
    if X is not None:
        _dev(X, torch.bfloat16, "X")
        if X.dim() != 2 or X.shape[1] != d or not X.is_contiguous():
            raise ValueError("X must be contiguous [n, d_in]")
        n_tok = X.shape[0]
    if n_tok is None:
        raise ValueError("n_tok is required when H is given")
    p = params.to_c()
    _check(lib().sgpt_prune_layer(_ptr(W), r, d, ldw, _ptr(X), n_tok, _ptr(H), _ptr(U), ctypes.byref(p),
                                  _ptr(mask), _ptr(values), _ptr(meta), _ptr(row_loss), _ptr(ws),
                                  ws.numel(), _ptr(dev_info), _stream(stream)), "sgpt_prune_layer")


# --------------------------------------------------------------- conveniences

@dataclass
class LayerBuffers:
    """Device buffers for pruning one layer shape (allocated once, reused)."""
    d_out: int
    d_in: int
    n_tok: int
    H: torch.Tensor
    U: torch.Tensor
    mask: torch.Tensor
    values: torch.Tensor
    meta: torch.Tensor
    row_loss: torch.Tensor
    ws: torch.Tensor
    info: torch.Tensor

    @classmethod
    def sharing(cls, other: "LayerBuffers", d_out: int, device="cuda", nm=(2, 4)) -> "LayerBuffers":
        """Buffers for another weight matrix that reads the same input: it
        shares H and U (factor once, sweep each matrix) and has its own
        outputs and workspace."""
        mine = cls.allocate(d_out, other.d_in, 0, device, with_hu=False, nm=nm)
        mine.H, mine.U, mine.n_tok = other.H, other.U, other.n_tok
        return mine

    @classmethod
    def allocate(cls, d_out: int, d_in: int, n_tok: int, device="cuda", with_hu: bool = True,
                 nm=(2, 4)) -> "LayerBuffers":
        """nm: the (N, M) the packed outputs are sized for."""
        f32 = dict(dtype=torch.float32, device=device)
        i32 = dict(dtype=torch.int32, device=device)
        hu = (d_in, d_in) if with_hu else (0, 0)
        n, m = nm
        words = max(pack_nm_meta_words(d_in, n, m), 0)
        return cls(d_out, d_in, n_tok,
                   H=torch.empty(hu, **f32), U=torch.empty(hu, **f32),
                   mask=torch.empty((d_out, d_in // 32), **i32),
                   values=torch.empty((d_out, d_in * n // m), **f32),
                   meta=torch.empty((d_out, words), **i32),
                   row_loss=torch.empty(d_out, **f32),
                   ws=workspace(d_out, d_in, n_tok, device=device),
                   info=new_info(device))

    def packs(self, params: Params) -> bool:
        """Whether the packed outputs are sized for this pattern."""
        if not params.is_nm:
            return False
        n, m = params.nm
        return self.values.shape[1] == self.d_in * n // m and \
            self.meta.shape[1] == pack_nm_meta_words(self.d_in, n, m)

    def run(self, W: torch.Tensor, X: torch.Tensor | None, params: Params, stream=None):
        pack = self.packs(params)
        prune_layer(W, self.H, self.U, params, self.mask, self.ws, self.info, X=X,
                    n_tok=self.n_tok, values=self.values if pack else None,
                    meta=self.meta if pack else None, row_loss=self.row_loss, stream=stream)


class LayerGraphs:
    """The four phases of one layer prune captured as CUDA graphs.

    hessian (H = X^T X), factor, prune (row loss cleared + sweep) and,
    for 2:4, pack. Replaying them in order does exactly what
    LayerBuffers.run does, with the launch overhead of one graph per phase.
    Capture reads no data: buffers are bound by address, so W and X must
    stay where they were at capture time. Replay on the current stream with
    replay(), or phase by phase through .graphs.
    """

    PHASES = ("hessian", "factor", "prune", "pack")

    def __init__(self, bufs: LayerBuffers, W: torch.Tensor, X: torch.Tensor | None, params: Params,
                 phases=PHASES):
        self.bufs, self.W, self.X, self.params = bufs, W, X, params
        self.phases = tuple(ph for ph in phases if not (ph == "pack" and not bufs.packs(params)))
        # one eager pass first: per-process kernel attributes are set outside capture
        self._eager()
        torch.cuda.synchronize()
        self.graphs = {}
        self.kernels = {}        # libsgpt kernels captured in each graph
        for name in self.phases:
            g = torch.cuda.CUDAGraph()
            before = kernel_launches()
            with torch.cuda.graph(g):
                self._phase(name)
            self.kernels[name] = kernel_launches() - before
            self.graphs[name] = g

    def _phase(self, name: str):
        b, p = self.bufs, self.params
        if name == "hessian":
            info_clear(b.info)
            hessian_compute(b.H, self.X, b.ws, b.info)
        elif name == "factor":
            factor(b.H, b.n_tok, p.damp, b.U, b.ws, b.info)
        elif name == "prune":
            b.row_loss.zero_()
            prune(self.W, b.U, p, b.mask, b.ws, b.info, row_loss=b.row_loss)
        elif name == "pack":
            pack_nm(self.W, b.mask, *p.nm, b.values, b.meta, b.info)

    def _eager(self):
        for name in self.phases:
            self._phase(name)

    def replay(self):
        for g in self.graphs.values():
            g.replay()


class HostPruner:
    """End-to-end pruning from host memory through the public API.

    Owns the device buffers of one layer shape and pinned host outputs.
    run() copies W and X from (pinned) host memory to the device, prunes the
    layer from X with sgpt_prune_layer, copies the pruned weights, the mask
    and (for the N:M pattern it was sized for, 2:4 by default) the packed
    values and metadata back to the host, and checks the device status. All
    copies are enqueued on the current stream.
    """

    def __init__(self, d_out: int, d_in: int, n_tok: int, device="cuda", nm=(2, 4)):
        self.bufs = LayerBuffers.allocate(d_out, d_in, n_tok, device, nm=nm)
        self.W = torch.empty((d_out, d_in), dtype=torch.float32, device=device)
        self.X = torch.empty((n_tok, d_in), dtype=torch.bfloat16, device=device)
        pin = dict(pin_memory=True)
        self.W_out = torch.empty((d_out, d_in), dtype=torch.float32, **pin)
        self.mask_out = torch.empty((d_out, d_in // 32), dtype=torch.int32, **pin)
        self.values_out = torch.empty(self.bufs.values.shape, dtype=torch.float32, **pin)
        self.meta_out = torch.empty(self.bufs.meta.shape, dtype=torch.int32, **pin)

    def h2d_bytes(self) -> int:
        return self.W.numel() * 4 + self.X.numel() * 2

    def d2h_bytes(self, params: Params) -> int:
        b = self.W_out.numel() * 4 + self.mask_out.numel() * 4
        if self.bufs.packs(params):
            b += self.values_out.numel() * 4 + self.meta_out.numel() * 4
        return b

    def enqueue(self, W_host: torch.Tensor, X_host: torch.Tensor | None, params: Params, stream=None,
                X_device: torch.Tensor | None = None):
        """Copies and pruning, all asynchronous. X_host None reuses the X on
        the device from the previous call; X_device prunes from an X already
        on the device (for example another pruner's, when several layers read
        the same input)."""
        self.W.copy_(W_host, non_blocking=True)
        if X_device is None and X_host is not None:
            self.X.copy_(X_host, non_blocking=True)
        self.bufs.run(self.W, self.X if X_device is None else X_device, params, stream=stream)
        self.W_out.copy_(self.W, non_blocking=True)
        self.mask_out.copy_(self.bufs.mask, non_blocking=True)
        if self.bufs.packs(params):
            self.values_out.copy_(self.bufs.values, non_blocking=True)
            self.meta_out.copy_(self.bufs.meta, non_blocking=True)

    def run(self, W_host: torch.Tensor, X_host: torch.Tensor, params: Params, stream=None):
        self.enqueue(W_host, X_host, params, stream)
        raise_on_info(self.bufs.info, stream, "HostPruner.run")
        if self.bufs.packs(params):
            return self.W_out, self.mask_out, self.values_out, self.meta_out
        return self.W_out, self.mask_out, None, None
