"""The C-ABI library loads and exports every entry point include/sgpt.h
declares; argument errors are rejected before anything touches a GPU."""

import ctypes
import os
import re

import pytest

import post_pruning_b200 as pp
from post_pruning_b200 import sgpt as S

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "sgpt.h")


def _declared():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"^\s*(?:const\s+char\s*\*|sgpt_status|int|int64_t|size_t|uint64_t)\s+(sgpt_\w+)\s*\(",
                                 src, flags=re.M)))


def test_header_declares_the_binding_exports():
    assert _declared() == sorted(pp.EXPORTS)


def test_library_exports_every_declared_symbol():
    L = pp.lib()
    for name in _declared():
        assert hasattr(L, name), name
    assert L.sgpt_abi_version() == 2


def test_status_strings():
    L = pp.lib()
    for code in range(0, 9):
        assert L.sgpt_status_string(code)
    assert L.sgpt_status_string(123) == b"unknown status"


def test_workspace_bytes():
    p = S.Params("2:4").to_c()
    L = pp.lib()
    ws = L.sgpt_workspace_bytes(4096, 11008, 131072, ctypes.byref(p))
    # at least the factor's d x d scratch
    assert ws >= 11008 * 11008 * 4
    assert L.sgpt_workspace_bytes(4096, 100, 0, ctypes.byref(p)) == 0      # d_in % 32
    assert L.sgpt_workspace_bytes(0, 256, 0, ctypes.byref(p)) == 0          # d_out
    assert pp.workspace_bytes(256, 256, 2048) > 0


FAKE = 1 << 20          # an aligned non-null address; never dereferenced
MISALIGNED = FAKE + 4


@pytest.mark.parametrize("case", [
    "null_W", "bad_din", "bad_ldw", "bad_blocksize", "bad_sparsity", "nm_unsupported",
    "misaligned", "bad_pattern", "negative_damp", "nm_blocksize", "nm_din", "nm_n_above_m",
])
def test_prune_rejects_bad_arguments(case):
    L = pp.lib()
    p = S.Params("2:4").to_c()
    args = dict(W=FAKE, r=64, d=256, ldw=256, U=FAKE, mask=FAKE)
    if case == "null_W":
        args["W"] = None
    elif case == "bad_din":
        args["d"] = 250
        args["ldw"] = 252
    elif case == "bad_ldw":
        args["ldw"] = 255
    elif case == "bad_blocksize":
        p.blocksize = 100
    elif case == "bad_sparsity":
        p = S.Params("unstructured:1.0").to_c()
    elif case == "nm_unsupported":
        p = S.Params("3:6").to_c()              # M not a power of two
    elif case == "nm_blocksize":
        p = S.Params("16:128", blocksize=64).to_c()
    elif case == "nm_din":
        p = S.Params("16:128").to_c()
        args["d"] = args["ldw"] = 320
    elif case == "nm_n_above_m":
        p = S.Params("8:4").to_c()
    elif case == "misaligned":
        args["mask"] = MISALIGNED
    elif case == "bad_pattern":
        p.pattern = 7
    elif case == "negative_damp":
        p.damp = -0.5
    st = L.sgpt_prune(args["W"], args["r"], args["d"], args["ldw"], args["U"], ctypes.byref(p),
                      args["mask"], None, FAKE, 1 << 30, FAKE, None)
    expected = 6 if case == "nm_unsupported" else 1
    assert st == expected, (case, st)


def test_other_entry_points_validate():
    L = pp.lib()
    assert L.sgpt_factor(None, 10, 256, 0.01, FAKE, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_factor(FAKE, 0, 256, 0.01, FAKE, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_factor(FAKE, 10, 256, 0.01, FAKE, FAKE, 16, FAKE, None) == 8     # workspace
    assert L.sgpt_factor(FAKE, 10, 256, 0.01, FAKE, FAKE + 16, 1 << 30, FAKE, None) == 8
    assert L.sgpt_hessian_accumulate(FAKE, MISALIGNED, 100, 256, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_hessian_accumulate(FAKE, FAKE, 100, 96 + 8, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_pack24(FAKE, 8, 64, 64, FAKE, FAKE, None, FAKE, None) == 1
    assert L.sgpt_recon_error(FAKE, FAKE, 8, 64, 60, FAKE, FAKE, None, 0, None) == 1
    assert L.sgpt_recon_error(FAKE, FAKE, 8, 64, 64, FAKE, FAKE, None, 0, None) == 8     # workspace
    # prune_layer checks W, the mask and ldw before anything is launched
    p24 = S.Params("2:4").to_c()
    assert L.sgpt_prune_layer(None, 8, 64, 64, None, 10, FAKE, FAKE + 4096, ctypes.byref(p24), FAKE, None,
                              None, None, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_prune_layer(FAKE, 8, 64, 60, None, 10, FAKE, FAKE + 4096, ctypes.byref(p24), FAKE, None,
                              None, None, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_prune_layer(FAKE, 8, 64, 64, None, 10, FAKE, FAKE + 4096, ctypes.byref(p24), MISALIGNED,
                              None, None, None, FAKE, 1 << 30, FAKE, None) == 1


def test_hessian_without_tokens():
    """n_tok == 0: X may be NULL and the accumulation is a no-op (nothing is
    launched, so this runs without a GPU); a negative count or a NULL X with
    tokens is refused."""
    L = pp.lib()
    assert L.sgpt_hessian_accumulate(FAKE, None, 0, 256, None, 0, FAKE, None) == 0
    assert L.sgpt_hessian_accumulate(FAKE, None, 5, 256, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_hessian_accumulate(FAKE, FAKE, -1, 256, FAKE, 1 << 30, FAKE, None) == 1


def test_sparse24_meta_tiles_sizes_and_validation():
    L = pp.lib()
    # 4 KB per 256 rows and 128 columns of K, both rounded up
    assert L.sgpt_sparse24_meta_tiles_bytes(256, 128) == 4096
    assert L.sgpt_sparse24_meta_tiles_bytes(5120, 25600) == 20 * 200 * 4096
    assert L.sgpt_sparse24_meta_tiles_bytes(257, 160) == 2 * 2 * 4096
    assert L.sgpt_sparse24_meta_tiles_bytes(256, 100) == 0            # d_in % 32
    assert L.sgpt_sparse24_meta_tiles_bytes(0, 128) == 0
    assert L.sgpt_sparse24_tile_meta(FAKE, 256, 128, MISALIGNED, None) == 1
    assert L.sgpt_sparse24_tile_meta(None, 256, 128, FAKE, None) == 1
    assert L.sgpt_sparse24_linear(FAKE, MISALIGNED, 256, 128, FAKE, 10, FAKE, FAKE, None) == 1
    assert L.sgpt_sparse24_linear(FAKE, FAKE, 256, 128, FAKE, 0, FAKE, FAKE, None) == 1


def test_pack_nm_sizes_and_validation():
    L = pp.lib()
    assert L.sgpt_pack_nm_meta_words(64, 2, 4) == 2          # = d_in / 32, as pack24
    assert L.sgpt_pack_nm_meta_words(32, 16, 32) == 3        # 16 x 5 bits
    assert L.sgpt_pack_nm_meta_words(256, 16, 128) == 7      # 2 x 16 x 7 bits
    assert L.sgpt_pack_nm_meta_words(64, 4, 8) == 3          # 8 groups x 4 x 3 bits = 96
    assert L.sgpt_pack_nm_meta_words(64, 3, 6) == -1
    assert L.sgpt_pack_nm_meta_words(96, 16, 64) == -1       # d_in % m
    assert L.sgpt_pack_nm(FAKE, 8, 64, 64, FAKE, 3, 6, FAKE, FAKE, FAKE, None) == 6
    assert L.sgpt_pack_nm(FAKE, 8, 96, 96, FAKE, 16, 64, FAKE, FAKE, FAKE, None) == 1
    assert L.sgpt_pack_nm(FAKE, 8, 64, 64, FAKE, 9, 8, FAKE, FAKE, FAKE, None) == 1
    assert L.sgpt_pack_nm(FAKE, 8, 64, 64, FAKE, 4, 8, MISALIGNED, FAKE, FAKE, None) == 1


def test_wait_limit_setting():
    L = pp.lib()
    default = 4000000000
    assert pp.set_wait_limit(1000) == default
    assert pp.set_wait_limit(0) == 1000
    assert pp.set_wait_limit(-5) == default
    assert L.sgpt_set_wait_limit(0) == default
    assert L.sgpt_info_clear(None, None) == 1
    assert L.sgpt_sync_status(None, None) == 1
    p = S.Params("2:4").to_c()
    # H and U must not alias; values without meta is an error
    assert L.sgpt_prune_layer(FAKE, 8, 64, 64, None, 10, FAKE, FAKE, ctypes.byref(p), FAKE, None, None,
                              None, FAKE, 1 << 30, FAKE, None) == 1
    assert L.sgpt_prune_layer(FAKE, 8, 64, 64, None, 10, FAKE, FAKE + 4096, ctypes.byref(p), FAKE, FAKE,
                              None, None, FAKE, 1 << 30, FAKE, None) == 1


def test_python_binding_requires_cuda_tensors():
    import torch
    W = torch.zeros(4, 64)
    with pytest.raises(TypeError):
        pp.hessian_zero(W)
