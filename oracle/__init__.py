"""Double-precision CPU oracle of the SparseGPT layer solver.

Test infrastructure: only the tests, the smoke check and the CPU-baseline leg
of the bench use it. See ``sparsegpt_ref`` for what it computes and which
passages of the pages each step follows.
"""

from . import mlp_block_ref  # noqa: F401
from .sparsegpt_ref import (  # noqa: F401
    NotPositiveDefinite,
    bits_to_mask,
    damp,
    hessian,
    inverse_cholesky_upper,
    mask_bits,
    pack24,
    pack_nm,
    parse_pattern,
    prune_layer,
    quant_grid,
    quantize,
    recon_error,
    sweep,
    unpack24,
    unpack_nm,
)
