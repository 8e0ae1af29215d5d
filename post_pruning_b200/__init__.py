"""B200-native SparseGPT layer solver: Python binding of the libsgpt C ABI.

The solver (Hessian accumulation, damped factorisation, blocked OBS sweep
with 2:4 or unstructured masks, 2:4 packing) runs in hand-written sm_100a CUDA
kernels inside ``libsgpt.so``; see ``include/sgpt.h`` for the contract.
"""

from .sgpt import (  # noqa: F401
    DRIVER_PARALLEL,
    DRIVER_SEQUENTIAL,
    EXPORTS,
    HostPruner,
    LIB_PATH,
    LayerBuffers,
    LayerGraphs,
    Params,
    SgptError,
    factor,
    hessian_accumulate,
    hessian_compute,
    hessian_zero,
    info_clear,
    kernel_launches,
    lib,
    linear_bf16,
    mlp_block_workspace,
    new_info,
    pack24,
    pack_nm,
    pack_nm_meta_words,
    prune,
    prune_layer,
    prune_mlp_block,
    prune_noalloc,
    quant_grid,
    raise_on_info,
    recon_error,
    set_wait_limit,
    sparse24_linear,
    sparse24_meta_tiles,
    sync_status,
    to_bf16,
    workspace,
    workspace_bytes,
)
