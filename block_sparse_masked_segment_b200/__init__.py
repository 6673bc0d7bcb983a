"""One-Pass to Reason masked attention on B200 (sm_100a).

Thin Python binding over ``lib/libopr.so`` (C ABI in ``include/opr.h``).
PyTorch only provides device memory and streams; every step of the path
(layout, RoPE, attention forward and backward) runs in the library's CUDA
kernels.  There is no fallback: if the library is missing or the device is
not a B200, the calls raise.
"""

from ._abi import (  # noqa: F401
    OprError,
    Layout,
    load_library,
    library_path,
    opr_build_layout,
    opr_rope,
    opr_attn_fwd,
    opr_attn_bwd,
    opr_attn_bwd_stages,
    opr_attn_bwd_noalloc,
    opr_duplication_index,
    opr_gather_rows,
    opr_fold_rows,
    opr_kpass,
    opr_loss_rows,
    opr_cross_entropy,
    KPass,
    BWD_ROW_TERMS,
    BWD_DQ,
    BWD_DKDV,
    opr_layout_workspace_bytes,
    opr_attn_bwd_workspace_bytes,
    opr_attn_bwd_min_workspace_bytes,
    opr_version,
    read_status,
    layout_table_offsets,
    EXPORTED_SYMBOLS,
)
from .pipeline import OnePassAttention, one_pass_forward, one_pass_backward, useful_flops  # noqa: F401

__version__ = "0.1.0"
