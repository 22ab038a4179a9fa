"""DELTA decode attention stack for NVIDIA B200 (sm_100a).

The compute path is libdelta_attn.so (include/delta_attn.h); this package is a thin
binding over it plus the per-step stack schedule.  There is no CPU fallback: importing
the binding fails when the library is missing.
"""
from . import _native  # noqa: F401  (fails loudly if the library is not built)
from ._native import (  # noqa: F401
    DELTA_BF16, DELTA_F32, DELTA_HEAD_MAX, DELTA_HEAD_SUM, DeltaDesc, DeltaError, DeltaPageTable,
    DeltaSelectParams, choose_layers, full_attn, full_attn_noalloc, kv_append, kv_append_layers, layer_shift, read_device_error, sel_capacity, select_attn, sparse_attn, sparse_attn_settled,
    status_string, workspace_init, workspace_size, workspace_size_reduce,
)
