"""Routed top-k MoE layer over codebook-quantised experts, for B200 (sm_100a).

The compute lives in libredlite_moe.so (C ABI, include/redlite_moe.h); this
package is a thin ctypes binding plus a buffer-owning convenience class."""

from ._native import (  # noqa: F401
    EXPORTS,
    LIB_PATH,
    REDLITE_EAGAIN,
    REDLITE_EINVAL,
    REDLITE_ENOMEM,
    REDLITE_EUNSUPPORTED,
    REDLITE_ECUDA,
    REDLITE_OK,
    REDLITE_Q_IQ1M_STYLE,
    REDLITE_Q_IQ2XS_STYLE,
    REDLITE_STATUS_BAD_EXPERT,
    REDLITE_STATUS_BAD_ID,
    REDLITE_STATUS_TIMEOUT,
    SlotPool,
    launches_per_call,
    lib,
    redlite_moe_dequant,
    redlite_moe_expand_grids,
    redlite_moe_expert,
    redlite_moe_grids_bytes,
    redlite_moe_layer,
    redlite_moe_layer_noalloc,
    redlite_moe_matrix_bytes,
    redlite_moe_block,
    redlite_moe_block_scratch_bytes,
    redlite_moe_pack_matrix,
    redlite_proj_gemv,
    redlite_proj_matrix_bytes,
    redlite_moe_pool_counters,
    redlite_moe_route_topk,
    redlite_moe_table,
    redlite_moe_upload_counters,
    redlite_moe_upload_experts,
    redlite_moe_workspace_bytes,
    redlite_moe_workspace_reset,
)
from .layer import MoeLayer  # noqa: F401
