"""MC-Sparse (Meta-Cached Sparse Attention) hot path for NVIDIA B200 (sm_100a).

The CUDA library (libmcs.so, C ABI in include/mcs.h) does all the work; this
package is its Python binding.  Import is cheap: the library is loaded on the
first call.
"""
from .api import (  # noqa: F401
    BlockMeta,
    Meta,
    alloc_workspace,
    compact_residual,
    dense,
    last_device_status,
    plan,
    plan_group,
    plan_residual,
    plan_scores,
    plan_select,
    plan_stats,
    plan_topk,
    pooled_scores,
    select_block_indices,
    select_blocks,
    select_topk,
    selftest_wait_timeout,
    set_wait_limit_ns,
    sparse_step,
    sparse_step_blocks,
    sparse_step_compact,
    union_pairs,
    validate_meta,
    workspace_size,
    workspace_views,
)
from .denoise import Schedule, fidelity  # noqa: F401,E402
