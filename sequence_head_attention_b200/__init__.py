"""B200-native sequence/head-parallel exact attention: a C-ABI CUDA library (libspattn.so) and its binding.

Importing the package loads nothing; the shared library is loaded on the first call of any entry point
and every entry point raises if it is missing (there is no CPU path).  See ``spattn`` for the binding,
``synth`` for the seeded synthetic inputs and ``build`` for the nvcc build.
"""
from .spattn import (  # noqa: F401
    SP_BF16, SP_F32, SP_OK, SP_ERR_CUDA, SP_ERR_INVALID_ARG, SP_ERR_TIMEOUT, SP_ERR_UNSUPPORTED, SP_TILE,
    SpError, sp_attn_bwd, sp_attn_bwd_partial, sp_attn_fwd, sp_attn_fwd_items, sp_attn_fwd_partial,
    sp_attn_fwd_partial_merge, sp_attn_fwd_seq_sharded, sp_attn_fwd_sparse_noalloc, sp_attn_fwd_workspace_bytes,
    sp_build_tile_list, sp_check_device_error, sp_convert_f32_to_bf16, sp_dbsp_plan, sp_dbsp_rank_items,
    sp_dbsp_unit_costs, sp_debug_wait_timeout, sp_head_to_seq_relayout, sp_merge_partials,
    sp_merge_heads, sp_seq_to_head_relayout, sp_set_wait_timeout_ns, sp_split_heads, sp_status_string, sp_version,
)
