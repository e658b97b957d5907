"""Persistent decode/prefill megakernel for one B200 (sm_100a).

The compute path is ``libwpk.so`` (CUDA, built in-tree by
``python -m streaming_persistent_sm_b200.build``); this package only binds it.
"""
from .wpk import (  # noqa: F401
    Engine,
    OP_NAMES,
    TRACE_DTYPE,
    WPK_MEGAKERNEL,
    WPK_PER_OP_GRAPH,
    WpkError,
    load_library,
    model_cfg,
    plan_cfg,
    wpk_build_graph,
    wpk_debug_break_counter,
    wpk_destroy,
    wpk_get_edges,
    wpk_get_error_info,
    wpk_get_tile_ops,
    wpk_get_trace,
    wpk_graph_stats_get,
    wpk_last_error,
    wpk_load_weights,
    wpk_prefill,
    wpk_select_program,
    wpk_set_block_table,
    wpk_simulate,
    wpk_step,
    wpk_verify_graph,
    wpk_workspace_size,
)
