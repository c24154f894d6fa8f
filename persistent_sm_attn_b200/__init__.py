"""Deterministic attention backward for B200 (sm_100a) with DASH schedules.

The compute path lives in the C-ABI library ``libdash_attn.so`` (CUDA kernels
and host runtime under ``csrc/``); ``binding`` marshals arguments to it.  The
binding is loaded on first use of one of its names, so that
``persistent_sm_attn_b200.inputs`` can be imported without the library.
"""
from __future__ import annotations

_BINDING_NAMES = {
    "dash_attn_fwd", "dash_attn_bwd", "dash_attn_sync_status", "dash_status_string",
    "dash_sched_simulate", "dash_sched_table", "dash_dag_longest_path", "dash_set_spin_limit_us",
    "dash_bwd_num_ctas", "dash_release_workspace", "dash_profile_begin", "dash_profile_end", "dash_trace_bwd", "dash_attn_bwd_noalloc", "dash_inject_fault", "SCHEDULES", "DashError", "load",
}


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
