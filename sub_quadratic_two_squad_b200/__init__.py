"""SQuad-Attention for B200 (sm_100a): a C-ABI CUDA library (include/squad_attn.h) and its binding.

The local pass attends inside windows that span all frames; the global pass attends, per slot,
across all windows with the local output as values (SQuad paper §3.2, appendix "Reachability").
"""
from .api import (  # noqa: F401
    HostRunner,
    SquadError,
    full_attn_flops,
    full_attn_fwd,
    make_kpass_params,
    make_params,
    squad_attention,
    squad_attn_bwd,
    squad_attn_bwd_kernels,
    squad_attn_bwd_workspace_bytes,
    squad_attn_flops,
    squad_window_solve,
    squad_attn_fwd,
    squad_attn_fwd_host,
    squad_attn_fwd_host_workspace_bytes,
    squad_attn_fwd_noalloc,
    squad_attn_fwd_status,
    squad_attn_fwd_workspace_bytes,
    squad_kpass_attention,
    squad_kpass_bwd,
    squad_kpass_flops,
    squad_kpass_fwd,
    squad_kpass_pass_params,
    squad_kpass_status,
    squad_seqpar_reorder,
)
