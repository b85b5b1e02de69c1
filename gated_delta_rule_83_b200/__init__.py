"""B200-native Kimi Delta Attention (KDA) operator: chunked prefill and decode (libkda.so, sm_100a).

Public API (a thin binding of the C ABI in include/kda.h):

    out, S_final = chunk_fwd(q, k, v, log_alpha, beta, S0=None, cu_seqlens=None)
    out, S_final = chunk_fwd_host(q, k, v, log_alpha, beta)  # host tensors, pipelined copies
    chunk_fwd_noalloc(q, k, v, log_alpha, beta, S0, out, S_final)  # no device allocation at all
    grads = chunk_bwd(q, k, v, log_alpha, beta, dout, S0=None, dS_final=None)   # training backward
    out = decode_step(q, k, v, log_alpha, beta, S)        # S updated in place
    check()                                               # raise on a device-side error
"""
from .kda import (PROLOGUE_BETA_LOGITS, PROLOGUE_GATE_BF16, PROLOGUE_GATE_LOGITS, PROLOGUE_L2NORM_QK,  # noqa: F401
                  KdaError,
                  bwd_workspace_size, check, chunk_bwd, chunk_fwd, chunk_fwd_host, chunk_fwd_noalloc, decode_step, gated_rmsnorm,
                  load_library, profile_begin, profile_end, release_host_resources, release_workspaces, version,
                  workspace_size)

__all__ = ["chunk_fwd", "chunk_fwd_host", "chunk_fwd_noalloc", "chunk_bwd", "decode_step", "gated_rmsnorm", "check",
           "workspace_size", "bwd_workspace_size", "release_workspaces", "release_host_resources", "load_library",
           "version", "KdaError"]
