"""Exact softmax attention (forward and training backward) for NVIDIA B200 (sm_100a).

The computation lives in libfa.so (hand-written tcgen05/TMA kernels behind the C ABI of
include/fa.h); this package only builds it (``build``) and binds it (``fa``).
"""
from .fa import (FAError, attention_backward, attention_forward, default_scale, fa_bwd,
                 fa_bwd_alibi, fa_bwd_dkdv, fa_bwd_dq, fa_bwd_noalloc, fa_bwd_preprocess,
                 fa_bwd_workspace_bytes, fa_debug_set_fault, fa_debug_status, fa_fwd,
                 fa_fwd_alibi, fa_status_string, fa_version, fa_window_t)

__all__ = ["FAError", "attention_backward", "attention_forward", "default_scale", "fa_bwd",
           "fa_bwd_alibi", "fa_bwd_dkdv", "fa_bwd_dq", "fa_bwd_noalloc", "fa_bwd_preprocess",
           "fa_bwd_workspace_bytes", "fa_debug_set_fault", "fa_debug_status", "fa_fwd",
           "fa_fwd_alibi", "fa_status_string", "fa_version", "fa_window_t"]
