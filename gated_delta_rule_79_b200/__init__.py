"""Gated delta rule token mixers (GDN, KDA) on B200: Python binding of libgdr.

    from gated_delta_rule_79_b200 import gdn_prefill, kda_prefill, gdn_decode, kda_decode

The names resolve lazily to ``_lib`` so that ``python -m
gated_delta_rule_79_b200.build`` works before the library exists; using any of
them without a built ``libgdr.so`` raises ImportError (there is no fallback).
"""

_PUBLIC = ("gdn_prefill", "kda_prefill", "gdn_decode", "kda_decode", "gdn_verify", "kda_verify",
           "gdn_prefill_varlen", "kda_prefill_varlen", "gdn_backward", "kda_backward",
           "backward_workspace_bytes", "PROLOGUE_L2NORM_QK", "PROLOGUE_GATE_LOGIT",
           "VERIFY_MAX_TOKENS", "prefill_workspace",
           "workspace_status", "check_status", "noalloc_status", "prefill_path", "timing_start", "timing_stop", "GdrError", "lib", "LIB_PATH", "EXPORTS", "GDR_OK",
           "GDR_ERR_INVALID_ARG", "GDR_ERR_UNSUPPORTED", "GDR_ERR_CUDA", "GDR_ERR_TIMEOUT",
           "GDR_F32", "GDR_BF16", "CHUNK")

__all__ = list(_PUBLIC)


def __getattr__(name):
    if name in _PUBLIC:
        from . import _lib
        return getattr(_lib, name)
    raise AttributeError(name)
