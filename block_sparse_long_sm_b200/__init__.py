"""Block-sparse long-context attention prefill for B200 (sm_100a).

Selection (AnchorAttention anchor/stripe test or SALE relative-score test),
sparse causal attention and decode-shaped reuse of the selection run in the CUDA library ``lib/libspa.so`` behind
the C ABI of ``include/spa.h``; ``binding`` is its Python binding.  The
binding is imported on first use of any of its names, so ``build`` can run
before the library exists; using the binding without the library raises
ImportError (there is no fallback).
"""

import importlib

_BINDING_NAMES = (
    "EXPORTED", "LIB_PATH", "MODES", "SPA_DEBUG_STALL_ATTN",
    "SPA_ERR_CUDA", "SPA_ERR_INVALID", "SPA_ERR_TIMEOUT", "SPA_ERR_UNSUPPORTED",
    "SPA_ERR_WORKSPACE", "SPA_MODE_ANCHOR", "SPA_MODE_DENSE", "SPA_MODE_SALE", "SPA_OK",
    "SpaError", "SpaParams", "SpaStats", "check", "kept_flops", "make_params",
    "sparse_decode_attn", "sparse_decode_prepare", "sparse_decode_scratch_bytes",
    "sparse_fp8_quantize", "sparse_fp8_scales_floats", "sparse_fp8_scratch_bytes",
    "sparse_key_mass", "sparse_prefill_attn", "sparse_prefill_attn_fp8", "sparse_prefill_plan",
    "sparse_prefill_plan_static", "sparse_prefill_stats", "sparse_prefill_status_string",
    "sparse_prefill_workspace_bytes")

__all__ = list(_BINDING_NAMES)


def __getattr__(name):
    if name in _BINDING_NAMES:
        return getattr(importlib.import_module(".binding", __name__), name)
    raise AttributeError(name)
