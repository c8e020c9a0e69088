"""Attention over a paged KV cache on B200 (sm_100a): Python binding.

The work happens in ``libtfpaged.so`` (hand-written CUDA kernels behind the
C ABI declared in ``include/tf_paged.h``).  This package only marshals torch
tensors into that ABI; it has no fallback: the first use of any ``tf_*`` name
without the built library raises ImportError, and every call runs the CUDA
kernels or fails.  ``verify_paged_gqa_b200.build`` compiles the library and
imports without it.
"""
_EXPORTS = (
    "TF_DEV_BAD_LEN", "TF_DEV_BAD_PAGE", "TF_DEV_TIMEOUT", "TF_EINVAL", "TF_ENOSPACE",
    "TF_ECUDA", "TF_EUNSUPPORTED", "TF_OK", "TFError", "library_path", "raw",
    "tf_kv_copy_state", "tf_kv_put_rows", "tf_paged_attn_decode", "tf_paged_attn_prompt", "tf_paged_attn_verify",
    "tf_paged_attn_verify_tree", "tf_paged_attn_workspace_bytes", "tf_status_str",
    "tf_workspace_status", "tf_testing_paged_attn",
)
__all__ = list(_EXPORTS)


def __getattr__(name):
    if name in _EXPORTS:
        from . import _abi
        return getattr(_abi, name)
    raise AttributeError(f"module {__name__!r} has no attribute {name!r}")
