"""Batch-invariant forward kernels for B200 (sm_100a) behind a C-ABI library.

The ops (``bi_rmsnorm``, ``bi_gemm``, ``bi_lora_shrink``, ``bi_lora_expand``,
``bi_decode_attn``) live in ``binding``; importing them loads the in-tree
``libbi.so`` and fails loudly if it has not been built.
"""
__version__ = "0.1.0"

_BINDING_NAMES = ("bi_rmsnorm", "bi_gemm", "bi_lora_shrink", "bi_lora_expand", "bi_decode_attn",
                  "library", "BIError")


def __getattr__(name):
    if name in _BINDING_NAMES:
        from . import binding
        return getattr(binding, name)
    raise AttributeError(name)
