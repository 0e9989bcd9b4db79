"""MLA prefill attention + o_proj for NVIDIA B200 (sm_100a).

The compute lives in hand-written CUDA kernels behind a C ABI
(``include/mla.h``, built into ``libmla_b200.so`` next to this file);
``mla_causal_attention_attn_b200.binding`` is a thin ctypes layer over it.
Importing the package does not load the library; the first call does, and
fails loudly if it is missing.
"""
from . import inputs  # noqa: F401  (seeded synthetic inputs, no arithmetic)

__all__ = ["inputs"]
