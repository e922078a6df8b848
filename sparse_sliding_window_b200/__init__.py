"""Longformer self-attention (sliding window + dilation + causal + symmetric
global attention) for NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``liblf_attn.so`` built from ``csrc/``
(hand-written CUDA kernels); ``lf_attn`` is its thin ctypes binding.  Importing
this package loads nothing; the library is loaded on first use of ``lf_attn``.
"""
__all__ = ["lf_attn", "synth"]
