"""Flint sink-aware sliding/full GQA attention for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``libflint_attn.so`` (C ABI in
``include/flint_attn.h``); ``flint_attn`` is its thin ctypes binding.
"""
