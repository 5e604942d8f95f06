"""Exact ring attention (blockwise self-attention over D virtual ring positions) for
NVIDIA B200 (sm_100a).

The compute path is a C-ABI shared library (``libringattn.so``, declared in
``include/ring_attn.h``) of hand-written CUDA kernels; ``ring_attn`` is its thin ctypes
binding (argument marshalling only).  ``workloads`` holds the seeded synthetic inputs.

Import ``long_context_exact_fwd_b200.ring_attn`` for the operations; it raises at import
time when the CUDA library has not been built.
"""
__all__ = ["ring_attn", "workloads", "build"]
