"""sbsa: dynamic block-sparse self-attention for B200 (sm_100a).

The compute lives in ``libsbsa.so`` (hand-written CUDA behind a C ABI declared in
``include/sbsa.h``).  ``video_dit_dynamic_b200.sbsa`` is the thin ctypes binding;
importing this package does not load the library, calling any entry point does, and
it raises if the library is missing -- there is no CPU fallback.
"""
__all__ = ["sbsa", "inputs"]
