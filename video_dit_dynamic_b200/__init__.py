"""sbsa: dynamic block-sparse self-attention for B200 (sm_100a).

The compute lives in ``libsbsa.so`` (hand-written CUDA behind a C ABI declared in
``include/sbsa.h``).  ``video_dit_dynamic_b200.sbsa`` is the thin ctypes binding;
``video_dit_dynamic_b200.ulysses`` drives Light-Ulysses sequence parallelism (buffers,
the head-level pipeline, the NCCL or peer-put exchange); ``inputs`` draws the seeded
synthetic workloads.  Importing this package does not load the library, calling any entry
point does, and it raises if the library is missing -- there is no CPU fallback.
"""
__all__ = ["sbsa", "inputs", "ulysses"]
