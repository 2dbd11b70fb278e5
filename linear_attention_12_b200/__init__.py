"""B200-native Gated DeltaNet (GDN) layer: chunked prefill and decode step.

The compute lives in ``libgdn.so`` (hand-written CUDA for sm_100a behind a
C ABI declared in ``include/gdn.h``).  ``linear_attention_12_b200.gdn`` is a
thin ctypes binding with the same call names; it only marshals arguments.
Importing this package does not load the library; the first call does, and
fails loudly when the library is missing or no GPU is present.
"""

__all__ = ["gdn", "inputs"]
