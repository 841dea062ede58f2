"""B200-native joint (prefix-LM) attention for pi0 / pi0.5-style VLA models.

The compute lives in ``libpiattn.so`` (CUDA for sm_100a, built from ``csrc/``),
reached through a C ABI declared in ``include/pi_attn.h``.  ``binding`` wraps
that ABI for torch tensors (argument marshalling only); ``workloads`` produces
seeded synthetic inputs.  Importing this package loads nothing; the library is
opened on first use and its absence is an error, never a fallback.
"""

__all__ = ["binding", "workloads"]
