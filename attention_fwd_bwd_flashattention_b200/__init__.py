"""Exact relative-position attention (T5, Shaw, Transformer-XL, DeBERTa), forward
and backward, as hand-written sm_100a CUDA behind a C ABI (include/relpos_attn.h).

``binding`` is the thin ctypes layer over the compiled library; ``inputs`` holds the
seeded synthetic workloads.  Importing the package does not load the library.
"""
__all__ = ["binding", "inputs", "build"]
