"""CKDA (Complex Kimi Delta Attention) for NVIDIA B200: chunked forward and
decode step as hand-written sm_100a CUDA kernels behind a C ABI.

``ckda`` is the Python binding of that ABI; ``inputs`` draws the seeded
synthetic workloads; ``build`` compiles the library in-tree.
"""
from . import ckda, inputs  # noqa: F401

__all__ = ["ckda", "inputs"]
