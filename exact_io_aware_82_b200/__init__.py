"""Exact IO-aware attention for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``libattn.so`` built from ``csrc/``; ``attn`` is its thin
ctypes binding.  Importing the package does not load the library; the first call does, and it
raises if the library is missing or no CUDA device is present.
"""

from . import accounting  # noqa: F401

__all__ = ["accounting"]
