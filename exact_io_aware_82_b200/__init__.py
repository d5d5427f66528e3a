"""Exact IO-aware attention for NVIDIA B200 (sm_100a).

The compute lives in the CUDA library ``libattn.so`` built from ``csrc/`` (``build.py``);
``attn`` is its thin ctypes binding.  Importing the package does not load the library; the
first call does, and raises if the library is missing or no sm_100 device is present.
"""

from . import accounting  # noqa: F401
from .attn import (MASK_CAUSAL, MASK_FULL, MASK_LOCAL_GLOBAL, MASK_SLIDING,  # noqa: F401
                   AttnError, attn_bwd, attn_bwd_workspace_bytes, attn_decode,
                   attn_decode_noalloc, attn_decode_num_splits, attn_decode_paged,
                   attn_decode_workspace_bytes, attn_fwd, attn_fwd_block_sparse, attn_fwd_f32,
                   attn_fwd_fp8, attn_fwd_varlen, attn_get_device_error)
