"""Gated delta-rule recurrence (Gated DeltaNet / Gated DeltaNet-2) for B200 (sm_100a).

The compute path is libgdn.so (CUDA kernels behind the C ABI in include/gdn.h); this package
only marshals arguments.  See gdn.py for the calls.
"""
from .gdn import (GdnError, gdn_chunk_bwd, gdn_chunk_fwd, gdn_chunk_fwd_noalloc, gdn_decode_step,
                  gdn_layer_core_fwd, load)

__all__ = ["GdnError", "gdn_chunk_fwd", "gdn_chunk_fwd_noalloc", "gdn_chunk_bwd", "gdn_decode_step", "gdn_layer_core_fwd",
           "load"]
