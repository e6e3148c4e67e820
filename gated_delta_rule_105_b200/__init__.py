"""B200-native chunked gated delta rule (GDN) and Gated Delta Rule-2 forward pass.

The compute lives in ``libgdn.so`` (hand-written sm_100a CUDA behind a C ABI declared in
``include/gdn.h``); :mod:`.binding` marshals torch tensors into it.  :mod:`.inputs` draws seeded
synthetic inputs of the shapes the method is measured on.
"""
from .binding import (GdnError, check_error, chunk_gated_delta_rule, gdn2_chunk_fwd, gdn_chunk_fwd,
                      gdn_chunk_fwd_noalloc, last_kernel, load_library, profile_enable, profile_take, set_kernel,
                      workspace_bytes)

__all__ = ["GdnError", "check_error", "chunk_gated_delta_rule", "gdn2_chunk_fwd", "gdn_chunk_fwd",
           "gdn_chunk_fwd_noalloc", "last_kernel", "load_library", "profile_enable", "profile_take", "set_kernel",
           "workspace_bytes"]
