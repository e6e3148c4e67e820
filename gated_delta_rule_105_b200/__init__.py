"""B200-native chunked gated delta rule (GDN), Gated Delta Rule-2 and KDA: forward, backward and decode.

The compute lives in ``libgdn.so`` (hand-written sm_100a CUDA behind a C ABI declared in
``include/gdn.h``); :mod:`.binding` marshals torch tensors into it.  :mod:`.inputs` draws seeded
synthetic inputs of the shapes the method is measured on.
"""
from .binding import (GdnError, bwd_workspace_bytes, check_error, chunk_gated_delta_rule, decode_fwd, gdn2_chunk_fwd,
                      gdn2_bwd_workspace_bytes, gdn2_chunk_bwd, gdn2_workspace_bytes, gdn_chunk_bwd,
                      gdn_chunk_fwd, gdn_chunk_fwd_noalloc, gdn_kda_chunk_bwd, gdn_kda_chunk_fwd, last_kernel, load_library,
                      output_gate_fwd, prelude_fwd, profile_enable, profile_take, set_kernel, workspace_bytes)

__all__ = ["GdnError", "bwd_workspace_bytes", "check_error", "chunk_gated_delta_rule", "decode_fwd", "gdn2_chunk_fwd",
           "gdn2_bwd_workspace_bytes", "gdn2_chunk_bwd", "gdn2_workspace_bytes", "gdn_chunk_bwd",
           "gdn_chunk_fwd", "gdn_chunk_fwd_noalloc", "gdn_kda_chunk_bwd", "gdn_kda_chunk_fwd", "last_kernel", "load_library",
           "output_gate_fwd", "prelude_fwd", "profile_enable", "profile_take", "set_kernel", "workspace_bytes"]
