"""Gated DeltaNet (gated delta rule) hot path on NVIDIA B200 (sm_100a).

The computation lives in the C-ABI library libgdn.so (include/gdn.h); this
package holds its build script, a thin ctypes binding (`gdn`) and the seeded
synthetic input generators (`inputs`).
"""
from .gdn import (  # noqa: F401
    GdnError,
    debug_device_errors,
    debug_set_spin_limit,
    gdn_ba_gates,
    gdn_chunk_prefill,
    gdn_chunk_prefill_workspace_bytes,
    gdn_flag_clear,
    gdn_fold,
    gdn_stash_seq_floats,
    gdn_verify_parent,
    gdn_verify_woa,
    version,
)
