"""fp64 CPU oracle for LISA (Linear-Indexed Sparse Attention).

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this package: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline legs of ``bench.py`` do.  It shares no code with the CUDA path.
"""

from .lisa_ref import (
    indexer_scores,
    topm_select,
    window_select,
    topm_threshold,
    borderline_mask,
    sparse_attention,
    linear_update,
    linear_readout,
    gate_fuse,
    decode_step,
    prefill,
    indexer_kl,
    PROJ_FIELDS,
    proj_widths,
    project_in,
    project_out,
)

__all__ = [
    "indexer_scores",
    "topm_select",
    "window_select",
    "topm_threshold",
    "borderline_mask",
    "sparse_attention",
    "linear_update",
    "linear_readout",
    "gate_fuse",
    "decode_step",
    "prefill",
    "indexer_kl",
    "PROJ_FIELDS",
    "proj_widths",
    "project_in",
    "project_out",
]
