"""fp64 CPU oracle of the frame-wise delta-rule memory (VDA).

Test infrastructure only: imported by the tests, the smoke check and the
benchmark's CPU-baseline leg, never by the product path.
"""
from .vda import (  # noqa: F401
    bridge_factors,
    bridged_readout,
    chunk_maps,
    chunk_readout,
    frame_stats,
    frame_update,
    gated_rmsnorm,
    is_anchor,
    num_chunks,
    readout_state,
    rel_frobenius,
    scan_states,
    stream_bridge_tail,
    stream_segment,
    text_state,
    transition,
    vda_head,
)
