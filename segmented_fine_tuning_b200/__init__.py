"""B200-native HGA per-segment attention step.

The compute lives in libhga.so (hand-written sm_100a kernels behind a C ABI,
include/hga.h).  This package is its thin binding plus the buffer plumbing of
one attention step (``step.AttentionStep``) and of the full segmented pass
(``segmented.SegmentedPass``).
"""
from ._binding import (  # noqa: F401
    BlockCache, Dims, HgaError, LIB_PATH, hga_append_segment, hga_attn_bwd, hga_attn_uses_tensor_cores, hga_attn_bwd_dkdv, hga_attn_bwd_sparse, spaco_sample_blocks, hga_attn_bwd_noalloc, hga_attn_bwd_dq, hga_attn_bwd_preprocess,
    hga_attn_bwd_workspace_size, hga_attn_fwd, hga_block_summaries, hga_cache_segment, hga_decode_attn,
    hga_decode_select, hga_decode_workspace_size,
    hga_device_status, hga_fetch_blocks, hga_gather_blocks_mapped, hga_fetch_blocks_cached, hga_offload_segment, hga_remap_idx, hga_segment_summaries, hga_select_topk, hga_selftest_attn_fwd_stalled,
    hga_selftest_umma, hga_set_forward_heads_per_cta,
    hga_status_string, load_library,
)
