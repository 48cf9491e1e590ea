"""Two-stage bucketed approximate top-k on B200 (sm_100a).

Method: "Approximate Top-k for Increased Parallelism" (arXiv 2412.04358): rows
are split into b interleaved buckets (element i -> bucket i mod b), each bucket
keeps its exact top-k_b, and a final exact top-k runs when the b*k_b
candidates exceed k.

The Python names mirror the C ABI in include/topk_b200.h; all work runs in the
CUDA library libtopk_b200.so (build: `python -m approximate_top_selection_b200.build`).
"""
from ._binding import (  # noqa: F401
    TOPK_EINVAL, TOPK_ECUDA, TOPK_ESCRATCH, TOPK_EUNSUPPORTED, TOPK_EWORKSPACE, TOPK_OK, TOPK_OP_BUCKETED,
    TOPK_OP_BUCKETED_BF16, TOPK_OP_EXACT, TOPK_OP_SCORE, TopkError, library_path, load_library, score_rerank, score_topk,
    topk_bucketed, topk_bucketed_bf16, topk_bucketed_merge, topk_bucketed_noalloc, topk_sample, topk_sample_rows, topk_device_status, topk_exact, topk_selftest_wait_timeout, topk_status_string, topk_workspace_bytes)
