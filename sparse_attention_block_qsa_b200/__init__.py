"""QSA (Qwen Sparse Attention) MQA indexer score for NVIDIA B200 (sm_100a).

Hand-written CUDA kernels behind a C ABI (``include/qsa.h``, ``libqsa.so``):
paged decode / spec-decode scores over a bf16, fp16 or fp8 E4M3 key cache,
packed prefill scores with per-row key intervals, per-row top-k selection,
the fused prefill + top-k path, mixed decode + prefill batches from the
paged cache in one call, and the core-attention stage after it
(block-to-token index expansion, sparse attention over paged K/V).  This package is the thin Python binding over
that library.
"""
from ._abi import (SCALE, QSAError, device_error, expand_block_indices, lib, mqa_decode, mqa_decode_fp8,
                   mqa_paged_batch, mqa_prefill, mqa_prefill_topk, mqa_prefill_topk_noalloc,
                   paged_batch_workspace_size, prefill_intervals, prefill_topk_workspace_size, selftest_bounded_wait, sparse_attention,
                   sparse_attention_workspace_size, topk, topk_workspace_size)

__all__ = ["SCALE", "QSAError", "device_error", "expand_block_indices", "lib", "mqa_decode", "mqa_decode_fp8",
           "mqa_paged_batch", "mqa_prefill", "mqa_prefill_topk", "paged_batch_workspace_size", "mqa_prefill_topk_noalloc", "prefill_intervals",
           "prefill_topk_workspace_size", "selftest_bounded_wait", "sparse_attention",
           "sparse_attention_workspace_size", "topk", "topk_workspace_size"]
