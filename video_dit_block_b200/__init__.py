"""Training-free block-sparse self-attention for video DiTs, native to B200 (sm_100a).

The compute path is a C-ABI CUDA library (include/sba.h, csrc/); this package is its
Python binding.  See `sba` for the calls.
"""
from .sba import (SbaError, attention, attention_compensated, attention_mean_compensated, attention_paired,
                  attention_to_shards, block_means, dense_attention, device_status, gather_tokens, keep_count,
                  keep_count_budget, keep_token_count, kmax_for, lib, lse_workspace_size,
                  mean_compensation_workspace_size, pair_query_blocks, pool_select, pool_select_lse,
                  pool_select_means, qk_norm_rope_pool, set_attention_kernel, set_wait_limit, sparse_attention,
                  token_prune, workspace_size)

__all__ = ["SbaError", "attention", "attention_compensated", "attention_mean_compensated", "attention_paired",
           "attention_to_shards", "block_means", "dense_attention", "device_status", "gather_tokens", "keep_count",
           "keep_count_budget", "keep_token_count", "kmax_for", "lib", "lse_workspace_size",
           "mean_compensation_workspace_size", "pair_query_blocks", "pool_select", "pool_select_lse",
           "pool_select_means", "qk_norm_rope_pool", "set_attention_kernel", "set_wait_limit", "sparse_attention",
           "token_prune", "workspace_size"]
