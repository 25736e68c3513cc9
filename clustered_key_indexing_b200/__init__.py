"""B200 (sm_100a) Latent Sparse Attention: indexer + attention path.

Thin PyTorch-facing binding of liblsa.so (include/lsa.h).  PyTorch only
allocates device memory and provides streams; every step runs in the
library's CUDA kernels.  See `api` for the calls.
"""
from .api import (Cache, Config, Decode, KernelTimer, Tree, attn_backward, build_buckets, build_tree, check_device_error,
                  fit_pca, lse_combine, prefill, prefill_chunk, prefill_host, prefill_workspace_bytes, query_latent,
                  select, select_attn, select_attn_workspace_bytes, select_workspace_bytes, shard_build_buckets,
                  shard_cand_cap, shard_candidates, shard_merge, sparse_attn, sparse_attn_partial)

__all__ = ["Cache", "Config", "Decode", "KernelTimer", "Tree", "attn_backward", "build_buckets", "build_tree", "check_device_error",
           "fit_pca", "lse_combine", "prefill", "prefill_chunk", "prefill_host", "prefill_workspace_bytes",
           "query_latent", "select", "select_attn", "select_attn_workspace_bytes", "select_workspace_bytes",
           "shard_build_buckets", "shard_cand_cap", "shard_candidates", "shard_merge", "sparse_attn",
           "sparse_attn_partial"]
