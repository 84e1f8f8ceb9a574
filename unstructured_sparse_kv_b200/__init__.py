"""B200-native (sm_100a) Mustafar hot path: per-token magnitude pruning of the K/V caches,
bitmap compression, runtime append and decode attention over the compressed caches.

The compute runs in ``libmustafar.so`` (hand-written CUDA); this package only marshals
torch tensors into its C ABI (see ``include/mustafar.h``).
"""
from ._lib import (ABI_SYMBOLS, DEVERR_LEN_RANGE, DEVERR_POS_RANGE, HEAD_DIM, WINDOW_TOKENS, CompressedCache,
                   MustafarError, load, mustafar_append, mustafar_cache_sizes, mustafar_cache_sizes_channel,
                   mustafar_cache_sizes_per_head, mustafar_compress, mustafar_decode_attn,
                   mustafar_decode_attn_noalloc, mustafar_decode_plan_cluster, mustafar_decode_plan_splits,
                   mustafar_decode_step,
                   mustafar_decode_workspace_bytes, mustafar_dense_decode_attn, mustafar_keep_count,
                   mustafar_keep_count_channel, PreparedCall, prepare_decode_step, capture_decode_steps)

__all__ = ["ABI_SYMBOLS", "DEVERR_LEN_RANGE", "DEVERR_POS_RANGE", "HEAD_DIM", "WINDOW_TOKENS", "CompressedCache",
           "MustafarError", "load", "mustafar_append", "mustafar_cache_sizes", "mustafar_cache_sizes_channel",
           "mustafar_cache_sizes_per_head", "mustafar_compress", "mustafar_decode_attn",
           "mustafar_decode_attn_noalloc", "mustafar_decode_plan_cluster", "mustafar_decode_plan_splits",
           "mustafar_decode_step",
           "mustafar_decode_workspace_bytes", "mustafar_dense_decode_attn", "mustafar_keep_count",
           "mustafar_keep_count_channel", "PreparedCall", "prepare_decode_step", "capture_decode_steps"]
