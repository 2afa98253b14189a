"""SparK on B200: query-aware unstructured key-cache channel pruning at
prefill and recover-then-attend decode attention, as hand-written sm_100a
CUDA kernels behind a C ABI (include/spark.h), with a thin ctypes binding.

Method: SparK (arXiv 2508.15212), as described by the paper walkthrough
"KV Cache 还能再砍一刀：SparK 在通道维度上做了一件被忽略多年的事" (sections
3.1-3.3, Fig. 3) and the AMD blog "AAAI 2026 AMD论文Spark方法揭秘".
"""
from .binding import (  # noqa: F401
    KCache, SparkError, lib, spark_cache_bytes, spark_cache_sizes, spark_decode_attn,
    spark_device_status, spark_lambda_to_T, spark_prune, spark_prune_noalloc, spark_prune_grouped, spark_group_budget, spark_prune_values, spark_prune_think, spark_prune_topp,
    spark_decode_attn_topp, spark_topp_offsets_bytes, spark_topp_vals_used, spark_selftest_wait_timeout,
    spark_decode_attn_kv, spark_workspace_bytes_kv, spark_snapkv_evict, spark_snapkv_evict_rows, spark_pyramid_keep, spark_tail_append, spark_workspace_bytes,
    status_str, workspace, SPARK_BF16, SPARK_F32, SPARK_OP_DECODE, SPARK_OP_PRUNE, SPARK_OP_SNAPKV, SPARK_OP_THINK, SPARK_OP_TOPP,
    SPARK_F_DEGENERATE, SPARK_F_GAUSSIAN, SPARK_F_EXPONENTIAL, EXPORTS,
)
