"""B200-native sparse-V decode attention over a block-quantized KV cache.

The compute lives in ``libkvq.so`` (CUDA for sm_100a, C ABI declared in
``include/kvq.h``); this package is its Python binding plus a small cache
wrapper that owns device memory through PyTorch.
"""
from ._binding import (  # noqa: F401
    FORMATS, KVQ_ERR_CUDA, KVQ_ERR_DEVICE, KVQ_ERR_INVALID_ARG, KVQ_ERR_UNSUPPORTED,
    KVQ_ERR_WORKSPACE, KVQ_FLAG_BAD_PAGE, KVQ_FLAG_BAD_SEQLEN, KVQ_FLAG_TIMEOUT, KVQ_FMT_LUT4,
    KVQ_FMT_Q4_0, KVQ_FMT_Q8_0, KVQ_FMT_NVFP4, KVQ_MAX_BATCH, KVQ_OPT_SHARED_MAX, KVQ_OPT_GLOBAL_MAX, KVQ_OPT_V_KEPT_ONLY, KVQ_OPT_V_WITH_K, KVQ_MAX_GROUP, KVQ_MAX_SPLIT_TOKENS, KVQ_OK,
    KvqCacheDesc, KvqError, LIB_PATH, kvq_code_row_bytes, kvq_combine, kvq_decode_attn, kvq_decode_attn_noalloc, KVQ_NOALLOC_SCRATCH_BYTES, kvq_noalloc_read_flags,
    kvq_lloyd_max_codebook, kvq_quantize, kvq_quantize_kv, kvq_read_device_flags, kvq_resolve_split, kvq_resolve_cluster,
    kvq_scale_row_count, kvq_selftest_wait, kvq_status_string, kvq_workspace_init, kvq_workspace_size, make_desc)
from .cache import QuantizedKVCache  # noqa: F401
