"""TurboQuant-style compressed KV cache for NVIDIA B200 (sm_100a).

The compute lives in the C-ABI library ``libtq_b200.so`` (include/tq.h);
this package is its thin Python binding plus the seeded synthetic workloads.
"""
from ._lib import (TQ_DEV_CHANNEL_RANGE, TQ_DEV_LEN_RANGE, TQ_DEV_NORM_OVERFLOW, TQ_DEV_POS_RANGE, TQ_F16,
                   TQ_F32, TQ_MAX_OUTLIERS, Codebook, KVDesc, TQError, lib)
from .api import (Cache, VOutliers, alloc_cache, alloc_outliers, alloc_workspace, cache_shapes,
                  codebook_arrays, decode_attention, decode_attention_multi, decode_attention_multi_v2,
                  decode_attention_multi_v3, decode_attention_noalloc, decode_attention_v2, decode_attention_v3, decode_step, decode_workspace_size, encode_kv,
                  encode_kv_v2, encode_kv_v3, kv_desc, make_codebook, make_tcq_codebook, outlier_row,
                  pick_outlier_channels, read_device_status, sign_vector)

__all__ = [
    "Cache", "Codebook", "KVDesc", "TQError", "TQ_F16", "TQ_F32", "TQ_DEV_CHANNEL_RANGE", "TQ_DEV_LEN_RANGE",
    "TQ_DEV_NORM_OVERFLOW", "TQ_DEV_POS_RANGE", "TQ_MAX_OUTLIERS", "VOutliers", "alloc_cache", "alloc_outliers",
    "alloc_workspace", "cache_shapes", "codebook_arrays", "decode_attention", "decode_attention_multi",
    "decode_attention_multi_v2", "decode_attention_multi_v3", "decode_attention_noalloc", "decode_attention_v2", "decode_attention_v3", "decode_step",
    "decode_workspace_size", "encode_kv", "encode_kv_v2", "encode_kv_v3", "kv_desc", "lib", "make_codebook",
    "make_tcq_codebook", "outlier_row", "pick_outlier_channels", "read_device_status", "sign_vector",
]
