"""TurboQuant compressed-KV hot path for NVIDIA B200 (sm_100a).

Python face of the C ABI in ``include/tq.h`` (``libtq.so``, built in-tree by
``kv_cache_vector_05_b200.build``): two-stage K/V compression (rotation,
Lloyd-Max codes, 1-bit QJL residual signs, value group quantization, bit
packing) and decode attention read straight from the packed cache.
"""
from ._lib import (  # noqa: F401
    Context, TQError, tq_codebook_load, tq_free, tq_compress_kv, tq_compress_kv_slots, tq_decode_attention,
    tq_decode_attention_paged, tq_decode_attention_partial, tq_merge_attention,
    tq_decode_workspace_bytes, tq_decompress, tq_haar_from_gaussian, tq_lloyd_max_codebook,
    tq_status_string, tq_set_profile_events, tq_check_device, tq_decode_attention_static,
    tq_decode_static_scratch_capacity, tq_set_decode_kernel, tq_decode_kernel_for, EXPORTED, LIB_PATH, TQ_F32,
    TQ_BF16, TQ_ROT_HADAMARD, TQ_ROT_HAAR, TQ_DECODE_AUTO, TQ_DECODE_TCGEN05, TQ_DECODE_MMA, TQ_DECODE_CUDA_CORE,
    DECODE_KERNEL_NAMES,
)
