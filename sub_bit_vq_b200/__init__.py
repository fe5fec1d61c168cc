"""LoopVQ decode hot path for NVIDIA B200 (sm_100a).

The work happens in ``libloopvq.so`` (hand-written CUDA); this package only
loads it and marshals arguments. Importing it without the built library
raises ``ImportError``: there is no CPU fallback.
"""
from .binding import (  # noqa: F401
    LOOPVQ_DECODE_STATUS_BAD_PAGE,
    LOOPVQ_ENCODE_STATUS_TIMEOUT,
    LOOPVQ_ENCODE_STATUS_UNDRAINED,
    LOOPVQ_ENCODE_STATUS_BAD_SLOT,
    LOOPVQ_DECODE_STATUS_RANGE,
    LOOPVQ_DECODE_STATUS_SHARED_BASE,
    LOOPVQ_DECODE_STATUS_TIMEOUT,
    LOOPVQ_DECODE_STATUS_UNDRAINED,
    LOOPVQ_DTYPE_BF16,
    LOOPVQ_DTYPE_F32,
    LoopVQConfig,
    LOOPVQ_STATIC_SCRATCH_BYTES,
    LoopVQError,
    loopvq_bf16_decode_attn,
    loopvq_bf16_decode_workspace_bytes,
    loopvq_cache_layout,
    loopvq_decode_attn,
    loopvq_decode_attn_noalloc,
    loopvq_decode_workspace_bytes,
    loopvq_encode,
    loopvq_encode_evict,
    loopvq_encode_status,
    loopvq_kmeans_assign_bytes,
    loopvq_kmeans_step,
    loopvq_prefill_attn,
    loopvq_prefill_workspace_bytes,
    loopvq_status_string,
)
