"""LightTransfer-Test prefill hot path on B200 (sm_100a).

A thin Python binding over the C ABI of ``liblt.so`` (declared in
``include/lt.h``).  Every function keeps the C name and only marshals
arguments: it checks tensor dtypes/devices/shapes, allocates outputs with
PyTorch when the caller passes none, and calls the library on the current CUDA
stream.  All arithmetic runs in the library's CUDA kernels; if the library is
missing the calls raise instead of falling back to anything else.
``PrefillStep`` (sharded.py) enqueues these calls for every layer of a
prefill, on one GPU or with the heads split over a process group.
"""
from __future__ import annotations

from .binding import (  # noqa: F401
    LT_ERR_CUDA,
    LT_ERR_INVALID_ARG,
    LT_ERR_TIMEOUT,
    LT_ERR_UNSUPPORTED,
    LT_OK,
    LtError,
    LtShape,
    library,
    library_path,
    lt_compact_kv,
    lt_attn_schedule,
    lt_device_status,
    lt_layer_score,
    lt_lazy_ratio,
    lt_prefill_attn,
    lt_prefill_attn_ratio,
    lt_prefill_attn_ratio_push,
    lt_queue_create,
    lt_queue_destroy,
    lt_queue_push,
    lt_queue_size,
    lt_select_layers,
    lt_selftest_wait_timeout,
    lt_status_string,
    lt_version,
    LayerQueue,
    DeviceQueue,
    layer_pointer_table,
    lt_compact_kv_pending,
    lt_compact_kv_layers,
    lt_dqueue_error,
    lt_dqueue_init,
    lt_dqueue_push,
    lt_dqueue_push_gathered,
    lt_dqueue_result,
    lt_dqueue_slots,
    lt_dqueue_state_bytes,
    lt_kv_pool_commit,
    lt_stream_append,
    lt_stream_decode,
    lt_decode_attn,
    lt_decode_attn_splitk,
    lt_decode_attn_splitk_noalloc,
    lt_decode_splitk_noalloc_capacity_bytes,
    lt_decode_splitk_workspace_bytes,
    lt_stream_ring_init,
)
from .build import build  # noqa: F401
from .sharded import (  # noqa: F401
    PrefillStep,
    gather_ratios,
    head_ratios,
    head_shard,
    pack_sequences,
    sequence_shard,
)
