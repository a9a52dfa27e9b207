"""Block-causal sink + window TwinCache attention for B200 (sm_100a).

The compute lives in ``libsa.so`` (CUDA kernels behind a C ABI, include/sa.h).
``_binding`` exposes each C entry point under its own name; ``StreamingAttention``
is a small convenience wrapper that owns the device buffer (allocated through
PyTorch) and passes tensors' device pointers and the current CUDA stream.
"""

from ._binding import (  # noqa: F401
    SA_OK, SA_ERR_INVALID_ARG, SA_ERR_STATE, SA_ERR_UNSUPPORTED, SA_ERR_CUDA, SA_ERR_TIMEOUT,
    SA_ERR_RANGE, SA_ERR_BOUNDS, SA_BUILD_DEVICE_CHECKS, sa_build_info,
    SA_TIER_NOISY, SA_TIER_CLEAN, SaConfig, SaError, make_config, lib, header_symbols,
    sa_validate_config, sa_required_bytes, sa_create, sa_destroy, sa_reset, sa_append_chunk,
    sa_append_chunk_frames, sa_set_reference, sa_attend, sa_attend_frames, sa_attend_aligned,
    sa_stage_keys,
    sa_stage_keys_frames, sa_attend_staged, sa_debug_attend_simt, sa_attend_noalloc, sa_debug_exp2,
    sa_debug_attend_stalled, sa_attend_sparse, sa_block_grid,
    sa_chunk_count, sa_debug_inject_cuda_error, sa_debug_kernel_clock, sa_debug_layout, sa_plan, sa_stream_plan, sa_slot_of,
    sa_get_status, last_error, SA_PAYLOAD_FP8, SA_PAYLOAD_BF16, sa_exchange_block_bytes,
    sa_exchange_pack, sa_exchange_unpack, sa_exchange_pack_to, sa_ipc_handle, sa_ipc_open,
    sa_ipc_close, sa_ipc_alloc, sa_ipc_free,
)
from .stream import StreamingAttention  # noqa: F401
