"""B200-native paged KV-cache append and paged decode attention.

The compute path is libpa.so (hand-written CUDA for sm_100a behind the C ABI
declared in include/pa.h); this package is its thin Python binding.
"""
from .binding import (  # noqa: F401
    PA_FLAG_CHECK, PA_FLAG_PDL, PA_FLAG_SELFTEST_STALL, PA_KV_BF16, PA_KV_E4M3, PA_PREFILL_AUTO, PA_PREFILL_TCGEN05, PA_PREFILL_TCGEN05_WS, PA_PREFILL_MMA, PA_KERNEL_AUTO, PA_KERNEL_SIMT, PA_KERNEL_TENSOR, PA_KERNEL_TENSOR_SPLIT, PA_OK, BlockManager, BlockPool,
    CacheDesc, DecodeOptions, DecodePlanInfo, PaError, declared_symbols, lib, pa_append_decode, pa_append_kv, pa_append_kv_e4m3, pa_copy_blocks,
    pa_decode, pa_decode_describe, pa_prefill,
    pa_decode_max_splits, pa_decode_noalloc, pa_decode_status, pa_decode_workspace_size, pa_rope_append_kv,
    pa_slot_mapping,
    pa_status_string,
)
