"""B200-native (sm_100a) single-token MLA decode over the latent KV cache.

The compute lives in ``libmla_b200.so`` (hand-written CUDA kernels behind the C
ABI declared in ``include/mla.h``); ``binding`` marshals torch tensors to it.
"""
from .binding import (  # noqa: F401
    PAGE_ROWS, Dims, DecodeStep, MLAError, absorb_q, cache_append, cache_append_fp8,
    cache_append_paged, cache_append_workspace_bytes, cache_fp8_row_bytes, cache_row_elems,
    combine, debug_inject_wait, decode, decode_default_splits, decode_fp8, decode_paged,
    decode_workspace_bytes, fold_output_weights, get_device_status, load_library,
    merge_partials, out_proj, out_proj_folded, out_proj_folded_workspace_bytes, prefill,
    prefill_workspace_bytes,
)
