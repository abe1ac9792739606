"""Paged GQA decode attention for B200 (sm_100a).

The compute lives in libpgd.so (hand-written CUDA, C ABI in include/pgd.h);
this package only marshals torch tensors to it.  `kvp` splits one sequence's
KV over the ranks of a process group.
"""
from ._binding import (  # noqa: F401
    PGD_KV_BF16, PGD_KV_FP8_E4M3, PGDError, LIB_PATH, lib_path, load_library, kv_append,
    kv_append_quant, paged_decode_attention, paged_decode_attention_ex,
    paged_decode_attention_noalloc, paged_decode_partial, kvp_plan, decode_step,
    merge_partials, decode_workspace_bytes, get_device_error, shutdown, set_decode_math,
    get_decode_math, debug_set_wait_limit_ns, debug_get_wait_limit_ns, decode_grid,
)
from . import kvp  # noqa: F401,E402

__all__ = ["kv_append", "kv_append_quant", "paged_decode_attention", "paged_decode_attention_ex",
           "paged_decode_attention_noalloc", "paged_decode_partial", "kvp_plan", "decode_step",
           "merge_partials", "decode_workspace_bytes", "get_device_error", "shutdown",
           "set_decode_math", "get_decode_math", "debug_set_wait_limit_ns",
           "debug_get_wait_limit_ns", "decode_grid", "PGDError", "load_library", "lib_path", "kvp",
           "PGD_KV_BF16", "PGD_KV_FP8_E4M3"]
