"""fp64 CPU oracle for paged GQA decode attention (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the bench's CPU-baseline leg use
this package.  It wraps ``pgd_oracle.c`` (plain C, single-threaded, fp64) via
ctypes and never touches the CUDA library.
"""
from .oracle import (  # noqa: F401
    BF16, E4M3, build_oracle, lib_path, bf16_to_double, e4m3_to_double,
    kv_append, paged_decode, paged_decode_rows, paged_decode_tiled,
    merge_partials, OracleError, e4m3_from_double, kv_append_quant, paged_decode_window,
    paged_decode_multi,
)
