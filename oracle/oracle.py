"""ctypes binding of the fp64 C oracle (test infrastructure only).

The oracle follows the plain definition of attention on the page
"attention kernels" (froggydisk, LLM serving / decoding), section "standard
attention", read through the block table of "batching and attention"
(beengineer500), section 3.4 PagedAttention.  See ``pgd_oracle.c`` for the
per-function citations.  Arrays are numpy; bf16 data travels as uint16 bit
patterns and FP8 E4M3 as uint8 bytes, so both sides read identical bytes.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

BF16 = 0
E4M3 = 1

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "pgd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lib = None


class OracleError(RuntimeError):
    pass


def lib_path() -> str:
    return _LIB


def build_oracle(force: bool = False) -> str:
    """Compile pgd_oracle.c with gcc into oracle/liboracle.so (in-tree)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-std=c99", "-fPIC", "-shared", "-Wall",
                               "-Wextra", "-fno-fast-math", "-ffp-contract=off",
                               "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def configure(lib):
    """Declare the C signatures on a loaded oracle library."""
    P = ctypes.c_void_p
    i32, i64, dbl = ctypes.c_int32, ctypes.c_int64, ctypes.c_double
    lib.pgdo_bf16_to_double.restype = dbl
    lib.pgdo_bf16_to_double.argtypes = [ctypes.c_uint16]
    lib.pgdo_e4m3_to_double.restype = dbl
    lib.pgdo_e4m3_to_double.argtypes = [ctypes.c_uint8]
    lib.pgdo_decode_bf16_array.argtypes = [P, P, i64]
    lib.pgdo_decode_e4m3_array.argtypes = [P, P, i64]
    lib.pgdo_kv_append.restype = ctypes.c_int
    lib.pgdo_kv_append.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32, i32]
    args = [P, P, P, i32, P, P, P, i32, P, i32, i32, i32, i32, i32, i32, dbl]
    lib.pgdo_paged_decode.restype = ctypes.c_int
    lib.pgdo_paged_decode.argtypes = args + [P, P]
    lib.pgdo_paged_decode_multi.restype = ctypes.c_int
    lib.pgdo_paged_decode_multi.argtypes = args + [i32, i32, P, P]
    lib.pgdo_paged_decode_window.restype = ctypes.c_int
    lib.pgdo_paged_decode_window.argtypes = args + [i32, P, P]
    lib.pgdo_paged_decode_rows.restype = ctypes.c_int
    lib.pgdo_paged_decode_rows.argtypes = args + [P, P, i32, P, P]
    lib.pgdo_paged_decode_tiled.restype = ctypes.c_int
    lib.pgdo_paged_decode_tiled.argtypes = args + [i32, i32, P, P]
    lib.pgdo_merge_partials.restype = ctypes.c_int
    lib.pgdo_merge_partials.argtypes = [P, P, i32, i32, i32, P, P]
    lib.pgdo_e4m3_from_double.restype = ctypes.c_uint8
    lib.pgdo_e4m3_from_double.argtypes = [dbl]
    lib.pgdo_encode_e4m3_array.argtypes = [P, P, i64]
    lib.pgdo_kv_append_quant.restype = ctypes.c_int
    lib.pgdo_kv_append_quant.argtypes = [P, P, P, i32, P, P, P, P, i32, i32, i32, i32]
    return lib


def set_library(lib):
    """Swap the loaded library (used by the mutation test); returns the old one."""
    global _lib
    old, _lib = _lib, lib
    return old


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        _lib = configure(ctypes.CDLL(_LIB))
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def _c(a, dtype):
    return None if a is None else np.ascontiguousarray(a, dtype=dtype)


def bf16_to_double(bits: np.ndarray) -> np.ndarray:
    bits = _c(bits, np.uint16)
    out = np.empty(bits.shape, np.float64)
    _load().pgdo_decode_bf16_array(_ptr(bits), _ptr(out), bits.size)
    return out


def e4m3_to_double(bits: np.ndarray) -> np.ndarray:
    bits = _c(bits, np.uint8)
    out = np.empty(bits.shape, np.float64)
    _load().pgdo_decode_e4m3_array(_ptr(bits), _ptr(out), bits.size)
    return out


def kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, block_size):
    """Returns new (k_cache, v_cache) arrays; inputs are not modified.

    k_new/v_new: [N_tok][Hkv][D] uint16 (bf16 bits) or uint8 (e4m3 bytes);
    caches: [num_blocks][Hkv][bs][D] of the same element type.
    """
    k_cache = np.array(k_cache, copy=True, order="C")
    v_cache = np.array(v_cache, copy=True, order="C")
    k_new = np.ascontiguousarray(k_new)
    v_new = np.ascontiguousarray(v_new)
    assert k_new.dtype == k_cache.dtype and v_new.dtype == v_cache.dtype
    slots = _c(slot_mapping, np.int64)
    nb, hkv, bs, d = k_cache.shape
    assert bs == block_size
    rc = _load().pgdo_kv_append(_ptr(k_new), _ptr(v_new), _ptr(slots), len(slots),
                                _ptr(k_cache), _ptr(v_cache), hkv, d, bs, nb,
                                k_cache.dtype.itemsize)
    if rc:
        raise OracleError(f"pgdo_kv_append rc={rc}")
    return k_cache, v_cache


def _decode_args(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                 k_scale=None, v_scale=None):
    q = _c(q, np.uint16)
    kv_dtype = BF16 if k_cache.dtype == np.uint16 else E4M3
    k_cache = np.ascontiguousarray(k_cache)
    v_cache = np.ascontiguousarray(v_cache)
    bt = _c(block_table, np.int32)
    cl = _c(context_lens, np.int32)
    ks = _c(k_scale, np.float32)
    vs = _c(v_scale, np.float32)
    B, Hq, D = q.shape
    nb, hkv, bs, d2 = k_cache.shape
    assert hkv == num_kv_heads and d2 == D and bt.shape[0] == B
    keep = (q, k_cache, v_cache, bt, cl, ks, vs)
    args = [_ptr(q), _ptr(k_cache), _ptr(v_cache), kv_dtype, _ptr(ks), _ptr(vs), _ptr(bt),
            bt.shape[1], _ptr(cl), B, Hq, hkv, D, bs, nb, float(scale)]
    return args, keep, (B, Hq, D)


def paged_decode(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                 k_scale=None, v_scale=None):
    """Plain definition; returns (out fp64 [B][Hq][D], lse fp64 [B][Hq])."""
    args, keep, (B, Hq, D) = _decode_args(q, k_cache, v_cache, block_table, context_lens,
                                          num_kv_heads, scale, k_scale, v_scale)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().pgdo_paged_decode(*args, _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_paged_decode rc={rc}")
    del keep
    return out, lse


def paged_decode_rows(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                      rows_seq, rows_head, k_scale=None, v_scale=None):
    """Plain definition on selected (seq, q head) rows only."""
    args, keep, (B, Hq, D) = _decode_args(q, k_cache, v_cache, block_table, context_lens,
                                          num_kv_heads, scale, k_scale, v_scale)
    rs = _c(rows_seq, np.int32)
    rh = _c(rows_head, np.int32)
    out = np.empty((len(rs), D), np.float64)
    lse = np.empty((len(rs),), np.float64)
    rc = _load().pgdo_paged_decode_rows(*args, _ptr(rs), _ptr(rh), len(rs), _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_paged_decode_rows rc={rc}")
    del keep
    return out, lse


def paged_decode_tiled(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                       tile_tokens, partition_tokens, k_scale=None, v_scale=None):
    """Online-softmax tiles inside partitions, then the LSE merge."""
    args, keep, (B, Hq, D) = _decode_args(q, k_cache, v_cache, block_table, context_lens,
                                          num_kv_heads, scale, k_scale, v_scale)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().pgdo_paged_decode_tiled(*args, int(tile_tokens), int(partition_tokens),
                                         _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_paged_decode_tiled rc={rc}")
    del keep
    return out, lse


def merge_partials(o_part, lse_part):
    """o_part [P][rows][D], lse_part [P][rows] -> (out [rows][D], lse [rows])."""
    o_part = _c(o_part, np.float64)
    lse_part = _c(lse_part, np.float64)
    P, R, D = o_part.shape
    out = np.empty((R, D), np.float64)
    lse = np.empty((R,), np.float64)
    rc = _load().pgdo_merge_partials(_ptr(o_part), _ptr(lse_part), P, R, D, _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_merge_partials rc={rc}")
    return out, lse


def e4m3_from_double(x: np.ndarray) -> np.ndarray:
    """Nearest E4M3 bytes (ties to even, saturating at +-448)."""
    x = _c(x, np.float64)
    out = np.empty(x.shape, np.uint8)
    _load().pgdo_encode_e4m3_array(_ptr(x), _ptr(out), x.size)
    return out


def kv_append_quant(k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, block_size):
    """bf16 rows (uint16 bits) [N][Hkv][D] -> E4M3 cache bytes; returns new
    (k_cache, v_cache); inputs are not modified."""
    k_cache = np.array(k_cache, dtype=np.uint8, copy=True, order="C")
    v_cache = np.array(v_cache, dtype=np.uint8, copy=True, order="C")
    kn, vn = _c(k_new, np.uint16), _c(v_new, np.uint16)
    ks, vs = _c(k_scale, np.float32), _c(v_scale, np.float32)
    slots = _c(slot_mapping, np.int64)
    nb, hkv, bs, d = k_cache.shape
    assert bs == block_size
    rc = _load().pgdo_kv_append_quant(_ptr(kn), _ptr(vn), _ptr(slots), len(slots), _ptr(k_cache),
                                      _ptr(v_cache), _ptr(ks), _ptr(vs), hkv, d, bs, nb)
    if rc:
        raise OracleError(f"pgdo_kv_append_quant rc={rc}")
    return k_cache, v_cache


def paged_decode_window(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                        window, k_scale=None, v_scale=None):
    """Plain definition restricted to each sequence's last `window` tokens
    (0 = full context)."""
    args, keep, (B, Hq, D) = _decode_args(q, k_cache, v_cache, block_table, context_lens,
                                          num_kv_heads, scale, k_scale, v_scale)
    out = np.empty((B, Hq, D), np.float64)
    lse = np.empty((B, Hq), np.float64)
    rc = _load().pgdo_paged_decode_window(*args, int(window), _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_paged_decode_window rc={rc}")
    del keep
    return out, lse


def paged_decode_multi(q, k_cache, v_cache, block_table, context_lens, num_kv_heads, scale,
                       window=0, k_scale=None, v_scale=None):
    """Several query tokens per sequence: q [B][L][Hq][D] (uint16 bf16 bits);
    returns out [B][L][Hq][D], lse [B][L][Hq]."""
    q = _c(q, np.uint16)
    B, L, Hq, D = q.shape
    args, keep, _ = _decode_args(q.reshape(B, L * Hq, D), k_cache, v_cache, block_table,
                                 context_lens, num_kv_heads, scale, k_scale, v_scale)
    args[10] = Hq                    # num_q_heads (the flattened view used L * Hq)
    out = np.empty((B, L, Hq, D), np.float64)
    lse = np.empty((B, L, Hq), np.float64)
    rc = _load().pgdo_paged_decode_multi(*args, int(L), int(window), _ptr(out), _ptr(lse))
    if rc:
        raise OracleError(f"pgdo_paged_decode_multi rc={rc}")
    del keep
    return out, lse
