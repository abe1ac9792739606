"""ctypes binding of libpgd.so (argument marshalling only).

Every function takes torch tensors that already live on the current CUDA
device, checks their dtype/shape/contiguity, and passes raw pointers and the
current stream to the C ABI declared in include/pgd.h.  All computation runs
in the library's CUDA kernels; there is no fallback path.  If libpgd.so has
not been built, loading raises ImportError.

Every function that enqueues work also takes prepare=True: it then checks
and marshals its arguments once and returns a Prepared call that re-issues
the same C call (same buffers, sizes and stream) each time it is called.
"""
from __future__ import annotations

import ctypes
import os
from typing import Optional

import numpy as np
import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libpgd.so")

PGD_KV_BF16 = 0
PGD_KV_FP8_E4M3 = 1

STATUS = {0: "PGD_OK", 1: "PGD_ERR_INVALID_ARG", 2: "PGD_ERR_UNSUPPORTED", 3: "PGD_ERR_CUDA",
          4: "PGD_ERR_DEVICE_BOUNDS", 5: "PGD_ERR_TIMEOUT", 6: "PGD_ERR_WORKSPACE"}

_lib = None


class PGDError(RuntimeError):
    def __init__(self, status: int, where: str):
        self.status = status
        super().__init__(f"{where}: {STATUS.get(status, status)}")


def lib_path() -> str:
    return LIB_PATH


def load_library():
    """Load libpgd.so once; raise ImportError if it is missing."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run `python -m paged_gqa_decode_07_b200.build`")
    lib = ctypes.CDLL(LIB_PATH)
    P, i32, i64, f32, sz = (ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_float,
                            ctypes.c_size_t)
    st = ctypes.c_int
    lib.pgd_status_string.restype = ctypes.c_char_p
    lib.pgd_status_string.argtypes = [st]
    lib.pgd_version.restype = ctypes.c_char_p
    lib.pgd_version.argtypes = []
    lib.pgd_kv_append.restype = st
    lib.pgd_kv_append.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32, st, P]
    lib.pgd_kv_append_quant.restype = st
    lib.pgd_kv_append_quant.argtypes = [P, P, P, i32, P, P, P, P, i32, i32, i32, i32, P]
    lib.pgd_decode_workspace_bytes.restype = sz
    lib.pgd_decode_workspace_bytes.argtypes = [i32, i32, i32, i32]
    lib.pgd_paged_decode_attention.restype = st
    lib.pgd_paged_decode_attention.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                               i32, f32, st, P, P, P, P, P, sz, i32, P]
    lib.pgd_paged_decode_attention_ex.restype = st
    lib.pgd_paged_decode_attention_ex.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32,
                                                  i32, i32, i32, i32, f32, st, P, P, P, P, P, sz,
                                                  i32, P]
    lib.pgd_paged_decode_partial.restype = st
    lib.pgd_paged_decode_partial.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                             i32, f32, st, P, P, P, P, P, sz, i32, P]
    lib.pgd_set_decode_math.restype = st
    lib.pgd_set_decode_math.argtypes = [st]
    lib.pgd_get_decode_math.restype = st
    lib.pgd_get_decode_math.argtypes = []
    lib.pgd_debug_set_wait_limit_ns.restype = st
    lib.pgd_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.pgd_debug_get_wait_limit_ns.restype = ctypes.c_uint64
    lib.pgd_debug_get_wait_limit_ns.argtypes = []
    lib.pgd_kvp_plan.restype = st
    lib.pgd_kvp_plan.argtypes = [P, i32, i32, i32, i32, P, P]
    lib.pgd_decode_grid.restype = ctypes.c_int64
    lib.pgd_decode_grid.argtypes = [i32] * 9
    lib.pgd_decode_step.restype = st
    lib.pgd_decode_step.argtypes = [P, P, P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32, i32,
                                    f32, st, P, P, P, P, P, sz, i32, P]
    lib.pgd_paged_decode_attention_noalloc.restype = st
    lib.pgd_paged_decode_attention_noalloc.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32,
                                                       i32, i32, i32, f32, st, P, P, P, P, i32, P]
    lib.pgd_merge_partials.restype = st
    lib.pgd_merge_partials.argtypes = [P, P, i32, i32, i32, P, P, P]
    lib.pgd_get_device_error.restype = st
    lib.pgd_get_device_error.argtypes = [P, ctypes.POINTER(ctypes.c_uint32)]
    lib.pgd_shutdown.restype = st
    lib.pgd_shutdown.argtypes = []
    lib.kv_append.restype = st
    lib.kv_append.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32, P]
    lib.paged_decode_attention.restype = st
    lib.paged_decode_attention.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                           f32, P, P]
    del i64
    _lib = lib
    return lib


def _check(status: int, where: str):
    if status != 0:
        raise PGDError(status, where)


class Prepared:
    """One library call with its arguments checked and marshalled once.

    A serving loop issues the same call with the same buffers every step
    (persistent q / out / cache tensors whose contents change); the
    per-call checks and the conversion of ~25 arguments to C types then cost
    more host time than a small batch's kernel takes on the GPU.  Calling a
    Prepared object re-issues the C call with the pointers, sizes and stream
    it was prepared with and returns what the original call returned.  The
    tensors must stay alive and keep their storage while it is in use."""

    __slots__ = ("_fn", "_args", "_name", "result")

    def __init__(self, fn, args, name, result):
        conv = []
        for t, a in zip(fn.argtypes, args):
            conv.append(a if a is None or isinstance(a, t) else t(a))
        self._fn, self._args, self._name, self.result = fn, tuple(conv), name, result

    def __call__(self):
        st = self._fn(*self._args)
        if st:
            raise PGDError(st, self._name)
        return self.result


def _issue(fn, name: str, args, prepare: bool, result=None):
    """Run the C call now, or return it prepared (see Prepared)."""
    if prepare:
        return Prepared(fn, args, name, result)
    _check(fn(*args), name)
    return result


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream) -> ctypes.c_void_p:
    if stream is None:
        stream = torch.cuda.current_stream()
    return ctypes.c_void_p(stream.cuda_stream if hasattr(stream, "cuda_stream") else int(stream))


def _kv_dtype(cache: torch.Tensor) -> int:
    if cache.dtype == torch.bfloat16:
        return PGD_KV_BF16
    if cache.dtype in (torch.uint8, torch.float8_e4m3fn):
        return PGD_KV_FP8_E4M3
    raise TypeError(f"KV cache dtype {cache.dtype} is not bf16 / FP8 E4M3")


def _need(t: torch.Tensor, name: str, dtypes, dim: Optional[int] = None):
    if not isinstance(t, torch.Tensor):
        raise TypeError(f"{name} must be a torch.Tensor")
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if dtypes and t.dtype not in dtypes:
        raise TypeError(f"{name} has dtype {t.dtype}, expected one of {dtypes}")
    if dim is not None and t.dim() != dim:
        raise ValueError(f"{name} must have {dim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")


_KV_DTYPES = (torch.bfloat16, torch.uint8, torch.float8_e4m3fn)


def kv_append(k_new, v_new, slot_mapping, k_cache, v_cache, *, stream=None, prepare=False):
    """Scatter new tokens' K/V rows into their cache slots (pgd_kv_append).

    k_new/v_new [N][Hkv][D] and caches [num_blocks][Hkv][bs][D] share one
    dtype (bf16, or uint8 / float8_e4m3fn bytes); slot_mapping int64 [N].
    """
    lib = load_library()
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(k_new, "k_new", (k_cache.dtype,), 3)
    _need(v_new, "v_new", (k_cache.dtype,), 3)
    _need(slot_mapping, "slot_mapping", (torch.int64,), 1)
    nb, hkv, bs, d = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape != v_new.shape or \
            k_new.shape[1:] != (hkv, d) or slot_mapping.shape[0] != k_new.shape[0]:
        raise ValueError("kv_append: inconsistent shapes")
    return _issue(lib.pgd_kv_append, "pgd_kv_append",
                  (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), k_new.shape[0], _ptr(k_cache),
                   _ptr(v_cache), hkv, d, bs, nb, _kv_dtype(k_cache), _stream(stream)), prepare)


def kv_append_quant(k_new, v_new, slot_mapping, k_cache, v_cache, k_scale, v_scale, *,
                    stream=None, prepare=False):
    """Quantise bf16 K/V rows of new tokens into an FP8 E4M3 cache
    (pgd_kv_append_quant): byte = E4M3(x / scale[kv head])."""
    lib = load_library()
    _need(k_cache, "k_cache", (torch.uint8, torch.float8_e4m3fn), 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(k_new, "k_new", (torch.bfloat16,), 3)
    _need(v_new, "v_new", (torch.bfloat16,), 3)
    _need(slot_mapping, "slot_mapping", (torch.int64,), 1)
    _need(k_scale, "k_scale", (torch.float32,), 1)
    _need(v_scale, "v_scale", (torch.float32,), 1)
    nb, hkv, bs, d = k_cache.shape
    if v_cache.shape != k_cache.shape or k_new.shape != v_new.shape or \
            k_new.shape[1:] != (hkv, d) or slot_mapping.shape[0] != k_new.shape[0] or \
            k_scale.shape != (hkv,) or v_scale.shape != (hkv,):
        raise ValueError("kv_append_quant: inconsistent shapes")
    return _issue(lib.pgd_kv_append_quant, "pgd_kv_append_quant",
                  (_ptr(k_new), _ptr(v_new), _ptr(slot_mapping), k_new.shape[0], _ptr(k_cache),
                   _ptr(v_cache), _ptr(k_scale), _ptr(v_scale), hkv, d, bs, nb,
                   _stream(stream)), prepare)


def decode_workspace_bytes(num_seqs: int, num_q_heads: int, num_kv_heads: int,
                           head_dim: int) -> int:
    return int(load_library().pgd_decode_workspace_bytes(num_seqs, num_q_heads, num_kv_heads,
                                                         head_dim))


def paged_decode_attention(q, k_cache, v_cache, block_table, context_lens, num_q_heads: int,
                           num_kv_heads: int, head_dim: int, block_size: int, scale: float,
                           out: Optional[torch.Tensor] = None, *, max_context_len: int = 0,
                           k_scale=None, v_scale=None, lse_out=None, workspace=None,
                           num_ctas: int = 0, stream=None, prepare=False):
    """One decode step of paged GQA attention (pgd_paged_decode_attention).

    q bf16 [B][Hq][D]; caches [num_blocks][Hkv][bs][D] (bf16 or E4M3 bytes);
    block_table int32 [B][max_blocks]; context_lens int32 [B]; FP8 caches take
    fp32 k_scale / v_scale [Hkv].  Returns out (bf16 [B][Hq][D]); lse_out
    (fp32 [B][Hq]) is filled when given.
    """
    lib = load_library()
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_table, "block_table", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B = q.shape[0]
    if q.shape != (B, num_q_heads, head_dim) or tuple(k_cache.shape[1:]) != (
            num_kv_heads, block_size, head_dim) or v_cache.shape != k_cache.shape or \
            block_table.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("paged_decode_attention: inconsistent shapes")
    kvd = _kv_dtype(k_cache)
    if kvd == PGD_KV_FP8_E4M3:
        _need(k_scale, "k_scale", (torch.float32,), 1)
        _need(v_scale, "v_scale", (torch.float32,), 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (torch.bfloat16,), 3)
    if lse_out is not None:
        _need(lse_out, "lse_out", (torch.float32,), 2)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", None)
        ws_bytes = workspace.numel() * workspace.element_size()
    return _issue(lib.pgd_paged_decode_attention, "pgd_paged_decode_attention", (
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), B, int(max_context_len), num_q_heads, num_kv_heads, head_dim,
        block_size, k_cache.shape[0], float(scale), kvd, _ptr(k_scale), _ptr(v_scale), _ptr(out),
        _ptr(lse_out), _ptr(workspace), ws_bytes, int(num_ctas), _stream(stream)), prepare, out)


def paged_decode_attention_ex(q, k_cache, v_cache, block_table, context_lens, num_q_heads: int,
                              num_kv_heads: int, head_dim: int, block_size: int, scale: float,
                              out: Optional[torch.Tensor] = None, *, window: int = 0,
                              max_context_len: int = 0, k_scale=None, v_scale=None, lse_out=None,
                              workspace=None, num_ctas: int = 0, stream=None, prepare=False):
    """Decode attention for q_len query tokens per sequence with an optional
    sliding window (pgd_paged_decode_attention_ex).

    q bf16 [B][q_len][Hq][D]: the q_len newest tokens of each sequence, already
    counted in context_lens; token j sees positions below
    context_lens - q_len + 1 + j, and with window > 0 only the last `window` of
    them.  Returns out (bf16 [B][q_len][Hq][D]); lse_out (fp32 [B][q_len][Hq])
    is filled when given.  Other arguments as paged_decode_attention.
    """
    lib = load_library()
    _need(q, "q", (torch.bfloat16,), 4)
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_table, "block_table", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B, L = q.shape[0], q.shape[1]
    if q.shape != (B, L, num_q_heads, head_dim) or tuple(k_cache.shape[1:]) != (
            num_kv_heads, block_size, head_dim) or v_cache.shape != k_cache.shape or \
            block_table.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("paged_decode_attention_ex: inconsistent shapes")
    kvd = _kv_dtype(k_cache)
    if kvd == PGD_KV_FP8_E4M3:
        _need(k_scale, "k_scale", (torch.float32,), 1)
        _need(v_scale, "v_scale", (torch.float32,), 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (torch.bfloat16,), 4)
    if lse_out is not None:
        _need(lse_out, "lse_out", (torch.float32,), 3)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", None)
        ws_bytes = workspace.numel() * workspace.element_size()
    return _issue(lib.pgd_paged_decode_attention_ex, "pgd_paged_decode_attention_ex", (
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), B, int(max_context_len), L, int(window), num_q_heads, num_kv_heads,
        head_dim, block_size, k_cache.shape[0], float(scale), kvd, _ptr(k_scale), _ptr(v_scale),
        _ptr(out), _ptr(lse_out), _ptr(workspace), ws_bytes, int(num_ctas), _stream(stream)),
        prepare, out)


def paged_decode_partial(q, k_cache, v_cache, block_table, context_lens, num_q_heads: int,
                         num_kv_heads: int, head_dim: int, block_size: int, scale: float,
                         o_part: Optional[torch.Tensor] = None,
                         lse_part: Optional[torch.Tensor] = None, *, max_context_len: int = 0,
                         k_scale=None, v_scale=None, workspace=None, num_ctas: int = 0,
                         stream=None, prepare=False):
    """Decode of one KV slice left unrounded for a merge
    (pgd_paged_decode_partial): returns (o_part fp32 [B][Hq][D],
    lse_part fp32 [B][Hq], natural log)."""
    lib = load_library()
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_table, "block_table", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B = q.shape[0]
    if q.shape != (B, num_q_heads, head_dim) or tuple(k_cache.shape[1:]) != (
            num_kv_heads, block_size, head_dim) or v_cache.shape != k_cache.shape or \
            block_table.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("paged_decode_partial: inconsistent shapes")
    kvd = _kv_dtype(k_cache)
    if kvd == PGD_KV_FP8_E4M3:
        _need(k_scale, "k_scale", (torch.float32,), 1)
        _need(v_scale, "v_scale", (torch.float32,), 1)
    if o_part is None:
        o_part = torch.empty((B, num_q_heads, head_dim), dtype=torch.float32, device=q.device)
    if lse_part is None:
        lse_part = torch.empty((B, num_q_heads), dtype=torch.float32, device=q.device)
    _need(o_part, "o_part", (torch.float32,), 3)
    _need(lse_part, "lse_part", (torch.float32,), 2)
    if o_part.shape != (B, num_q_heads, head_dim) or lse_part.shape != (B, num_q_heads):
        raise ValueError("paged_decode_partial: output shapes")
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", None)
        ws_bytes = workspace.numel() * workspace.element_size()
    return _issue(lib.pgd_paged_decode_partial, "pgd_paged_decode_partial", (
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), B, int(max_context_len), num_q_heads, num_kv_heads, head_dim,
        block_size, k_cache.shape[0], float(scale), kvd, _ptr(k_scale), _ptr(v_scale),
        _ptr(o_part), _ptr(lse_part), _ptr(workspace), ws_bytes, int(num_ctas), _stream(stream)),
        prepare, (o_part, lse_part))


_MATH = {"tensor_core": 0, "cuda_core": 1}


def set_decode_math(math: str) -> None:
    """Consumer math of the decode kernels, process-wide (pgd_set_decode_math):
    "tensor_core" (default) or "cuda_core" (FMA + warp shuffles; bf16,
    head_dim 128, at most 8 query rows per KV head)."""
    if math not in _MATH:
        raise ValueError(f"math must be one of {sorted(_MATH)}")
    _check(load_library().pgd_set_decode_math(_MATH[math]), "pgd_set_decode_math")


def get_decode_math() -> str:
    v = int(load_library().pgd_get_decode_math())
    return {b: a for a, b in _MATH.items()}[v]


def debug_set_wait_limit_ns(limit_ns: int) -> None:
    """Limit of the decode kernels' pipeline waits, in ns, for the launches
    that follow (pgd_debug_set_wait_limit_ns); 0 restores the default 1 s.
    A test hook for the timeout path."""
    _check(load_library().pgd_debug_set_wait_limit_ns(int(limit_ns)),
           "pgd_debug_set_wait_limit_ns")


def debug_get_wait_limit_ns() -> int:
    return int(load_library().pgd_debug_get_wait_limit_ns())


def decode_grid(sms: int, ctas_per_sm: int, num_seqs: int, num_kv_heads: int, head_dim: int,
                block_size: int, max_blocks_per_seq: int, max_context_len: int = 0,
                fp8: bool = False) -> int:
    """CTA count of the decode entry points' automatic grid (pgd_decode_grid;
    host only, no CUDA call).  Raises ValueError for invalid arguments."""
    g = int(load_library().pgd_decode_grid(int(sms), int(ctas_per_sm), int(num_seqs),
                                           int(num_kv_heads), int(head_dim), int(block_size),
                                           int(max_blocks_per_seq), int(max_context_len),
                                           1 if fp8 else 0))
    if g <= 0:
        raise ValueError("pgd_decode_grid: invalid arguments")
    return g


def kvp_plan(context_lens, block_size: int, world_size: int, rank: int):
    """Host-side KV-parallel slice of every sequence held by `rank`
    (pgd_kvp_plan): returns (block_start, slice_len), int32 numpy [B]."""
    lib = load_library()
    cl = np.ascontiguousarray(np.asarray(context_lens, dtype=np.int32))
    B = int(cl.shape[0])
    start = np.zeros(B, np.int32)
    length = np.zeros(B, np.int32)
    _check(lib.pgd_kvp_plan(cl.ctypes.data_as(ctypes.c_void_p), B, int(block_size),
                            int(world_size), int(rank), start.ctypes.data_as(ctypes.c_void_p),
                            length.ctypes.data_as(ctypes.c_void_p)), "pgd_kvp_plan")
    return start, length


def decode_step(q, k_new, v_new, k_cache, v_cache, block_table, context_lens, num_q_heads: int,
                num_kv_heads: int, head_dim: int, block_size: int, scale: float,
                out: Optional[torch.Tensor] = None, *, max_context_len: int = 0, k_scale=None,
                v_scale=None, lse_out=None, workspace=None, num_ctas: int = 0,
                stream=None, prepare=False):
    """One decode step in one launch (pgd_decode_step): writes each sequence's
    newest K/V row (k_new / v_new [B][Hkv][D], cache dtype) at position
    context_lens[s] - 1, then computes paged decode attention over the
    updated cache.  Same as kv_append + paged_decode_attention."""
    lib = load_library()
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(k_new, "k_new", (k_cache.dtype,), 3)
    _need(v_new, "v_new", (k_cache.dtype,), 3)
    _need(block_table, "block_table", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B = q.shape[0]
    if q.shape != (B, num_q_heads, head_dim) or tuple(k_cache.shape[1:]) != (
            num_kv_heads, block_size, head_dim) or v_cache.shape != k_cache.shape or \
            k_new.shape != (B, num_kv_heads, head_dim) or v_new.shape != k_new.shape or \
            block_table.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("decode_step: inconsistent shapes")
    kvd = _kv_dtype(k_cache)
    if kvd == PGD_KV_FP8_E4M3:
        _need(k_scale, "k_scale", (torch.float32,), 1)
        _need(v_scale, "v_scale", (torch.float32,), 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (torch.bfloat16,), 3)
    if lse_out is not None:
        _need(lse_out, "lse_out", (torch.float32,), 2)
    ws_bytes = 0
    if workspace is not None:
        _need(workspace, "workspace", None)
        ws_bytes = workspace.numel() * workspace.element_size()
    return _issue(lib.pgd_decode_step, "pgd_decode_step", (
        _ptr(q), _ptr(k_new), _ptr(v_new), _ptr(k_cache), _ptr(v_cache), _ptr(block_table),
        block_table.shape[1], _ptr(context_lens), B, int(max_context_len), num_q_heads,
        num_kv_heads, head_dim, block_size, k_cache.shape[0], float(scale), kvd, _ptr(k_scale),
        _ptr(v_scale), _ptr(out), _ptr(lse_out), _ptr(workspace), ws_bytes, int(num_ctas),
        _stream(stream)), prepare, out)


def paged_decode_attention_noalloc(q, k_cache, v_cache, block_table, context_lens,
                                   num_q_heads: int, num_kv_heads: int, head_dim: int,
                                   block_size: int, scale: float,
                                   out: Optional[torch.Tensor] = None, *,
                                   max_context_len: int = 0, k_scale=None, v_scale=None,
                                   lse_out=None, num_ctas: int = 0, stream=None) -> torch.Tensor:
    """The decode step of paged_decode_attention for callers that cannot let
    the library allocate device memory (pgd_paged_decode_attention_noalloc):
    its scratch is a fixed static device array, so the call allocates
    nothing.  Same arguments minus the workspace; the output is passed in or
    allocated here by torch before the call."""
    lib = load_library()
    _need(q, "q", (torch.bfloat16,), 3)
    _need(k_cache, "k_cache", _KV_DTYPES, 4)
    _need(v_cache, "v_cache", (k_cache.dtype,), 4)
    _need(block_table, "block_table", (torch.int32,), 2)
    _need(context_lens, "context_lens", (torch.int32,), 1)
    B = q.shape[0]
    if q.shape != (B, num_q_heads, head_dim) or tuple(k_cache.shape[1:]) != (
            num_kv_heads, block_size, head_dim) or v_cache.shape != k_cache.shape or \
            block_table.shape[0] != B or context_lens.shape[0] != B:
        raise ValueError("paged_decode_attention_noalloc: inconsistent shapes")
    kvd = _kv_dtype(k_cache)
    if kvd == PGD_KV_FP8_E4M3:
        _need(k_scale, "k_scale", (torch.float32,), 1)
        _need(v_scale, "v_scale", (torch.float32,), 1)
    if out is None:
        out = torch.empty_like(q)
    _need(out, "out", (torch.bfloat16,), 3)
    if lse_out is not None:
        _need(lse_out, "lse_out", (torch.float32,), 2)
    _check(lib.pgd_paged_decode_attention_noalloc(
        _ptr(q), _ptr(k_cache), _ptr(v_cache), _ptr(block_table), block_table.shape[1],
        _ptr(context_lens), B, int(max_context_len), num_q_heads, num_kv_heads, head_dim,
        block_size, k_cache.shape[0], float(scale), kvd, _ptr(k_scale), _ptr(v_scale), _ptr(out),
        _ptr(lse_out), int(num_ctas), _stream(stream)), "pgd_paged_decode_attention_noalloc")
    return out


def merge_partials(o_part, lse_part, out=None, lse_out=None, *, stream=None, prepare=False):
    """LSE merge of split results: o_part fp32 [P][rows][D], lse_part fp32
    [P][rows] (natural log) -> out bf16 [rows][D] (pgd_merge_partials)."""
    lib = load_library()
    _need(o_part, "o_part", (torch.float32,), 3)
    _need(lse_part, "lse_part", (torch.float32,), 2)
    P, R, D = o_part.shape
    if lse_part.shape != (P, R):
        raise ValueError("merge_partials: inconsistent shapes")
    if out is None:
        out = torch.empty((R, D), dtype=torch.bfloat16, device=o_part.device)
    _need(out, "out", (torch.bfloat16,), 2)
    if lse_out is not None:
        _need(lse_out, "lse_out", (torch.float32,), 1)
    return _issue(lib.pgd_merge_partials, "pgd_merge_partials",
                  (_ptr(o_part), _ptr(lse_part), P, R, D, _ptr(out), _ptr(lse_out),
                   _stream(stream)), prepare, out)


def get_device_error(*, stream=None) -> int:
    """Wait for the stream, then read and clear the device flag bits."""
    flags = ctypes.c_uint32(0)
    status = load_library().pgd_get_device_error(_stream(stream), ctypes.byref(flags))
    if status == 3:
        raise PGDError(status, "pgd_get_device_error")
    return int(flags.value)


def shutdown() -> None:
    _check(load_library().pgd_shutdown(), "pgd_shutdown")
