"""Seeded synthetic inputs for paged GQA decode attention.

This module only draws inputs: context lengths, a shuffled block table, Q/K/V
values rounded to the storage format, the KV append payload, and NaN poison in
every cache slot that no sequence owns.  It holds none of the attention
arithmetic; the CUDA path and the fp64 oracle both read the arrays it returns
(bf16 as uint16 bit patterns, FP8 E4M3 as uint8 bytes).

Workload shapes follow the pages: a Llama-3-style 32/8 head split ("batching
and attention", section 2.4), long contexts ("attention kernels", section "what
to check": measure near the service's maximum context), GQA groups 4-16 and
head_dim 128/256 (potato-ai, principles 1 and 2), FP8 KV read directly
("attention kernels", sections "paged KV and kernels" and "what to check").
No dataset is involved: every value is drawn from a seeded generator.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import numpy as np
import torch

BF16_NAN = np.uint16(0x7FC0)
E4M3_NAN = np.uint8(0x7F)
E4M3_MAX = 448.0


def to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """fp32 -> bf16 (round to nearest even) as uint16 bit patterns."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.bfloat16).view(torch.int16).numpy().view(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << 16).view(np.float32)


def to_e4m3_bytes(x: np.ndarray) -> np.ndarray:
    """fp32 -> FP8 E4M3 bytes via torch's float8_e4m3fn cast (RNE); |x| <= 448."""
    t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32))
    return t.to(torch.float8_e4m3fn).view(torch.uint8).numpy()


@dataclass
class Workload:
    name: str
    num_q_heads: int
    num_kv_heads: int
    head_dim: int
    block_size: int
    kv_dtype: str                      # "bf16" | "e4m3"
    context_lens: np.ndarray           # int32 [B]
    block_table: np.ndarray            # int32 [B][max_blocks_per_seq]
    q: np.ndarray                      # uint16 (bf16 bits) [B][Hq][D]
    k_cache: np.ndarray                # uint16 | uint8 [num_blocks][Hkv][bs][D]
    v_cache: np.ndarray
    scale: float
    k_scale: Optional[np.ndarray] = None   # float32 [Hkv] (FP8 only)
    v_scale: Optional[np.ndarray] = None
    # KV append payload applied before the decode (may be empty)
    k_new: Optional[np.ndarray] = None     # [N_tok][Hkv][D], cache element type
    v_new: Optional[np.ndarray] = None
    slot_mapping: Optional[np.ndarray] = None   # int64 [N_tok]
    meta: dict = field(default_factory=dict)

    @property
    def num_seqs(self) -> int:
        return int(self.context_lens.shape[0])

    @property
    def num_blocks(self) -> int:
        return int(self.k_cache.shape[0])

    @property
    def max_blocks_per_seq(self) -> int:
        return int(self.block_table.shape[1])

    @property
    def max_context_len(self) -> int:
        return int(self.context_lens.max()) if self.num_seqs else 0

    @property
    def group(self) -> int:
        return self.num_q_heads // self.num_kv_heads

    @property
    def elem_bytes(self) -> int:
        return 2 if self.kv_dtype == "bf16" else 1

    @property
    def num_tokens(self) -> int:
        return int(self.context_lens.astype(np.int64).sum())

    def visible_ranges(self, q_len: int = 1, window: int = 0):
        """Per sequence, the positions [lo, n) that some query row sees when
        the q_len newest tokens are queried (token j sees positions below
        n - q_len + 1 + j) with an optional window of `window` positions."""
        n = self.context_lens.astype(np.int64)
        if window <= 0:
            return np.zeros_like(n), n
        return np.maximum(0, n - q_len + 1 - window), n

    def algorithmic_bytes(self, q_len: int = 1, window: int = 0) -> dict:
        """Bytes one decode step must move at minimum (see the design notes):
        every visible K and V row once per (sequence, KV head), Q in, out back,
        the block-table entries of the visible blocks, the context lengths,
        the FP8 scales and, when present, the append payload read and
        written."""
        B, Hq, Hkv, D = self.num_seqs, self.num_q_heads, self.num_kv_heads, self.head_dim
        lo, n = self.visible_ranges(q_len, window)
        kv = int((n - lo).sum()) * Hkv * D * 2 * self.elem_bytes
        bs = self.block_size
        blocks = int(np.where(n > lo, (n - 1) // bs - lo // bs + 1, 0).sum())
        qo = 2 * B * q_len * Hq * D * 2
        meta = blocks * 4 + B * 4 + (2 * Hkv * 4 if self.kv_dtype == "e4m3" else 0)
        app = 0
        if self.slot_mapping is not None and len(self.slot_mapping):
            n = len(self.slot_mapping)
            app = 2 * (n * Hkv * D * 2 * self.elem_bytes) + n * 8
        return {"kv": kv, "qo": qo, "meta": meta, "append": app,
                "decode_total": kv + qo + meta, "step_total": kv + qo + meta + app}

    def flops(self) -> int:
        return 4 * self.num_q_heads * self.head_dim * self.num_tokens


def multi_query(w: Workload, q_len: int, seed: int = 0) -> np.ndarray:
    """Query rows for q_len tokens per sequence, bf16 bits [B][q_len][Hq][D],
    N(0, 1) from np.random.default_rng(seed + 7_000_001)."""
    rng = np.random.default_rng(seed + 7_000_001)
    return to_bf16_bits(rng.standard_normal((w.num_seqs, q_len, w.num_q_heads, w.head_dim),
                                            dtype=np.float32))


def _assign_blocks(rng, ctx: np.ndarray, bs: int, pool: int):
    nblk = (ctx.astype(np.int64) + bs - 1) // bs
    used = int(nblk.sum())
    assert used <= pool, (used, pool)
    perm = rng.permutation(pool).astype(np.int32)
    width = max(1, int(nblk.max()) if len(nblk) else 1)
    spare = perm[used:]
    fill = int(spare[0]) if len(spare) else 0
    table = np.full((len(ctx), width), fill, np.int32)
    pos = 0
    for s, n in enumerate(nblk):
        table[s, :n] = perm[pos:pos + n]
        pos += n
    return table, perm[:used], spare


def _poison(cache: np.ndarray, ctx: np.ndarray, table: np.ndarray, spare: np.ndarray,
            bs: int, nan):
    cache[spare] = nan
    for s, n in enumerate(ctx):
        n = int(n)
        if n % bs:
            cache[table[s, n // bs], :, n % bs:, :] = nan


def make_case(context_lens, num_q_heads: int, num_kv_heads: int, head_dim: int,
              block_size: int, kv_dtype: str = "bf16", seed: int = 0,
              pool: Optional[int] = None, spare_frac: float = 0.10,
              scale: Optional[float] = None, key_boost_frac: float = 0.0,
              key_boost: float = 8.0, append_last: bool = False, name: str = "case",
              table_width: Optional[int] = None) -> Workload:
    """Draw one paged-decode case.

    Order of draws from ``np.random.default_rng(seed)``: block permutation,
    Q, K pool, V pool, key-boost mask, append payload.  Values are N(0, 1) in
    fp32, rounded to bf16 (RNE) or quantised to E4M3 with a per-KV-head scale
    amax / 448 over that head's live rows.  With ``append_last`` the last token
    of every sequence is not in the cache yet: its K/V rows come as the append
    payload and its slot holds NaN until the append writes it.
    """
    rng = np.random.default_rng(seed)
    ctx = np.asarray(context_lens, dtype=np.int32)
    B, bs, D, Hkv = len(ctx), block_size, head_dim, num_kv_heads
    nblk = (ctx.astype(np.int64) + bs - 1) // bs
    used = int(nblk.sum())
    if pool is None:
        pool = used + max(1, int(math.ceil(spare_frac * used)))
    table, _, spare = _assign_blocks(rng, ctx, bs, pool)
    if table_width is not None and table_width > table.shape[1]:
        fill = int(spare[0]) if len(spare) else 0
        wide = np.full((B, table_width), fill, np.int32)
        wide[:, :table.shape[1]] = table
        table = wide
    q = to_bf16_bits(rng.standard_normal((B, num_q_heads, D), dtype=np.float32))
    kf = rng.standard_normal((pool, Hkv, bs, D), dtype=np.float32)
    vf = rng.standard_normal((pool, Hkv, bs, D), dtype=np.float32)
    if key_boost_frac > 0:
        # per (sequence, position) mask; the boost applies to every KV head
        # and dim of that position's key (x8 is exact in bf16).
        for s in range(B):
            n = int(ctx[s])
            mask = rng.random(n) < key_boost_frac
            for t in np.nonzero(mask)[0]:
                kf[table[s, t // bs], :, t % bs, :] *= key_boost
    k_scale = v_scale = None
    if kv_dtype == "bf16":
        k_cache = to_bf16_bits(kf)
        v_cache = to_bf16_bits(vf)
        nan = BF16_NAN
    elif kv_dtype == "e4m3":
        live = np.zeros((pool, bs), bool)
        for s in range(B):
            n = int(ctx[s])
            for j in range(int(nblk[s])):
                live[table[s, j], :min(bs, n - j * bs)] = True
        k_scale = np.empty(Hkv, np.float32)
        v_scale = np.empty(Hkv, np.float32)
        for h in range(Hkv):
            ka = np.abs(kf[:, h][live]).max() if live.any() else 1.0
            va = np.abs(vf[:, h][live]).max() if live.any() else 1.0
            k_scale[h] = np.float32(ka / E4M3_MAX) if ka > 0 else np.float32(1.0)
            v_scale[h] = np.float32(va / E4M3_MAX) if va > 0 else np.float32(1.0)
        k_cache = to_e4m3_bytes(np.clip(kf / k_scale[None, :, None, None], -E4M3_MAX, E4M3_MAX))
        v_cache = to_e4m3_bytes(np.clip(vf / v_scale[None, :, None, None], -E4M3_MAX, E4M3_MAX))
        nan = E4M3_NAN
    else:
        raise ValueError(kv_dtype)
    k_cache = k_cache.reshape(pool, Hkv, bs, D)
    v_cache = v_cache.reshape(pool, Hkv, bs, D)
    _poison(k_cache, ctx, table, spare, bs, nan)
    _poison(v_cache, ctx, table, spare, bs, nan)
    k_new = v_new = slots = None
    if append_last:
        live_seqs = [s for s in range(B) if ctx[s] > 0]
        slots = np.array([int(table[s, (ctx[s] - 1) // bs]) * bs + int((ctx[s] - 1) % bs)
                          for s in live_seqs], np.int64)
        blk, off = slots // bs, slots % bs
        k_new = k_cache[blk, :, off, :].copy()
        v_new = v_cache[blk, :, off, :].copy()
        k_cache[blk, :, off, :] = nan
        v_cache[blk, :, off, :] = nan
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    return Workload(name=name, num_q_heads=num_q_heads, num_kv_heads=Hkv, head_dim=D,
                    block_size=bs, kv_dtype=kv_dtype, context_lens=ctx, block_table=table,
                    q=q, k_cache=k_cache, v_cache=v_cache, scale=float(scale),
                    k_scale=k_scale, v_scale=v_scale, k_new=k_new, v_new=v_new,
                    slot_mapping=slots, meta={"seed": seed, "pool": pool})


# --------------------------------------------------------------------------- #
# The five named workloads.                                                   #
# --------------------------------------------------------------------------- #
WORKLOADS = {
    "tiny": "4 seqs, context_lens {1,17,64,200}, 8 q / 2 kv heads (g 4), D 128, bs 16, "
            "pool 64 blocks",
    "llama3_8b_decode": "64 seqs, context U[512,4096], 32 q / 8 kv heads (g 4), D 128, bs 16, "
                        "+ kv_append of 64 new tokens",
    "long_context": "4 seqs x 131072, 64 q / 8 kv heads (g 8), D 128, bs 64",
    "wide_heads": "32 seqs, context lognormal(median 8192, sigma 1) capped 32768, "
                  "32 q / 2 kv heads (g 16), D 256, bs 32, 5% of keys x8",
    "fp8_mixed": "256 seqs, context Pareto(alpha 1.2, x_m 16) clipped [16,65536], "
                 "64 q / 8 kv heads (g 8), D 128, bs 16, FP8 E4M3 KV + per-head scales",
}


def context_lens_for(name: str, seed: int = 0) -> np.ndarray:
    rng = np.random.default_rng(seed + 1_000_003)
    if name == "tiny":
        return np.array([1, 17, 64, 200], np.int32)
    if name == "llama3_8b_decode":
        return rng.integers(512, 4096, size=64, endpoint=True).astype(np.int32)
    if name == "long_context":
        return np.full(4, 131072, np.int32)
    if name == "wide_heads":
        x = np.rint(rng.lognormal(math.log(8192.0), 1.0, size=32))
        return np.clip(x, 1, 32768).astype(np.int32)
    if name == "fp8_mixed":
        x = np.floor(16.0 * (1.0 + rng.pareto(1.2, size=256)))
        return np.clip(x, 16, 65536).astype(np.int32)
    raise KeyError(name)


def make_workload(name: str, seed: int = 0, shape_seed: Optional[int] = None) -> Workload:
    """The named workload.  `shape_seed` (default `seed`) draws the context
    lengths; `seed` draws the block permutation and the values, so replicas
    that share a shape_seed have the same shape and their own data."""
    ctx = context_lens_for(name, seed if shape_seed is None else shape_seed)
    if name == "tiny":
        return make_case(ctx, 8, 2, 128, 16, "bf16", seed, pool=64, name=name)
    if name == "llama3_8b_decode":
        return make_case(ctx, 32, 8, 128, 16, "bf16", seed, append_last=True, name=name)
    if name == "long_context":
        return make_case(ctx, 64, 8, 128, 64, "bf16", seed, name=name)
    if name == "wide_heads":
        return make_case(ctx, 32, 2, 256, 32, "bf16", seed, key_boost_frac=0.05, name=name)
    if name == "fp8_mixed":
        return make_case(ctx, 64, 8, 128, 16, "e4m3", seed, name=name)
    raise KeyError(name)
