"""KV parallelism (KVP): one sequence's KV split along its length over the
ranks of a process group.

Models with few KV heads cannot spread attention over more GPUs than KV
heads by tensor parallelism; attention then shards each sequence's KV by
length instead (the co-design page's "Principle 4", KVP / Helix).  Each rank
holds a contiguous run of every sequence's blocks (pgd_kvp_plan), decodes its
run into an unrounded split result (pgd_paged_decode_partial), the ranks
all-gather those results (NCCL over NVLink on GPUs, gloo in host tests), and
the log-sum-exp merge kernel (pgd_merge_partials) combines them exactly as
the splits inside one GPU are combined ("attention kernels", section
"prefill and decode attention").  The exchange is num_seqs * num_q_heads *
(head_dim + 1) fp32 per rank.
"""
from __future__ import annotations

import numpy as np
import torch
import torch.distributed as dist

from . import _binding as B


def local_block_table(block_table: np.ndarray, block_start: np.ndarray, slice_len: np.ndarray,
                      block_size: int) -> np.ndarray:
    """Block table of a rank's slice: row s lists the global table's blocks
    block_start[s] .. block_start[s] + ceil(slice_len[s] / block_size) - 1
    (unused entries 0, never read).  Host set-up, done when the table
    changes, not per step."""
    bt = np.asarray(block_table, dtype=np.int32)
    nblk = (np.asarray(slice_len, np.int64) + block_size - 1) // block_size
    width = max(1, int(nblk.max(initial=0)))
    out = np.zeros((bt.shape[0], width), np.int32)
    for s in range(bt.shape[0]):
        n = int(nblk[s])
        if n:
            b0 = int(block_start[s])
            out[s, :n] = bt[s, b0:b0 + n]
    return out


def _world(group) -> int:
    return dist.get_world_size(group) if dist.is_available() and dist.is_initialized() else 1


def _rank(group) -> int:
    return dist.get_rank(group) if dist.is_available() and dist.is_initialized() else 0


def gather_partials(o_part: torch.Tensor, lse_part: torch.Tensor, o_all: torch.Tensor,
                    lse_all: torch.Tensor, group=None) -> None:
    """All-gather every rank's split result: o_part [rows][D] (any shape with
    rows * D elements) and lse_part [rows] into o_all [W][rows][D] and
    lse_all [W][rows], rank r at index r.  o_part / lse_part may already be
    this rank's slots of o_all / lse_all (then nothing is copied locally)."""
    W, r = _world(group), _rank(group)
    if o_all.shape[0] != W or lse_all.shape[0] != W:
        raise ValueError("gather buffers must have one slot per rank")
    for part, full in ((o_part, o_all), (lse_part, lse_all)):
        in_place = part.data_ptr() == full[r].data_ptr()
        if W == 1:
            if not in_place:
                full[0].view(-1).copy_(part.reshape(-1))
            continue
        src = part.reshape(-1)
        if in_place and dist.get_backend(group) != "nccl":
            src = src.clone()          # only NCCL gathers in place
        dist.all_gather_into_tensor(full.view(-1), src, group=group)


class KVPDecoder:
    """Decode attention with every sequence's KV split over the ranks of
    `group`.  Buffers for one batch shape are allocated once; step() runs
    the rank's slice decode, the exchange and the merge on the current
    stream and returns the merged bf16 output [B][Hq][D] (identical on every
    rank)."""

    def __init__(self, num_seqs: int, num_q_heads: int, num_kv_heads: int, head_dim: int,
                 block_size: int, group=None, device=None):
        self.B, self.Hq, self.Hkv, self.D, self.bs = (num_seqs, num_q_heads, num_kv_heads,
                                                      head_dim, block_size)
        self.group = group
        self.world = _world(group)
        dev = torch.device("cuda") if device is None else torch.device(device)
        rows = num_seqs * num_q_heads
        f32 = dict(dtype=torch.float32, device=dev)
        self.o_all = torch.empty((self.world, rows, head_dim), **f32)
        self.lse_all = torch.empty((self.world, rows), **f32)
        # this rank's split result is decoded straight into its gather slot
        r = _rank(group)
        self.o_local = self.o_all[r].view(num_seqs, num_q_heads, head_dim)
        self.lse_local = self.lse_all[r].view(num_seqs, num_q_heads)
        self.out = torch.empty((num_seqs, num_q_heads, head_dim), dtype=torch.bfloat16,
                               device=dev)
        self.lse = torch.empty((rows,), **f32)

    def exchange_bytes(self) -> int:
        """fp32 bytes each rank contributes to the all-gather."""
        return self.B * self.Hq * (self.D + 1) * 4

    def step(self, q: torch.Tensor, k_cache: torch.Tensor, v_cache: torch.Tensor,
             block_table: torch.Tensor, slice_lens: torch.Tensor, scale: float, *,
             max_context_len: int = 0, k_scale=None, v_scale=None,
             num_ctas: int = 0) -> torch.Tensor:
        """q [B][Hq][D] (the same on every rank); the caches, block_table and
        slice_lens describe this rank's slice (pgd_kvp_plan)."""
        B.paged_decode_partial(q, k_cache, v_cache, block_table, slice_lens, self.Hq, self.Hkv,
                               self.D, self.bs, scale, self.o_local, self.lse_local,
                               max_context_len=max_context_len, k_scale=k_scale,
                               v_scale=v_scale, num_ctas=num_ctas)
        gather_partials(self.o_local, self.lse_local, self.o_all, self.lse_all, self.group)
        B.merge_partials(self.o_all, self.lse_all, self.out.view(self.B * self.Hq, self.D),
                         self.lse)
        return self.out


def plan(context_lens, block_size: int, world_size: int, rank: int):
    """(block_start, slice_len) of `rank` for every sequence (pgd_kvp_plan)."""
    return B.kvp_plan(context_lens, block_size, world_size, rank)


__all__ = ["plan", "local_block_table", "gather_partials", "KVPDecoder"]
