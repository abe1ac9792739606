"""Helpers shared by the GPU parity tests: move a seeded workload to the
device, run the CUDA path through the binding, and compute the oracle's
expectation on the same host arrays."""
from __future__ import annotations

import numpy as np
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd

# tolerances stated for the two KV formats: |err| <= atol + rtol * |ref|
TOL = {"bf16": (2e-3, 1e-2), "e4m3": (2e-2, 5e-2)}


def dev_bf16(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).cuda()


def dev_cache(a: np.ndarray) -> torch.Tensor:
    if a.dtype == np.uint16:
        return dev_bf16(a)
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host_bits(t: torch.Tensor) -> np.ndarray:
    t = t.cpu()
    if t.dtype == torch.bfloat16:
        return t.view(torch.int16).numpy().view(np.uint16)
    return t.numpy()


def to_f64(t: torch.Tensor) -> np.ndarray:
    return t.float().cpu().numpy().astype(np.float64)


class Dev:
    """A workload resident on the GPU."""

    def __init__(self, w):
        self.w = w
        self.q = dev_bf16(w.q)
        self.k = dev_cache(w.k_cache)
        self.v = dev_cache(w.v_cache)
        self.bt = torch.from_numpy(w.block_table).cuda()
        self.cl = torch.from_numpy(w.context_lens).cuda()
        self.ks = torch.from_numpy(w.k_scale).cuda() if w.k_scale is not None else None
        self.vs = torch.from_numpy(w.v_scale).cuda() if w.v_scale is not None else None
        self.kn = self.vn = self.slots = None
        if w.slot_mapping is not None:
            self.kn = dev_cache(w.k_new)
            self.vn = dev_cache(w.v_new)
            self.slots = torch.from_numpy(w.slot_mapping).cuda()

    def append(self):
        if self.slots is not None:
            pgd.kv_append(self.kn, self.vn, self.slots, self.k, self.v)

    def decode(self, num_ctas=0, lse=True, out=None, max_context_len=None):
        w = self.w
        lse_t = torch.empty((w.num_seqs, w.num_q_heads), dtype=torch.float32,
                            device="cuda") if lse else None
        mcl = w.max_context_len if max_context_len is None else max_context_len
        out = pgd.paged_decode_attention(self.q, self.k, self.v, self.bt, self.cl,
                                         w.num_q_heads, w.num_kv_heads, w.head_dim,
                                         w.block_size, w.scale, out, max_context_len=mcl,
                                         k_scale=self.ks, v_scale=self.vs, lse_out=lse_t,
                                         num_ctas=num_ctas)
        return out, lse_t


def oracle_caches(w):
    """Caches after the append, computed by the oracle."""
    if w.slot_mapping is None:
        return w.k_cache, w.v_cache
    return oracle.kv_append(w.k_new, w.v_new, w.slot_mapping, w.k_cache, w.v_cache, w.block_size)


def oracle_full(w):
    kc, vc = oracle_caches(w)
    return oracle.paged_decode(w.q, kc, vc, w.block_table, w.context_lens, w.num_kv_heads,
                               w.scale, w.k_scale, w.v_scale)


def oracle_rows(w, rows_seq, rows_head):
    kc, vc = oracle_caches(w)
    return oracle.paged_decode_rows(w.q, kc, vc, w.block_table, w.context_lens, w.num_kv_heads,
                                    w.scale, rows_seq, rows_head, w.k_scale, w.v_scale)


def assert_close(got: np.ndarray, ref: np.ndarray, kv_dtype: str, what: str = ""):
    atol, rtol = TOL[kv_dtype]
    err = np.abs(got - ref)
    bound = atol + rtol * np.abs(ref)
    bad = ~(err <= bound)
    if bad.any():
        idx = np.argwhere(bad)[:5]
        raise AssertionError(
            f"{what}: {int(bad.sum())} of {bad.size} elements outside tolerance "
            f"(atol {atol}, rtol {rtol}); max err {float(np.nanmax(err)):.3e}; first "
            f"{[(tuple(i), float(got[tuple(i)]), float(ref[tuple(i)])) for i in idx]}")


def rel_l2(got: np.ndarray, ref: np.ndarray) -> float:
    return float(np.linalg.norm(got - ref) / max(np.linalg.norm(ref), 1e-30))
