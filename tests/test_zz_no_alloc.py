"""The decode entry point that allocates nothing.

Callers such as a serving engine that has reserved nearly all HBM for its
KV-cache pool, or a host that routes every device byte through its own
allocator, cannot let the library cudaMalloc its scratch.  For them
pgd_paged_decode_attention_noalloc keeps that scratch in a fixed static device
array.  These tests call it through the C ABI and check that two calls in a
row give the same answer as the allocating entry point, within the tolerances
the parity tests use, and that requests past the array's limits are refused
before anything is enqueued.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes on its own in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, assert_close, to_f64
from workloads import make_case

pytestmark = pytest.mark.gpu

CASES = [  # (context lens, Hq, Hkv, D, bs, kv dtype)
    ([1, 15, 16, 17, 200, 1000, 2049, 0, 333], 32, 8, 128, 16, "bf16"),
    ([700, 5, 3000], 32, 2, 256, 32, "bf16"),
    ([64, 900, 17, 4000], 64, 8, 128, 16, "e4m3"),
]


@pytest.mark.parametrize("ctx,Hq,Hkv,D,bs,dt", CASES,
                         ids=[f"g{c[1] // c[2]}-D{c[3]}-{c[5]}" for c in CASES])
def test_noalloc_matches_allocating_entry_point_twice(ctx, Hq, Hkv, D, bs, dt):
    assert torch.cuda.is_available()
    w = make_case(ctx, Hq, Hkv, D, bs, dt, seed=101 + D + Hq)
    d = Dev(w)
    ref, ref_lse = d.decode()
    torch.cuda.synchronize()
    ref = to_f64(ref)
    ref_lse = ref_lse.cpu().numpy()
    for call in range(2):
        lse = torch.full((w.num_seqs, Hq), float("nan"), dtype=torch.float32, device="cuda")
        out = torch.full_like(d.q, float("nan"))
        torch.cuda.synchronize()
        free_before = torch.cuda.mem_get_info()[0]
        pgd.paged_decode_attention_noalloc(d.q, d.k, d.v, d.bt, d.cl, Hq, Hkv, D, bs, w.scale,
                                           out, max_context_len=w.max_context_len,
                                           k_scale=d.ks, v_scale=d.vs, lse_out=lse)
        torch.cuda.synchronize()
        free_after = torch.cuda.mem_get_info()[0]
        if call == 1:
            # the first call on a device may commit the static array; from
            # then on a call leaves the device's free memory as it was
            assert free_after == free_before, \
                f"noalloc call changed free device memory by {free_before - free_after} bytes"
        got = to_f64(out)
        assert np.all(np.isfinite(got)), f"call {call}: non-finite output"
        assert_close(got, ref, dt, f"noalloc call {call}")
        gl = lse.cpu().numpy()
        live = np.isfinite(ref_lse)
        assert np.array_equal(np.isneginf(gl), ~live)
        assert np.max(np.abs(gl[live] - ref_lse[live])) <= 1e-3
    assert pgd.get_device_error() == 0


def test_noalloc_refuses_requests_past_its_limits():
    lib = pgd.load_library()
    w = make_case([40, 70], 8, 2, 128, 16, "bf16", seed=7)
    d = Dev(w)
    P = lambda t: ctypes.c_void_p(t.data_ptr())  # noqa: E731
    out = torch.empty_like(d.q)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    base = [P(d.q), P(d.k), P(d.v), P(d.bt), w.max_blocks_per_seq, P(d.cl)]
    tail = [8, 2, 128, 16, w.num_blocks, w.scale, 0, None, None, P(out), None]
    # more (sequence, KV head) pairs than the counter array holds: refused on
    # the host, nothing is read or launched
    assert lib.pgd_paged_decode_attention_noalloc(*base, 40000, 0, *tail, 0, stream) == 6
    # an explicit grid whose partials do not fit in the static array
    assert lib.pgd_paged_decode_attention_noalloc(*base, w.num_seqs, 0, *tail, 1 << 20,
                                                  stream) == 6
    # within the limits the same call succeeds
    assert lib.pgd_paged_decode_attention_noalloc(*base, w.num_seqs, 0, *tail, 0, stream) == 0
    torch.cuda.synchronize()
    assert pgd.get_device_error() == 0
