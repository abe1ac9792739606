"""GPU parity of the KV-parallel path on one GPU: the W ranks' slices are
decoded one after another (pgd_paged_decode_partial; no kernel waits on
another), stacked as the all-gather would stack them, and merged by
pgd_merge_partials; each slice's split result is compared with the oracle's
decode of that slice and the merged output with the oracle's unsplit
decode."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from paged_gqa_decode_07_b200 import kvp
from tests.gpu_helpers import Dev, assert_close, to_f64
from workloads import make_case

pytestmark = pytest.mark.gpu

# split results are fp32: tighter than the bf16 output tolerance
PART_TOL = {"bf16": (2e-4, 2e-3), "e4m3": (2e-2, 5e-2)}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    yield
    assert pgd.get_device_error() == 0


def run_kvp(w, W, num_ctas=0):
    d = Dev(w)
    rows = w.num_seqs * w.num_q_heads
    o_all = torch.empty((W, rows, w.head_dim), dtype=torch.float32, device="cuda")
    lse_all = torch.empty((W, rows), dtype=torch.float32, device="cuda")
    slices = []
    for r in range(W):
        start, length = kvp.plan(w.context_lens, w.block_size, W, r)
        table = kvp.local_block_table(w.block_table, start, length, w.block_size)
        o, lse = pgd.paged_decode_partial(
            d.q, d.k, d.v, torch.from_numpy(table).cuda(), torch.from_numpy(length).cuda(),
            w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size, w.scale,
            max_context_len=int(length.max(initial=0)), k_scale=d.ks, v_scale=d.vs,
            num_ctas=num_ctas)
        o_all[r].copy_(o.view(rows, -1))
        lse_all[r].copy_(lse.view(-1))
        slices.append((table, length))
    out = torch.empty((rows, w.head_dim), dtype=torch.bfloat16, device="cuda")
    lse_out = torch.empty((rows,), dtype=torch.float32, device="cuda")
    pgd.merge_partials(o_all, lse_all, out, lse_out)
    torch.cuda.synchronize()
    return d, slices, o_all, lse_all, out, lse_out


def check_kvp(w, W, num_ctas=0):
    d, slices, o_all, lse_all, out, lse_out = run_kvp(w, W, num_ctas)
    rows = w.num_seqs * w.num_q_heads
    for r, (table, length) in enumerate(slices):
        ref, rl = oracle.paged_decode(w.q, w.k_cache, w.v_cache, table, length, w.num_kv_heads,
                                      w.scale, w.k_scale, w.v_scale)
        got = o_all[r].double().cpu().numpy()
        assert_close_tol(got, ref.reshape(rows, -1), PART_TOL[w.kv_dtype], f"slice {r}/{W}")
        gl = lse_all[r].double().cpu().numpy()
        live = np.isfinite(rl.reshape(-1))
        assert np.all(np.isneginf(gl[~live])) and np.all(got[~live] == 0)
        assert np.max(np.abs(gl[live] - rl.reshape(-1)[live]), initial=0) <= 1e-3
    ref, rl = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                  w.num_kv_heads, w.scale, w.k_scale, w.v_scale)
    assert_close(to_f64(out), ref.reshape(rows, -1), w.kv_dtype, f"kvp merged W={W}")
    live = np.isfinite(rl.reshape(-1))
    gl = lse_out.double().cpu().numpy()
    assert np.max(np.abs(gl[live] - rl.reshape(-1)[live]), initial=0) <= 1e-3
    return d, out


def assert_close_tol(got, ref, tol, what):
    atol, rtol = tol
    bad = ~(np.abs(got - ref) <= atol + rtol * np.abs(ref))
    assert not bad.any(), f"{what}: {int(bad.sum())} of {bad.size} outside ({atol}, {rtol})"


CTX = [1, 15, 16, 17, 200, 1000, 2049, 0, 333, 5000]


@pytest.mark.parametrize("W", [2, 3, 4, 8])
def test_kvp_bf16(W):
    check_kvp(make_case(CTX, 32, 8, 128, 16, "bf16", seed=1000 + W, name="kvp-bf16"), W)


@pytest.mark.parametrize("W", [2, 5])
def test_kvp_fp8_and_d256(W):
    check_kvp(make_case(CTX, 64, 8, 128, 32, "e4m3", seed=1100 + W, name="kvp-fp8"), W)
    check_kvp(make_case(CTX, 16, 2, 256, 64, "bf16", seed=1200 + W, name="kvp-d256"), W)


def test_kvp_long_sequences_many_ranks():
    """Few long sequences split over 8 ranks, the case KV parallelism is for
    (one KV head: tensor parallelism over heads would stop at 1 GPU)."""
    w = make_case([32768, 20000, 65, 31999], 8, 1, 128, 16, "bf16", seed=1300, name="kvp-long")
    check_kvp(w, 8)


def test_partial_rounds_to_the_plain_decode_bits():
    """The fp32 split result of a whole sequence, rounded to bf16, is the
    plain decode's output bit for bit (same arithmetic, rounding last)."""
    w = make_case(CTX, 32, 8, 128, 16, "bf16", seed=1400, name="partial-bits")
    d = Dev(w)
    a, la = d.decode()
    o, lo = pgd.paged_decode_partial(d.q, d.k, d.v, d.bt, d.cl, w.num_q_heads, w.num_kv_heads,
                                     w.head_dim, w.block_size, w.scale,
                                     max_context_len=w.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), o.to(torch.bfloat16).view(torch.int16))
    assert torch.equal(la, lo)


def test_decoder_single_rank_matches_plain_decode():
    """KVPDecoder with a world of one: the slice is the whole sequence."""
    w = make_case(CTX, 32, 8, 128, 16, "bf16", seed=1500, name="kvp-decoder")
    d = Dev(w)
    dec = kvp.KVPDecoder(w.num_seqs, w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size)
    out = dec.step(d.q, d.k, d.v, d.bt, d.cl, w.scale, max_context_len=w.max_context_len)
    ref, _ = d.decode()
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
