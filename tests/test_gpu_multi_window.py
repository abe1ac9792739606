"""GPU parity for several query tokens per sequence and sliding windows
(pgd_paged_decode_attention_ex) against the oracle's multi-token decode:
query token j of a sequence with n tokens sees positions below
n - q_len + 1 + j, and with a window W only the last W of them."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, assert_close, dev_bf16, host_bits, to_f64
from workloads import make_case, to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    yield
    assert pgd.get_device_error() == 0


def multi_q(B, L, Hq, D, seed):
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal((B, L, Hq, D), dtype=np.float32))


def run_ex(d, qm, window, num_ctas=0):
    w = d.w
    B, L = qm.shape[:2]
    lse = torch.empty((B, L, w.num_q_heads), dtype=torch.float32, device="cuda")
    out = pgd.paged_decode_attention_ex(dev_bf16(qm), d.k, d.v, d.bt, d.cl, w.num_q_heads,
                                        w.num_kv_heads, w.head_dim, w.block_size, w.scale,
                                        window=window, max_context_len=w.max_context_len,
                                        k_scale=d.ks, v_scale=d.vs, lse_out=lse,
                                        num_ctas=num_ctas)
    torch.cuda.synchronize()
    return out, lse


def check_multi(w, qm, window, num_ctas=0, lse_tol=1e-3):
    d = Dev(w)
    out, lse = run_ex(d, qm, window, num_ctas)
    ref, ref_lse = oracle.paged_decode_multi(qm, w.k_cache, w.v_cache, w.block_table,
                                             w.context_lens, w.num_kv_heads, w.scale,
                                             window=window, k_scale=w.k_scale,
                                             v_scale=w.v_scale)
    got = to_f64(out)
    assert np.all(np.isfinite(got)), "non-finite output (masked slot read?)"
    assert_close(got, ref, w.kv_dtype, f"{w.name} q_len={qm.shape[1]} W={window}")
    gl = lse.cpu().numpy().astype(np.float64)
    live = np.isfinite(ref_lse)
    assert np.all(np.isneginf(gl[~live])), "rows that see nothing must have lse -inf"
    assert np.all(got[~live] == 0), "rows that see nothing must be zero"
    assert np.max(np.abs(gl[live] - ref_lse[live]), initial=0) <= lse_tol
    return d, out, lse


# ragged contexts: shorter than q_len, block edges, several tiles per sequence
CTX = [1, 3, 15, 16, 17, 64, 65, 200, 1000, 2049, 0, 333]

MULTI = [  # (Hq, Hkv, D, bs, dtype, q_len)
    (8, 2, 128, 16, "bf16", 2), (8, 2, 128, 16, "bf16", 4), (4, 2, 128, 32, "bf16", 8),
    (8, 8, 128, 64, "bf16", 8), (16, 2, 128, 16, "bf16", 2), (12, 4, 128, 16, "bf16", 3),
    (8, 2, 256, 32, "bf16", 4), (4, 4, 256, 16, "bf16", 5), (32, 8, 128, 16, "e4m3", 4),
    (16, 8, 128, 64, "e4m3", 8), (8, 1, 128, 32, "e4m3", 2),
    # 17 to 32 rows per KV head: two row groups of consumer warps, one pass
    # over K/V (Llama shape g 4 with q_len 5-8; g 8 with q_len 3-4; g 16 at
    # head_dim 256 with q_len 2)
    (32, 8, 128, 16, "bf16", 8), (32, 8, 128, 16, "bf16", 5), (64, 8, 128, 64, "bf16", 4),
    (64, 8, 128, 16, "e4m3", 4), (24, 8, 128, 32, "e4m3", 7), (32, 2, 256, 32, "bf16", 2),
    (16, 2, 256, 16, "bf16", 3), (20, 4, 128, 64, "bf16", 6), (8, 1, 128, 16, "bf16", 3),
]


@pytest.mark.parametrize("Hq,Hkv,D,bs,dt,L", MULTI,
                         ids=[f"g{a // b}-L{f}-D{c}-bs{d}-{e}" for a, b, c, d, e, f in MULTI])
def test_multi_token_causal(Hq, Hkv, D, bs, dt, L):
    w = make_case(CTX, Hq, Hkv, D, bs, dt, seed=900 + Hq + L * 7 + D + bs, name=f"multi-{dt}")
    check_multi(w, multi_q(len(CTX), L, Hq, D, seed=901 + L), 0)


WINDOWS = [1, 5, 16, 17, 100, 1024, 5000]


@pytest.mark.parametrize("W", WINDOWS)
@pytest.mark.parametrize("dt,D,bs", [("bf16", 128, 16), ("bf16", 256, 64), ("e4m3", 128, 32)])
def test_sliding_window_single_token(W, dt, D, bs):
    w = make_case(CTX, 16, 4, D, bs, dt, seed=930 + W + bs, name=f"window-{dt}")
    check_multi(w, multi_q(len(CTX), 1, 16, D, seed=931), W)


@pytest.mark.parametrize("L,W", [(2, 3), (4, 16), (8, 33), (4, 1), (2, 700)])
def test_sliding_window_multi_token(L, W):
    w = make_case(CTX, 8, 4, 128, 16, "bf16", seed=950 + L + W, name="window-multi")
    check_multi(w, multi_q(len(CTX), L, 8, 128, seed=951), W)


@pytest.mark.parametrize("Hq,Hkv,D,bs,dt,L,W", [
    (32, 8, 128, 16, "bf16", 8, 33), (64, 8, 128, 16, "e4m3", 4, 100),
    (32, 2, 256, 32, "bf16", 2, 1000), (32, 8, 128, 64, "bf16", 8, 1)])
def test_sliding_window_32_rows(Hq, Hkv, D, bs, dt, L, W):
    w = make_case(CTX, Hq, Hkv, D, bs, dt, seed=955 + L + W, name=f"window-32rows-{dt}")
    check_multi(w, multi_q(len(CTX), L, Hq, D, seed=956), W)


@pytest.mark.parametrize("num_ctas", [1, 3, 29, 148, 1000])
def test_multi_window_split_count_invariance(num_ctas):
    w = make_case([5000, 17, 640, 1, 0, 2222], 8, 2, 128, 16, "bf16", seed=960,
                  name="multi-split")
    check_multi(w, multi_q(6, 4, 8, 128, seed=961), 300, num_ctas=num_ctas)


@pytest.mark.parametrize("num_ctas", [1, 7, 296, 1000])
def test_32_rows_split_count_invariance(num_ctas):
    """32 rows per KV head (g 4, q_len 8): units split over many CTAs are
    merged by the two-pass column loop of the split merge."""
    w = make_case([5000, 17, 640, 1, 0, 2222], 32, 8, 128, 16, "bf16", seed=962,
                  name="multi-split-32")
    check_multi(w, multi_q(6, 8, 32, 128, seed=963), 0, num_ctas=num_ctas)
    check_multi(w, multi_q(6, 8, 32, 128, seed=964), 300, num_ctas=num_ctas)


def test_single_token_no_window_is_the_plain_decode():
    """q_len 1 and window 0 give the bits of pgd_paged_decode_attention."""
    w = make_case(CTX, 32, 8, 128, 16, "bf16", seed=970, name="ex-plain")
    d = Dev(w)
    a, la = d.decode()
    b, lb = run_ex(d, w.q[:, None], 0)
    assert torch.equal(a.view(torch.int16), b[:, 0].view(torch.int16))
    assert torch.equal(la, lb[:, 0])


def test_window_covering_the_context_is_bit_identical_to_no_window():
    w = make_case(CTX, 8, 2, 128, 32, "bf16", seed=971, name="ex-wide-window")
    d = Dev(w)
    qm = multi_q(len(CTX), 4, 8, 128, seed=972)
    a, la = run_ex(d, qm, 0)
    b, lb = run_ex(d, qm, int(max(CTX)) + 8)
    assert np.array_equal(host_bits(a), host_bits(b))
    assert torch.equal(la, lb)


def test_window_never_reads_blocks_before_it():
    """Blocks wholly before every row's window hold NaN: the result must
    still match, so they are neither read into the softmax nor multiplied."""
    ctx = [700, 333, 64]
    w = make_case(ctx, 8, 2, 128, 16, "bf16", seed=973, name="window-poison")
    W, L = 40, 2
    k = w.k_cache.copy()
    v = w.v_cache.copy()
    for s, n in enumerate(ctx):
        first = max(0, n - L + 1 - W) // 16         # first block any row can see
        for b in w.block_table[s, :first]:
            k[b] = 0x7FC0
            v[b] = 0x7FC0
    w.k_cache, w.v_cache = k, v
    check_multi(w, multi_q(3, L, 8, 128, seed=974), W)


def test_multi_token_full_size_long_context():
    """A long-context batch at the sizes of the decode benchmark's long case,
    four query tokens per sequence, g * q_len = 16 rows per KV head, and
    eight (32 rows)."""
    ctx = [32768, 16384, 8192, 4096, 1, 31999]
    w = make_case(ctx, 32, 8, 128, 16, "bf16", seed=980, name="multi-long")
    check_multi(w, multi_q(len(ctx), 4, 32, 128, seed=981), 0)
    check_multi(w, multi_q(len(ctx), 4, 32, 128, seed=982), 4096)
    check_multi(w, multi_q(len(ctx), 8, 32, 128, seed=983), 0)
    check_multi(w, multi_q(len(ctx), 8, 32, 128, seed=984), 4096)


def test_32_rows_repeat_and_permutation_bits():
    """Two row groups merge in a fixed order: repeated runs, and the same
    blocks placed elsewhere in the pool, give identical bits."""
    w = make_case([3000, 700, 65, 1], 32, 8, 128, 16, "bf16", seed=985, name="multi-bits")
    qm = multi_q(4, 8, 32, 128, seed=986)
    d = Dev(w)
    a, la = run_ex(d, qm, 0, num_ctas=41)
    b, lb = run_ex(d, qm, 0, num_ctas=41)
    assert np.array_equal(host_bits(a), host_bits(b)) and torch.equal(la, lb)
    rng = np.random.default_rng(987)
    perm = rng.permutation(w.num_blocks)
    k2 = np.empty_like(w.k_cache)
    v2 = np.empty_like(w.v_cache)
    k2[perm], v2[perm] = w.k_cache, w.v_cache
    w.k_cache, w.v_cache, w.block_table = k2, v2, perm[w.block_table].astype(np.int32)
    c, lc = run_ex(Dev(w), qm, 0, num_ctas=41)
    assert np.array_equal(host_bits(a), host_bits(c)) and torch.equal(la, lc)
