"""GPU parity: the CUDA path (through the C ABI) against the fp64 oracle on the
same seeded inputs, element by element, within the stated tolerances
(bf16 KV: 2e-3 + 1e-2*|ref|; FP8 E4M3 KV: 2e-2 + 5e-2*|ref|); kv_append
bit-exact over the whole pool."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, assert_close, host_bits, oracle_caches, oracle_full, to_f64
from workloads import make_case, make_workload

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    yield
    assert pgd.get_device_error() == 0


def check_case(w, num_ctas=0, lse_tol=1e-3):
    d = Dev(w)
    d.append()
    out, lse = d.decode(num_ctas=num_ctas)
    torch.cuda.synchronize()
    ref, ref_lse = oracle_full(w)
    got = to_f64(out)
    assert np.all(np.isfinite(got)), "non-finite output (poisoned slot read?)"
    assert_close(got, ref, w.kv_dtype, w.name)
    gl = lse.cpu().numpy().astype(np.float64)
    live = np.isfinite(ref_lse)
    assert np.all(np.isneginf(gl[~live]))
    assert np.max(np.abs(gl[live] - ref_lse[live]), initial=0) <= lse_tol
    return d, got, ref


# --------------------------------------------------------------------------- #
def test_tiny_workload():
    check_case(make_workload("tiny"))


SHAPES = [  # (Hq, Hkv, D, bs, dtype)
    (8, 2, 128, 16, "bf16"), (32, 8, 128, 16, "bf16"), (64, 8, 128, 64, "bf16"),
    (32, 2, 256, 32, "bf16"), (16, 16, 128, 32, "bf16"), (8, 1, 128, 64, "bf16"),
    (16, 8, 256, 16, "bf16"), (32, 2, 128, 16, "bf16"), (64, 4, 256, 64, "bf16"),
    (64, 8, 128, 16, "e4m3"), (32, 2, 128, 32, "e4m3"), (8, 8, 128, 64, "e4m3"),
    (16, 1, 128, 16, "e4m3"),
    # groups that are not powers of two (7: 28 query heads over 4 KV heads)
    (28, 4, 128, 16, "bf16"), (12, 4, 128, 32, "e4m3"), (20, 2, 256, 64, "bf16"),
    (5, 1, 128, 16, "bf16"),
]
CTX = [1, 15, 16, 17, 63, 64, 65, 200, 1000, 2049, 0, 333]


@pytest.mark.parametrize("Hq,Hkv,D,bs,dt", SHAPES,
                         ids=[f"g{a // b}-D{c}-bs{d}-{e}" for a, b, c, d, e in SHAPES])
def test_ragged_batch(Hq, Hkv, D, bs, dt):
    w = make_case(CTX, Hq, Hkv, D, bs, dt, seed=Hq * 7 + D + bs, name=f"ragged-{dt}")
    check_case(w)


@pytest.mark.parametrize("num_ctas", [1, 2, 3, 7, 64, 296, 1000])
def test_split_count_invariance(num_ctas):
    w = make_case([5, 700, 3000, 64, 1], 32, 8, 128, 16, "bf16", seed=5)
    check_case(w, num_ctas=num_ctas)


def test_split_count_invariance_fp8_g16():
    w = make_case([900, 17, 4000], 32, 2, 128, 16, "e4m3", seed=6)
    for n in (1, 5, 100):
        check_case(w, num_ctas=n)


def test_block_permutation_gives_identical_bits():
    w = make_case([300, 1500, 77], 32, 8, 128, 16, "bf16", seed=8)
    d = Dev(w)
    a, la = d.decode(num_ctas=37)
    rng = np.random.default_rng(9)
    perm = rng.permutation(w.num_blocks)
    k2 = np.empty_like(w.k_cache); v2 = np.empty_like(w.v_cache)
    k2[perm] = w.k_cache; v2[perm] = w.v_cache
    w2 = make_case([300, 1500, 77], 32, 8, 128, 16, "bf16", seed=8)
    w2.k_cache, w2.v_cache, w2.block_table = k2, v2, perm[w.block_table].astype(np.int32)
    b, lb = Dev(w2).decode(num_ctas=37)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert torch.equal(la, lb)


def test_repeat_runs_are_bit_identical():
    w = make_case([4000, 123, 2500, 16], 64, 8, 128, 64, "bf16", seed=10)
    d = Dev(w)
    outs = [d.decode()[0].clone() for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


def test_empty_contexts():
    w = make_case([0, 0, 0], 16, 4, 128, 16, "bf16", seed=11, pool=8)
    w.context_lens[:] = 0
    d = Dev(w)
    out, lse = d.decode(max_context_len=0)
    torch.cuda.synchronize()
    assert torch.count_nonzero(out.float()) == 0
    assert torch.all(torch.isneginf(lse))


def test_peaked_softmax_planted_key():
    """One key planted parallel to query head 0 so its score dominates every
    other by > 30: head 0's output must be that token's V row."""
    from workloads import bf16_bits_to_f32, to_bf16_bits
    w = make_case([5000], 16, 2, 128, 16, "bf16", seed=12)
    t = 1234
    pb, row = w.block_table[0, t // 16], t % 16
    q0 = bf16_bits_to_f32(w.q[0, 0])
    w.k_cache[pb, 0, row] = to_bf16_bits(q0 * 4.0)
    d, got, ref = check_case(w)
    v_t = bf16_bits_to_f32(w.v_cache[pb, 0, row]).astype(np.float64)
    np.testing.assert_allclose(got[0, 0], v_t, rtol=1e-2, atol=1e-3)
    w2 = make_case([5000, 3000], 32, 2, 256, 32, "bf16", seed=13, key_boost_frac=0.05)
    check_case(w2)


@pytest.mark.parametrize("qexp", [-20, 17, 0])
def test_fp8_query_magnitudes_outside_f16_range(qexp):
    """The FP8 path multiplies in f16, whose range is far narrower than
    bf16's.  Query rows scaled by 2^qexp with the softmax scale scaled by
    2^-qexp give the same logits; at 2^17 |q| passes f16's largest value
    (65504) and at 2^-20 it falls into f16's subnormals, yet the result must
    match the oracle as the unscaled case does."""
    from workloads import bf16_bits_to_f32, to_bf16_bits
    w = make_case(CTX, 64, 8, 128, 16, "e4m3", seed=40 + qexp, name=f"fp8-q2^{qexp}")
    w.q = to_bf16_bits(bf16_bits_to_f32(w.q) * np.float32(2.0 ** qexp))   # exact in bf16
    w.scale = w.scale * 2.0 ** -qexp
    assert np.abs(bf16_bits_to_f32(w.q)).max() > (65504 if qexp > 0 else 0)
    check_case(w)


def test_one_token_contexts_return_v0():
    w = make_case([1] * 9, 32, 8, 128, 16, "bf16", seed=14)
    d, got, ref = check_case(w)
    # exact: a single weight of 1 gives V_0 rounded to bf16, which is V_0
    assert np.array_equal(got, ref)


def test_kv_append_bit_exact_whole_pool():
    for dt in ("bf16", "e4m3"):
        w = make_case([1, 16, 17, 100, 513], 16, 4, 128, 16, dt, seed=15, append_last=True)
        w.slot_mapping = np.concatenate([w.slot_mapping, np.array([-1], np.int64)])
        w.k_new = np.concatenate([w.k_new, np.zeros_like(w.k_new[:1])])
        w.v_new = np.concatenate([w.v_new, np.zeros_like(w.v_new[:1])])
        d = Dev(w)
        d.append()
        torch.cuda.synchronize()
        ek, ev = oracle_caches(w)
        assert np.array_equal(host_bits(d.k), ek) and np.array_equal(host_bits(d.v), ev)


def test_merge_partials_kernel():
    rng = np.random.default_rng(16)
    P, R, D = 5, 37, 128
    o = rng.standard_normal((P, R, D)).astype(np.float32)
    lse = (rng.standard_normal((P, R)) * 3).astype(np.float32)
    lse[1, :5] = -np.inf
    lse[:, 7] = -np.inf
    ref, ref_lse = oracle.merge_partials(o.astype(np.float64), lse.astype(np.float64))
    lse_t = torch.empty(R, dtype=torch.float32, device="cuda")
    out = pgd.merge_partials(torch.from_numpy(o).cuda(), torch.from_numpy(lse).cuda(),
                             lse_out=lse_t)
    got = to_f64(out)
    assert_close(got, ref, "bf16", "merge")
    gl = lse_t.cpu().numpy()
    assert np.isneginf(gl[7])
    live = np.isfinite(ref_lse)
    assert np.max(np.abs(gl[live] - ref_lse[live])) < 1e-4


# --------------------------------------------------------------------------- #
# full-size workloads, in the launch configuration the bench times (automatic
# grid): every (sequence, query head) row against the oracle
# --------------------------------------------------------------------------- #
def oracle_every_row(w):
    """The oracle's out / lse for every (sequence, query head) row of a
    workload.  The unchanged single-threaded oracle runs on chunks of rows in
    a thread pool: its ctypes calls release the GIL, so the chunks run on all
    host cores at once (threads, not processes: nothing is forked after the
    GPU is in use)."""
    import os
    from concurrent.futures import ThreadPoolExecutor
    kc, vc = oracle_caches(w)
    B, Hq = w.num_seqs, w.num_q_heads
    rs_all = np.repeat(np.arange(B, dtype=np.int32), Hq)
    rh_all = np.tile(np.arange(Hq, dtype=np.int32), B)
    # chunks of similar cost: rows sorted by context length, dealt round robin
    order = np.argsort(-w.context_lens[rs_all], kind="stable")
    nthreads = max(1, os.cpu_count() or 1)
    nchunks = min(len(order), 4 * nthreads)
    chunks = [order[i::nchunks] for i in range(nchunks)]

    def run(idx):
        return idx, oracle.paged_decode_rows(w.q, kc, vc, w.block_table, w.context_lens,
                                             w.num_kv_heads, w.scale, rs_all[idx],
                                             rh_all[idx], w.k_scale, w.v_scale)

    out = np.empty((B * Hq, w.head_dim), np.float64)
    lse = np.empty(B * Hq, np.float64)
    with ThreadPoolExecutor(max_workers=nthreads) as ex:
        for idx, (o, l) in ex.map(run, chunks):
            out[idx], lse[idx] = o, l
    return out.reshape(B, Hq, w.head_dim), lse.reshape(B, Hq)


@pytest.mark.parametrize("name", ["llama3_8b_decode", "long_context", "wide_heads", "fp8_mixed"])
def test_full_size_every_row(name):
    w = make_workload(name)
    d = Dev(w)
    d.append()
    out, lse = d.decode()
    torch.cuda.synchronize()
    got = to_f64(out)
    assert np.all(np.isfinite(got))
    ref, ref_lse = oracle_every_row(w)
    assert_close(got, ref, w.kv_dtype, f"{name}: all {w.num_seqs * w.num_q_heads} rows")
    # per-row relative L2 error and lse, reported over every row
    err = np.linalg.norm(got - ref, axis=-1) / np.maximum(np.linalg.norm(ref, axis=-1), 1e-30)
    live = w.context_lens > 0
    assert err[live].max() < (1e-2 if w.kv_dtype == "bf16" else 5e-2), err[live].max()
    gl = lse.cpu().numpy().astype(np.float64)
    assert np.max(np.abs(gl[live] - ref_lse[live])) < 1e-3
    print(f"{name}: {w.num_seqs * w.num_q_heads} rows checked; max rel L2 "
          f"{err[live].max():.2e}; max |dlse| {np.max(np.abs(gl[live] - ref_lse[live])):.2e}")
    if w.slot_mapping is not None:
        ek, ev = oracle_caches(w)
        assert np.array_equal(host_bits(d.k), ek) and np.array_equal(host_bits(d.v), ev)
        # the launch the decode-step benchmark times: append fused into the
        # decode (pgd_decode_step), same bits as the two launches above
        from tests.gpu_helpers import dev_cache
        kn, vn = _step_payload(w)
        d2 = Dev(w)
        lse2 = torch.empty_like(lse)
        out2 = pgd.decode_step(d2.q, dev_cache(kn), dev_cache(vn), d2.k, d2.v, d2.bt, d2.cl,
                               w.num_q_heads, w.num_kv_heads, w.head_dim, w.block_size,
                               w.scale, max_context_len=w.max_context_len, k_scale=d2.ks,
                               v_scale=d2.vs, lse_out=lse2)
        torch.cuda.synchronize()
        assert torch.equal(out2.view(torch.int16), out.view(torch.int16))
        assert torch.equal(lse2, lse)
        assert np.array_equal(host_bits(d2.k), ek) and np.array_equal(host_bits(d2.v), ev)


# --------------------------------------------------------------------------- #
# device-side bounds checks: flagged, never faulting
# --------------------------------------------------------------------------- #
def test_out_of_range_inputs_are_flagged_not_faulting():
    w = make_case([40, 70], 8, 2, 128, 16, "bf16", seed=18)
    d = Dev(w)
    assert pgd.get_device_error() == 0
    d.bt[1, 2] = w.num_blocks + 5           # block id past the pool
    d.decode()
    assert pgd.get_device_error() & 1
    d.bt.copy_(torch.from_numpy(w.block_table).cuda())
    d.cl[0] = w.max_blocks_per_seq * w.block_size + 1   # context past the table
    d.decode()
    assert pgd.get_device_error() & 2
    d.cl.copy_(torch.from_numpy(w.context_lens).cuda())
    kn = torch.zeros((1, 2, 128), dtype=torch.bfloat16, device="cuda")
    pgd.kv_append(kn, kn, torch.tensor([w.num_blocks * 16], dtype=torch.int64, device="cuda"),
                  d.k, d.v)
    assert pgd.get_device_error() & 4
    # the context is still usable and results are right again
    out, _ = d.decode()
    torch.cuda.synchronize()
    ref, _ = oracle_full(w)
    assert_close(to_f64(out), ref, "bf16", "after flags")


# --------------------------------------------------------------------------- #
# fused decode step: append of each sequence's newest token + decode, one launch
# --------------------------------------------------------------------------- #
def _step_payload(w):
    """k_new / v_new [B][Hkv][D] for pgd_decode_step from the append payload
    (one row per live sequence, zeros for empty ones)."""
    live = [s for s in range(w.num_seqs) if w.context_lens[s] > 0]
    kn = np.zeros((w.num_seqs,) + w.k_new.shape[1:], w.k_new.dtype)
    vn = np.zeros_like(kn)
    kn[live] = w.k_new
    vn[live] = w.v_new
    return kn, vn


STEP_CASES = [  # (ctx, Hq, Hkv, D, bs, dtype, num_ctas)
    ([1, 15, 16, 17, 200, 1000, 2049, 0, 333], 32, 8, 128, 16, "bf16", 0),
    ([1, 15, 16, 17, 200, 1000, 2049, 0, 333], 32, 8, 128, 16, "bf16", 7),
    ([700, 5, 3000, 64], 32, 2, 256, 32, "bf16", 0),
    ([64, 900, 17, 4000, 1], 64, 8, 128, 16, "e4m3", 0),
    ([65, 128, 129], 16, 2, 128, 64, "bf16", 3),
]


@pytest.mark.parametrize("ctx,Hq,Hkv,D,bs,dt,nctas", STEP_CASES,
                         ids=[f"g{c[1] // c[2]}-D{c[3]}-bs{c[4]}-{c[5]}-n{c[6]}" for c in STEP_CASES])
def test_fused_decode_step(ctx, Hq, Hkv, D, bs, dt, nctas):
    from tests.gpu_helpers import dev_cache
    w = make_case(ctx, Hq, Hkv, D, bs, dt, seed=200 + D + bs, append_last=True)
    kn, vn = _step_payload(w)
    # fused path
    d1 = Dev(w)
    lse1 = torch.empty((w.num_seqs, Hq), dtype=torch.float32, device="cuda")
    out1 = pgd.decode_step(d1.q, dev_cache(kn), dev_cache(vn), d1.k, d1.v, d1.bt, d1.cl, Hq, Hkv,
                           D, bs, w.scale, max_context_len=w.max_context_len, k_scale=d1.ks,
                           v_scale=d1.vs, lse_out=lse1, num_ctas=nctas)
    # two-launch path on a fresh copy
    d2 = Dev(w)
    d2.append()
    out2, lse2 = d2.decode(num_ctas=nctas)
    torch.cuda.synchronize()
    ek, ev = oracle_caches(w)
    assert np.array_equal(host_bits(d1.k), ek) and np.array_equal(host_bits(d1.v), ev)
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert torch.equal(lse1, lse2)
    ref, ref_lse = oracle_full(w)
    got = to_f64(out1)
    assert np.all(np.isfinite(got))
    assert_close(got, ref, dt, "fused step")


# --------------------------------------------------------------------------- #
# quantising append: bf16 rows -> E4M3 cache, bit-exact with the oracle
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("D,bs", [(128, 16), (256, 32), (128, 64)])
def test_kv_append_quant_bit_exact(D, bs):
    from workloads import to_bf16_bits
    rng = np.random.default_rng(300 + D + bs)
    N, Hkv, nb = 57, 4, 40
    x = rng.standard_normal((2, N, Hkv, D)).astype(np.float32) * 3
    x[:, :5] *= 1e3                      # saturate
    x[:, 5:10] *= 1e-4                   # subnormal codes
    x[:, 10, :, :4] = [1.0625, 1.1875, -3.25, 0.0]   # exact midpoints at scale 1
    kb, vb = to_bf16_bits(x[0]), to_bf16_bits(x[1])
    ks = np.array([1.0, 0.0071, 0.02, 0.5], np.float32)
    vs = np.array([0.003, 1.0, 0.25, 2.0], np.float32)
    slots = rng.choice(nb * bs, size=N, replace=False).astype(np.int64)
    slots[3] = -1
    kc0 = rng.integers(0, 256, size=(nb, Hkv, bs, D)).astype(np.uint8)
    vc0 = rng.integers(0, 256, size=(nb, Hkv, bs, D)).astype(np.uint8)
    ek, ev = oracle.kv_append_quant(kb, vb, slots, kc0, vc0, ks, vs, bs)
    from tests.gpu_helpers import dev_bf16
    kc = torch.from_numpy(kc0.copy()).cuda()
    vc = torch.from_numpy(vc0.copy()).cuda()
    pgd.kv_append_quant(dev_bf16(kb), dev_bf16(vb), torch.from_numpy(slots).cuda(), kc, vc,
                        torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda())
    torch.cuda.synchronize()
    assert np.array_equal(kc.cpu().numpy(), ek) and np.array_equal(vc.cpu().numpy(), ev)


def test_quantised_append_then_fp8_decode():
    """bf16 K/V quantised by the library, then decoded from the FP8 cache."""
    from tests.gpu_helpers import dev_bf16
    from workloads import to_bf16_bits
    w = make_case([70, 300, 16, 1], 32, 4, 128, 16, "e4m3", seed=310)
    rng = np.random.default_rng(311)
    live = [s for s in range(w.num_seqs) if w.context_lens[s] > 0]
    slots = np.array([int(w.block_table[s, (w.context_lens[s] - 1) // 16]) * 16 +
                      int((w.context_lens[s] - 1) % 16) for s in live], np.int64)
    kb = to_bf16_bits(rng.standard_normal((len(slots), 4, 128)).astype(np.float32))
    vb = to_bf16_bits(rng.standard_normal((len(slots), 4, 128)).astype(np.float32))
    ek, ev = oracle.kv_append_quant(kb, vb, slots, w.k_cache, w.v_cache, w.k_scale, w.v_scale, 16)
    d = Dev(w)
    pgd.kv_append_quant(dev_bf16(kb), dev_bf16(vb), torch.from_numpy(slots).cuda(), d.k, d.v,
                        d.ks, d.vs)
    out, _ = d.decode()
    torch.cuda.synchronize()
    assert np.array_equal(d.k.cpu().numpy(), ek) and np.array_equal(d.v.cpu().numpy(), ev)
    w.k_cache, w.v_cache = ek, ev
    ref, _ = oracle_full(w)
    assert_close(to_f64(out), ref, "e4m3", "quantised append + decode")


# --------------------------------------------------------------------------- #
# prepared calls: the same C call re-issued with the arguments marshalled once
# --------------------------------------------------------------------------- #
def test_prepared_calls_give_the_same_bits():
    w = make_case([1, 17, 64, 200, 999], 32, 8, 128, 16, "bf16", seed=19, append_last=True)
    kn, vn = _step_payload(w)
    from tests.gpu_helpers import dev_cache
    d1, d2 = Dev(w), Dev(w)
    kn_d, vn_d = dev_cache(kn), dev_cache(vn)
    out1 = pgd.decode_step(d1.q, kn_d, vn_d, d1.k, d1.v, d1.bt, d1.cl, 32, 8, 128, 16, w.scale,
                           max_context_len=w.max_context_len)
    out2 = torch.empty_like(out1)
    call = pgd.decode_step(d2.q, kn_d, vn_d, d2.k, d2.v, d2.bt, d2.cl, 32, 8, 128, 16, w.scale,
                           out2, max_context_len=w.max_context_len, prepare=True)
    for _ in range(3):
        assert call() is out2
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    # the prepared call reads the buffers' current contents on every call
    d2.q.copy_(d2.q.flip(0))
    call()
    out3 = pgd.decode_step(d1.q.flip(0).contiguous(), kn_d, vn_d, d1.k, d1.v, d1.bt, d1.cl, 32,
                           8, 128, 16, w.scale, max_context_len=w.max_context_len)
    torch.cuda.synchronize()
    assert torch.equal(out2.view(torch.int16), out3.view(torch.int16))
