"""Pins for the fp64 oracle: each test checks it against something other than
itself -- the pages' worked example, closed forms, invariants the pages state,
textbook library routines, or brute force on tiny inputs.

Pages cited:
  "attention kernels" (froggydisk), sections "standard attention",
  "FlashAttention", "prefill and decode attention", "paged KV and kernels";
  "Optimization 1: batching and attention" (beengineer500), sections 2.2, 2.4,
  3.4.
"""
import json
import math
import os

import numpy as np
import pytest
import torch

import oracle
from workloads import make_case, to_bf16_bits, to_e4m3_bytes, bf16_bits_to_f32

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


# --------------------------------------------------------------------------- #
# helpers                                                                     #
# --------------------------------------------------------------------------- #
def contiguous_case(ctx, Hq, Hkv, D, bs, seed=0, kv="bf16"):
    """K/V drawn per sequence as [ctx][Hkv][D]; the cache places block j of
    sequence s at physical block s * W + j (identity table)."""
    rng = np.random.default_rng(seed)
    B = len(ctx)
    W = max(1, max((n + bs - 1) // bs for n in ctx))
    q = to_bf16_bits(rng.standard_normal((B, Hq, D), dtype=np.float32))
    kseq, vseq = [], []
    for n in ctx:
        kseq.append(rng.standard_normal((W * bs, Hkv, D), dtype=np.float32))
        vseq.append(rng.standard_normal((W * bs, Hkv, D), dtype=np.float32))
    kf = np.stack(kseq)  # [B][W*bs][Hkv][D]
    vf = np.stack(vseq)
    ks = vs = None
    if kv == "bf16":
        kb, vb = to_bf16_bits(kf), to_bf16_bits(vf)
    else:
        ks = (np.abs(kf).max(axis=(0, 1, 3)) / 448.0).astype(np.float32)
        vs = (np.abs(vf).max(axis=(0, 1, 3)) / 448.0).astype(np.float32)
        kb = to_e4m3_bytes(np.clip(kf / ks[None, None, :, None], -448, 448))
        vb = to_e4m3_bytes(np.clip(vf / vs[None, None, :, None], -448, 448))
    kb = kb.reshape(B, W * bs, Hkv, D)
    vb = vb.reshape(B, W * bs, Hkv, D)

    def to_cache(x):
        return np.ascontiguousarray(
            x.reshape(B, W, bs, Hkv, D).transpose(0, 1, 3, 2, 4).reshape(B * W, Hkv, bs, D))

    table = (np.arange(B)[:, None] * W + np.arange(W)[None, :]).astype(np.int32)
    return dict(q=q, kseq=kb, vseq=vb, k_cache=to_cache(kb), v_cache=to_cache(vb),
                table=table, ctx=np.asarray(ctx, np.int32), ks=ks, vs=vs)


def dec(bits):
    if bits.dtype == np.uint16:
        return torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double()
    return torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).double()


def sdpa_reference(c, Hq, Hkv, scale):
    """torch's scaled_dot_product_attention (float64, CPU) on each sequence's
    contiguous K/V, with KV heads repeated to the query heads (GQA group of
    contiguous query heads, "batching and attention" section 2.4)."""
    g = Hq // Hkv
    outs, lses = [], []
    q = dec(c["q"])
    for s, n in enumerate(c["ctx"]):
        k = dec(c["kseq"][s, :n])  # [n][Hkv][D]
        v = dec(c["vseq"][s, :n])
        if c["ks"] is not None:
            k = k * torch.from_numpy(c["ks"]).double()[None, :, None]
            v = v * torch.from_numpy(c["vs"]).double()[None, :, None]
        k = k.permute(1, 0, 2).repeat_interleave(g, dim=0)  # [Hq][n][D]
        v = v.permute(1, 0, 2).repeat_interleave(g, dim=0)
        qs = q[s][:, None, :]                                # [Hq][1][D]
        o = torch.nn.functional.scaled_dot_product_attention(qs, k, v, scale=scale)
        lse = torch.logsumexp(torch.matmul(qs, k.transpose(1, 2)) * scale, dim=-1)
        outs.append(o[:, 0, :].numpy())
        lses.append(lse[:, 0].numpy())
    return np.stack(outs), np.stack(lses)


def run_oracle(c, Hkv, scale, tiled=None):
    if tiled is None:
        return oracle.paged_decode(c["q"], c["k_cache"], c["v_cache"], c["table"], c["ctx"],
                                   Hkv, scale, c["ks"], c["vs"])
    return oracle.paged_decode_tiled(c["q"], c["k_cache"], c["v_cache"], c["table"], c["ctx"],
                                     Hkv, scale, tiled[0], tiled[1], c["ks"], c["vs"])


# --------------------------------------------------------------------------- #
# number formats                                                              #
# --------------------------------------------------------------------------- #
def test_bf16_decoder_all_patterns(oracle_lib):
    bits = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    ours = oracle.bf16_to_double(bits)
    ref = torch.from_numpy(bits.view(np.int16).copy()).view(torch.bfloat16).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert np.array_equal(ours[~nan], ref[~nan])
    # format definition spot values
    assert oracle.bf16_to_double(np.array([0x3F80], np.uint16))[0] == 1.0
    assert oracle.bf16_to_double(np.array([0x0001], np.uint16))[0] == 2.0 ** -133
    assert oracle.bf16_to_double(np.array([0xC040], np.uint16))[0] == -3.0


def test_e4m3_decoder_all_bytes(oracle_lib):
    bits = np.arange(256, dtype=np.uint16).astype(np.uint8)
    ours = oracle.e4m3_to_double(bits)
    ref = torch.from_numpy(bits.copy()).view(torch.float8_e4m3fn).double().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(ours), nan)
    assert list(np.nonzero(nan)[0]) == [0x7F, 0xFF]
    assert np.array_equal(ours[~nan], ref[~nan])
    spot = {0x01: 2.0 ** -9, 0x07: 7 * 2.0 ** -9, 0x08: 2.0 ** -6, 0x38: 1.0,
            0x7E: 448.0, 0xFE: -448.0, 0x80: 0.0}
    for b, v in spot.items():
        assert oracle.e4m3_to_double(np.array([b], np.uint8))[0] == v


# --------------------------------------------------------------------------- #
# the page's worked example of the block table                                #
# --------------------------------------------------------------------------- #
def test_block_table_worked_example(oracle_lib):
    ex = json.load(open(os.path.join(GOLDEN, "block_table_example.json")))
    bs, table, n = ex["block_size"], ex["block_table"], ex["context_len"]
    D, Hkv, Hq, nb = 4, 1, 2, 8
    assert (n + bs - 1) // bs == len(table) and n - (len(table) - 1) * bs == ex["last_block_fill"]
    slots = np.array([table[t // bs] * bs + t % bs for t in range(n)], np.int64)
    assert list(slots) == ex["token_slots"]
    # append token t with K row = t+1 in dim 0, V row = one-hot-ish of t
    kn = np.zeros((n, Hkv, D), np.float32)
    vn = np.zeros((n, Hkv, D), np.float32)
    kn[:, 0, 0] = np.arange(1, n + 1)
    vn[:, 0, 1] = np.arange(n) * 0.5
    kz = np.full((nb, Hkv, bs, D), 0x7FC0, np.uint16)   # NaN everywhere
    vz = kz.copy()
    kc, vc = oracle.kv_append(to_bf16_bits(kn), to_bf16_bits(vn), slots, kz, vz, bs)
    # every appended token is at the slot the figure implies; the rest is untouched
    for t, sl in enumerate(ex["token_slots"]):
        assert np.array_equal(kc[sl // bs, 0, sl % bs], to_bf16_bits(kn[t, 0]))
    touched = np.zeros((nb, bs), bool)
    for sl in slots:
        touched[sl // bs, sl % bs] = True
    assert np.all(kc[:, 0][~touched] == 0x7FC0)
    # decode through the table: compare with SDPA on the contiguous sequence
    q = to_bf16_bits(np.array([[[0.25, 0, 0, 0], [-0.5, 1, 0, 0]]], np.float32))
    bt = np.array([table], np.int32)
    out, lse = oracle.paged_decode(q, kc, vc, bt, np.array([n], np.int32), Hkv, 1.0)
    k = torch.from_numpy(kn[:, 0].astype(np.float64))[None].expand(Hq, n, D)
    v = torch.from_numpy(vn[:, 0].astype(np.float64))[None].expand(Hq, n, D)
    qq = dec(q[0])[:, None, :]
    ref = torch.nn.functional.scaled_dot_product_attention(qq, k, v, scale=1.0)[:, 0]
    np.testing.assert_allclose(out[0], ref.numpy(), rtol=1e-13, atol=1e-15)
    assert np.all(np.isfinite(out))


# --------------------------------------------------------------------------- #
# closed forms                                                                #
# --------------------------------------------------------------------------- #
def _single_seq(krows, vrows, qrow, bs=4, scale=1.0):
    n, D = krows.shape
    W = (n + bs - 1) // bs
    kc = np.full((W + 1, 1, bs, D), 0x7FC0, np.uint16)
    vc = kc.copy()
    perm = np.arange(W)[::-1].copy() + 1          # reversed physical order
    for t in range(n):
        kc[perm[t // bs], 0, t % bs] = to_bf16_bits(krows[t])
        vc[perm[t // bs], 0, t % bs] = to_bf16_bits(vrows[t])
    q = to_bf16_bits(qrow[None, None, :])
    return oracle.paged_decode(q, kc, vc, perm[None].astype(np.int32),
                               np.array([n], np.int32), 1, scale)


def test_one_token_context_returns_v0(oracle_lib):
    D = 8
    k = np.zeros((1, D), np.float32); k[0, 0] = 3.0
    v = np.arange(D, dtype=np.float32)[None] * 0.25 - 1
    q = np.zeros(D, np.float32); q[0] = 2.0
    out, lse = _single_seq(k, v, q, scale=0.5)
    assert np.array_equal(out[0, 0], v[0].astype(np.float64))
    assert lse[0, 0] == 3.0          # 0.5 * (2 * 3)


def test_identical_keys_give_mean_of_v(oracle_lib):
    rng = np.random.default_rng(3)
    n, D = 37, 16
    k = np.tile(bf16_bits_to_f32(to_bf16_bits(rng.standard_normal(D, dtype=np.float32))), (n, 1))
    v = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((n, D), dtype=np.float32)))
    q = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal(D, dtype=np.float32)))
    out, lse = _single_seq(k, v, q, bs=8, scale=0.3)
    mean = v.astype(np.float64).mean(axis=0)
    np.testing.assert_allclose(out[0, 0], mean, rtol=1e-13, atol=1e-15)
    x = 0.3 * float(np.dot(q.astype(np.float64), k[0].astype(np.float64)))
    assert abs(lse[0, 0] - (x + math.log(n))) < 1e-12


def test_zero_scale_gives_mean_of_v(oracle_lib):
    rng = np.random.default_rng(4)
    n, D = 21, 8
    k = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((n, D), dtype=np.float32)))
    v = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((n, D), dtype=np.float32)))
    q = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal(D, dtype=np.float32)))
    out, lse = _single_seq(k, v, q, bs=4, scale=0.0)
    np.testing.assert_allclose(out[0, 0], v.astype(np.float64).mean(0), rtol=1e-13, atol=1e-15)
    assert abs(lse[0, 0] - math.log(n)) < 1e-13


def test_dominant_key_selects_its_value(oracle_lib):
    rng = np.random.default_rng(5)
    n, D = 40, 8
    k = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((n, D), dtype=np.float32)))
    k[17] = 0; k[17, 0] = 1024.0     # x_17 = 1024 vs |x_t| <= ~30 for the rest
    v = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal((n, D), dtype=np.float32)))
    q = np.zeros(D, np.float32); q[0] = 1.0
    q[1:] = bf16_bits_to_f32(to_bf16_bits(rng.standard_normal(D - 1, dtype=np.float32) * 0.01))
    out, lse = _single_seq(k, v, q, scale=1.0)
    assert np.array_equal(out[0, 0], v[17].astype(np.float64))
    assert lse[0, 0] == 1024.0


def test_empty_context(oracle_lib):
    c = contiguous_case([0, 5], 4, 2, 16, 4, seed=9)
    out, lse = run_oracle(c, 2, 0.25)
    assert np.all(out[0] == 0) and np.all(np.isneginf(lse[0]))
    assert np.all(np.isfinite(out[1]))


# --------------------------------------------------------------------------- #
# library special case and brute force                                        #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("Hq,Hkv,D,bs,ctx", [
    (8, 2, 64, 16, [1, 17, 64, 200]),     # GQA g = 4
    (4, 4, 32, 8, [9, 33, 1]),            # MHA (g = 1)
    (8, 1, 32, 16, [50, 3]),              # MQA (Hkv = 1)
    (16, 1, 16, 32, [70]),                # g = 16
])
def test_matches_torch_sdpa(oracle_lib, Hq, Hkv, D, bs, ctx):
    c = contiguous_case(ctx, Hq, Hkv, D, bs, seed=11)
    scale = 1.0 / math.sqrt(D)
    out, lse = run_oracle(c, Hkv, scale)
    ref, ref_lse = sdpa_reference(c, Hq, Hkv, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def test_fp8_matches_torch_sdpa_on_dequantised(oracle_lib):
    c = contiguous_case([5, 40, 129], 8, 2, 32, 16, seed=12, kv="e4m3")
    scale = 0.17
    out, lse = run_oracle(c, 2, scale)
    ref, ref_lse = sdpa_reference(c, 8, 2, scale)
    np.testing.assert_allclose(out, ref, rtol=1e-11, atol=1e-13)
    np.testing.assert_allclose(lse, ref_lse, rtol=1e-12, atol=1e-12)


def _brute_force_row(q, kc, vc, table, n, h, bs, scale):
    """Hand-expanded attention for one row: every score, every exponential
    and every weighted sum written as explicit Python loops."""
    D = len(q)
    keys = [[float(kc[table[t // bs]][h][t % bs][d]) for d in range(D)] for t in range(n)]
    vals = [[float(vc[table[t // bs]][h][t % bs][d]) for d in range(D)] for t in range(n)]
    xs = []
    for t in range(n):
        acc = 0.0
        for d in range(D):
            acc += q[d] * keys[t][d]
        xs.append(scale * acc)
    m = max(xs)
    ws = [math.exp(x - m) for x in xs]
    z = sum(ws)
    out = [sum(ws[t] * vals[t][d] for t in range(n)) / z for d in range(D)]
    return out, m + math.log(z)


def test_brute_force_tiny(oracle_lib):
    rng = np.random.default_rng(21)
    D, bs, Hkv, Hq = 4, 2, 2, 4
    ctx = np.array([1, 2, 3, 4, 5], np.int32)
    w = make_case(ctx, Hq, Hkv, D, bs, "bf16", seed=21, pool=20, scale=0.7)
    out, lse = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                   Hkv, w.scale)
    kf = bf16_bits_to_f32(w.k_cache).reshape(w.k_cache.shape)
    vf = bf16_bits_to_f32(w.v_cache).reshape(w.v_cache.shape)
    qf = bf16_bits_to_f32(w.q).reshape(w.q.shape)
    for s in range(len(ctx)):
        for i in range(Hq):
            ref, rl = _brute_force_row([float(x) for x in qf[s, i]], kf, vf, w.block_table[s],
                                       int(ctx[s]), i // (Hq // Hkv), bs, 0.7)
            np.testing.assert_allclose(out[s, i], ref, rtol=1e-13, atol=1e-15)
            assert abs(lse[s, i] - rl) < 1e-13
    del rng


# --------------------------------------------------------------------------- #
# invariants the pages state                                                  #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("tile,part", [(1, 1), (16, 16), (7, 13), (64, 64), (16, 10 ** 6),
                                       (5, 50), (1000, 3)])
def test_tiled_online_softmax_is_exact(oracle_lib, tile, part):
    """Online softmax over K tiles equals the full-row softmax ("attention
    kernels", section FlashAttention); splitting along the KV length and
    merging the splits changes nothing (section "prefill and decode")."""
    w = make_case([1, 17, 64, 200, 333], 8, 2, 32, 16, "bf16", seed=31, scale=0.2)
    w2 = make_case([45, 3], 32, 2, 16, 32, "bf16", seed=32, key_boost_frac=0.1, scale=1.0)
    for ww in (w, w2):
        a, la = oracle.paged_decode(ww.q, ww.k_cache, ww.v_cache, ww.block_table,
                                    ww.context_lens, ww.num_kv_heads, ww.scale)
        b, lb = oracle.paged_decode_tiled(ww.q, ww.k_cache, ww.v_cache, ww.block_table,
                                          ww.context_lens, ww.num_kv_heads, ww.scale, tile, part)
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lb, la, rtol=1e-13, atol=1e-13)


def test_split_count_invariance_fp8(oracle_lib):
    w = make_case([300, 17, 1000], 16, 2, 64, 16, "e4m3", seed=33)
    a, la = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                2, w.scale, w.k_scale, w.v_scale)
    for part in (16, 48, 333, 1000):
        b, lb = oracle.paged_decode_tiled(w.q, w.k_cache, w.v_cache, w.block_table,
                                          w.context_lens, 2, w.scale, 16, part,
                                          w.k_scale, w.v_scale)
        np.testing.assert_allclose(b, a, rtol=1e-12, atol=1e-14)
        np.testing.assert_allclose(lb, la, rtol=1e-13, atol=1e-13)


def test_block_permutation_invariance(oracle_lib):
    """Blocks are reached through the table, never by position ("batching and
    attention" section 3.4): permuting the physical pool and rewriting the
    table leaves every output bit unchanged."""
    w = make_case([1, 17, 64, 200], 8, 2, 32, 16, "bf16", seed=41)
    a, la = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                2, w.scale)
    rng = np.random.default_rng(42)
    perm = rng.permutation(w.num_blocks)          # new position of old block b
    k2 = np.empty_like(w.k_cache); v2 = np.empty_like(w.v_cache)
    k2[perm] = w.k_cache; v2[perm] = w.v_cache
    t2 = perm[w.block_table].astype(np.int32)
    b, lb = oracle.paged_decode(w.q, k2, v2, t2, w.context_lens, 2, w.scale)
    assert np.array_equal(a, b) and np.array_equal(la, lb)


def test_gqa_group_shares_kv_head(oracle_lib):
    """Query heads of one group read the same KV head ("batching and
    attention" 2.4): equal query rows inside a group give equal outputs, and
    equal query rows in different groups (different KV heads) do not."""
    w = make_case([50, 9], 8, 2, 32, 16, "bf16", seed=51)
    q = w.q.copy()
    q[:, 1] = q[:, 0]; q[:, 3] = q[:, 0]; q[:, 4] = q[:, 0]
    out, lse = oracle.paged_decode(q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                   2, w.scale)
    assert np.array_equal(out[:, 1], out[:, 0]) and np.array_equal(out[:, 3], out[:, 0])
    assert not np.allclose(out[:, 4], out[:, 0])


def test_merge_partials_closed_forms(oracle_lib):
    o = np.array([[[1.0, 2.0]], [[3.0, -2.0]], [[5.0, 5.0]]])
    lse = np.array([[0.5], [0.5], [-np.inf]])
    out, l = oracle.merge_partials(o, lse)
    np.testing.assert_allclose(out[0], [2.0, 0.0], rtol=0, atol=1e-15)
    assert abs(l[0] - (0.5 + math.log(2.0))) < 1e-15
    out, l = oracle.merge_partials(o[2:], lse[2:])
    assert np.all(out == 0) and np.isneginf(l[0])
    # weights follow exp(lse): lse differing by ln 3 gives weights 3:1
    out, l = oracle.merge_partials(o[:2], np.array([[math.log(3.0)], [0.0]]))
    np.testing.assert_allclose(out[0], [1.5, 1.0], rtol=1e-15, atol=1e-15)


def test_rows_api_matches_full(oracle_lib):
    w = make_case([30, 70, 5], 8, 2, 32, 16, "bf16", seed=61)
    a, la = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                2, w.scale)
    rs = np.array([2, 0, 1, 1], np.int32); rh = np.array([7, 0, 3, 4], np.int32)
    b, lb = oracle.paged_decode_rows(w.q, w.k_cache, w.v_cache, w.block_table,
                                     w.context_lens, 2, w.scale, rs, rh)
    assert np.array_equal(b, a[rs, rh]) and np.array_equal(lb, la[rs, rh])


# --------------------------------------------------------------------------- #
# kv_append                                                                   #
# --------------------------------------------------------------------------- #
@pytest.mark.parametrize("dtype", [np.uint16, np.uint8])
def test_kv_append_is_a_byte_copy(oracle_lib, dtype):
    rng = np.random.default_rng(71)
    nb, Hkv, bs, D, N = 6, 3, 4, 8, 9
    kc = rng.integers(0, 255, size=(nb, Hkv, bs, D)).astype(dtype)
    vc = rng.integers(0, 255, size=(nb, Hkv, bs, D)).astype(dtype)
    kn = rng.integers(0, 255, size=(N, Hkv, D)).astype(dtype)
    vn = rng.integers(0, 255, size=(N, Hkv, D)).astype(dtype)
    slots = rng.choice(nb * bs, size=N, replace=False).astype(np.int64)
    slots[3] = -1
    k2, v2 = oracle.kv_append(kn, vn, slots, kc, vc, bs)
    ek, ev = kc.copy(), vc.copy()
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        ek[sl // bs, :, sl % bs, :] = kn[t]
        ev[sl // bs, :, sl % bs, :] = vn[t]
    assert np.array_equal(k2, ek) and np.array_equal(v2, ev)
    with pytest.raises(oracle.OracleError):
        oracle.kv_append(kn, vn, np.array([nb * bs] * N, np.int64), kc, vc, bs)
