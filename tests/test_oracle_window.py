"""Pins for the oracle's sliding-window decode: the query at position n-1
sees only the last W tokens (sliding-window attention, named on the
co-design page (principle 3) and "batching and attention" 2.3 as a way to cut
the KV state a step reads)."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle import contiguous_case, dec
from workloads import make_case, bf16_bits_to_f32


def test_window_covering_context_is_the_full_decode(oracle_lib):
    w = make_case([1, 17, 64, 200], 8, 2, 32, 16, "bf16", seed=401)
    full, lf = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens, 2,
                                   w.scale)
    for W in (0, 200, 10 ** 6):
        a, la = oracle.paged_decode_window(w.q, w.k_cache, w.v_cache, w.block_table,
                                           w.context_lens, 2, w.scale, W)
        assert np.array_equal(a, full) and np.array_equal(la, lf)


def test_window_of_one_returns_last_value(oracle_lib):
    w = make_case([1, 17, 64, 200], 8, 2, 32, 16, "bf16", seed=402)
    a, la = oracle.paged_decode_window(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                       2, w.scale, 1)
    vf = bf16_bits_to_f32(w.v_cache).reshape(w.v_cache.shape)
    for s, n in enumerate(w.context_lens):
        t = n - 1
        for i in range(8):
            v_last = vf[w.block_table[s, t // 16], i // 4, t % 16].astype(np.float64)
            assert np.array_equal(a[s, i], v_last)


@pytest.mark.parametrize("W", [3, 16, 17, 50, 129])
def test_window_matches_sdpa_on_last_tokens(oracle_lib, W):
    c = contiguous_case([1, 17, 64, 200, 300], 8, 2, 64, 16, seed=403)
    scale = 1 / math.sqrt(64)
    out, lse = oracle.paged_decode_window(c["q"], c["k_cache"], c["v_cache"], c["table"],
                                          c["ctx"], 2, scale, W)
    q = dec(c["q"])
    for s, n in enumerate(c["ctx"]):
        lo = max(0, n - W)
        k = dec(c["kseq"][s, lo:n]).permute(1, 0, 2).repeat_interleave(4, dim=0)
        v = dec(c["vseq"][s, lo:n]).permute(1, 0, 2).repeat_interleave(4, dim=0)
        ref = torch.nn.functional.scaled_dot_product_attention(q[s][:, None, :], k, v,
                                                               scale=scale)[:, 0]
        rl = torch.logsumexp(torch.matmul(q[s][:, None, :], k.transpose(1, 2)) * scale, -1)[:, 0]
        np.testing.assert_allclose(out[s], ref.numpy(), rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(lse[s], rl.numpy(), rtol=1e-12, atol=1e-12)


def test_window_brute_force_tiny(oracle_lib):
    w = make_case([1, 2, 3, 4, 5, 9], 4, 2, 4, 2, "bf16", seed=404, pool=20, scale=0.7)
    W = 3
    out, lse = oracle.paged_decode_window(w.q, w.k_cache, w.v_cache, w.block_table,
                                          w.context_lens, 2, w.scale, W)
    kf = bf16_bits_to_f32(w.k_cache).reshape(w.k_cache.shape)
    vf = bf16_bits_to_f32(w.v_cache).reshape(w.v_cache.shape)
    qf = bf16_bits_to_f32(w.q).reshape(w.q.shape)
    for s, n in enumerate(w.context_lens):
        lo = max(0, int(n) - W)
        for i in range(4):
            h = i // 2
            ks = [[float(kf[w.block_table[s][t // 2]][h][t % 2][d]) for d in range(4)]
                  for t in range(lo, n)]
            vs = [[float(vf[w.block_table[s][t // 2]][h][t % 2][d]) for d in range(4)]
                  for t in range(lo, n)]
            xs = [0.7 * sum(float(qf[s, i, d]) * kk[d] for d in range(4)) for kk in ks]
            m = max(xs)
            ws = [math.exp(x - m) for x in xs]
            z = sum(ws)
            ref = [sum(ws[j] * vs[j][d] for j in range(len(ws))) / z for d in range(4)]
            np.testing.assert_allclose(out[s, i], ref, rtol=1e-13, atol=1e-15)
            assert abs(lse[s, i] - (m + math.log(z))) < 1e-13
