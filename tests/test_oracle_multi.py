"""Pins for the oracle's multi-token decode: the q_len newest tokens of a
sequence are queried together (speculative-decoding verification in the
inference lecture; long-prefix prefill on the co-design page), each seeing
the tokens up to and including itself, optionally only the last W of them."""
import math

import numpy as np
import pytest
import torch

import oracle
from tests.test_oracle import contiguous_case, dec
from workloads import make_case, to_bf16_bits


def _multi_q(B, L, Hq, D, seed):
    rng = np.random.default_rng(seed)
    return to_bf16_bits(rng.standard_normal((B, L, Hq, D)).astype(np.float32))


def test_single_token_is_the_decode(oracle_lib):
    w = make_case([1, 17, 64, 200], 8, 2, 32, 16, "bf16", seed=501)
    a, la = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens, 2,
                                w.scale)
    b, lb = oracle.paged_decode_multi(w.q[:, None], w.k_cache, w.v_cache, w.block_table,
                                      w.context_lens, 2, w.scale)
    assert np.array_equal(a, b[:, 0]) and np.array_equal(la, lb[:, 0])
    c, lc = oracle.paged_decode_window(w.q, w.k_cache, w.v_cache, w.block_table,
                                       w.context_lens, 2, w.scale, 21)
    d, ld = oracle.paged_decode_multi(w.q[:, None], w.k_cache, w.v_cache, w.block_table,
                                      w.context_lens, 2, w.scale, window=21)
    assert np.array_equal(c, d[:, 0]) and np.array_equal(lc, ld[:, 0])


@pytest.mark.parametrize("L,W", [(2, 0), (4, 0), (3, 5), (8, 17), (4, 1)])
def test_matches_sdpa_with_causal_band_mask(oracle_lib, L, W):
    c = contiguous_case([9, 17, 64, 130], 8, 2, 64, 16, seed=502)
    q = _multi_q(len(c["ctx"]), L, 8, 64, seed=503)
    scale = 1 / math.sqrt(64)
    out, lse = oracle.paged_decode_multi(q, c["k_cache"], c["v_cache"], c["table"], c["ctx"], 2,
                                         scale, window=W)
    qq = dec(q)
    for s, n in enumerate(c["ctx"]):
        k = dec(c["kseq"][s, :n]).permute(1, 0, 2).repeat_interleave(4, dim=0)   # [Hq][n][D]
        v = dec(c["vseq"][s, :n]).permute(1, 0, 2).repeat_interleave(4, dim=0)
        pos = torch.arange(n)
        hi = n - L + 1 + torch.arange(L)                                        # exclusive
        mask = pos[None, :] < hi[:, None]
        if W > 0:
            mask &= pos[None, :] >= (hi[:, None] - W)
        qs = qq[s].permute(1, 0, 2)                                            # [Hq][L][D]
        ref = torch.nn.functional.scaled_dot_product_attention(qs, k, v, attn_mask=mask,
                                                               scale=scale)
        sc = torch.matmul(qs, k.transpose(1, 2)) * scale
        rl = torch.logsumexp(sc.masked_fill(~mask, -math.inf), -1)
        np.testing.assert_allclose(out[s], ref.permute(1, 0, 2).numpy(), rtol=1e-11, atol=1e-13)
        np.testing.assert_allclose(lse[s], rl.permute(1, 0).numpy(), rtol=1e-12, atol=1e-12)


def test_query_token_equals_decode_of_truncated_context(oracle_lib):
    w = make_case([40, 77, 16], 8, 2, 32, 16, "bf16", seed=504)
    L = 5
    q = _multi_q(3, L, 8, 32, seed=505)
    out, lse = oracle.paged_decode_multi(q, w.k_cache, w.v_cache, w.block_table,
                                         w.context_lens, 2, w.scale)
    for i in range(L):
        ctx_i = (w.context_lens - L + 1 + i).astype(np.int32)
        a, la = oracle.paged_decode(q[:, i], w.k_cache, w.v_cache, w.block_table, ctx_i, 2,
                                    w.scale)
        assert np.array_equal(a, out[:, i]) and np.array_equal(la, lse[:, i])


def test_rows_before_the_sequence_start_are_empty(oracle_lib):
    w = make_case([2, 30], 4, 2, 32, 16, "bf16", seed=506)
    q = _multi_q(2, 4, 4, 32, seed=507)
    out, lse = oracle.paged_decode_multi(q, w.k_cache, w.v_cache, w.block_table,
                                         w.context_lens, 2, w.scale)
    # sequence 0 has 2 tokens but 4 query tokens: the first two see nothing
    assert np.all(out[0, :2] == 0) and np.all(np.isneginf(lse[0, :2]))
    assert np.all(np.isfinite(out[0, 2:])) and np.all(np.isfinite(lse[1]))
