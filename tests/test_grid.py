"""The automatic grid of the decode entry points (pgd_decode_grid, host only,
no GPU needed): one wave of resident CTAs, fewer for small batches, and a
whole number of pieces per (sequence, KV head) unit when there are fewer
units than CTAs."""
import numpy as np
import pytest

import paged_gqa_decode_07_b200 as pgd

B200 = 148   # SMs


def grid(num_seqs, hkv, d, bs, max_ctx, fp8=False, occ=None, sms=B200, max_blocks=None):
    occ = occ if occ is not None else (2 if d == 128 else 1)
    mb = max_blocks if max_blocks is not None else max(1, -(-max_ctx // bs))
    return pgd.decode_grid(sms, occ, num_seqs, hkv, d, bs, mb, max_ctx, fp8)


@pytest.mark.parametrize("case,expected", [
    # the workloads the bench times
    (dict(num_seqs=4, hkv=2, d=128, bs=16, max_ctx=200), 8),            # tiny: one unit per CTA
    (dict(num_seqs=64, hkv=8, d=128, bs=16, max_ctx=4096), 296),        # llama3-shaped: full wave
    (dict(num_seqs=4, hkv=8, d=128, bs=64, max_ctx=131072), 288),       # long context: 9 per unit
    (dict(num_seqs=32, hkv=2, d=256, bs=32, max_ctx=32768), 148),       # wide heads: 148 % 64 > 1/8
    (dict(num_seqs=256, hkv=8, d=128, bs=16, max_ctx=65536, fp8=True), 296),   # FP8 mixed
    # small batches measured with forced grids
    (dict(num_seqs=1, hkv=8, d=128, bs=16, max_ctx=4096), 128),
    (dict(num_seqs=8, hkv=8, d=128, bs=16, max_ctx=1024), 256),
    (dict(num_seqs=2, hkv=8, d=128, bs=16, max_ctx=256), 16),
    (dict(num_seqs=16, hkv=8, d=128, bs=16, max_ctx=256), 128),
    (dict(num_seqs=11, hkv=8, d=128, bs=16, max_ctx=2048), 264),
    # many one-block units: the unit cost fills the wave
    (dict(num_seqs=256, hkv=8, d=128, bs=16, max_ctx=16, fp8=True), 296),
])
def test_workload_grids(case, expected):
    assert grid(**case) == expected


def test_rule_properties():
    """Random shapes: never above one wave, never below one CTA; with fewer
    units than CTAs the grid is the wave itself or a whole number of pieces
    per unit, and a multiple taken from a full wave loses at most 1/8."""
    rng = np.random.default_rng(7)
    for _ in range(3000):
        d = int(rng.choice([128, 256]))
        bs = int(rng.choice([16, 32, 64]))
        fp8 = bool(rng.integers(2)) and d == 128
        occ = int(rng.integers(1, 4))
        sms = int(rng.integers(1, 200))
        b, hkv = int(rng.integers(1, 300)), int(rng.integers(1, 17))
        max_ctx = int(rng.integers(1, 200000))
        g = grid(b, hkv, d, bs, max_ctx, fp8=fp8, occ=occ, sms=sms)
        wave, units = sms * occ, b * hkv
        assert 1 <= g <= wave
        if units < g:
            assert g == wave or g % units == 0
        # a long batch has a full wave's worth of work: the wave or its
        # largest multiple of the units within 1/8
        if max_ctx >= 4 * 64 * wave and units < wave:
            assert g == wave or (g % units == 0 and wave - g <= wave // 8)


@pytest.mark.parametrize("bad", [
    dict(sms=0), dict(occ=0), dict(num_seqs=-1), dict(hkv=0), dict(d=64), dict(bs=8),
    dict(max_blocks=0), dict(max_ctx=-5),
])
def test_invalid_arguments(bad):
    args = dict(num_seqs=4, hkv=2, d=128, bs=16, max_ctx=200)
    kw = {}
    for k, v in bad.items():
        if k in ("sms", "occ", "max_blocks"):
            kw[k] = v
        else:
            args[k] = v
    with pytest.raises(ValueError):
        grid(**args, **kw)
    lib = pgd.load_library()
    assert lib.pgd_decode_grid(148, 2, 4, 2, 128, 16, 13, 200, 2) == 0   # fp8 must be 0 or 1
