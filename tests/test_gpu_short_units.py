"""GPU parity on batches made mostly of short (sequence, KV head) units:
many units that lie whole in one CTA's range and fit in one 64-token stage,
next to a few long ones (the continuous-batching mix of the "attention
kernels" page, section "paged KV and kernels": short and long sequences in
one launch).  The batches are compared with the oracle row by row in every
output form: bf16 out and lse, the fp32 split result of
pgd_paged_decode_partial, several query tokens, a window, the fused append,
and both KV formats; the short units' results must also be identical across
repeated runs and grids of every size."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, assert_close, dev_bf16, dev_cache, host_bits, to_f64
from tests.test_gpu_parity import check_case
from workloads import make_case, to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    yield
    assert pgd.get_device_error() == 0


def short_mix(n, seed, longest=64, long_ones=(3000,)):
    """n sequences of 1..longest tokens and a few long ones among them."""
    rng = np.random.default_rng(seed)
    ctx = rng.integers(1, longest + 1, size=n)
    ctx[rng.choice(n, size=min(5, n), replace=False)] = 0
    for i, L in enumerate(long_ones):
        ctx[(i * 97) % n] = L
    return ctx.astype(np.int32)


SHAPES = [  # (Hq, Hkv, bs, dtype)
    (64, 8, 16, "e4m3"), (64, 8, 16, "bf16"), (32, 8, 16, "bf16"), (32, 8, 32, "e4m3"),
    (8, 8, 64, "bf16"), (12, 4, 16, "bf16"), (8, 1, 32, "e4m3"), (16, 2, 64, "e4m3"),
]


@pytest.mark.parametrize("Hq,Hkv,bs,dt", SHAPES,
                         ids=[f"g{a // b}-bs{c}-{d}" for a, b, c, d in SHAPES])
def test_many_short_units(Hq, Hkv, bs, dt):
    w = make_case(short_mix(300, 1100 + Hq + bs), Hq, Hkv, 128, bs, dt,
                  seed=1101 + Hq + bs, name=f"short-{dt}")
    check_case(w)


@pytest.mark.parametrize("num_ctas", [1, 5, 64, 296, 1000])
def test_short_units_any_grid(num_ctas):
    """The cut decides which units are whole in a CTA and which are split
    (pieces merged by log-sum-exp): every grid must give the oracle's
    result."""
    w = make_case(short_mix(200, 1110, longest=80, long_ones=(5000, 700)), 64, 8, 128, 16,
                  "e4m3", seed=1111, name="short-grid")
    check_case(w, num_ctas=num_ctas)


def test_short_units_repeat_bits():
    w = make_case(short_mix(256, 1120), 64, 8, 128, 16, "e4m3", seed=1121, name="short-bits")
    d = Dev(w)
    outs = [d.decode()[0].clone() for _ in range(3)]
    for o in outs[1:]:
        assert torch.equal(o.view(torch.int16), outs[0].view(torch.int16))


@pytest.mark.parametrize("dt", ["bf16", "e4m3"])
@pytest.mark.parametrize("L,W", [(2, 0), (2, 20), (1, 9)])
def test_short_units_multi_token_and_window(L, W, dt):
    """Several query tokens and a window on short units, both KV formats."""
    w = make_case(short_mix(150, 1130 + L + W), 16, 4, 128, 16, dt, seed=1131 + L,
                  name="short-multi")
    rng = np.random.default_rng(1132)
    qm = to_bf16_bits(rng.standard_normal((w.num_seqs, L, 16, 128), dtype=np.float32))
    d = Dev(w)
    lse = torch.empty((w.num_seqs, L, 16), dtype=torch.float32, device="cuda")
    out = pgd.paged_decode_attention_ex(dev_bf16(qm), d.k, d.v, d.bt, d.cl, 16, 4, 128, 16,
                                        w.scale, window=W, max_context_len=w.max_context_len,
                                        k_scale=d.ks, v_scale=d.vs, lse_out=lse)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.paged_decode_multi(qm, w.k_cache, w.v_cache, w.block_table,
                                             w.context_lens, w.num_kv_heads, w.scale, window=W,
                                             k_scale=w.k_scale, v_scale=w.v_scale)
    got = to_f64(out)
    assert np.all(np.isfinite(got))
    assert_close(got, ref, dt, f"short multi L={L} W={W}")
    gl = lse.cpu().numpy().astype(np.float64)
    live = np.isfinite(ref_lse)
    assert np.all(np.isneginf(gl[~live]))
    assert np.max(np.abs(gl[live] - ref_lse[live])) <= 1e-3


@pytest.mark.parametrize("num_ctas", [1, 3, 37, 296, 2000])
def test_short_unit_runs_next_to_split_ones(num_ctas):
    """Runs of one-stage units between units that CTA ranges split, at grids
    that cut the runs at every offset; the units of 1, 16, 17, 63 and 64
    tokens cover a stage's partial and full 16-token sub-tiles."""
    ctx = np.array([1, 16, 17, 63, 64, 2000, 5, 64, 33, 700, 48, 2, 64, 64, 0, 9, 3000, 31]
                   * 6, np.int32)
    w = make_case(ctx, 64, 8, 128, 16, "e4m3", seed=1160, name="short-runs")
    check_case(w, num_ctas=num_ctas)


@pytest.mark.parametrize("dt", ["bf16", "e4m3"])
def test_short_units_fp32_split_result(dt):
    """pgd_paged_decode_partial writes the unrounded fp32 result of every
    short unit."""
    w = make_case(short_mix(120, 1140), 32, 8, 128, 16, dt, seed=1141, name="short-f32")
    d = Dev(w)
    o, lse = pgd.paged_decode_partial(d.q, d.k, d.v, d.bt, d.cl, 32, 8, 128, 16, w.scale,
                                      max_context_len=w.max_context_len, k_scale=d.ks,
                                      v_scale=d.vs)
    torch.cuda.synchronize()
    ref, ref_lse = oracle.paged_decode(w.q, w.k_cache, w.v_cache, w.block_table, w.context_lens,
                                       w.num_kv_heads, w.scale, w.k_scale, w.v_scale)
    tol = {"bf16": (2e-4, 2e-3), "e4m3": (2e-2, 5e-2)}[dt]
    got = o.cpu().numpy().astype(np.float64)
    err = np.abs(got - ref)
    assert np.all(err <= tol[0] + tol[1] * np.abs(ref)), float(err.max())
    gl = lse.cpu().numpy().astype(np.float64)
    live = np.isfinite(ref_lse)
    assert np.all(np.isneginf(gl[~live]))
    assert np.max(np.abs(gl[live] - ref_lse[live])) <= 1e-3


def test_short_units_fused_append():
    w = make_case(short_mix(200, 1150, long_ones=(1500,)), 64, 8, 128, 16, "e4m3", seed=1151,
                  append_last=True, name="short-step")
    live = [s for s in range(w.num_seqs) if w.context_lens[s] > 0]
    kn = np.zeros((w.num_seqs,) + w.k_new.shape[1:], w.k_new.dtype)
    vn = np.zeros_like(kn)
    kn[live], vn[live] = w.k_new, w.v_new
    d1 = Dev(w)
    out1 = pgd.decode_step(d1.q, dev_cache(kn), dev_cache(vn), d1.k, d1.v, d1.bt, d1.cl, 64, 8,
                           128, 16, w.scale, max_context_len=w.max_context_len, k_scale=d1.ks,
                           v_scale=d1.vs)
    d2 = Dev(w)
    d2.append()
    out2, _ = d2.decode()
    torch.cuda.synchronize()
    assert torch.equal(out1.view(torch.int16), out2.view(torch.int16))
    assert np.array_equal(host_bits(d1.k), host_bits(d2.k))
    kc, vc = oracle.kv_append(w.k_new, w.v_new, w.slot_mapping, w.k_cache, w.v_cache, 16)
    ref, _ = oracle.paged_decode(w.q, kc, vc, w.block_table, w.context_lens, 8, w.scale,
                                 w.k_scale, w.v_scale)
    assert_close(to_f64(out1), ref, "e4m3", "short fused step")
