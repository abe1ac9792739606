"""The timeout path of the decode kernels, forced without hanging anything.

Every wait inside a decode launch is bounded.  No correct input makes one run
out, so these tests shorten the limit of the pipeline waits with the test
hook pgd_debug_set_wait_limit_ns (a few ns up to a few µs): the waits give
up, the kernel raises flag 8, its warps leave together, and the producer
still waits (with its own fixed limit) for every copy it issued before the
CTA exits.  Each test then checks that

  * the call returned and the device reports PGD_ERR_TIMEOUT (flag 8) when
    the limit is 1 ns (longer limits may or may not run out);
  * pgd_get_device_error cleared the flags and the arrival counters, so a
    normal call right after gives exactly the bits of a fresh run.

Nothing here waits on a flag that nothing sets for longer than the limit, and
every copy in flight still lands: the GPU stays usable throughout.
"""
import ctypes

import numpy as np
import pytest
import torch

import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, dev_bf16, dev_cache
from workloads import make_case, to_bf16_bits

pytestmark = pytest.mark.gpu

TIMEOUT_FLAG = 8
PGD_ERR_TIMEOUT = 5
LIMITS_NS = [1, 300, 3000]


@pytest.fixture(autouse=True)
def _restore():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    pgd.debug_set_wait_limit_ns(0)
    assert pgd.get_device_error() == 0
    yield
    pgd.debug_set_wait_limit_ns(0)
    pgd.set_decode_math("tensor_core")
    torch.cuda.synchronize()
    pgd.get_device_error()


def _status_and_flags():
    """pgd_get_device_error through the C ABI: (status, flag bits)."""
    lib = pgd.load_library()
    flags = ctypes.c_uint32(0)
    st = lib.pgd_get_device_error(ctypes.c_void_p(torch.cuda.current_stream().cuda_stream),
                                  ctypes.byref(flags))
    return int(st), int(flags.value)


def _bits(t):
    return t.view(torch.int32 if t.dtype == torch.float32 else torch.int16).clone()


def _exercise(run):
    """run() enqueues one decode and returns its output tensors.  The result
    of a normal run, then for each short limit: one run that may time out,
    the device status, and a normal run that must give the first bits."""
    ref = [_bits(t) for t in run()]
    torch.cuda.synchronize()
    assert pgd.get_device_error() == 0
    for limit in LIMITS_NS:
        pgd.debug_set_wait_limit_ns(limit)
        run()
        torch.cuda.synchronize()
        st, flags = _status_and_flags()
        pgd.debug_set_wait_limit_ns(0)
        assert flags & ~TIMEOUT_FLAG == 0, f"limit {limit} ns: unexpected flags {flags}"
        if limit == 1:
            assert flags == TIMEOUT_FLAG and st == PGD_ERR_TIMEOUT, \
                f"a 1 ns limit must run out: status {st}, flags {flags}"
        else:
            assert st == (PGD_ERR_TIMEOUT if flags else 0)
        # flags and counters were cleared: the next call is a fresh run
        got = run()
        torch.cuda.synchronize()
        assert pgd.get_device_error() == 0, f"limit {limit} ns: flags left behind"
        for a, b in zip(ref, got):
            assert torch.equal(a, _bits(b)), f"limit {limit} ns: the next call differs"


# (context lens, Hq, Hkv, D, bs, kv dtype, forced grid) -- several CTAs share
# the long units, so split units, their merges and the arrival counters are
# all on the path that times out
CASES = [
    ([4096, 1, 17, 3000, 0, 900, 2049, 64] * 2, 32, 8, 128, 16, "bf16", 0),
    ([4096, 1, 17, 3000, 0, 900, 2049, 64] * 2, 32, 8, 128, 16, "bf16", 37),
    ([5000, 700, 64, 3000], 32, 2, 256, 32, "bf16", 0),
    ([4000, 64, 900, 17, 1], 64, 8, 128, 16, "e4m3", 0),
    ([8192, 8192], 64, 8, 128, 64, "bf16", 0),
]


@pytest.mark.parametrize("ctx,Hq,Hkv,D,bs,dt,nctas", CASES,
                         ids=[f"g{c[1] // c[2]}-D{c[3]}-bs{c[4]}-{c[5]}-n{c[6]}" for c in CASES])
def test_decode_timeout_then_clean(ctx, Hq, Hkv, D, bs, dt, nctas):
    w = make_case(ctx, Hq, Hkv, D, bs, dt, seed=900 + D + bs)
    d = Dev(w)
    lse = torch.empty((w.num_seqs, Hq), dtype=torch.float32, device="cuda")
    out = torch.empty_like(d.q)

    def run():
        pgd.paged_decode_attention(d.q, d.k, d.v, d.bt, d.cl, Hq, Hkv, D, bs, w.scale, out,
                                   max_context_len=w.max_context_len, k_scale=d.ks,
                                   v_scale=d.vs, lse_out=lse, num_ctas=nctas)
        return out, lse

    _exercise(run)


def test_fused_step_timeout_then_clean():
    """The appender warp's handoff waits time out too; the append is
    idempotent, so the cache ends the same either way."""
    w = make_case([4096, 1, 17, 3000, 900, 2049, 64, 513], 32, 8, 128, 16, "bf16", seed=910,
                  append_last=True)
    d = Dev(w)
    kn = np.zeros((w.num_seqs,) + w.k_new.shape[1:], w.k_new.dtype)
    vn = np.zeros_like(kn)
    kn[:], vn[:] = w.k_new, w.v_new          # every sequence is live here
    kn_d, vn_d = dev_cache(kn), dev_cache(vn)
    out = torch.empty_like(d.q)

    def run():
        pgd.decode_step(d.q, kn_d, vn_d, d.k, d.v, d.bt, d.cl, w.num_q_heads, w.num_kv_heads,
                        w.head_dim, w.block_size, w.scale, out,
                        max_context_len=w.max_context_len)
        return out, d.k, d.v

    _exercise(run)


def test_multi_token_window_timeout_then_clean():
    w = make_case([3000, 40, 1500, 777], 16, 4, 128, 32, "bf16", seed=920)
    d = Dev(w)
    rng = np.random.default_rng(921)
    qm = dev_bf16(to_bf16_bits(rng.standard_normal((w.num_seqs, 4, 16, 128),
                                                   dtype=np.float32)))
    out = torch.empty_like(qm)

    def run():
        pgd.paged_decode_attention_ex(qm, d.k, d.v, d.bt, d.cl, 16, 4, 128, 32, w.scale, out,
                                      window=1000, max_context_len=w.max_context_len)
        return (out,)

    _exercise(run)


def test_cuda_core_variant_timeout_then_clean():
    w = make_case([4096, 1, 17, 3000, 0, 900], 32, 8, 128, 16, "bf16", seed=930)
    d = Dev(w)
    pgd.set_decode_math("cuda_core")
    out = torch.empty_like(d.q)

    def run():
        pgd.paged_decode_attention(d.q, d.k, d.v, d.bt, d.cl, 32, 8, 128, 16, w.scale, out,
                                   max_context_len=w.max_context_len)
        return (out,)

    _exercise(run)
