"""GPU parity of the CUDA-core decode variant (pgd_set_decode_math
"cuda_core": FMA dot products and warp-shuffle sums instead of mma.sync)
against the oracle, on the shapes it covers: bf16, head_dim 128, up to 8
query rows per KV head."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import Dev, assert_close, dev_bf16, to_f64
from tests.test_gpu_parity import check_case
from workloads import make_case, to_bf16_bits

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda_core():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    pgd.set_decode_math("cuda_core")
    yield
    pgd.set_decode_math("tensor_core")
    assert pgd.get_device_error() == 0


CTX = [1, 15, 16, 17, 63, 64, 65, 200, 1000, 2049, 0, 333]
SHAPES = [(8, 8, 16), (8, 4, 32), (8, 2, 16), (32, 8, 64), (16, 2, 16), (24, 4, 32),
          (8, 1, 64), (5, 1, 16)]


@pytest.mark.parametrize("Hq,Hkv,bs", SHAPES, ids=[f"g{a // b}-bs{c}" for a, b, c in SHAPES])
def test_cuda_core_ragged_batch(Hq, Hkv, bs):
    assert pgd.get_decode_math() == "cuda_core"
    check_case(make_case(CTX, Hq, Hkv, 128, bs, "bf16", seed=2000 + Hq + bs, name="cc-ragged"))


@pytest.mark.parametrize("num_ctas", [1, 7, 296, 1000])
def test_cuda_core_split_count_invariance(num_ctas):
    w = make_case([5000, 17, 640, 1, 0, 2222], 32, 8, 128, 16, "bf16", seed=2100, name="cc-split")
    check_case(w, num_ctas=num_ctas)


def test_cuda_core_multi_token_and_window():
    w = make_case(CTX, 8, 4, 128, 16, "bf16", seed=2200, name="cc-multi")
    rng = np.random.default_rng(2201)
    qm = to_bf16_bits(rng.standard_normal((len(CTX), 4, 8, 128), dtype=np.float32))
    d = Dev(w)
    for W in (0, 37):
        lse = torch.empty((len(CTX), 4, 8), dtype=torch.float32, device="cuda")
        out = pgd.paged_decode_attention_ex(dev_bf16(qm), d.k, d.v, d.bt, d.cl, 8, 4, 128, 16,
                                            w.scale, window=W, max_context_len=w.max_context_len,
                                            lse_out=lse)
        torch.cuda.synchronize()
        ref, rl = oracle.paged_decode_multi(qm, w.k_cache, w.v_cache, w.block_table,
                                            w.context_lens, 4, w.scale, window=W)
        assert_close(to_f64(out), ref, "bf16", f"cuda-core multi W={W}")


def test_cuda_core_close_to_tensor_core_and_reproducible():
    w = make_case(CTX, 32, 8, 128, 16, "bf16", seed=2300, name="cc-vs-tc")
    d = Dev(w)
    a, _ = d.decode()
    b, _ = d.decode()
    pgd.set_decode_math("tensor_core")
    try:
        c, _ = d.decode()
    finally:
        pgd.set_decode_math("cuda_core")
    torch.cuda.synchronize()
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    assert float((a.float() - c.float()).abs().max()) < 2e-2


@pytest.mark.parametrize("kw", [dict(D=256), dict(dt="e4m3"), dict(Hq=32, Hkv=2)])
def test_cuda_core_rejects_shapes_it_does_not_cover(kw):
    D = kw.get("D", 128)
    dt = kw.get("dt", "bf16")
    w = make_case([40, 7], kw.get("Hq", 8), kw.get("Hkv", 2), D, 16, dt, seed=2400, name="cc-no")
    d = Dev(w)
    with pytest.raises(pgd.PGDError) as e:
        d.decode()
    assert e.value.status == 2
