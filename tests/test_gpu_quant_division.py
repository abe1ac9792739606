"""The quantising append's per-element division, bit for bit against the
oracle (the IEEE single-precision quotient x / s, then its E4M3 code): every
bf16 value (NaN payloads aside) divided by scales that put quotients on and
within a few ulps of E4M3 rounding midpoints, at and past the ends of the
range where the kernel's reciprocal-and-correction path gives way to IEEE
division, and at random."""
import numpy as np
import pytest
import torch

import oracle
import paged_gqa_decode_07_b200 as pgd
from tests.gpu_helpers import dev_bf16

pytestmark = pytest.mark.gpu

HKV, D, BS = 16, 128, 16


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    pgd.load_library()
    yield
    assert pgd.get_device_error() == 0


def all_bf16_but_nan():
    b = np.arange(65536, dtype=np.uint32).astype(np.uint16)
    exp, man = (b >> 7) & 0xFF, b & 0x7F
    return b[~((exp == 0xFF) & (man != 0))]


def near_midpoint(m):
    """Scales s with 1 / s = m (1 + j 2^-24), j = -8 .. 7: quotients of 1.0
    (and of its powers of two) on and around the E4M3 midpoint m."""
    j = np.arange(-8, 8, dtype=np.float64)
    return (1.0 / (m * (1.0 + j * 2.0 ** -24))).astype(np.float32)


SCALE_SETS = {
    "random": (2.0 ** np.random.default_rng(1234).uniform(-30, 30, HKV)).astype(np.float32),
    # midpoints between E4M3 codes: 1 | 1.125, 1.125 | 1.25, 3 | 3.5, and the
    # subnormal pair 1 * 2^-9 | 2 * 2^-9
    "mid_1.0625": near_midpoint(1.0625),
    "mid_1.1875": near_midpoint(1.1875),
    "mid_3.25": near_midpoint(3.25),
    "mid_sub": near_midpoint(1.5 * 2.0 ** -9),
    # powers of two, the ends of the fast path's scale range (2^-125, 2^125)
    # and past them, a subnormal and a huge scale, everyday scales
    "edges": np.array([1.0, 2.0, 0.5, 2.0 ** -125, 2.0 ** 125, 2.0 ** -126, 2.0 ** 126, 1e-40,
                       3e38, 1.5 * 2.0 ** -124, 448 / 3.0, 0.0071, 1 / 448, 7.0, 1e-20, 1e20],
                      np.float32),
    # scales at and near the ends of the fast path's range [2^-40, 2^40], whose
    # quotients of the largest and smallest fast-path values (2^+-60) reach
    # 2^+-100
    "fast_edges": np.array([2.0 ** 40, 2.0 ** -40, 2.0 ** 40 * (1 - 2.0 ** -24),
                            2.0 ** -40 * (1 + 2.0 ** -23), 1.37 * 2.0 ** 39, 1.9 * 2.0 ** -39,
                            1e12, 1e-12, 3.0, 5.0, 0.3, 0.7, 1.1e-7, 9.9e6, 2.0 ** 20 + 1,
                            3 * 2.0 ** -20], np.float32),
}


@pytest.mark.parametrize("name", list(SCALE_SETS))
def test_every_bf16_value_against_ieee_division(name):
    vals = all_bf16_but_nan()
    n_tok = -(-vals.size // D)
    flat = np.zeros(n_tok * D, np.uint16)
    flat[:vals.size] = vals
    rows = flat.reshape(n_tok, 1, D)
    kb = np.ascontiguousarray(np.broadcast_to(rows, (n_tok, HKV, D)))
    vb = np.ascontiguousarray(kb[::-1])              # other token order for V
    ks = SCALE_SETS[name]
    vs = np.ascontiguousarray(ks[::-1])
    nb = -(-n_tok // BS)
    slots = np.arange(n_tok, dtype=np.int64)
    kc0 = np.zeros((nb, HKV, BS, D), np.uint8)
    vc0 = np.zeros_like(kc0)
    ek, ev = oracle.kv_append_quant(kb, vb, slots, kc0, vc0, ks, vs, BS)
    kc = torch.from_numpy(kc0.copy()).cuda()
    vc = torch.from_numpy(vc0.copy()).cuda()
    pgd.kv_append_quant(dev_bf16(kb), dev_bf16(vb), torch.from_numpy(slots).cuda(), kc, vc,
                        torch.from_numpy(ks).cuda(), torch.from_numpy(vs).cuda())
    torch.cuda.synchronize()
    gk, gv = kc.cpu().numpy(), vc.cpu().numpy()
    bad = int((gk != ek).sum() + (gv != ev).sum())
    assert bad == 0, f"{bad} codes differ from the IEEE quotient's"
