"""Pins for the oracle's E4M3 quantiser and the quantising KV append.

The format (OCP FP8 E4M3, "fn": bias 7, subnormals m * 2^-9, S.1111.111 NaN,
largest finite 448) fixes every code; rounding is to nearest with ties to the
even mantissa, and magnitudes past 448 saturate (the quantiser's reading).
The quantising append divides by the per-KV-head scale in fp32 first."""

import numpy as np
import pytest
import torch

import oracle
from workloads import to_bf16_bits, bf16_bits_to_f32


def finite_codes():
    b = np.arange(256, dtype=np.uint16).astype(np.uint8)
    v = oracle.e4m3_to_double(b)
    keep = ~np.isnan(v)
    return b[keep], v[keep]


def test_every_finite_code_round_trips(oracle_lib):
    b, v = finite_codes()
    assert np.array_equal(oracle.e4m3_from_double(v), b)


def test_midpoints_round_to_even_mantissa(oracle_lib):
    b, v = finite_codes()
    pos = np.argsort(v)
    vals, codes = v[pos], b[pos]
    keep = vals >= 0
    vals, codes = vals[keep], codes[keep]
    vals, idx = np.unique(vals, return_index=True)   # +0 and -0
    codes = codes[idx]
    for i in range(len(vals) - 1):
        mid = (vals[i] + vals[i + 1]) / 2
        got = oracle.e4m3_from_double(np.array([mid]))[0]
        even = codes[i] if codes[i] % 2 == 0 else codes[i + 1]
        assert got == even, (vals[i], vals[i + 1], got)
        # just off the midpoint goes to the nearer value
        up = oracle.e4m3_from_double(np.array([np.nextafter(mid, np.inf)]))[0]
        dn = oracle.e4m3_from_double(np.array([np.nextafter(mid, -np.inf)]))[0]
        assert up == codes[i + 1] and dn == codes[i]


def test_saturation_and_special_values(oracle_lib):
    x = np.array([448.0, 449.0, 463.9, 464.0, 1e9, -500.0, np.inf, -np.inf, np.nan, 0.0, -0.0,
                  2.0 ** -10, 2.0 ** -9 * 1.5, 2.0 ** -9 * 2.5])
    got = oracle.e4m3_from_double(x)
    assert list(got[:8]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0x7E, 0xFE]
    assert got[8] == 0x7F and got[9] == 0x00 and got[10] == 0x80
    # 2^-10 is halfway between 0 and 2^-9: ties to even -> 0
    assert got[11] == 0x00
    # 1.5 * 2^-9 -> 2 * 2^-9 (even); 2.5 * 2^-9 -> 2 * 2^-9 (even)
    assert got[12] == 0x02 and got[13] == 0x02


def test_matches_torch_cast_in_range(oracle_lib):
    rng = np.random.default_rng(3)
    x = np.concatenate([rng.standard_normal(20000) * 50,
                        rng.uniform(-448, 448, 20000),
                        rng.standard_normal(20000) * 1e-2]).astype(np.float32)
    ref = torch.from_numpy(x).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    got = oracle.e4m3_from_double(x.astype(np.float64))
    assert np.array_equal(got, ref)


def test_kv_append_quant_divides_in_fp32_then_rounds(oracle_lib):
    rng = np.random.default_rng(4)
    N, Hkv, D, bs, nb = 7, 3, 16, 4, 6
    kf = rng.standard_normal((N, Hkv, D)).astype(np.float32) * 3
    vf = rng.standard_normal((N, Hkv, D)).astype(np.float32)
    kb, vb = to_bf16_bits(kf), to_bf16_bits(vf)
    ks = np.array([0.0071, 0.02, 0.5], np.float32)
    vs = np.array([0.003, 1.0, 0.25], np.float32)
    slots = rng.choice(nb * bs, size=N, replace=False).astype(np.int64)
    slots[2] = -1
    kc0 = np.full((nb, Hkv, bs, D), 0x55, np.uint8)
    vc0 = kc0.copy()
    kc, vc = oracle.kv_append_quant(kb, vb, slots, kc0, vc0, ks, vs, bs)
    kx = bf16_bits_to_f32(kb).reshape(kb.shape)
    vx = bf16_bits_to_f32(vb).reshape(vb.shape)
    for t, sl in enumerate(slots):
        if sl < 0:
            continue
        qk = (kx[t] / ks[:, None]).astype(np.float32)      # fp32 division
        qv = (vx[t] / vs[:, None]).astype(np.float32)
        ek = torch.from_numpy(np.clip(qk, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8)
        ev = torch.from_numpy(np.clip(qv, -448, 448)).to(torch.float8_e4m3fn).view(torch.uint8)
        assert np.array_equal(kc[sl // bs, :, sl % bs], ek.numpy())
        assert np.array_equal(vc[sl // bs, :, sl % bs], ev.numpy())
    touched = np.zeros((nb, bs), bool)
    for sl in slots[slots >= 0]:
        touched[sl // bs, sl % bs] = True
    assert np.all(kc.transpose(0, 2, 1, 3)[~touched] == 0x55)
    # power-of-two scale: quantising x / 2^k equals quantising x, decoded * 2^k
    x = np.array([[[1.0, -3.5, 96.0, 0.0078125]]], np.float32)   # all exact after / 0.25
    kc, _ = oracle.kv_append_quant(to_bf16_bits(x), to_bf16_bits(x), np.array([0], np.int64),
                                   np.zeros((1, 1, 1, 4), np.uint8), np.zeros((1, 1, 1, 4), np.uint8),
                                   np.array([0.25], np.float32), np.array([1.0], np.float32), 1)
    assert np.allclose(oracle.e4m3_to_double(kc[0, 0, 0]) * 0.25, x[0, 0])
