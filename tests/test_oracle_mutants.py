"""Plant plausible mistakes in copies of the oracle's C source (CPU only) and
check that the pins in test_oracle.py catch every one of them.  The committed
oracle is never modified; each mutant is compiled to a temporary library."""
import ctypes
import os
import subprocess

import pytest

import oracle
from oracle import oracle as ormod
import tests.test_oracle as pins
import tests.test_oracle_quant as qpins
import tests.test_oracle_window as wpins
import tests.test_oracle_multi as mpins

SRC = os.path.join(os.path.dirname(ormod.__file__), "pgd_oracle.c")

# (name, text in the source, replacement, occurrence to replace: 0 = first)
MUTANTS = [
    ("head map i % Hkv", "const int32_t h = i / g;", "const int32_t h = i % a->num_kv_heads;", 0),
    ("dropped softmax scale", "return scale * acc;", "return acc;", 0),
    ("token offset off by one", "int32_t off = t % a->block_size;",
     "int32_t off = (t + 1) % a->block_size;", 0),
    ("NHD instead of HND address",
     "((int64_t)pb * a->num_kv_heads + h) * a->block_size + off",
     "((int64_t)pb * a->block_size + off) * a->num_kv_heads + h", 0),
    ("lse sign", "*lse = M + log(Z);", "*lse = M - log(Z);", 0),
    ("no max subtraction", "x[t] = exp(x[t] - M);", "x[t] = exp(x[t]);", 0),
    ("missing normalisation", "for (int32_t d = 0; d < D; ++d) out[d] /= Z;", "", 0),
    ("V read from K cache", "gather_row(a, a->v_cache, a->v_scale, s, h, t, row);\n        for",
     "gather_row(a, a->k_cache, a->k_scale, s, h, t, row);\n        for", 0),
    ("e4m3 bias 8", "expo - 7", "expo - 8", 0),
    ("e4m3 subnormal scale", "ldexp((double)man, -9)", "ldexp((double)man, -10)", 0),
    ("bf16 mantissa width", "/ 128.0", "/ 256.0", 0),
    ("fp8 scale ignored", "* sc;", ";", 0),
    ("online rescale of acc dropped", "for (int32_t d = 0; d < D; ++d) acc[d] *= alpha;", "", 0),
    ("online rescale of l dropped", "l *= alpha;", "", 0),
    ("merge weight sign", "double w = exp(l - M);", "double w = exp(M - l);", 0),
    ("append keeps padding", "if (slot < 0) continue;", "if (slot < 0) slot = 0;", 0),
    ("dot product drops last dim", "for (int32_t d = 0; d < D; ++d) acc += qrow[d] * krow[d];",
     "for (int32_t d = 0; d + 1 < D; ++d) acc += qrow[d] * krow[d];", 0),
    ("q row of wrong head", "+ i) * a->head_dim;", "+ i / 2) * a->head_dim;", 0),
    ("e4m3 ties away from zero", "nearbyint((ldexp(a, -E) - 1.0) * 8.0)",
     "round((ldexp(a, -E) - 1.0) * 8.0)", 0),
    ("e4m3 subnormal ties away", "nearbyint(ldexp(a, 9))", "round(ldexp(a, 9))", 0),
    ("e4m3 NaN instead of saturation", "if (a >= 448.0) return (uint8_t)(sign | 0x7E);",
     "if (a >= 448.0) return 0x7F;", 0),
    ("quant K with V scale", "float ky = kx / k_scale[h];", "float ky = kx / v_scale[h];", 0),
    ("window one token short", "? n - a->window : 0;", "? n - a->window + 1 : 0;", 0),
    ("window ignored", "    a.window = window;\n", "", 0),
    ("plain q row of wrong head", "+ i) * a->head_dim, lo, n", "+ i / 2) * a->head_dim, lo, n", 0),
    ("causal limit one short", "context_lens[s] - q_len + 1 + it;", "context_lens[s] - q_len + it;", 0),
    ("multi query token order", "((int64_t)s * q_len + it) * num_q_heads + i;",
     "((int64_t)s * q_len + (q_len - 1 - it)) * num_q_heads + i;", 0),
]

PIN_CALLS = [
    ("bf16 decoder", lambda: pins.test_bf16_decoder_all_patterns(None)),
    ("e4m3 decoder", lambda: pins.test_e4m3_decoder_all_bytes(None)),
    ("worked example", lambda: pins.test_block_table_worked_example(None)),
    ("ctx 1", lambda: pins.test_one_token_context_returns_v0(None)),
    ("identical keys", lambda: pins.test_identical_keys_give_mean_of_v(None)),
    ("zero scale", lambda: pins.test_zero_scale_gives_mean_of_v(None)),
    ("dominant key", lambda: pins.test_dominant_key_selects_its_value(None)),
    ("sdpa g4", lambda: pins.test_matches_torch_sdpa(None, 8, 2, 64, 16, [1, 17, 64, 200])),
    ("sdpa mha", lambda: pins.test_matches_torch_sdpa(None, 4, 4, 32, 8, [9, 33, 1])),
    ("sdpa fp8", lambda: pins.test_fp8_matches_torch_sdpa_on_dequantised(None)),
    ("brute force", lambda: pins.test_brute_force_tiny(None)),
    ("tiled exact", lambda: pins.test_tiled_online_softmax_is_exact(None, 7, 13)),
    ("merge closed forms", lambda: pins.test_merge_partials_closed_forms(None)),
    ("kv append", lambda: pins.test_kv_append_is_a_byte_copy(None, __import__("numpy").uint16)),
    ("e4m3 round trip", lambda: qpins.test_every_finite_code_round_trips(None)),
    ("e4m3 midpoints", lambda: qpins.test_midpoints_round_to_even_mantissa(None)),
    ("e4m3 saturation", lambda: qpins.test_saturation_and_special_values(None)),
    ("quant append", lambda: qpins.test_kv_append_quant_divides_in_fp32_then_rounds(None)),
    ("window of one", lambda: wpins.test_window_of_one_returns_last_value(None)),
    ("window sdpa", lambda: wpins.test_window_matches_sdpa_on_last_tokens(None, 17)),
    ("multi sdpa", lambda: mpins.test_matches_sdpa_with_causal_band_mask(None, 4, 0)),
    ("multi window sdpa", lambda: mpins.test_matches_sdpa_with_causal_band_mask(None, 3, 5)),
]


def _compile(src_text, tmp_path, name):
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"{name}.so"
    c.write_text(src_text)
    subprocess.check_call(["gcc", "-O1", "-std=c99", "-fPIC", "-shared", "-o", str(so),
                           str(c), "-lm"])
    return ormod.configure(ctypes.CDLL(str(so)))


def test_unmutated_copy_passes_every_pin(tmp_path, oracle_lib):
    lib = _compile(open(SRC).read(), tmp_path, "clean")
    old = ormod.set_library(lib)
    try:
        for _, call in PIN_CALLS:
            call()
    finally:
        ormod.set_library(old)


@pytest.mark.parametrize("name,old,new,occ", MUTANTS, ids=[m[0] for m in MUTANTS])
def test_mutant_is_caught(tmp_path, oracle_lib, name, old, new, occ):
    src = open(SRC).read()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    idx = -1
    for _ in range(occ + 1):
        idx = src.index(old, idx + 1)
    mutated = src[:idx] + new + src[idx + len(old):]
    lib = _compile(mutated, tmp_path, "mutant")
    old_lib = ormod.set_library(lib)
    caught = []
    try:
        for pin, call in PIN_CALLS:
            try:
                call()
            except Exception:  # noqa: BLE001 - any failure counts as caught
                caught.append(pin)
    finally:
        ormod.set_library(old_lib)
    assert caught, f"no pin caught the planted mistake '{name}'"
