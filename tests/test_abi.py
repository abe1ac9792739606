"""C ABI checks that need no GPU: the library builds for sm_100a, loads,
exports every entry point include/pgd.h declares, and rejects bad arguments
on the host before any CUDA call."""
import ctypes
import os
import re
import subprocess

import pytest

from paged_gqa_decode_07_b200 import build as pgd_build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "pgd.h")

OK, INVALID, UNSUPPORTED, CUDA, BOUNDS, TIMEOUT, WORKSPACE = range(7)


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return re.findall(r"^\s*(?:pgd_status|pgd_decode_math|size_t|uint64_t|const\s+char\s*\*)"
                      r"\s*\**\s*(\w+)\s*\(",
                      text, flags=re.M)


@pytest.fixture(scope="module")
def lib():
    path = pgd_build.build()
    L = ctypes.CDLL(path)
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    L.pgd_kv_append.argtypes = [P, P, P, i32, P, P, i32, i32, i32, i32, ctypes.c_int, P]
    L.pgd_paged_decode_attention.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                             i32, f32, ctypes.c_int, P, P, P, P, P, sz, i32, P]
    L.pgd_paged_decode_attention_ex.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32,
                                                i32, i32, i32, i32, f32, ctypes.c_int, P, P, P, P,
                                                P, sz, i32, P]
    L.pgd_merge_partials.argtypes = [P, P, i32, i32, i32, P, P, P]
    L.pgd_status_string.restype = ctypes.c_char_p
    L.pgd_version.restype = ctypes.c_char_p
    return L


def test_every_declared_symbol_is_exported(lib):
    names = declared_functions()
    assert {"pgd_kv_append", "pgd_paged_decode_attention", "kv_append",
            "paged_decode_attention", "pgd_merge_partials"} <= set(names)
    out = subprocess.run(["nm", "-D", "--defined-only", pgd_build.LIB], capture_output=True,
                         text=True, check=True).stdout
    exported = {ln.split()[-1] for ln in out.splitlines() if " T " in ln}
    for n in names:
        assert n in exported, n
        assert hasattr(lib, n), n


def test_built_for_sm100a_only():
    # the build step passes exactly one -gencode: compute_100a -> sm_100a
    assert pgd_build.ARCH == ["-gencode", "arch=compute_100a,code=sm_100a"]


def test_status_strings(lib):
    assert lib.pgd_status_string(0) == b"ok"
    assert b"workspace" in lib.pgd_status_string(WORKSPACE)
    assert lib.pgd_version().count(b".") == 2


# fake, never-dereferenced device addresses (all checks below fail on the host)
A = ctypes.c_void_p(0x10000)
MIS = ctypes.c_void_p(0x10002)


def decode(lib, **kw):
    args = dict(q=A, k=A, v=A, bt=A, mbps=8, cl=A, B=2, maxctx=0, Hq=8, Hkv=2, D=128, bs=16,
                nb=16, scale=0.1, dt=0, ks=None, vs=None, out=A, lse=None, ws=None, wsb=0,
                nctas=0)
    args.update(kw)
    a = args
    return lib.pgd_paged_decode_attention(a["q"], a["k"], a["v"], a["bt"], a["mbps"], a["cl"],
                                          a["B"], a["maxctx"], a["Hq"], a["Hkv"], a["D"],
                                          a["bs"], a["nb"], a["scale"], a["dt"], a["ks"],
                                          a["vs"], a["out"], a["lse"], a["ws"], a["wsb"],
                                          a["nctas"], None)


@pytest.mark.parametrize("kw,status", [
    (dict(Hq=6, Hkv=4), INVALID),          # heads not a multiple
    (dict(Hq=34, Hkv=2), UNSUPPORTED),     # group 17
    (dict(Hq=64, Hkv=2), UNSUPPORTED),     # group 32
    (dict(D=64), UNSUPPORTED),
    (dict(bs=8), UNSUPPORTED),
    (dict(dt=1, D=256, ks=A, vs=A), UNSUPPORTED),
    (dict(dt=1), INVALID),                 # FP8 without scales
    (dict(dt=7), INVALID),
    (dict(q=None), INVALID),
    (dict(out=None), INVALID),
    (dict(k=MIS), INVALID),                # TMA needs 16-byte aligned caches
    (dict(q=ctypes.c_void_p(0x10002)), INVALID),
    (dict(B=-1), INVALID),
    (dict(nb=0), INVALID),
    (dict(mbps=0), INVALID),
    (dict(scale=float("nan")), INVALID),
    (dict(ws=None, wsb=64), INVALID),
    (dict(nctas=-3), INVALID),
    (dict(B=0, q=None, k=None), OK),       # empty batch: nothing to do
])
def test_decode_host_validation(lib, kw, status):
    assert decode(lib, **kw) == status


def decode_ex(lib, q_len, window, **kw):
    args = dict(q=A, k=A, v=A, bt=A, mbps=8, cl=A, B=2, maxctx=0, Hq=8, Hkv=2, D=128, bs=16,
                nb=16, scale=0.1, dt=0, ks=None, vs=None, out=A, lse=None, ws=None, wsb=0,
                nctas=0)
    args.update(kw)
    a = args
    return lib.pgd_paged_decode_attention_ex(a["q"], a["k"], a["v"], a["bt"], a["mbps"], a["cl"],
                                             a["B"], a["maxctx"], q_len, window, a["Hq"],
                                             a["Hkv"], a["D"], a["bs"], a["nb"], a["scale"],
                                             a["dt"], a["ks"], a["vs"], a["out"], a["lse"],
                                             a["ws"], a["wsb"], a["nctas"], None)


@pytest.mark.parametrize("q_len,window,kw,status", [
    (0, 0, {}, INVALID),                   # no query token
    (1, -1, {}, INVALID),                  # negative window
    (9, 0, {}, UNSUPPORTED),               # g * q_len = 36 rows > 32
    (3, 0, dict(Hq=16, Hkv=1), UNSUPPORTED),
    (4, 3, dict(out=MIS), INVALID),
    (4, 3, dict(B=0, q=None), OK),
    (8, 0, dict(Hq=4, Hkv=2, B=0), OK),    # 16 rows: accepted
    (8, 0, dict(B=0), OK),                 # 32 rows (g 4, q_len 8): accepted
    (2, 0, dict(Hq=16, Hkv=1, D=256, B=0), OK),   # 32 rows at head_dim 256
])
def test_decode_ex_host_validation(lib, q_len, window, kw, status):
    assert decode_ex(lib, q_len, window, **kw) == status


@pytest.mark.parametrize("kw,status", [
    (dict(n=-1), INVALID), (dict(D=96), UNSUPPORTED), (dict(bs=128), UNSUPPORTED),
    (dict(dt=3), INVALID), (dict(kn=None), INVALID), (dict(kn=MIS), INVALID),
    (dict(n=0, kn=None), OK), (dict(Hkv=65537), UNSUPPORTED), (dict(Hkv=65537, n=0), UNSUPPORTED),
])
def test_kv_append_host_validation(lib, kw, status):
    a = dict(kn=A, vn=A, sl=A, n=4, kc=A, vc=A, Hkv=2, D=128, bs=16, nb=8, dt=0)
    a.update(kw)
    assert lib.pgd_kv_append(a["kn"], a["vn"], a["sl"], a["n"], a["kc"], a["vc"], a["Hkv"],
                             a["D"], a["bs"], a["nb"], a["dt"], None) == status


def test_merge_host_validation(lib):
    assert lib.pgd_merge_partials(A, A, 0, 4, 128, A, None, None) == INVALID
    assert lib.pgd_merge_partials(A, A, 2, 4, 100, A, None, None) == UNSUPPORTED
    assert lib.pgd_merge_partials(A, A, 2, 0, 128, A, None, None) == OK
    # the merge reads float4 columns and writes 8-byte groups
    assert lib.pgd_merge_partials(MIS, A, 2, 4, 128, A, None, None) == INVALID
    assert lib.pgd_merge_partials(A, A, 2, 4, 128, MIS, None, None) == INVALID


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    import paged_gqa_decode_07_b200._binding as b
    monkeypatch.setattr(b, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(b, "_lib", None)
    with pytest.raises(ImportError):
        b.load_library()


def test_partial_decode_needs_lse(lib):
    P, i32, f32, sz = ctypes.c_void_p, ctypes.c_int32, ctypes.c_float, ctypes.c_size_t
    lib.pgd_paged_decode_partial.argtypes = [P, P, P, P, i32, P, i32, i32, i32, i32, i32, i32,
                                             i32, f32, ctypes.c_int, P, P, P, P, P, sz, i32, P]
    args = [A, A, A, A, 8, A, 2, 0, 8, 2, 128, 16, 16, 0.1, 0, None, None]
    assert lib.pgd_paged_decode_partial(*args, A, None, None, 0, 0, None) == INVALID
    assert lib.pgd_paged_decode_partial(*args, MIS, A, None, 0, 0, None) == INVALID
    args[6] = 0   # empty batch
    assert lib.pgd_paged_decode_partial(*args, None, None, None, 0, 0, None) == OK


def test_decode_math_setting_is_host_only(lib):
    lib.pgd_set_decode_math.argtypes = [ctypes.c_int]
    lib.pgd_get_decode_math.restype = ctypes.c_int
    assert lib.pgd_get_decode_math() == 0
    assert lib.pgd_set_decode_math(1) == OK and lib.pgd_get_decode_math() == 1
    assert lib.pgd_set_decode_math(7) == INVALID and lib.pgd_get_decode_math() == 1
    assert lib.pgd_set_decode_math(0) == OK and lib.pgd_get_decode_math() == 0


def test_wait_limit_hook_is_host_only(lib):
    lib.pgd_debug_set_wait_limit_ns.argtypes = [ctypes.c_uint64]
    lib.pgd_debug_get_wait_limit_ns.restype = ctypes.c_uint64
    assert lib.pgd_debug_get_wait_limit_ns() == 1_000_000_000
    assert lib.pgd_debug_set_wait_limit_ns(5) == OK and lib.pgd_debug_get_wait_limit_ns() == 5
    # 0 restores the default
    assert lib.pgd_debug_set_wait_limit_ns(0) == OK
    assert lib.pgd_debug_get_wait_limit_ns() == 1_000_000_000
