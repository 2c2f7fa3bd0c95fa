"""C-ABI checks that need no GPU: the library loads, exports what include/art.h
declares, and rejects bad arguments with the documented status before making
any CUDA call (descriptors here point at never-dereferenced fake addresses)."""
import ctypes
import os
import re
import subprocess

import pytest

from kv_cache_early_art_b200 import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "art.h")


@pytest.fixture(scope="module")
def art():
    build.build_library()
    import kv_cache_early_art_b200 as pkg
    return pkg


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(art_[a-z_]+)\s*\(", src)))


def test_header_declares_the_boundary():
    names = declared_functions()
    for n in ("art_decode_attention", "art_decode_attention_ex", "art_build_order_sink_recency",
              "art_strerror", "art_version"):
        assert n in names


def test_library_exports_every_declared_symbol(art):
    out = subprocess.run(["nm", "-D", "--defined-only", art.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = set(re.findall(r"\s[TW]\s+(\w+)$", out, flags=re.M))
    missing = [n for n in declared_functions() if n not in exported]
    assert not missing, missing
    lib = ctypes.CDLL(art.LIB_PATH)
    for n in declared_functions():
        assert getattr(lib, n) is not None


def test_strerror_and_version(art):
    for code in range(-8, 1):
        s = art.art_strerror(code)
        assert s and s != "unknown status"
    assert art.art_strerror(-99) == "unknown status"
    assert art.art_version() >= 100


FAKE = 0x7f0000000000   # 1 MiB aligned, never dereferenced: checks fail first


def T(shape, dtype, stride=None, data=FAKE):
    t = __import__("kv_cache_early_art_b200").ArtTensor()
    t.data = data
    t.dtype = dtype
    t.ndim = len(shape)
    if stride is None:
        stride, acc = [], 1
        for s in reversed(shape):
            stride.insert(0, acc)
            acc *= s
    for i, s in enumerate(shape):
        t.shape[i] = s
        t.stride[i] = stride[i]
    return t


def good(B=2, Hq=8, Hkv=2, d=128, page=64, NP=10, MB=5, dt=1):
    return dict(q=T([B, Hq, d], dt), k=T([NP, Hkv, page, d], dt), v=T([NP, Hkv, page, d], dt),
                pt=T([B, MB], 2), bo=T([B, MB], 2), sl=T([B], 2), out=T([B, Hq, d], 0), st=T([B, Hkv], 2))


def call(art, a, eps_m=1e-3, eps_d=1e-4, P=2, mb=1):
    lib = art.raw_library()
    r = ctypes.byref
    return lib.art_decode_attention(r(a["q"]), r(a["k"]), r(a["v"]), r(a["pt"]), r(a["bo"]), r(a["sl"]),
                                    eps_m, eps_d, P, mb, r(a["out"]), r(a["st"]), None)


def test_null_pointers(art):
    a = good()
    a["k"].data = None
    assert call(art, a) == -1
    lib = art.raw_library()
    assert lib.art_decode_attention(None, None, None, None, None, None, 0.0, 0.0, 0, 0, None, None, None) == -1
    assert lib.art_decode_attention_ex(None, None) == -1


@pytest.mark.parametrize("mut,code", [
    (lambda a: setattr(a["q"], "ndim", 2), -2),
    (lambda a: a["k"].shape.__setitem__(3, 64), -2),                    # d mismatch
    (lambda a: a["v"].shape.__setitem__(1, 3), -2),                     # v shape != k shape
    (lambda a: a["out"].shape.__setitem__(1, 4), -2),
    (lambda a: a["st"].shape.__setitem__(1, 8), -2),
    (lambda a: a["bo"].shape.__setitem__(1, 6), -2),
    (lambda a: a["q"].stride.__setitem__(2, 2), -2),                    # d not contiguous
    (lambda a: a["k"].stride.__setitem__(2, 100), -2),                  # 200-byte row stride: not 16-aligned
    (lambda a: setattr(a["k"], "data", FAKE + 8), -2),                  # misaligned base
    (lambda a: setattr(a["k"], "dtype", 0), -3),                        # f32 cache with bf16 q
    (lambda a: setattr(a["out"], "dtype", 1), -3),
    (lambda a: setattr(a["pt"], "dtype", 0), -3),
])
def test_shape_and_dtype_errors(art, mut, code):
    a = good()
    mut(a)
    assert call(art, a) == code


def test_unsupported_sizes(art):
    assert call(art, good(d=96)) == -2 or call(art, good(d=96)) == -4
    a = good(d=96)
    assert call(art, a) == -4
    assert call(art, good(page=32)) == -4
    assert call(art, good(Hq=18, Hkv=2)) == -4          # G = 9
    assert call(art, good(Hq=9, Hkv=2)) == -2           # Hq % Hkv != 0


@pytest.mark.parametrize("eps_m,eps_d,P,mb", [(float("nan"), 1e-3, 1, 1), (1e-3, -1.0, 1, 1),
                                              (1e-3, 1e-3, -1, 1), (1e-3, 1e-3, 1, -2)])
def test_parameter_errors(art, eps_m, eps_d, P, mb):
    assert call(art, good(), eps_m, eps_d, P, mb) == -5


def test_ex_option_errors(art):
    a = good()
    p = art.ArtParams()
    for name, key in (("q", "q"), ("k_cache", "k"), ("v_cache", "v"), ("page_table", "pt"),
                      ("block_order", "bo"), ("seq_lens", "sl"), ("out", "out"), ("stop_block", "st")):
        setattr(p, name, a[key])
    lib = art.raw_library()
    for field, val in (("engine", 3), ("cluster_size", 17), ("stages", 9), ("stages", 1), ("window", 65),
                       ("compute_warps", 7), ("window", 7), ("debug_flags", 2), ("timeout_ns", -1),
                       ("prefetch", -2), ("prefetch", 65)):
        setattr(p, field, val)
        assert lib.art_decode_attention_ex(ctypes.byref(p), None) == -5, field
        setattr(p, field, 0)
    p.sm_scale = float("inf")
    assert lib.art_decode_attention_ex(ctypes.byref(p), None) == -5
    p.sm_scale = 0.0
    # tensor-core engine needs bf16
    f = good(dt=0)
    for name, key in (("q", "q"), ("k_cache", "k"), ("v_cache", "v")):
        setattr(p, name, f[key])
    p.engine = 2
    assert lib.art_decode_attention_ex(ctypes.byref(p), None) == -4


def test_order_builder_errors(art):
    lib = art.raw_library()
    sl, bo = T([4], 2), T([4, 10], 2)
    assert lib.art_build_order_sink_recency(ctypes.byref(sl), 0, ctypes.byref(bo), None) == -5
    bad = T([3, 10], 2)
    assert lib.art_build_order_sink_recency(ctypes.byref(sl), 64, ctypes.byref(bad), None) == -2
    f = T([4, 10], 0)
    assert lib.art_build_order_sink_recency(ctypes.byref(sl), 64, ctypes.byref(f), None) == -3
    assert lib.art_build_order_sink_recency(None, 64, ctypes.byref(bo), None) == -1


def test_binding_refuses_cpu_tensors(art):
    import torch
    q = torch.zeros(1, 4, 64)
    with pytest.raises(ValueError):
        art.art_decode_attention(q, q, q, q, q, q, 0.0, 0.0, 0, 0)
