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
              "art_page_summary", "art_build_order_importance", "art_strerror", "art_version"):
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
    for code in range(-9, 1):
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
    for field, val in (("engine", 3), ("cluster_size", 17), ("stages", 9), ("stages", 1), ("window", 129),
                       ("compute_warps", 7), ("window", 7), ("debug_flags", 2), ("timeout_ns", -1),
                       ("prefetch", -2), ("prefetch", 65), ("detector_off", 2), ("detector_off", -1),
                       ("merge_cta", 3), ("merge_cta", -2), ("workspace_bytes", -1)):
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


def _summary_call(art, k, pt, sl, summ, status=None):
    r = ctypes.byref
    return art.raw_library().art_page_summary(r(k), r(pt), r(sl), r(summ), status, None)


def test_page_summary_errors(art):
    k, pt, sl, sm = T([10, 2, 64, 128], 1), T([2, 5], 2), T([2], 2), T([10, 2, 128], 0)
    assert art.raw_library().art_page_summary(None, None, None, None, None, None) == -1
    k0 = T([10, 2, 64, 128], 1, data=None)
    assert _summary_call(art, k0, pt, sl, sm) == -1
    assert _summary_call(art, k, pt, sl, T([10, 2, 64], 0)) == -2          # d mismatch
    assert _summary_call(art, k, pt, sl, T([9, 2, 128], 0)) == -2          # page count mismatch
    assert _summary_call(art, k, T([3, 5], 2), sl, sm) == -2               # table rows != B
    assert _summary_call(art, k, pt, sl, T([10, 2, 128], 2)) == -3         # int summary
    assert _summary_call(art, k, T([2, 5], 0), sl, sm) == -3               # float page table
    assert _summary_call(art, T([10, 2, 64, 96], 1), pt, sl, T([10, 2, 96], 0)) == -4
    assert _summary_call(art, T([10, 2, 64, 128], 1, data=FAKE + 8), pt, sl, sm) == -2
    assert _summary_call(art, k, pt, sl, T([10, 2, 128], 0, data=FAKE + 4)) == -2
    assert _summary_call(art, k, pt, sl, sm, status=FAKE + 2) == -2        # misaligned status word


def _imp_call(art, q, sm, pt, sl, page, scale, sc, bo):
    r = ctypes.byref
    return art.raw_library().art_build_order_importance(r(q), r(sm), r(pt), r(sl), page, scale, r(sc), r(bo),
                                                        None, None)


def test_importance_order_errors(art):
    q, sm, pt, sl = T([2, 8, 128], 1), T([10, 2, 128], 0), T([2, 5], 2), T([2], 2)
    sc, bo = T([2, 5], 0), T([2, 5], 2)
    lib = art.raw_library()
    assert lib.art_build_order_importance(None, None, None, None, 64, 0.0, None, None, None, None) == -1
    assert _imp_call(art, q, sm, pt, sl, 64, 0.0, sc, T([2, 5], 2, data=None)) == -1
    assert _imp_call(art, q, sm, pt, sl, 0, 0.0, sc, bo) == -5                 # page
    assert _imp_call(art, q, sm, pt, sl, 64, float("nan"), sc, bo) == -5
    assert _imp_call(art, q, sm, pt, sl, 64, float("inf"), sc, bo) == -5
    assert _imp_call(art, T([2, 7, 128], 1), sm, pt, sl, 64, 0.0, sc, bo) == -2   # Hq % Hkv
    assert _imp_call(art, q, T([10, 2, 64], 0), pt, sl, 64, 0.0, sc, bo) == -2    # d mismatch
    assert _imp_call(art, q, sm, pt, sl, 64, 0.0, T([2, 6], 0), bo) == -2          # scores shape
    assert _imp_call(art, q, sm, pt, sl, 64, 0.0, sc, T([3, 5], 2)) == -2          # order shape
    assert _imp_call(art, q, sm, pt, sl, 64, 0.0, T([2, 5], 2), bo) == -3          # int scores
    assert _imp_call(art, q, sm, pt, sl, 64, 0.0, sc, T([2, 5], 0)) == -3          # float order
    assert _imp_call(art, T([2, 8, 96], 1), T([10, 2, 96], 0), pt, sl, 64, 0.0, sc, bo) == -4
    big_q, big_s = T([2, 256, 128], 1), T([10, 256, 128], 0)                       # Hkv * d > 16384
    assert _imp_call(art, big_q, big_s, pt, sl, 64, 0.0, sc, bo) == -4


def test_importance_binding_refuses_cpu_tensors(art):
    import torch
    z = torch.zeros(2, 5, dtype=torch.int32)
    with pytest.raises(ValueError):
        art.art_page_summary(torch.zeros(10, 2, 64, 128), z, torch.zeros(2, dtype=torch.int32))
    with pytest.raises(ValueError):
        art.art_build_order_importance(torch.zeros(2, 8, 128), torch.zeros(10, 2, 128), z,
                                       torch.zeros(2, dtype=torch.int32), 64)


def multi_params(art, B=2, T_=2, Hq=8, Hkv=2, d=128, page=64, NP=10, MB=5, dt=1):
    """art_params_t for art_decode_attention_multi over fake (never read) buffers."""
    import kv_cache_early_art_b200 as pkg
    p = pkg.ArtParams()
    p.q = T([B, T_, Hq, d], dt)
    p.k_cache, p.v_cache = T([NP, Hkv, page, d], dt), T([NP, Hkv, page, d], dt)
    p.page_table, p.seq_lens = T([B, MB], 2), T([B], 2)
    p.out, p.stop_block = T([B, T_, Hq, d], 0), T([B, T_, Hkv], 2)
    p.eps_m, p.eps_d, p.P, p.min_blocks = 1e-3, 1e-4, 2, 1
    return p


def test_multi_query_host_errors(art):
    lib = art.raw_library()
    lib.art_decode_attention_multi.argtypes = [ctypes.c_void_p, ctypes.c_int32, ctypes.c_void_p]
    r = lambda p, n=2: lib.art_decode_attention_multi(ctypes.addressof(p), n, None)
    assert lib.art_decode_attention_multi(None, 2, None) == -1
    assert r(multi_params(art), 3) == -4                      # only 1 or 2 tokens per walk
    assert r(multi_params(art), 0) == -4
    assert r(multi_params(art, T_=1), 2) == -2                # token dimension differs from n_queries
    assert r(multi_params(art, Hq=10, Hkv=2)) == -4           # 2 tokens x 5 heads > 8 rows
    assert r(multi_params(art, d=64)) == -4                   # head dim 128 only
    p = multi_params(art)
    p.q.ndim = 3
    assert r(p) == -2                                         # q must be [B, T, Hq, d]
    p = multi_params(art)
    p.out.shape[1] = 3
    assert r(p) == -2                                         # token count differs
    p = multi_params(art)
    p.stop_block.shape[2] = 3
    assert r(p) == -2                                         # stop_block [B, T, Hkv]
    p = multi_params(art)
    p.q.stride[1] = 8 * 128 + 4                               # token stride not 16-byte aligned
    p.q.stride[0] = 2 * p.q.stride[1]
    assert r(p) == -2
    p = multi_params(art)
    p.k_cache.dtype = 0
    assert r(p) == -3                                         # cache dtype differs from q


def test_packed_params_equal_field_by_field(art):
    """The binding packs art_params_t in one struct call; the bytes must be
    those of the same structure filled field by field through ctypes, for
    every tensor rank the entry points take and for every option."""
    import torch
    from kv_cache_early_art_b200 import binding as B
    g = torch.Generator().manual_seed(5)
    q = torch.zeros(3, 8, 128, dtype=torch.bfloat16)[:, :, :]
    k = torch.zeros(20, 2, 64, 128, dtype=torch.bfloat16)
    v = torch.zeros(20, 2, 64, 128, dtype=torch.bfloat16).transpose(0, 1).contiguous().transpose(0, 1)
    pt = torch.zeros(3, 7, dtype=torch.int32)
    bo = torch.zeros(3, 7, dtype=torch.int32)
    sl = torch.zeros(3, dtype=torch.int32)
    out = torch.zeros(3, 8, 128)
    st = torch.zeros(3, 2, dtype=torch.int32)
    em = torch.zeros(3)
    orig = B._need_cuda
    B._need_cuda = lambda *a: None
    try:
        for trial in range(6):
            opts = [int(x) for x in torch.randint(0, 9, (11,), generator=g)]
            args = (q, k, v, pt, bo if trial % 2 else None, sl, out, st, 1e-3 * trial, 2e-4, opts[0], opts[1],
                    0.25 * trial, em, None if trial % 3 else em, sl, None, sl if trial > 2 else None, sl, opts[2],
                    opts[3], opts[4], opts[5], opts[6], 12345678901 * trial, opts[7] % 2, opts[8], opts[9] % 2,
                    opts[10] % 3 - 1)
            p, _ = B._params(*args, want_info=False)
            ref = B.ArtParams()
            for name, t in zip(("q", "k_cache", "v_cache", "page_table", "block_order", "seq_lens", "out",
                                "stop_block"), args[:8]):
                if t is not None:
                    setattr(ref, name, B.descriptor(t))
            for name, val in zip(("eps_m", "eps_d", "P", "min_blocks", "sm_scale"), args[8:13]):
                setattr(ref, name, val)
            for name, t in zip(("eps_m_per_seq", "eps_d_per_seq", "P_per_seq", "min_blocks_per_seq",
                                "blocks_fetched", "device_status"), args[13:19]):
                setattr(ref, name, t.data_ptr() if t is not None else None)
            for name, val in zip(("engine", "cluster_size", "stages", "compute_warps", "window", "timeout_ns",
                                  "debug_flags", "prefetch", "detector_off", "merge_cta"), args[19:]):
                setattr(ref, name, val)
            assert bytes(p) == bytes(ref), trial
    finally:
        B._need_cuda = orig
