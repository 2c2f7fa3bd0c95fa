"""art_decode_attention_no_alloc (include/art.h): the workspace walk run
through a fixed scratch array inside the library, for callers that cannot
allocate device memory (a serving engine whose pool owns nearly all of it, a
decode loop that may not stall on cudaMalloc/cudaFree, a plug-in that may not
grow its host application's footprint).  The paper has no counterpart; the
walk it runs is the one the other tests check against the oracle.

The GPU tests call it through the C ABI twice in a row (the second call finds
the first one's leftovers in the shared array) and compare both results with
art_decode_attention_ex's on the same inputs.  This file is collected last."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from kv_cache_early_art_b200.workloads import make_custom, make_workload
from tests import parity
from tests.test_gpu_parity import run_gpu
from tests.test_abi import good

SCRATCH_SIZE = -9


def _no_alloc(art, w, out, stop, fetched, status):
    """One call with caller-owned outputs and accounting buffers."""
    g = w.to("cuda")
    return art.art_decode_attention_no_alloc(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order, g.seq_lens,
                                             eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d, P_per_seq=g.P,
                                             min_blocks_per_seq=g.min_blocks, blocks_fetched=fetched,
                                             device_status=status, out=out, stop_block=stop, want_info=True)


def _ragged():
    lens = [2900, 17, 64 * 40 + 5, 0, 64 * 3, 1, 1800]
    return make_custom(B=len(lens), Hq=14, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=lens, seed=990,
                       keys="recency", planted=3, planted_gain=5.0, order="random", eps_m=2e-2, eps_d=2e-3,
                       P=[1, 2, 3, 0, 2, 1, 4], min_blocks=[1, 3, 0, 1, 2, 1, 5], spare_pages=5)


@pytest.mark.gpu
@pytest.mark.parametrize("case", ["qwen7b_b4", "ragged"])
def test_no_alloc_two_calls_match_ex(cuda_lib, case):
    w = make_workload("qwen7b_b4") if case == "qwen7b_b4" else _ragged()
    wc = w.to("cpu")
    out_ex, stop_ex, _, status_ex, _ = run_gpu(cuda_lib, w)
    assert status_ex == 0
    adm = oracle.run(wc, want_out=False).admissible
    tol = parity.TOL[torch.bfloat16]
    B, Hq, d, Hkv = w.B, w.Hq, w.d, w.Hkv
    out = torch.empty(B, Hq, d, dtype=torch.float32, device="cuda")
    stop = torch.empty(B, Hkv, dtype=torch.int32, device="cuda")
    fetched = torch.zeros(B * Hkv, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    results = []
    for call in range(2):
        out.fill_(float("nan"))
        stop.fill_(-7)
        fetched.zero_()
        _, _, info = _no_alloc(cuda_lib, w, out, stop, fetched, status)
        torch.cuda.synchronize()
        assert int(status.item()) == 0, call
        assert info["merge_cta"] == 2 and 16 <= info["ring_slots"] <= 128
        results.append((out.clone(), stop.clone()))
        # stops: equal to the existing entry point's, or another stop the
        # oracle admits where a statistic sits on a threshold
        st, se = stop.cpu().numpy(), stop_ex.cpu().numpy()
        for u in range(B * Hkv):
            b, h = divmod(u, Hkv)
            if st[b, h] != se[b, h]:
                assert len(adm[u]) > 1 and int(st[b, h]) in [int(x) for x in adm[u]], (call, b, h)
        same = torch.from_numpy((st == se).all(axis=1)).to("cuda")
        assert int(same.sum()) >= B - 1
        err = float((out[same] - out_ex[same]).abs().max()) if bool(same.any()) else 0.0
        assert err <= tol, (call, err)
        fe = fetched.view(B, Hkv).cpu().numpy()
        assert (fe >= st).all() and (fe <= st + info["window"]).all()
    assert torch.equal(results[0][1], results[1][1]) and torch.equal(results[0][0], results[1][0])
    parity.check(wc, results[1][0], results[1][1])


@pytest.mark.gpu
def test_no_alloc_refuses_too_large(cuda_lib):
    """70 units with 8 query heads per kv head need about 4.7 MB even with
    the smallest ring: more than the array holds, so the call is refused
    before anything is launched; other walks are refused where they are not
    built."""
    w = make_custom(B=35, Hq=16, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 4] * 35, seed=991)
    g = w.to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_no_alloc(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens)
    assert e.value.status == SCRATCH_SIZE
    f = make_custom(B=2, Hq=4, Hkv=1, d=64, page=16, dtype="f32", seq_lens=[100, 40], seed=992).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_no_alloc(f.q, f.k_cache, f.v_cache, f.page_table, None, f.seq_lens)
    assert e.value.status == -4


def test_no_alloc_host_errors():
    """Refusals that need no GPU: the caller may not bring a workspace or
    ask for another walk; a NULL parameter block; the new status has a
    message."""
    from kv_cache_early_art_b200 import build
    build.build_library()
    import kv_cache_early_art_b200 as art
    lib = art.raw_library()
    assert lib.art_decode_attention_no_alloc(None, None) == -1
    a = good()
    p = art.ArtParams()
    for name, key in (("q", "q"), ("k_cache", "k"), ("v_cache", "v"), ("page_table", "pt"),
                      ("block_order", "bo"), ("seq_lens", "sl"), ("out", "out"), ("stop_block", "st")):
        setattr(p, name, a[key])
    for field, val in (("workspace", 0x7f0000000000), ("workspace_bytes", 1 << 20), ("merge_cta", 1),
                       ("merge_cta", -1)):
        setattr(p, field, val)
        assert lib.art_decode_attention_no_alloc(ctypes.byref(p), None) == -5, field
        setattr(p, field, None if field == "workspace" else 0)
    p.eps_m = -1.0
    assert lib.art_decode_attention_no_alloc(ctypes.byref(p), None) == -5
    assert art.art_strerror(SCRATCH_SIZE) != "unknown status"
    assert art.STATUS[SCRATCH_SIZE] == "ART_ERR_SCRATCH_SIZE"
