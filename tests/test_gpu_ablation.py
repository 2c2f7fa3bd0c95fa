"""GPU parity for the ablation modes (ART explainer, Technical Summary §4:
removing the scale or the direction criterion, or the patience mechanism),
the undecided band around a threshold (§2.2 thresholds; the acceptance
rule's 1e-4 relative band), and launch-option and length edge cases."""
import numpy as np
import pytest
import torch

import oracle
from kv_cache_early_art_b200.workloads import make_custom
from tests import parity
from tests.test_gpu_parity import _full, assert_fetch_bound, run_gpu

pytestmark = pytest.mark.gpu

INF = float("inf")


# ------------------------------------------------------ ablations, full size ----

@pytest.mark.parametrize("name", ["llama8b_b32", "mistral7b_b128"])
def test_scale_only_full_size(cuda_lib, name):
    """Direction criterion removed (eps_d = +inf, the workload's own eps_m):
    only the magnitude change decides.  Every unit against the oracle."""
    s, w, stop = _full(cuda_lib, name, eps_d=INF)
    # the magnitude test alone stops some walks early on these workloads
    assert s["blocks_consumed"] < s["blocks_total"]


@pytest.mark.parametrize("name", ["llama8b_b32", "mistral7b_b128"])
def test_direction_only_full_size(cuda_lib, name):
    """Magnitude criterion removed (eps_m = +inf)."""
    _full(cuda_lib, name, eps_m=INF)


@pytest.mark.parametrize("name", ["llama8b_b32", "mistral7b_b128", "qwen7b_b4"])
def test_no_patience_full_size(cuda_lib, name):
    """Patience removed (P = 1): the first stable block stops the walk."""
    _full(cuda_lib, name, P=1)


# ------------------------------------------------------------ undecided band ----

@pytest.mark.parametrize("dtype,engine,G,d,page,which", [
    ("bf16", 2, 4, 128, 64, "dir"), ("bf16", 2, 7, 128, 64, "scale"), ("bf16", 1, 4, 128, 64, "dir"),
    ("f32", 1, 4, 64, 16, "dir"), ("f32", 1, 1, 64, 16, "scale")])
def test_threshold_on_a_statistic(cuda_lib, dtype, engine, G, d, page, which):
    """Each sequence gets a threshold equal (in binary32) to one of its own
    blocks' statistics, so the oracle marks that block undecided ('?') and
    admits two stops: the one with the block stable (j + 1, forced by
    min_blocks = j + 1 and P = 1) and a later one.  The GPU's fp32 statistic
    may fall on either side; its stop must be one the oracle admits, and its
    output must match the oracle's output at that stop."""
    lens = [page * 40 + 3, page * 37, page * 52 + page // 2, page * 45]
    B = len(lens)
    w = make_custom(B=B, Hq=G, Hkv=1, d=d, page=page, dtype=dtype, seq_lens=lens, seed=700 + G + len(which),
                    keys="recency", planted=2, planted_gain=3.0, order="random", eps_m=1.0, eps_d=1.0, P=1)
    r = oracle.run(w, eps_m=0.0, eps_d=0.0, want_stats=True, want_out=False)
    stat = r.dd if which == "dir" else r.ds
    eps_m, eps_d, minb = [], [], []
    for b in range(B):
        j = 6 + 3 * b
        x = float(np.float32(stat[b, 0, j]))
        assert x > 0.0
        eps_m.append(INF if which == "dir" else x)
        eps_d.append(x if which == "dir" else INF)
        minb.append(j + 1)
    w.eps_m = torch.tensor(eps_m, dtype=torch.float32)
    w.eps_d = torch.tensor(eps_d, dtype=torch.float32)
    w.P = torch.ones(B, dtype=torch.int32)
    w.min_blocks = torch.tensor(minb, dtype=torch.int32)
    r2 = oracle.run(w, want_stats=True, want_out=False)
    for b in range(B):
        j = minb[b] - 1
        assert chr(r2.flag[b, 0, j]) == "?"
        adm = [int(x) for x in r2.admissible[b]]
        assert j + 1 in adm and len(adm) >= 2, adm
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, engine=engine)
    assert status == 0
    s = parity.check(w, out, stop)
    assert s["ambiguous"] >= B
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])


# ----------------------------------------------------- launch-option edge cases ----

@pytest.mark.parametrize("nw,st", [(2, 0), (3, 0), (4, 0), (0, 4), (0, 6), (0, 2), (5, 0), (6, 0)])
def test_one_launch_option_given(cuda_lib, nw, st):
    """Only one of compute_warps / stages fixed: the library completes the
    other (stages a multiple of the warps) instead of refusing, on a few-unit
    bf16 d = 128, 64-token page case and on a many-unit one; the result
    equals the automatic launch bit for bit."""
    for B, Hkv in ((2, 2), (40, 8)):
        w = make_custom(B=B, Hq=4 * Hkv, Hkv=Hkv, d=128, page=64, dtype="bf16",
                        seq_lens=[64 * (20 + 3 * b) + b for b in range(B)], seed=40 + B, planted=2,
                        planted_gain=5.0, order="random", eps_m=5e-3, eps_d=5e-4, P=2)
        out0, stop0, _, status0, _ = run_gpu(cuda_lib, w)
        out, stop, fetched, status, info = run_gpu(cuda_lib, w, compute_warps=nw, stages=st)
        assert status0 == 0 and status == 0
        if nw:
            assert info["compute_warps"] == nw and info["stages"] % nw == 0
        if st:
            assert info["stages"] == st and st % info["compute_warps"] == 0
        assert torch.equal(stop, stop0) and torch.equal(out, out0)
        assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])
    parity.check(w, out, stop)


def test_mismatched_warps_and_stages_refused(cuda_lib):
    w = make_custom(B=1, Hq=4, Hkv=1, d=128, page=64, dtype="bf16", seq_lens=[500], seed=41).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens,
                                         compute_warps=3, stages=4)
    assert e.value.status == -5


def test_length_near_int32_max_reported(cuda_lib):
    """A sequence length of INT32_MAX tokens is longer than any page table:
    the unit reports stop -1 and the bad-index status (the block count is
    formed without overflow), the other sequences are exact."""
    w = make_custom(B=3, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[700, 300, 64 * 5], seed=42,
                    planted=2, planted_gain=5.0, eps_m=5e-3, eps_d=5e-4, P=2)
    g = w.to("cuda")
    g.seq_lens[2] = 2 ** 31 - 1
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens,
                                                 eps_m=5e-3, eps_d=5e-4, P=2, min_blocks=1,
                                                 device_status=status)
    order = cuda_lib.art_build_order_sink_recency(g.seq_lens, 64, max_blocks=g.page_table.shape[1])
    torch.cuda.synchronize()
    assert int(status.item()) == -8
    assert stop[2].tolist() == [-1, -1]
    assert (out[2] == 0).all()
    assert order[2, 0].item() == 0 and (order[2, 1:] > 0).all()
    ok = parity.subset_sequences(w, [0, 1])
    parity.check(ok, out[:2], stop[:2])


# ----------------------------------------------------------- detector off ----

@pytest.mark.parametrize("case", ["llama8b_b8", "qwen7b_b4", "tiny_fp32", "many_g8", "many_g4"])
def test_detector_off_equals_eps0(cuda_lib, case):
    """The walk built without the detector (no statistic, no patience, no
    early stop) gives the eps = 0 walk's stops and output bit for bit, in the
    same launch shape; and both equal the oracle's full softmax attention."""
    from kv_cache_early_art_b200.workloads import make_workload
    if case == "many_g8":
        w = make_custom(B=40, Hq=28, Hkv=4, d=128, page=64, dtype="bf16",
                        seq_lens=[64 * (10 + b) + 7 * b for b in range(40)], seed=61)
    elif case == "many_g4":
        w = make_custom(B=48, Hq=16, Hkv=4, d=128, page=64, dtype="bf16",
                        seq_lens=[64 * (5 + 2 * b) + b for b in range(48)], seed=62)
    else:
        w = make_workload(case)
    g = w.to("cuda")
    zero = torch.zeros(w.B, dtype=torch.float32, device="cuda")
    kw = dict(eps_m_per_seq=zero, eps_d_per_seq=zero, P_per_seq=g.P, min_blocks_per_seq=g.min_blocks)
    out0, stop0, info0 = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens,
                                                          want_info=True, **kw)
    fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    out1, stop1, info1 = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens,
                                                          detector_off=1, blocks_fetched=fetched, want_info=True,
                                                          **kw)
    torch.cuda.synchronize()
    assert info0 == info1
    N = w.n_blocks().numpy()[:, None]
    assert (stop1.cpu().numpy() == N).all() and (fetched.view(w.B, w.Hkv).cpu().numpy() == N).all()
    assert torch.equal(stop0, stop1) and torch.equal(out0, out1)
    wc = w.to("cpu")
    wc.eps_m, wc.eps_d = torch.zeros(w.B), torch.zeros(w.B)
    parity.check(wc, out1, stop1)


def test_detector_off_where_not_built(cuda_lib):
    """Shapes without a detector-off build, and the shared walk, refuse it."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[300, 200], seed=63).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens,
                                         detector_off=1, engine=1)
    assert e.value.status == -4
    qm = torch.stack([w.q, w.q], dim=1)
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_multi(qm, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens,
                                            detector_off=1)
    assert e.value.status == -4
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens,
                                         detector_off=2)
    assert e.value.status == -5
