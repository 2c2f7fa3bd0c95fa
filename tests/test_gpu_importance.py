"""GPU parity of the importance-first order (art_page_summary,
art_build_order_importance) against the fp64 oracle in oracle/importance.py,
and ART walks over that order.

Tolerances follow from fp32 arithmetic (unit roundoff u = 2^-24):
* a page mean of n <= page keys: |err| <= (n + 1) u * mean |k| per channel,
  plus one rounding to bf16 (2^-8 relative) for a bf16 summary;
* a block score: the group sums of q (G terms) and a dot product of Hkv*d
  terms split over 32 lanes and a 5-level butterfly, so |err| <= (G + Hkv*d/32
  + 8) u * A with A = scale * sum |q_i| |kbar| (the same sum of magnitudes).
The order is integer work decided by those scores: it must be a permutation
with block 0 first, sorted by the oracle's fp64 scores except between blocks
whose scores lie within the summed tolerances (either order is correct
there), and exactly sorted by the scores the kernel returns.
"""
import math

import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import make_custom, make_workload, sink_recency_order
import oracle
from oracle import importance as imp
from tests import parity

pytestmark = pytest.mark.gpu

U32 = 2.0 ** -24


def _case(name):
    if name == "tiny_fp32":
        return make_workload("tiny_fp32")
    if name == "bf16_g4":
        return make_custom(B=3, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[4096, 1000, 64], seed=1,
                           planted=5, eps_m=5e-4, eps_d=5e-5, P=3)
    if name == "bf16_g7":
        return make_custom(B=2, Hq=28, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[8192, 3001], seed=2,
                           planted=8, eps_m=2e-4, eps_d=2e-5, P=4, min_blocks=4)
    if name == "f32_d64_p16_ragged":
        return make_custom(B=5, Hq=4, Hkv=2, d=64, page=16, dtype="f32", seq_lens=[1, 17, 500, 0, 33], seed=3,
                           planted=3, eps_m=1e-3, eps_d=1e-4, P=2, spare_pages=4)
    if name == "f32_d256":
        return make_custom(B=2, Hq=4, Hkv=2, d=256, page=16, dtype="f32", seq_lens=[300, 47], seed=4, planted=2)
    if name == "bf16_d16":
        return make_custom(B=2, Hq=6, Hkv=3, d=16, page=64, dtype="bf16", seq_lens=[1000, 65], seed=5, planted=2)
    raise KeyError(name)


ALL = ["tiny_fp32", "bf16_g4", "bf16_g7", "f32_d64_p16_ragged", "f32_d256", "bf16_d16"]
WALKABLE = ["tiny_fp32", "bf16_g4", "bf16_g7", "f32_d64_p16_ragged"]


def _referenced(w):
    N = w.n_blocks().cpu().numpy()
    pt = w.page_table.cpu().numpy()
    return sorted({int(pt[b, j]) for b in range(w.B) for j in range(int(N[b]))})


def _page_abs_mean(w):
    """mean |k| over each referenced page's valid tokens: [num_pages, Hkv, d]."""
    k = w.k_cache.cpu().double().abs().numpy()
    pt, L = w.page_table.cpu().numpy(), w.seq_lens.cpu().numpy()
    out = np.zeros(k.shape[:2] + k.shape[3:])
    for b in range(w.B):
        for j in range(int(w.n_blocks()[b])):
            n = min(w.page, int(L[b]) - j * w.page)
            out[pt[b, j]] = k[pt[b, j], :, :n].mean(axis=1)
    return out


def _score_bound(w, summ64, scale):
    """A[b, j] = scale * sum_i sum_c |q_ic| |kbar_c| (the magnitude sum behind
    the score's rounding bound)."""
    q = w.q.cpu().double().abs().numpy()
    qa = q.reshape(w.B, w.Hkv, w.G, w.d).sum(2)          # [B, Hkv, d]
    pt = w.page_table.cpu().numpy()
    A = np.zeros(pt.shape)
    for b in range(w.B):
        for j in range(int(w.n_blocks()[b])):
            A[b, j] = scale * float((qa[b] * np.abs(summ64[pt[b, j]])).sum())
    return A


def _score_tol(w, A):
    return (w.G + w.Hkv * w.d / 32 + 8) * U32 * A + 1e-30


def _assert_valid_order(w, order, s64, tol):
    """Permutation, sink first, -1 after N_b, and sorted by the fp64 scores
    wherever they differ by more than the two blocks' tolerances."""
    N = w.n_blocks().cpu().numpy()
    for b in range(w.B):
        n = int(N[b])
        o = order[b]
        assert (o[n:] == -1).all()
        if n == 0:
            continue
        assert o[0] == 0 and sorted(o[:n].tolist()) == list(range(n))
        if n <= 2:
            continue
        s, t = s64[b, o[1:n]], tol[b, o[1:n]]
        # for positions p < r: s[p] + t[p] >= s[r] - t[r]; i.e. the running
        # minimum of (s + t) over the prefix stays above each later (s - t)
        lo = np.minimum.accumulate(s + t)[:-1]
        hi = (s - t)[1:]
        bad = np.nonzero(lo < hi)[0]
        assert bad.size == 0, f"sequence {b}: block at order position {bad[0] + 2} sorts out of place"


def _sorted_by_own_scores(w, order, sc):
    N = w.n_blocks().cpu().numpy()
    for b in range(w.B):
        n = int(N[b])
        if n < 2:
            continue
        rest = sorted(range(1, n), key=lambda j: (-float(sc[b, j]) if sc[b, j] != 0 else 0.0, -j))
        assert order[b, 1:n].tolist() == rest


@pytest.mark.parametrize("sdt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name", ALL)
def test_page_summary_parity(cuda_lib, name, sdt):
    w = _case(name)
    g = w.to("cuda")
    NP = w.k_cache.shape[0]
    sentinel = 7.0
    summ = torch.full((NP, w.Hkv, w.d), sentinel, dtype=sdt, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    cuda_lib.art_page_summary(g.k_cache, g.page_table, g.seq_lens, summ, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    got = summ.double().cpu().numpy()
    ref = imp.page_summary(w.k_cache, w.page_table, w.seq_lens)
    used = _referenced(w)
    absm = _page_abs_mean(w)
    tol = (w.page + 1) * U32 * absm + U32 * np.abs(ref)
    if sdt == torch.bfloat16:
        tol = tol + 2.0 ** -8 * np.abs(np.nan_to_num(ref))
    err = np.abs(got[used] - ref[used])
    assert (err <= tol[used]).all(), float((err - tol[used]).max())
    unused = sorted(set(range(NP)) - set(used))
    assert (got[unused] == sentinel).all()


@pytest.mark.parametrize("sdt", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("name", ALL)
def test_scores_and_order_parity(cuda_lib, name, sdt):
    """Scores from a given summary (the oracle's, stored as sdt) against the
    oracle's fp64 scores from the same stored values; the order against
    those scores."""
    w = _case(name)
    scale = 1.0 / math.sqrt(w.d)
    ref_summ = np.nan_to_num(imp.page_summary(w.k_cache, w.page_table, w.seq_lens))
    stored = torch.from_numpy(ref_summ).to(sdt)
    s64 = imp.block_scores(w.q, stored, w.page_table, w.seq_lens, w.page, scale)
    o64 = imp.importance_order(s64, w.seq_lens, w.page)
    g = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    order, sc = cuda_lib.art_build_order_importance(g.q, stored.cuda(), g.page_table, g.seq_lens, w.page,
                                                    device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    sc, order = sc.cpu().numpy(), order.cpu().numpy()
    fin = np.isfinite(s64)
    assert (np.isneginf(sc) == ~fin).all()
    tol = _score_tol(w, _score_bound(w, stored.double().numpy(), scale))
    err = np.abs(sc[fin] - s64[fin])
    assert (err <= tol[fin]).all(), f"score error {float((err / tol[fin]).max()):.2f} x its bound"
    _assert_valid_order(w, order, s64, tol)
    _sorted_by_own_scores(w, order, sc)
    # small cases have no near ties: then the order is the oracle's exactly
    if name in ("tiny_fp32", "f32_d64_p16_ragged", "bf16_d16"):
        np.testing.assert_array_equal(order, o64)


def _importance_walk(cuda_lib, w, sdt=torch.float32):
    g = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    summ = cuda_lib.art_page_summary(g.k_cache, g.page_table, g.seq_lens, dtype=sdt, device_status=status)
    order, sc = cuda_lib.art_build_order_importance(g.q, summ, g.page_table, g.seq_lens, w.page,
                                                    device_status=status)
    fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, order, g.seq_lens,
                                                 eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d, P_per_seq=g.P,
                                                 min_blocks_per_seq=g.min_blocks, blocks_fetched=fetched,
                                                 device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    return out, stop, order.cpu().numpy(), sc.cpu().numpy()


def _composed_reference(w, sdt):
    """The oracle's order from its own summary (stored as sdt), its fp64
    scores, and a tolerance covering the GPU's summary and score rounding:
    the summary's per-channel bound (plus half a bf16 ulp when stored as
    bf16) carried through the dot product, plus the score's own bound."""
    scale = 1.0 / math.sqrt(w.d)
    summ = np.nan_to_num(imp.page_summary(w.k_cache, w.page_table, w.seq_lens))
    stored = torch.from_numpy(summ).to(sdt).double().numpy()
    s64 = imp.block_scores(w.q, stored, w.page_table, w.seq_lens, w.page, scale)
    o64 = imp.importance_order(s64, w.seq_lens, w.page)
    per_channel = (w.page + 1) * U32 * _page_abs_mean(w)
    if sdt == torch.bfloat16:
        per_channel = per_channel + 2.0 ** -8 * (np.abs(summ) + per_channel)
    tol = _score_tol(w, _score_bound(w, stored, scale)) + _score_bound(w, per_channel, scale)
    return o64, s64, tol


def _check_composed(w, out, stop, order_gpu, sdt=torch.float32, min_frac=1.0):
    """The walk's result depends only on the order's first `stop` entries.
    Units whose GPU order agrees with the oracle's over every admissible stop
    must match the oracle's walk over the oracle's own order; the GPU order
    must be a valid sort of the oracle's scores everywhere (near ties may go
    either way); at least min_frac of the units are compared."""
    o64, s64, tol = _composed_reference(w, sdt)
    _assert_valid_order(w, order_gpu, s64, tol)
    wo = w.to("cpu")
    wo.block_order = torch.from_numpy(o64)
    r = oracle.run(wo, want_out=False)
    units = []
    for u in range(w.B * w.Hkv):
        b = u // w.Hkv
        s_max = max([int(x) for x in r.admissible[u]] + [0])
        if (order_gpu[b, :s_max] == o64[b, :s_max]).all():
            units.append(u)
    U = w.B * w.Hkv
    assert len(units) >= min_frac * U, f"orders differ inside the consumed prefix for {U - len(units)} of {U} units"
    return parity.check(wo, out, stop, units=units)


@pytest.mark.parametrize("name", WALKABLE)
def test_walk_over_importance_order(cuda_lib, name):
    w = _case(name)
    out, stop, order, sc = _importance_walk(cuda_lib, w)
    _check_composed(w, out, stop, order)


def test_walk_over_importance_order_bf16_summary(cuda_lib):
    """A bf16 summary rounds the scores by up to 2^-8 relative, so near ties
    inside the consumed prefix may break either way; those units are checked
    for a valid order only."""
    w = _case("bf16_g7")
    out, stop, order, sc = _importance_walk(cuda_lib, w, sdt=torch.bfloat16)
    _check_composed(w, out, stop, order, sdt=torch.bfloat16, min_frac=0.5)


def test_qwen7b_b4_importance_full_size(cuda_lib):
    """Planted heavy hitters: the walk over the importance order stops after
    the planted blocks, the sink and P more blocks."""
    w = make_workload("qwen7b_b4")
    out, stop, order, sc = _importance_walk(cuda_lib, w)
    s = _check_composed(w, out, stop, order)
    st = stop.cpu().numpy()
    planted = [len(set((w.meta["planted_pos"][b] // w.page).tolist()) - {0}) for b in range(w.B)]
    for b in range(w.B):
        assert (st[b] <= planted[b] + 1 + int(w.P[b]) + 1).all(), (st[b], planted[b])
    assert s["blocks_consumed"] < 0.02 * s["blocks_total"]


def test_equal_scores_give_default_order(cuda_lib):
    """Identical pages: every score ties exactly, so the order is the sink then
    newest first."""
    w = make_custom(B=3, Hq=8, Hkv=2, d=64, page=16, dtype="bf16", seq_lens=[16 * 40, 16 * 3 + 2, 5], seed=6,
                    keys="noise")
    w.k_cache[:] = w.k_cache[0:1, :, 0:1]       # one key row per head everywhere: every page mean is exact
    g = w.to("cuda")
    summ = cuda_lib.art_page_summary(g.k_cache, g.page_table, g.seq_lens)
    order, sc = cuda_lib.art_build_order_importance(g.q, summ, g.page_table, g.seq_lens, w.page)
    torch.cuda.synchronize()
    ref = sink_recency_order(w.n_blocks().cpu(), w.max_blocks)
    assert torch.equal(order.cpu(), ref)


def test_importance_bitwise_deterministic(cuda_lib):
    w = _case("bf16_g7").to("cuda")
    runs = []
    for _ in range(3):
        summ = cuda_lib.art_page_summary(w.k_cache, w.page_table, w.seq_lens)
        order, sc = cuda_lib.art_build_order_importance(w.q, summ, w.page_table, w.seq_lens, w.page)
        runs.append((summ.clone(), order.clone(), sc.clone()))
    torch.cuda.synchronize()
    for r in runs[1:]:
        for a, b in zip(runs[0], r):
            assert torch.equal(a.view(torch.int32) if a.dtype == torch.float32 else a,
                               b.view(torch.int32) if b.dtype == torch.float32 else b)


def test_importance_bad_entries_reported(cuda_lib):
    """A page-table entry out of range and a sequence longer than its table:
    status BAD_INDEX, a NaN score for the bad block, and still a permutation."""
    w = _case("bf16_g4")
    g = w.to("cuda")
    pt = g.page_table.clone()
    pt[0, 3] = w.k_cache.shape[0]
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    summ = torch.zeros(w.k_cache.shape[0], w.Hkv, w.d, device="cuda")
    cuda_lib.art_page_summary(g.k_cache, pt, g.seq_lens, summ, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -8
    status.zero_()
    order, sc = cuda_lib.art_build_order_importance(g.q, summ, pt, g.seq_lens, w.page, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -8
    sc, order = sc.cpu().numpy(), order.cpu().numpy()
    assert math.isnan(sc[0, 3])
    N = w.n_blocks().cpu().numpy()
    for b in range(w.B):
        assert order[b, 0] == 0 and sorted(order[b, :N[b]].tolist()) == list(range(int(N[b])))
    # too long for the table
    status.zero_()
    sl = g.seq_lens.clone()
    sl[1] = w.max_blocks * w.page + 1
    cuda_lib.art_build_order_importance(g.q, summ, g.page_table, sl, w.page, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -8


def test_importance_strided_layouts(cuda_lib):
    """Cache pages, summary rows and the order/score rows with padding."""
    w = _case("bf16_g4")
    NP = w.k_cache.shape[0]
    big = torch.zeros(NP, w.Hkv + 1, w.page + 8, w.d + 64, dtype=w.k_cache.dtype)
    big[:, :w.Hkv, :w.page, :w.d] = w.k_cache
    k = big.cuda()[:, :w.Hkv, :w.page, :w.d]
    g = w.to("cuda")
    sbig = torch.zeros(NP, w.Hkv + 2, w.d + 8, device="cuda")
    summ = sbig[:, 1:w.Hkv + 1, :w.d]
    cuda_lib.art_page_summary(k, g.page_table, g.seq_lens, summ)
    ref = cuda_lib.art_page_summary(g.k_cache, g.page_table, g.seq_lens)
    torch.cuda.synchronize()
    used = _referenced(w)
    assert torch.equal(summ[used], ref[used])
    obig = torch.zeros(w.B, w.max_blocks + 5, dtype=torch.int32, device="cuda")
    scbig = torch.zeros(w.B, w.max_blocks + 3, device="cuda")
    order, sc = cuda_lib.art_build_order_importance(g.q, summ, g.page_table, g.seq_lens, w.page,
                                                    block_scores=scbig[:, :w.max_blocks],
                                                    block_order=obig[:, :w.max_blocks])
    o2, s2 = cuda_lib.art_build_order_importance(g.q, ref, g.page_table, g.seq_lens, w.page)
    torch.cuda.synchronize()
    assert torch.equal(order, o2) and torch.equal(sc, s2)
    assert (obig[:, w.max_blocks:] == 0).all()
