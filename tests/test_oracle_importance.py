"""Pins of the importance-first order oracle (oracle/importance.py), CPU only.

Each check rests on something other than the oracle's own formulas: a closed
form (pages built with a known mean key), the other route to the same score
(per-token logits averaged, against the mean key dotted), the tie rule reduced
to the default sink-then-recency order, exact symmetries (physical page
relabelling, positive query scaling, query negation) and planted keys whose
ranking is known in advance.
"""
import math

import numpy as np
import pytest
import torch

from kv_cache_early_art_b200 import workloads as W
from oracle import importance as imp


def _cache(num_pages, Hkv, page, d, dtype=torch.float32):
    return torch.zeros(num_pages, Hkv, page, d, dtype=dtype)


def test_summary_closed_form_masks_the_tail():
    """Tokens t < n carry c + (t - (n-1)/2) u, so their mean is exactly c;
    tokens past the sequence end hold 1e6 and must not count."""
    page, d, Hkv = 16, 8, 2
    lens = [16 * 3 + 5]                      # 4 blocks, the last with 5 tokens
    k = _cache(4, Hkv, page, d)
    pt = torch.tensor([[2, 0, 3, 1]], dtype=torch.int32)
    g = torch.Generator().manual_seed(3)
    want = {}
    for j in range(4):
        p = int(pt[0, j])
        n = min(page, lens[0] - j * page)
        c = torch.randint(-8, 9, (Hkv, d), generator=g).float() / 4
        u = torch.randint(-3, 4, (Hkv, d), generator=g).float()
        for t in range(page):
            k[p, :, t] = c + (t - (n - 1) / 2) * u if t < n else 1e6
        want[p] = c.double().numpy()
    kb = imp.page_summary(k, pt, torch.tensor(lens))
    for p, c in want.items():
        np.testing.assert_array_equal(kb[p], c)


def test_summary_unreferenced_pages_are_nan():
    k = torch.randn(5, 1, 4, 4)
    kb = imp.page_summary(k, torch.tensor([[3, 1]], dtype=torch.int32), torch.tensor([6]))
    assert np.isnan(kb[[0, 2, 4]]).all() and not np.isnan(kb[[1, 3]]).any()


@pytest.mark.parametrize("G", [1, 4, 7])
def test_score_equals_mean_of_head_summed_logits(G):
    """s[b,j] against the per-token route: logits q_i . k_t for every valid
    token and query head (query head i reads kv head i // G), summed over
    heads, averaged over the block's tokens."""
    Hkv, d, page = 2, 16, 8
    w = W.make_custom(B=2, Hq=Hkv * G, Hkv=Hkv, d=d, page=page, dtype="f32", seq_lens=[37, 8], seed=11,
                      keys="noise")
    scale = 1.0 / math.sqrt(d)
    kb = imp.page_summary(w.k_cache, w.page_table, w.seq_lens)
    s = imp.block_scores(w.q, kb, w.page_table, w.seq_lens, page, scale)
    q, k = w.q.double(), w.k_cache.double()
    for b in range(w.B):
        L = int(w.seq_lens[b])
        for j in range(int(w.n_blocks()[b])):
            p = int(w.page_table[b, j])
            n = min(page, L - j * page)
            logits = torch.stack([k[p, i // G, :n] @ q[b, i] for i in range(w.Hq)])   # [Hq, n]
            ref = scale * float(logits.sum(0).mean())
            assert abs(s[b, j] - ref) <= 1e-12 * max(1.0, abs(ref))
        assert np.all(np.isneginf(s[b, int(w.n_blocks()[b]):]))


def test_equal_scores_give_the_default_order():
    """Identical pages: every score ties, so the order is block 0 then newest
    first, the sink-then-recency order."""
    page, d = 4, 8
    lens = torch.tensor([4 * 9, 4 * 3 + 1, 4, 0])
    N = imp.n_blocks(lens, page)
    k = torch.ones(int(N.sum()), 2, page, d)
    pt = torch.full((4, 9), -1, dtype=torch.int32)
    off = 0
    for b in range(4):
        pt[b, :N[b]] = torch.arange(off, off + N[b], dtype=torch.int32)
        off += N[b]
    q = torch.randn(4, 4, d, generator=torch.Generator().manual_seed(0))
    order = imp.importance_walk_order(q, k, pt, lens, 0.5)
    ref = W.sink_recency_order(torch.as_tensor(N), 9).numpy()
    np.testing.assert_array_equal(order, ref)
    assert (order[3] == -1).all() and order[2, 0] == 0 and (order[2, 1:] == -1).all()


def test_planted_pages_rank_first_in_gain_order():
    """Pages whose keys point along +q (gains 3 > 2 > 1) come right after the
    sink in that order; a page along -q comes last; the rest (zero keys)
    tie and follow newest first."""
    page, d, N = 4, 8, 10
    g = torch.Generator().manual_seed(5)
    q = torch.randn(1, 2, d, generator=g)
    qhat = q[0].sum(0) / q[0].sum(0).norm()
    k = _cache(N, 1, page, d)
    pt = torch.randperm(N, generator=g).to(torch.int32).view(1, N)
    gains = {6: 3.0, 2: 2.0, 8: 1.0, 4: -1.0}
    for j, a in gains.items():
        k[int(pt[0, j]), 0] = a * qhat
    order = imp.importance_walk_order(q, k, pt, torch.tensor([N * page]), 1.0)
    assert order[0].tolist() == [0, 6, 2, 8, 9, 7, 5, 3, 1, 4]


def test_symmetries_relabel_scale_negate():
    w = W.make_custom(B=3, Hq=8, Hkv=2, d=32, page=16, dtype="f32", seq_lens=[300, 17, 129], seed=2,
                      keys="noise", spare_pages=3)
    page, scale = 16, 1.0 / math.sqrt(32)
    base_s = imp.block_scores(w.q, imp.page_summary(w.k_cache, w.page_table, w.seq_lens), w.page_table,
                              w.seq_lens, page, scale)
    base = imp.importance_order(base_s, w.seq_lens, page)
    N = imp.n_blocks(w.seq_lens, page)
    # relabel physical pages: cache rows permuted, table entries mapped along
    perm = torch.randperm(w.k_cache.shape[0], generator=torch.Generator().manual_seed(9))
    inv = torch.empty_like(perm)
    inv[perm] = torch.arange(perm.numel())
    k2 = w.k_cache[perm]
    pt2 = torch.where(w.page_table >= 0, inv[w.page_table.clamp(min=0).long()].to(torch.int32), w.page_table)
    np.testing.assert_array_equal(imp.importance_walk_order(w.q, k2, pt2, w.seq_lens, scale), base)
    # positive scaling of the query scales the scores, keeps the order
    s3 = imp.block_scores(w.q * 4, imp.page_summary(w.k_cache, w.page_table, w.seq_lens), w.page_table,
                          w.seq_lens, page, scale)
    fin = np.isfinite(base_s)
    np.testing.assert_allclose(s3[fin], 4 * base_s[fin], rtol=1e-12)
    np.testing.assert_array_equal(imp.importance_order(s3, w.seq_lens, page), base)
    # negating the query reverses blocks 1..N-1 (the scores are distinct here)
    neg = imp.importance_walk_order(-w.q, w.k_cache, w.page_table, w.seq_lens, scale)
    for b in range(w.B):
        n = int(N[b])
        assert len(set(base_s[b, 1:n].tolist())) == n - 1
        assert neg[b, 0] == 0 and neg[b, 1:n].tolist() == base[b, 1:n][::-1].tolist()


def test_order_is_a_permutation_with_the_sink_first():
    w = W.make_workload("tiny_fp32")
    order = imp.importance_walk_order(w.q, w.k_cache, w.page_table, w.seq_lens, 1 / 8)
    N = int(w.n_blocks()[0])
    assert order[0, 0] == 0 and sorted(order[0, :N].tolist()) == list(range(N))
    assert (order[0, N:] == -1).all()


def test_planted_heavy_hitters_lead_the_order():
    """Keys planted along the group query at known positions: their blocks
    (and only they) follow the sink, before every recency-only block."""
    w = W.make_custom(B=2, Hq=8, Hkv=2, d=64, page=16, dtype="bf16", seq_lens=[2048, 1500], seed=4,
                      planted=6)
    order = imp.importance_walk_order(w.q, w.k_cache, w.page_table, w.seq_lens, 1 / 8)
    for b in range(2):
        blocks = set((w.meta["planted_pos"][b] // 16).tolist()) - {0}
        assert set(order[b, 1:1 + len(blocks)].tolist()) == blocks
