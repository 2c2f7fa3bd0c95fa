"""Importance-first walk order: plain fp64 CPU oracle (test infrastructure).

Only the tests, ``__graft_entry__.smoke()`` and the CPU leg of ``bench.py``
use this module; the product library never does, and the two share no code.

Source: "ART: Attention Run-time Termination for Efficient Large Language
Model Decoding" (gist.science explainer), Technical Summary section 2.4 --
ART is an orthogonal control layer over a reordered traversal of the KV
blocks ("recency-first" or "importance-first"), with block 0 always
evaluated first.  The pages name importance-first traversal but define no
importance estimate; the estimate here is this library's own and is stated
in full:

* page summary: the mean key of the page's valid tokens, per kv-head,
      kbar[p, h, :] = (1/n) * sum_{t < n} K[p, h, t, :]
  where page p holds logical block j of sequence b and n = min(page,
  seq_len_b - j*page) tokens of it are valid;
* block score: the mean over the block's valid tokens of the attention
  logit summed over all query heads,
      s[b, j] = scale * sum_{i < Hq} q[b, i, :] . kbar[page_table[b, j], i // G, :]
  (by linearity, the dot product of each query head with its kv-head's
  mean key, summed over heads);
* order: block 0 first (the mandatory sink), then blocks 1 .. N_b-1 by
  decreasing score, equal scores newest (largest j) first, then -1 up to
  max_blocks.

Everything is IEEE double after an exact upcast of the stored values.
"""
from __future__ import annotations

import numpy as np
import torch


def _f64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.float64).numpy()
    return np.asarray(t, np.float64)


def _i64(t) -> np.ndarray:
    if isinstance(t, torch.Tensor):
        return t.detach().to("cpu").to(torch.int64).numpy()
    return np.asarray(t, np.int64)


def n_blocks(seq_lens, page: int) -> np.ndarray:
    L = _i64(seq_lens)
    return np.where(L <= 0, 0, (L + page - 1) // page)


def page_summary(k_cache, page_table, seq_lens) -> np.ndarray:
    """Mean key of each referenced page's valid tokens: [num_pages, Hkv, d]
    float64.  Pages no sequence references are NaN."""
    k = _f64(k_cache)                       # [num_pages, Hkv, page, d]
    pt, L = _i64(page_table), _i64(seq_lens)
    num_pages, Hkv, page, d = k.shape
    out = np.full((num_pages, Hkv, d), np.nan)
    N = n_blocks(L, page)
    for b in range(pt.shape[0]):
        for j in range(int(N[b])):
            p = int(pt[b, j])
            n = min(page, int(L[b]) - j * page)
            acc = np.zeros((Hkv, d))
            for t in range(n):
                acc += k[p, :, t, :]
            out[p] = acc / n
    return out


def block_scores(q, summary, page_table, seq_lens, page: int, scale: float) -> np.ndarray:
    """Importance score of every block: [B, max_blocks] float64, -inf past N_b."""
    qq = _f64(q)                            # [B, Hq, d]
    kb = _f64(summary)                      # [num_pages, Hkv, d]
    pt = _i64(page_table)
    B, Hq, d = qq.shape
    Hkv = kb.shape[1]
    G = Hq // Hkv
    N = n_blocks(seq_lens, page)
    s = np.full(pt.shape, -np.inf)
    for b in range(B):
        for j in range(int(N[b])):
            p = int(pt[b, j])
            tot = 0.0
            for i in range(Hq):
                tot += float(np.dot(qq[b, i], kb[p, i // G]))
            s[b, j] = scale * tot
    return s


def importance_order(scores, seq_lens, page: int) -> np.ndarray:
    """Block 0, then blocks 1..N_b-1 by decreasing score (ties: larger index
    first), then -1: [B, max_blocks] int32."""
    s = _f64(scores)
    N = n_blocks(seq_lens, page)
    B, max_blocks = s.shape
    order = np.full((B, max_blocks), -1, np.int32)
    for b in range(B):
        n = int(N[b])
        if n == 0:
            continue
        rest = sorted(range(1, n), key=lambda j: (-s[b, j], -j))
        order[b, :n] = [0] + rest
    return order


def importance_walk_order(q, k_cache, page_table, seq_lens, scale: float) -> np.ndarray:
    """The three steps above in a row, from the cache itself."""
    page = int(k_cache.shape[2])
    kb = page_summary(k_cache, page_table, seq_lens)
    return importance_order(block_scores(q, kb, page_table, seq_lens, page, scale), seq_lens, page)
