"""GPU parity of several query tokens sharing one walk (art_decode_attention_multi).

Each token's result is defined as its own single-query ART walk, so every
token is checked against the oracle run on that token alone (the same
admissible-stop and output-tolerance rule as the single-query tests); the
shared walk must read no page past the latest token's stop plus the window.
"""
import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import draft_queries, make_custom, token_view
from tests import parity

pytestmark = pytest.mark.gpu


def run_multi(art, w, q_multi, **kw):
    g = w.to("cuda")
    qm = q_multi.to("cuda")
    fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    opts = dict(eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d, P_per_seq=g.P, min_blocks_per_seq=g.min_blocks)
    opts.update(kw)
    out, stop, info = art.art_decode_attention_multi(qm, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                     g.seq_lens, blocks_fetched=fetched, device_status=status,
                                                     want_info=True, **opts)
    torch.cuda.synchronize()
    return out, stop, fetched.view(w.B, w.Hkv), int(status.item()), info


def check_tokens(w, qm, out, stop, fetched, window):
    """Every token against the oracle on that token alone; fetch bound on the shared walk."""
    T = qm.shape[1]
    for t in range(T):
        parity.check(token_view(w, qm, t).to("cpu"), out[:, t], stop[:, t])
    N = w.n_blocks().numpy()[:, None]
    latest = stop.cpu().numpy().max(axis=1)               # [B, Hkv]
    fe = fetched.cpu().numpy()
    assert (fe >= latest).all()
    assert (fe <= np.minimum(N, latest + window)).all()


CASES = [
    # (seed, dtype, G, page, cluster)
    (300, "bf16", 4, 64, 0), (301, "bf16", 4, 16, 1), (302, "bf16", 2, 64, 2), (303, "bf16", 1, 16, 3),
    (304, "bf16", 3, 64, 1), (305, "f32", 4, 16, 0), (306, "f32", 1, 16, 2), (307, "f32", 3, 64, 1),
]


@pytest.mark.parametrize("seed,dtype,G,page,cluster", CASES)
def test_two_tokens_parity(cuda_lib, seed, dtype, G, page, cluster):
    """Ragged lengths (an empty sequence, partial pages), random orders,
    planted heavy hitters so the walks stop mid-way; the second token is the
    first plus noise, so the two tokens stop at different blocks."""
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in rng.integers(1, 40 * page, size=3)] + [0, page * 3, 1]
    w = make_custom(B=len(lens), Hq=G * 2, Hkv=2, d=128, page=page, dtype=dtype, seq_lens=lens, seed=seed,
                    keys="recency", planted=3, planted_gain=5.0, order="random" if seed % 2 else "sink_recency",
                    eps_m=2e-2, eps_d=2e-3, P=[1, 2, 3, 0, 2, 1], min_blocks=[1, 3, 0, 1, 2, 1], spare_pages=5)
    qm = draft_queries(w, 2, spread=0.7, seed=seed)
    out, stop, fetched, status, info = run_multi(cuda_lib, w, qm, cluster_size=cluster)
    assert status == 0
    check_tokens(w, qm, out, stop, fetched, info["window"] + info["prefetch"])
    assert stop[3].tolist() == [[0, 0], [0, 0]] and (out[3] == 0).all()


def test_tokens_stop_apart(cuda_lib):
    """A workload where the tokens' stops differ in most units, so a token is
    frozen while the walk goes on for the other, inside a batch and across
    batches."""
    w = make_custom(B=4, Hq=8, Hkv=2, d=128, page=16, dtype="bf16", seq_lens=[16 * 200, 16 * 150 + 3, 900, 16 * 64],
                    seed=41, keys="recency", planted=4, planted_gain=5.0, order="sink_recency",
                    eps_m=1e-2, eps_d=1e-3, P=2, min_blocks=1)
    qm = draft_queries(w, 2, spread=1.5, seed=41)
    out, stop, fetched, status, info = run_multi(cuda_lib, w, qm)
    assert status == 0
    s = stop.cpu()
    assert (s[:, 0] != s[:, 1]).sum() >= 2, s
    check_tokens(w, qm, out, stop, fetched, info["window"] + info["prefetch"])


def test_identical_tokens_agree_bitwise(cuda_lib):
    """Two copies of the same query: the same stop and bit-identical outputs."""
    w = make_custom(B=3, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[3000, 64, 777], seed=9, planted=3,
                    planted_gain=5.0, eps_m=5e-3, eps_d=5e-4, P=2)
    qm = torch.stack([w.q, w.q], dim=1)
    out, stop, fetched, status, _ = run_multi(cuda_lib, w, qm)
    assert status == 0
    assert torch.equal(stop[:, 0], stop[:, 1]) and torch.equal(out[:, 0], out[:, 1])
    parity.check(w, out[:, 0], stop[:, 0])


@pytest.mark.parametrize("P,minb", [(0, 0), (1, 1), (3, 2), (2, 50)])
def test_constant_values_closed_form(cuda_lib, P, minb):
    """Constant values: every token stops at min(N, max(min_blocks, P+1)) (P = 0: max(min_blocks, 1)), out = v."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 20 + 5, 64 * 3], seed=8,
                    value="constant", eps_m=1e-4, eps_d=1e-5, P=P, min_blocks=minb)
    qm = draft_queries(w, 2, seed=8)
    out, stop, fetched, status, info = run_multi(cuda_lib, w, qm)
    assert status == 0
    N = w.n_blocks().numpy()
    for b in range(2):
        assert (stop[b].cpu().numpy() == min(N[b], max(minb, P + 1))).all()
    check_tokens(w, qm, out, stop, fetched, info["window"] + info["prefetch"])


def test_full_attention_eps0(cuda_lib):
    """eps = 0: both tokens read everything and get plain softmax attention."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[3000, 777], seed=7,
                    eps_m=0.0, eps_d=0.0, P=1)
    qm = draft_queries(w, 2, seed=7)
    out, stop, fetched, status, info = run_multi(cuda_lib, w, qm)
    N = w.n_blocks().numpy()[:, None, None]
    assert status == 0 and (stop.cpu().numpy() == N).all()
    check_tokens(w, qm, out, stop, fetched, info["window"] + info["prefetch"])


def test_one_token_equals_single_query(cuda_lib):
    """n_queries = 1 on [B, 1, Hq, d] tensors is the single-query call, bit for bit."""
    w = make_custom(B=3, Hq=16, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[3000, 64, 777], seed=21,
                    planted=3, planted_gain=5.0, eps_m=5e-3, eps_d=5e-4, P=2)
    g = w.to("cuda")
    kw = dict(eps_m=5e-3, eps_d=5e-4, P=2, min_blocks=1)
    o1, s1 = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order, g.seq_lens,
                                              **kw)
    o2, s2 = cuda_lib.art_decode_attention_multi(g.q.unsqueeze(1), g.k_cache, g.v_cache, g.page_table,
                                                 g.block_order, g.seq_lens, **kw)
    torch.cuda.synchronize()
    assert o2.shape == (3, 1, 16, 128) and s2.shape == (3, 1, 4)
    assert torch.equal(o2[:, 0], o1) and torch.equal(s2[:, 0], s1)


def test_shared_walk_reads_once(cuda_lib):
    """Full attention on a long cache: the shared walk fetches every page once
    for both tokens (fetched = N per unit, not 2N)."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 300, 64 * 100 + 9], seed=12,
                    eps_m=0.0, eps_d=0.0, P=1)
    qm = draft_queries(w, 2, seed=12)
    out, stop, fetched, status, _ = run_multi(cuda_lib, w, qm)
    N = w.n_blocks().numpy()[:, None]
    assert status == 0 and (fetched.cpu().numpy() == N).all()


def test_unsupported_combinations(cuda_lib):
    w = make_custom(B=1, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[300], seed=1)
    qm = draft_queries(w, 2, seed=1)
    with pytest.raises(cuda_lib.ArtError, match="UNSUPPORTED"):
        run_multi(cuda_lib, w, qm, engine=1)            # bf16 multi-token runs on the tensor-core engine only
    w5 = make_custom(B=1, Hq=10, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[300], seed=1)
    with pytest.raises(cuda_lib.ArtError, match="UNSUPPORTED"):
        run_multi(cuda_lib, w5, draft_queries(w5, 2, seed=1))   # 2 x 5 heads > 8 rows


def test_shared_walk_ignores_stale_shared_memory(cuda_lib):
    """Shared memory filled with NaN, then -inf, before each shared walk:
    padding rows (3 heads per token, 6 of the engine's 8 rows used) are never
    written and must not matter."""
    from tests import smem_poison
    w = make_custom(B=3, Hq=6, Hkv=2, d=128, page=16, dtype="bf16", seq_lens=[700, 333, 1000], seed=61, planted=2,
                    planted_gain=5.0, eps_m=1e-2, eps_d=1e-3, P=2, min_blocks=1)
    qm = draft_queries(w, 2, seed=61)
    wf = make_custom(B=3, Hq=6, Hkv=2, d=128, page=16, dtype="f32", seq_lens=[700, 333, 1000], seed=62, planted=2,
                     planted_gain=5.0, eps_m=1e-2, eps_d=1e-3, P=2, min_blocks=1)
    qf = draft_queries(wf, 2, seed=62)
    for ww, qq in ((w, qm), (wf, qf)):
        for pattern in (smem_poison.NAN, smem_poison.NEG_INF):
            smem_poison.poison(pattern)
            out, stop, fetched, status, info = run_multi(cuda_lib, ww, qq)
            assert status == 0 and torch.isfinite(out).all()
            check_tokens(ww, qq, out, stop, fetched, info["window"] + info["prefetch"])
