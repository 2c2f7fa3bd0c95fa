"""Seeded random configurations of the walk against the oracle.

Each seed draws a configuration the library supports -- element type, head
dim, page size, group size, kv heads, batch with ragged lengths (empty
sequences and partial pages included), random or default order, planted
heavy hitters or not, thresholds, patience, min_blocks, engine, cluster size
and sometimes an explicit launch shape -- runs it through the C ABI and holds
it to the same rule as the other parity tests.  Where two tokens fit one
unit (d = 128, 2G <= 8) the same draw also runs as a shared walk of two
tokens, each checked against the oracle on that token alone.
"""
import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import draft_queries, make_custom, token_view
from tests import parity
from tests.test_gpu_parity import assert_fetch_bound, run_gpu

pytestmark = pytest.mark.gpu

SHAPES = [(2, 2, 16), (3, 3, 24), (1, 2, 8), (4, 4, 16), (2, 4, 16)]


def draw(seed):
    rng = np.random.default_rng(1000 + seed)
    dtype = "bf16" if rng.random() < 0.7 else "f32"
    d = int(rng.choice([64, 128]))
    page = int(rng.choice([16, 64]))
    G = int(rng.integers(1, 9))
    Hkv = int(rng.integers(1, 4))
    B = int(rng.integers(1, 6))
    lens = [int(x) for x in rng.integers(0, 50 * page, size=B)]
    if rng.random() < 0.3:
        lens[int(rng.integers(0, B))] = 0
    eps_m = float(10 ** rng.uniform(-3, -1.3))
    eps_d = eps_m / 10 if rng.random() < 0.5 else float(10 ** rng.uniform(-4, -2))
    P = [int(x) for x in rng.integers(0, 5, size=B)]
    minb = [int(x) for x in rng.integers(0, 6, size=B)]
    planted = int(rng.integers(0, 4))
    order = "random" if rng.random() < 0.5 else "sink_recency"
    engine = int(rng.choice([0, 1, 2])) if dtype == "bf16" else int(rng.choice([0, 1]))
    cluster = int(rng.choice([0, 0, 1, 2, 3, 4]))
    shape = SHAPES[int(rng.integers(0, len(SHAPES)))] if rng.random() < 0.3 else None
    w = make_custom(B=B, Hq=G * Hkv, Hkv=Hkv, d=d, page=page, dtype=dtype, seq_lens=lens, seed=2000 + seed,
                    keys="recency", planted=planted, planted_gain=5.0, order=order, eps_m=eps_m, eps_d=eps_d,
                    P=P, min_blocks=minb, spare_pages=int(rng.integers(0, 6)))
    opts = dict(engine=engine, cluster_size=cluster)
    if shape is not None:
        opts.update(compute_warps=shape[0], stages=shape[1], window=shape[2])
    return w, opts


@pytest.mark.parametrize("seed", range(24))
def test_fuzz(cuda_lib, seed):
    w, opts = draw(seed)
    if w.k_cache.shape[0] == 0:
        # every sequence empty and no spare page: a cache without data is a
        # NULL required pointer, refused on the host
        with pytest.raises(cuda_lib.ArtError, match="NULL"):
            run_gpu(cuda_lib, w, **opts)
        return
    try:
        out, stop, fetched, status, info = run_gpu(cuda_lib, w, **opts)
    except cuda_lib.ArtError as e:
        # an explicit shape whose ring does not fit, or the CUDA-core-only
        # element type on the tensor-core engine: refused on the host
        assert "UNSUPPORTED" in str(e), e
        return
    assert status == 0
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])
    if w.d == 128 and 2 * w.G <= 8:       # the shared walk picks its engine by element type
        qm = draft_queries(w, 2, seed=seed)
        g = w.to("cuda")
        st2 = torch.zeros(1, dtype=torch.int32, device="cuda")
        out2, stop2 = cuda_lib.art_decode_attention_multi(
            qm.to("cuda"), g.k_cache, g.v_cache, g.page_table, g.block_order, g.seq_lens, eps_m_per_seq=g.eps_m,
            eps_d_per_seq=g.eps_d, P_per_seq=g.P, min_blocks_per_seq=g.min_blocks, device_status=st2,
            cluster_size=opts["cluster_size"])
        torch.cuda.synchronize()
        assert int(st2.item()) == 0
        for t in range(2):
            parity.check(token_view(w, qm, t), out2[:, t], stop2[:, t])
