"""GPU parity of the walk with a dedicated merge CTA (merge_cta = 1): the
first CTA of each cluster holds the block states and merges them in two
overlapping stages (fold warps, then a decision warp one batch behind), the
others fetch and compute.  Stops and outputs must follow the same sequential
rule as every other launch shape (ART explainer, Technical Summary 2.1-2.3)."""
import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import make_custom, make_workload
from tests import parity
from tests.test_gpu_parity import assert_fetch_bound, run_gpu

pytestmark = pytest.mark.gpu


def _case(seed, G, lens, **kw):
    base = dict(keys="recency", planted=3, planted_gain=5.0, order="random", eps_m=2e-2, eps_d=2e-3,
                P=[1, 2, 3, 0, 2, 1, 4, 2][:len(lens)], min_blocks=[1, 3, 0, 1, 2, 1, 5, 1][:len(lens)],
                spare_pages=5)
    base.update(kw)
    return make_custom(B=len(lens), Hq=G * 2, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=lens, seed=seed, **base)


@pytest.mark.parametrize("G", [4, 7, 8, 3])
@pytest.mark.parametrize("cluster", [2, 3, 5])
def test_merge_cta_random(cuda_lib, G, cluster):
    """Ragged lengths (partial pages, an empty sequence, one block), random
    orders, planted keys so walks stop mid-way: against the oracle, and equal
    to the one-kernel walk wherever both stops agree."""
    rng = np.random.default_rng(900 + G + 10 * cluster)
    lens = [int(x) for x in rng.integers(1, 3000, size=3)] + [0, 64 * 3, 1, 64 * 40 + 5]
    w = _case(900 + G, G, lens)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=cluster)
    assert status == 0 and info["merge_cta"] == 1 and info["cluster_size"] == cluster
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    assert stop[3].tolist() == [0, 0] and (out[3] == 0).all()
    out1, stop1, _, status1, info1 = run_gpu(cuda_lib, w, merge_cta=-1)
    assert status1 == 0 and info1["merge_cta"] == 0
    same = (stop == stop1).all(dim=1)
    assert torch.equal(out[same], out1[same])


@pytest.mark.parametrize("window", [8, 16, 24, 48, 80, 128])
def test_merge_cta_windows(cuda_lib, window):
    """Any window from one merge batch to 128 blocks (past the 48-slot ring: states wait for their slot): the same stops and
    outputs, and never more pages fetched past the stop than the window."""
    w = _case(950, 7, [64 * 90 + 7, 64 * 40, 1, 64 * 130 + 32])
    out0, stop0, _, status0, _ = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=4)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=4, window=window)
    assert status0 == 0 and status == 0 and info["window"] == window
    assert torch.equal(stop, stop0) and torch.equal(out, out0)
    assert_fetch_bound(w, stop, fetched, window)
    parity.check(w, out, stop)


def test_merge_cta_eps0_is_full_attention(cuda_lib):
    w = make_custom(B=3, Hq=28, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[5000, 64, 777], seed=951,
                    eps_m=0.0, eps_d=0.0, P=1)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=6)
    N = w.n_blocks().numpy()[:, None]
    assert status == 0 and (stop.cpu().numpy() == N).all() and (fetched.cpu().numpy() == N).all()
    parity.check(w, out, stop)
    # the walk built without the detector gives the same output bit for bit
    out2, stop2, _, status2, info2 = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=6, detector_off=1)
    assert status2 == 0 and info2 == info and torch.equal(stop2, stop) and torch.equal(out2, out)


@pytest.mark.parametrize("P,minb", [(0, 0), (1, 1), (3, 2), (6, 1), (2, 50), (9, 3)])
def test_merge_cta_constant_values(cuda_lib, P, minb):
    """Constant values: stop = min(N, max(min_blocks, P + 1)), out = v -- also
    where the stop falls in either of the two batches still undecided."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 20 + 5, 64 * 3], seed=952,
                    value="constant", eps_m=1e-4, eps_d=1e-5, P=P, min_blocks=minb)
    out, stop, _, status, _ = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=3)
    N = w.n_blocks().numpy()
    for b in range(2):
        assert (stop[b].cpu().numpy() == min(N[b], max(minb, P + 1))).all()
    parity.check(w, out, stop)


def test_merge_cta_bad_index_and_timeout(cuda_lib):
    """A bad page entry ends that unit with stop -1 and the bad-index status;
    the decision warp's bounded wait on a barrier nothing arrives on ends the
    call with the timeout status and leaves the context usable."""
    w = _case(953, 4, [1000, 1000, 500])
    g = w.to("cuda")
    g.page_table[0, 3] = 10 ** 6
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d,
                                                 P_per_seq=g.P, min_blocks_per_seq=g.min_blocks,
                                                 device_status=status, merge_cta=1, cluster_size=3)
    torch.cuda.synchronize()
    assert int(status.item()) == -8 and stop[0].tolist() == [-1, -1]
    parity.check(parity.subset_sequences(w, [1, 2]), out[1:], stop[1:])
    status.zero_()
    g.page_table[0, 3] = int(w.page_table[0, 3])
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m=1e-3, eps_d=1e-4, P=2, min_blocks=1,
                                                 device_status=status, merge_cta=1, cluster_size=3,
                                                 timeout_ns=20_000_000, debug_flags=1)
    torch.cuda.synchronize()
    assert int(status.item()) == -7 and (stop == -1).all()
    out2, stop2, _, status2, _ = run_gpu(cuda_lib, _case(954, 4, [700, 300]), merge_cta=1, cluster_size=3)
    assert status2 == 0


def test_merge_cta_refused_where_not_built(cuda_lib):
    w = make_custom(B=2, Hq=8, Hkv=2, d=64, page=64, dtype="bf16", seq_lens=[300, 200], seed=955).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens, merge_cta=1)
    assert e.value.status == -4
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[300, 200], seed=955).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens, merge_cta=1,
                                         cluster_size=1)
    assert e.value.status == -5


def test_qwen7b_b4_merge_cta_full_size(cuda_lib):
    """The few-unit long-context workload in both layouts: every unit against
    the oracle, and the two layouts agree."""
    w = make_workload("qwen7b_b4", device="cuda")
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, merge_cta=1)
    assert status == 0 and info["merge_cta"] == 1
    parity.check(w.to("cpu"), out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    out1, stop1, _, status1, _ = run_gpu(cuda_lib, w, merge_cta=-1)
    same = (stop == stop1).all(dim=1)
    assert int(same.sum()) >= w.B - 1
    assert torch.equal(out[same], out1[same])
