"""GPU parity of the walks with a dedicated merge CTA: merge_cta = 1 (the
first CTA of each cluster holds the block states and merges them in three
overlapping stages: share warp, fold warps, a decision warp one batch
behind; the others fetch and compute) and merge_cta = 2 (the same merge, the
states handed over through a workspace in global memory instead of a
cluster).  Stops and outputs must follow the same sequential rule as every
other launch shape (ART explainer, Technical Summary 2.1-2.3)."""
import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import make_custom, make_workload
from tests import parity
from tests.test_gpu_parity import assert_fetch_bound, run_gpu

pytestmark = pytest.mark.gpu

MODES = ["cluster", "workspace"]


def mode_kw(art, w, mode, **extra):
    """Options selecting the walk: merge_cta 1, or 2 with a fresh workspace
    of the size art_workspace_bytes asks for (filled with garbage: it needs
    no clearing)."""
    if mode == "cluster":
        return dict(merge_cta=1, **extra)
    g = w.to("cuda")
    n = art.art_workspace_bytes(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens, merge_cta=2,
                                **{k: v for k, v in extra.items() if k in ("cluster_size", "compute_warps", "stages")})
    assert n > 0
    ws = torch.randint(-2 ** 31, 2 ** 31 - 1, ((n + 3) // 4,), dtype=torch.int32, device="cuda")
    return dict(merge_cta=2, workspace=ws, **extra)


def _case(seed, G, lens, **kw):
    base = dict(keys="recency", planted=3, planted_gain=5.0, order="random", eps_m=2e-2, eps_d=2e-3,
                P=[1, 2, 3, 0, 2, 1, 4, 2][:len(lens)], min_blocks=[1, 3, 0, 1, 2, 1, 5, 1][:len(lens)],
                spare_pages=5)
    base.update(kw)
    return make_custom(B=len(lens), Hq=G * 2, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=lens, seed=seed, **base)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("G", [4, 7, 8, 3])
@pytest.mark.parametrize("cluster", [2, 3, 5])
def test_merge_cta_random(cuda_lib, G, cluster, mode):
    """Ragged lengths (partial pages, an empty sequence, one block), random
    orders, planted keys so walks stop mid-way: against the oracle, and equal
    to the one-kernel walk wherever both stops agree."""
    rng = np.random.default_rng(900 + G + 10 * cluster)
    lens = [int(x) for x in rng.integers(1, 3000, size=3)] + [0, 64 * 3, 1, 64 * 40 + 5]
    w = _case(900 + G, G, lens)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **mode_kw(cuda_lib, w, mode, cluster_size=cluster))
    assert status == 0 and info["merge_cta"] == (1 if mode == "cluster" else 2) and info["cluster_size"] == cluster
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    assert stop[3].tolist() == [0, 0] and (out[3] == 0).all()
    out1, stop1, _, status1, info1 = run_gpu(cuda_lib, w, merge_cta=-1)
    assert status1 == 0 and info1["merge_cta"] == 0
    same = (stop == stop1).all(dim=1)
    assert torch.equal(out[same], out1[same])


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("window", [8, 16, 24, 48, 80, 128])
def test_merge_cta_windows(cuda_lib, window, mode):
    """Any window from one merge batch to 128 blocks (past the 48-slot ring: states wait for their slot): the same stops and
    outputs, and never more pages fetched past the stop than the window."""
    w = _case(950, 7, [64 * 90 + 7, 64 * 40, 1, 64 * 130 + 32])
    out0, stop0, _, status0, _ = run_gpu(cuda_lib, w, **mode_kw(cuda_lib, w, mode, cluster_size=4))
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **mode_kw(cuda_lib, w, mode, cluster_size=4, window=window))
    assert status0 == 0 and status == 0 and info["window"] == window
    assert torch.equal(stop, stop0) and torch.equal(out, out0)
    assert_fetch_bound(w, stop, fetched, window)
    parity.check(w, out, stop)


@pytest.mark.parametrize("mode", MODES)
def test_merge_cta_eps0_is_full_attention(cuda_lib, mode):
    w = make_custom(B=3, Hq=28, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[5000, 64, 777], seed=951,
                    eps_m=0.0, eps_d=0.0, P=1)
    kw = mode_kw(cuda_lib, w, mode, cluster_size=6)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **kw)
    N = w.n_blocks().numpy()[:, None]
    assert status == 0 and (stop.cpu().numpy() == N).all() and (fetched.cpu().numpy() == N).all()
    parity.check(w, out, stop)
    # the walk built without the detector gives the same output bit for bit
    out2, stop2, _, status2, info2 = run_gpu(cuda_lib, w, detector_off=1, **kw)
    assert status2 == 0 and info2 == info and torch.equal(stop2, stop) and torch.equal(out2, out)


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("P,minb", [(0, 0), (1, 1), (3, 2), (6, 1), (2, 50), (9, 3)])
def test_merge_cta_constant_values(cuda_lib, P, minb, mode):
    """Constant values: stop = min(N, max(min_blocks, P + 1)), out = v -- also
    where the stop falls in either of the two batches still undecided."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 20 + 5, 64 * 3], seed=952,
                    value="constant", eps_m=1e-4, eps_d=1e-5, P=P, min_blocks=minb)
    out, stop, _, status, _ = run_gpu(cuda_lib, w, **mode_kw(cuda_lib, w, mode, cluster_size=3))
    N = w.n_blocks().numpy()
    for b in range(2):
        assert (stop[b].cpu().numpy() == min(N[b], max(minb, P + 1))).all()
    parity.check(w, out, stop)


@pytest.mark.parametrize("mode", MODES)
def test_merge_cta_bad_index_and_timeout(cuda_lib, mode):
    """A bad page entry ends that unit with stop -1 and the bad-index status;
    the decision warp's bounded wait on a barrier nothing arrives on ends the
    call with the timeout status and leaves the context usable."""
    w = _case(953, 4, [1000, 1000, 500])
    g = w.to("cuda")
    kw = mode_kw(cuda_lib, w, mode, cluster_size=3)
    g.page_table[0, 3] = 10 ** 6
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d,
                                                 P_per_seq=g.P, min_blocks_per_seq=g.min_blocks,
                                                 device_status=status, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == -8 and stop[0].tolist() == [-1, -1]
    parity.check(parity.subset_sequences(w, [1, 2]), out[1:], stop[1:])
    status.zero_()
    g.page_table[0, 3] = int(w.page_table[0, 3])
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m=1e-3, eps_d=1e-4, P=2, min_blocks=1,
                                                 device_status=status, timeout_ns=20_000_000, debug_flags=1, **kw)
    torch.cuda.synchronize()
    assert int(status.item()) == -7 and (stop == -1).all()
    w2 = _case(954, 4, [700, 300])
    out2, stop2, _, status2, _ = run_gpu(cuda_lib, w2, **mode_kw(cuda_lib, w2, mode, cluster_size=3))
    assert status2 == 0
    parity.check(w2, out2, stop2)


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


@pytest.mark.parametrize("mode", MODES)
def test_qwen7b_b4_merge_cta_full_size(cuda_lib, mode):
    """The few-unit long-context workload with a dedicated merge CTA, against
    the one-kernel walk: every unit against the oracle, and the layouts agree."""
    w = make_workload("qwen7b_b4", device="cuda")
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **mode_kw(cuda_lib, w, mode))
    assert status == 0 and info["merge_cta"] == (1 if mode == "cluster" else 2)
    parity.check(w.to("cpu"), out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    out1, stop1, _, status1, _ = run_gpu(cuda_lib, w, merge_cta=-1)
    same = (stop == stop1).all(dim=1)
    assert int(same.sum()) >= w.B - 1
    assert torch.equal(out[same], out1[same])


def test_workspace_reused_across_calls(cuda_lib):
    """One workspace serves call after call without clearing: the words a
    call leaves behind carry its epoch and are never taken for a later
    call's.  Two different batches alternate through the same workspace."""
    wa = _case(960, 7, [64 * 90 + 7, 64 * 40, 1, 64 * 130 + 32])
    wb = _case(961, 7, [64 * 70, 64 * 200 + 9, 64 * 5, 3])
    kw = mode_kw(cuda_lib, wa, "workspace", cluster_size=4)
    kw_b = dict(kw)
    ref = {}
    for name, w in (("a", wa), ("b", wb)):
        out, stop, _, status, _ = run_gpu(cuda_lib, w, merge_cta=1, cluster_size=4)
        assert status == 0
        ref[name] = (out, stop)
    for it in range(3):
        for name, w in (("a", wa), ("b", wb)):
            out, stop, fetched, status, info = run_gpu(cuda_lib, w, **kw_b)
            assert status == 0 and info["merge_cta"] == 2
            same = (stop == ref[name][1]).all(dim=1)
            assert int(same.sum()) >= w.B - 1
            assert torch.equal(out[same], ref[name][0][same])
            parity.check(w, out, stop)


def test_workspace_size_rules(cuda_lib):
    """The size query and its limits: the walk fits a smaller workspace with
    a smaller ring (at least 16 slots per unit), refuses one too small, and
    without a workspace the automatic choice is the cluster walk."""
    w = _case(962, 4, [3000, 2000, 500])
    g = w.to("cuda")
    n = cuda_lib.art_workspace_bytes(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens, merge_cta=2,
                                     cluster_size=3)
    assert n > 0
    small = torch.empty(n // 4 // 3, dtype=torch.int32, device="cuda")
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, merge_cta=2, cluster_size=3, workspace=small)
    assert status == 0 and info["merge_cta"] == 2 and 16 <= info["ring_slots"] < 128
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    tiny = torch.empty(64, dtype=torch.int32, device="cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        run_gpu(cuda_lib, w, merge_cta=2, cluster_size=3, workspace=tiny)
    assert e.value.status == -2
    with pytest.raises(cuda_lib.ArtError) as e:
        run_gpu(cuda_lib, w, merge_cta=2)
    assert e.value.status == -1
    # many units: the workspace walk does not apply and the size query says so
    wm = make_workload("llama8b_b32", device="cuda")
    assert cuda_lib.art_workspace_bytes(wm.q, wm.k_cache, wm.v_cache, wm.page_table, None, wm.seq_lens) == 0


@pytest.mark.parametrize("mode", MODES)
@pytest.mark.parametrize("G", [4, 8])
def test_single_unit_largest_cluster(cuda_lib, G, mode):
    """One (sequence, kv-head) unit: the automatic launch gives the dedicated
    merge CTA the largest cluster that fits (sixteen CTAs, fifteen fetching),
    or, through a workspace, every other CTA of the GPU.  A long sequence with
    planted keys stops mid-way; the same cache at eps = 0 is full attention.
    Both against the oracle."""
    L = 64 * 700 + 23
    w = make_custom(B=1, Hq=G, Hkv=1, d=128, page=64, dtype="bf16", seq_lens=[L], seed=970 + G, keys="recency",
                    planted=3, planted_gain=5.0, order="random", eps_m=2e-3, eps_d=2e-4, P=3, min_blocks=2)
    kw = {} if mode == "cluster" else mode_kw(cuda_lib, w, mode)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **kw)
    assert status == 0 and info["merge_cta"] == (1 if mode == "cluster" else 2) and info["cluster_size"] >= 8
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
    w0 = w.to("cpu")
    w0.eps_m, w0.eps_d = torch.zeros(1), torch.zeros(1)
    out0, stop0, fetched0, status0, info0 = run_gpu(cuda_lib, w0, **kw)
    assert status0 == 0 and int(stop0.item()) == int(w.n_blocks()[0])
    parity.check(w0, out0, stop0)


@pytest.mark.parametrize("mode", MODES)
def test_short_units_largest_cluster(cuda_lib, mode):
    """Very short sequences (1 to 9 blocks) on the largest clusters: most
    fetching CTAs get no block at all; stops and outputs as the oracle's."""
    lens = [1, 64, 65, 64 * 3 + 1, 64 * 5, 64 * 9 - 7]
    w = make_custom(B=len(lens), Hq=8, Hkv=1, d=128, page=64, dtype="bf16", seq_lens=lens, seed=975,
                    keys="recency", planted=1, planted_gain=4.0, order="random", eps_m=5e-3, eps_d=5e-4, P=1,
                    min_blocks=1)
    kw = {} if mode == "cluster" else mode_kw(cuda_lib, w, mode)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, **kw)
    assert status == 0 and info["merge_cta"] == (1 if mode == "cluster" else 2)
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"])
