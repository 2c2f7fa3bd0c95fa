"""GPU parity: the CUDA path (through the C ABI) against the CPU oracle."""
import math

import numpy as np
import pytest
import torch

from kv_cache_early_art_b200.workloads import make_custom, make_workload, sink_recency_order
from tests import parity

pytestmark = pytest.mark.gpu


def run_gpu(art, w, **kw):
    """Call art_decode_attention_ex on a CUDA copy of w with its per-sequence parameters."""
    g = w.to("cuda")
    fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    opts = dict(eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d, P_per_seq=g.P, min_blocks_per_seq=g.min_blocks)
    opts.update(kw)
    out, stop, info = art.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                  g.seq_lens, blocks_fetched=fetched, device_status=status,
                                                  want_info=True, **opts)
    torch.cuda.synchronize()
    return out, stop, fetched.view(w.B, w.Hkv), int(status.item()), info


def assert_fetch_bound(w, stop, fetched, window):
    """Pages fetched: at least the consumed ones, at most `window` beyond."""
    N = w.n_blocks().cpu().numpy()[:, None]
    st, fe = stop.cpu().numpy(), fetched.cpu().numpy()
    assert (fe >= st).all()
    assert (fe <= np.minimum(N, st + window)).all(), (fe - st).max()


def test_tiny_fp32_config(cuda_lib):
    w = make_workload("tiny_fp32")
    out, stop, fetched, status, info = run_gpu(cuda_lib, w)
    assert status == 0
    s = parity.check(w, out, stop)
    assert s["canonical_mismatch"] == 0
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])


@pytest.mark.parametrize("engine", [1, 2])
def test_llama8b_b8_config(cuda_lib, engine):
    w = make_workload("llama8b_b8")
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, engine=engine)
    assert status == 0 and info["engine"] == engine
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])


SWEEP = []
for i, (dtype, G, d, page) in enumerate([("f32", 1, 64, 16), ("f32", 4, 128, 64), ("f32", 7, 64, 64),
                                         ("f32", 8, 128, 16), ("bf16", 1, 64, 16), ("bf16", 4, 128, 64),
                                         ("bf16", 7, 128, 64), ("bf16", 8, 64, 16), ("bf16", 4, 64, 64),
                                         ("bf16", 3, 128, 16)]):
    for engine in ([1] if dtype == "f32" else [1, 2]):
        for cl in (1, 3):
            SWEEP.append((100 + i, dtype, G, d, page, engine, cl))


@pytest.mark.parametrize("seed,dtype,G,d,page,engine,cluster", SWEEP)
def test_random_sweep(cuda_lib, seed, dtype, G, d, page, engine, cluster):
    """Ragged lengths (partial last pages, an empty sequence), random page
    tables and walk orders, planted heavy hitters so walks stop mid-way."""
    rng = np.random.default_rng(seed)
    lens = [int(x) for x in rng.integers(1, 40 * page, size=3)] + [0, page * 3, 1]
    order = "random" if seed % 2 else "sink_recency"
    w = make_custom(B=len(lens), Hq=G * 2, Hkv=2, d=d, page=page, dtype=dtype, seq_lens=lens, seed=seed,
                    keys="recency", planted=3, planted_gain=5.0, order=order, eps_m=2e-2, eps_d=2e-3,
                    P=[1, 2, 3, 0, 2, 1], min_blocks=[1, 3, 0, 1, 2, 1], spare_pages=5)
    out, stop, fetched, status, info = run_gpu(cuda_lib, w, engine=engine, cluster_size=cluster)
    assert status == 0
    assert info["cluster_size"] == cluster
    s = parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])
    assert stop[3].tolist() == [0, 0] and (out[3] == 0).all()


@pytest.mark.parametrize("engine", [1, 2])
def test_full_attention_eps0(cuda_lib, engine):
    """eps = 0: the walk reads everything and equals plain softmax attention."""
    w = make_custom(B=3, Hq=16, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[3000, 64, 777], seed=7,
                    eps_m=0.0, eps_d=0.0, P=1)
    out, stop, fetched, status, _ = run_gpu(cuda_lib, w, engine=engine)
    N = w.n_blocks().numpy()[:, None]
    assert (stop.cpu().numpy() == N).all() and (fetched.cpu().numpy() == N).all()
    parity.check(w, out, stop)


@pytest.mark.parametrize("P,minb", [(0, 0), (0, 4), (1, 1), (3, 2), (6, 1), (2, 50)])
def test_constant_values_closed_form(cuda_lib, P, minb):
    """Constant values: stop = min(N, max(min_blocks, P+1)) (P = 0: max(min_blocks, 1)), out = v."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[64 * 20 + 5, 64 * 3],
                    seed=8, value="constant", eps_m=1e-4, eps_d=1e-5, P=P, min_blocks=minb)
    out, stop, _, status, _ = run_gpu(cuda_lib, w)
    N = w.n_blocks().numpy()
    for b in range(2):
        assert (stop[b].cpu().numpy() == min(N[b], max(minb, P + 1))).all()
    parity.check(w, out, stop)


def test_sink_order_builder(cuda_lib):
    lens = torch.tensor([0, 1, 64, 65, 1000, 4096], dtype=torch.int32)
    order = cuda_lib.art_build_order_sink_recency(lens.cuda(), 64, max_blocks=70)
    torch.cuda.synchronize()
    N = (lens.long() + 63) // 64
    assert torch.equal(order.cpu(), sink_recency_order(N, 70))


@pytest.mark.parametrize("cluster", [1, 2])
def test_default_order_on_the_fly(cuda_lib, cluster):
    """No block_order: the walk builds sink-then-newest-first itself, and the
    result equals the same walk given that order explicitly, bit for bit."""
    w = make_custom(B=4, Hq=16, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[3000, 64, 777, 1],
                    seed=21, planted=3, planted_gain=5.0, order="sink_recency", eps_m=5e-3, eps_d=5e-4, P=2)
    g = w.to("cuda")
    kw = dict(eps_m=5e-3, eps_d=5e-4, P=2, min_blocks=1, cluster_size=cluster)
    out0, stop0 = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens, **kw)
    out1, stop1 = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                   g.seq_lens, **kw)
    out2, stop2 = cuda_lib.art_decode_attention(g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens,
                                                5e-3, 5e-4, 2, 1)
    torch.cuda.synchronize()
    assert torch.equal(stop0, stop1) and torch.equal(out0, out1)
    assert torch.equal(stop0, stop2) and torch.equal(out0, out2)
    parity.check(w, out0, stop0)


def test_over_pruned_cache(cuda_lib):
    """ART on a StreamingLLM-style pruned cache (sink page + recent window,
    compacted page table): parity with the oracle on the same pruned view."""
    from kv_cache_early_art_b200.workloads import streaming_subset
    base = make_custom(B=3, Hq=16, Hkv=4, d=128, page=64, dtype="bf16", seq_lens=[5000, 700, 130], seed=22,
                       planted=4, planted_gain=5.0, eps_m=5e-3, eps_d=5e-4, P=2)
    w = streaming_subset(base, window_blocks=16)
    assert w.n_blocks().tolist() == [17, 11, 3]
    out, stop, fetched, status, info = run_gpu(cuda_lib, w)
    assert status == 0
    parity.check(w, out, stop)
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])


def test_strided_cache_layout(cuda_lib):
    """Cache stored as [num_pages, page, Hkv, d] and viewed with strides."""
    w = make_custom(B=2, Hq=8, Hkv=2, d=128, page=64, dtype="bf16", seq_lens=[900, 300], seed=9,
                    planted=2, planted_gain=5.0, eps_m=1e-2, eps_d=1e-3, P=2)
    g = w.to("cuda")
    k2 = g.k_cache.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    v2 = g.v_cache.permute(0, 2, 1, 3).contiguous().permute(0, 2, 1, 3)
    assert not k2.is_contiguous()
    out, stop = cuda_lib.art_decode_attention(g.q, k2, v2, g.page_table, g.block_order, g.seq_lens,
                                              1e-2, 1e-3, 2, 1)
    torch.cuda.synchronize()
    parity.check(w, out, stop)


def test_bitwise_deterministic(cuda_lib):
    w = make_workload("llama8b_b8")
    a = run_gpu(cuda_lib, w)
    b = run_gpu(cuda_lib, w)
    assert torch.equal(a[0], b[0]) and torch.equal(a[1], b[1])


def test_bad_index_reported(cuda_lib):
    """An out-of-range page entry and an over-long sequence: the unit gets
    stop -1 and the status word the bad-index code; other units are exact."""
    w = make_custom(B=3, Hq=4, Hkv=1, d=64, page=16, dtype="f32", seq_lens=[100, 100, 40], seed=10,
                    eps_m=1e-3, eps_d=1e-4, P=2)
    g = w.to("cuda")
    g.page_table[0, 3] = 10 ** 6
    g.seq_lens[2] = 16 * w.max_blocks + 1
    fetched = torch.zeros(3, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m=1e-3, eps_d=1e-4, P=2, min_blocks=1,
                                                 blocks_fetched=fetched, device_status=status)
    torch.cuda.synchronize()
    assert int(status.item()) == -8
    assert stop[0, 0].item() == -1 and stop[2, 0].item() == -1
    ok = parity.subset_sequences(w, [1])
    parity.check(ok, out[1:2], stop[1:2])


def test_bounded_wait_expires_cleanly(cuda_lib):
    """debug flag: the stop decision waits on a barrier nothing arrives on.
    The wait gives up after its limit, the call reports a timeout, and the
    context stays usable for the next call."""
    w = make_custom(B=1, Hq=4, Hkv=1, d=64, page=16, dtype="f32", seq_lens=[200], seed=11)
    g = w.to("cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop = cuda_lib.art_decode_attention_ex(g.q, g.k_cache, g.v_cache, g.page_table, g.block_order,
                                                 g.seq_lens, eps_m=1e-3, eps_d=1e-4, P=2, min_blocks=1,
                                                 device_status=status, timeout_ns=20_000_000, debug_flags=1,
                                                 cluster_size=1)
    torch.cuda.synchronize()
    assert int(status.item()) == -7
    assert stop[0, 0].item() == -1
    out2, stop2, *_ = run_gpu(cuda_lib, w)
    parity.check(w, out2, stop2)


def test_invalid_arguments_launch_nothing(cuda_lib):
    w = make_custom(B=1, Hq=4, Hkv=2, d=64, page=16, dtype="bf16", seq_lens=[50], seed=12).to("cuda")
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention(w.q, w.k_cache, w.v_cache, w.page_table, w.block_order, w.seq_lens,
                                      float("nan"), 1e-3, 2, 1)
    assert e.value.status == -5
    with pytest.raises(cuda_lib.ArtError) as e:
        cuda_lib.art_decode_attention(w.q.float(), w.k_cache, w.v_cache, w.page_table, w.block_order,
                                      w.seq_lens, 1e-3, 1e-3, 2, 1)
    assert e.value.status == -3


# ------------------------------------------------------------ full sizes ----

def _full(art, name, seqs=None, engine=0, **params):
    """A named workload at its full size, in the launch configuration the
    bench times (library-chosen shape, default order built inside the walk):
    every unit (or the listed sequences) against the oracle.  params
    overrides the per-sequence thresholds / patience (scalars)."""
    torch.manual_seed(0)
    w = make_workload(name, device="cuda")
    for key, val in params.items():
        dt = torch.int32 if key in ("P", "min_blocks") else torch.float32
        setattr(w, key, torch.full((w.B,), val, dtype=dt, device="cuda"))
    g = w
    fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device="cuda")
    status = torch.zeros(1, dtype=torch.int32, device="cuda")
    out, stop, info = art.art_decode_attention_ex(
        g.q, g.k_cache, g.v_cache, g.page_table, None, g.seq_lens, eps_m_per_seq=g.eps_m, eps_d_per_seq=g.eps_d,
        P_per_seq=g.P, min_blocks_per_seq=g.min_blocks, blocks_fetched=fetched, device_status=status,
        engine=engine, want_info=True)
    torch.cuda.synchronize()
    assert int(status.item()) == 0
    fetched = fetched.view(w.B, w.Hkv)
    if seqs is None:
        wc, o, st = w.to("cpu"), out, stop
    else:
        wc = parity.subset_sequences(w, seqs)
        idx = torch.as_tensor(seqs)
        o, st = out[idx], stop[idx]
    s = parity.check(wc, o, st)
    assert_fetch_bound(w, stop, fetched, info["window"] + info["prefetch"])
    return s, w, stop


def test_llama8b_b32_full_size(cuda_lib):
    """Every one of the 256 units of the B=32, L=32768 batch."""
    _full(cuda_lib, "llama8b_b32")


def test_llama8b_b32_eps0_full_size(cuda_lib):
    """The full-attention companion of the same batch (eps_m = eps_d = 0):
    every unit walks all 512 blocks and equals the oracle's full softmax."""
    s, w, stop = _full(cuda_lib, "llama8b_b32", eps_m=0.0, eps_d=0.0)
    N = w.n_blocks().cpu().numpy()[:, None]
    assert (stop.cpu().numpy() == N).all()
    assert s["blocks_consumed"] == s["blocks_total"]


def test_qwen7b_b4_full_size(cuda_lib):
    _full(cuda_lib, "qwen7b_b4")


def test_mistral7b_b128_full_size(cuda_lib):
    """Every one of the 1024 units of the ragged B=128 batch, per-sequence
    thresholds and patience."""
    _full(cuda_lib, "mistral7b_b128")


def test_llama8b_b8_full_size_default_order(cuda_lib):
    _full(cuda_lib, "llama8b_b8")


SHAPES = {
    # (cluster, compute warps, stages, window): every (warps, stages) pairing
    # the launch accepts, from the smallest ring to the deepest window
    "bf16": [(1, 1, 2, 8), (2, 2, 2, 16), (2, 3, 3, 24), (2, 4, 4, 24), (2, 5, 5, 28), (3, 2, 4, 16),
             (4, 1, 2, 8), (2, 2, 4, 32)],
    "f32": [(1, 1, 2, 8), (2, 5, 5, 28), (2, 6, 6, 16), (2, 3, 6, 16), (3, 2, 4, 24), (2, 4, 8, 16)],
}


@pytest.mark.parametrize("dtype,engine", [("bf16", 2), ("bf16", 1), ("f32", 1)])
def test_launch_shapes(cuda_lib, dtype, engine):
    """Explicit launch shapes: the stop and the output do not depend on how
    the walk is spread over CTAs, warps, stages and the window (block states
    are exact per block and the merge folds fixed batches in walk order), so
    every shape equals the library's own choice bit for bit, and that one
    matches the oracle."""
    page = 64 if dtype == "bf16" else 16
    w = make_custom(B=4, Hq=12, Hkv=3, d=128, page=page, dtype=dtype,
                    seq_lens=[page * 90 + 7, page * 40, 1, page * 130 + page // 2], seed=31, planted=3,
                    planted_gain=5.0, order="random", eps_m=5e-3, eps_d=5e-4, P=[2, 1, 3, 2],
                    min_blocks=[1, 2, 1, 4])
    out0, stop0, fetched0, status, info0 = run_gpu(cuda_lib, w, engine=engine)
    assert status == 0
    parity.check(w, out0, stop0)
    ran = 0
    for (cl, nw, st, win) in SHAPES[dtype]:
        try:
            out, stop, fetched, status, info = run_gpu(cuda_lib, w, engine=engine, cluster_size=cl,
                                                       compute_warps=nw, stages=st, window=win)
        except cuda_lib.ArtError as e:
            assert "UNSUPPORTED" in str(e), e     # this shape's ring does not fit in shared memory
            continue
        ran += 1
        assert status == 0
        assert (info["cluster_size"], info["compute_warps"], info["stages"], info["window"]) == (cl, nw, st, win)
        assert torch.equal(stop, stop0), (cl, nw, st, win)
        assert torch.equal(out, out0), (cl, nw, st, win)
        assert_fetch_bound(w, stop, fetched, win + info["prefetch"])
    assert ran >= len(SHAPES[dtype]) - 1


@pytest.mark.parametrize("dtype,G,d,page", [("bf16", 3, 128, 16), ("f32", 7, 64, 64), ("f32", 3, 128, 16),
                                            ("bf16", 7, 128, 64)])
def test_stale_shared_memory_is_ignored(cuda_lib, dtype, G, d, page):
    """Every SM's shared memory is filled with NaN (then -inf) right before
    the walk: a block state's padding rows (G below the engine's row count)
    are never written, and the result must not depend on what they hold."""
    from tests import smem_poison
    rng = np.random.default_rng(500 + G)
    lens = [int(x) for x in rng.integers(1, 40 * page, size=3)] + [page * 3, 1]
    w = make_custom(B=len(lens), Hq=G * 2, Hkv=2, d=d, page=page, dtype=dtype, seq_lens=lens, seed=500 + G,
                    keys="recency", planted=3, planted_gain=5.0, order="random", eps_m=2e-2, eps_d=2e-3,
                    P=[1, 2, 3, 2, 1], min_blocks=[1, 3, 0, 2, 1])
    for engine in ([1] if dtype == "f32" else [1, 2]):
        for pattern in (smem_poison.NAN, smem_poison.NEG_INF):
            smem_poison.poison(pattern)
            out, stop, fetched, status, info = run_gpu(cuda_lib, w, engine=engine)
            assert status == 0
            parity.check(w, out, stop)
            assert torch.isfinite(out).all()
