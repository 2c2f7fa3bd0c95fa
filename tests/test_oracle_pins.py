"""Pins for the CPU oracle: every check here is independent of the oracle's own
code -- closed forms derived by hand, a direct two-pass softmax attention and
torch's float64 scaled_dot_product_attention, brute-force recomputation of
every prefix, and invariants the method fixes (ART explainer, Technical
Summary section 2.4: permutation invariance of attention, mandatory sink
block; section 2.2: both criteria must hold; section 2.3: patience)."""
import math

import numpy as np
import pytest
import torch

import oracle
from kv_cache_early_art_b200.workloads import make_custom, sink_recency_order

pytestmark = pytest.mark.filterwarnings("ignore::UserWarning")


# ---------------------------------------------------------------- helpers ----

def _f64(t):
    return t.detach().cpu().to(torch.float64)


def direct_attention(w, b, h, blocks=None):
    """Two-pass softmax attention over the tokens of the given logical blocks
    (all blocks when None) of sequence b, kv-head h: [G, d] float64."""
    L = int(w.seq_lens[b])
    page, G, d = w.page, w.G, w.d
    N = (L + page - 1) // page
    blocks = range(N) if blocks is None else blocks
    ks, vs = [], []
    for lb in blocks:
        pp = int(w.page_table[b, lb])
        n = min(page, L - lb * page)
        ks.append(_f64(w.k_cache[pp, h, :n]))
        vs.append(_f64(w.v_cache[pp, h, :n]))
    K = torch.cat(ks)
    V = torch.cat(vs)
    q = _f64(w.q[b, h * G:(h + 1) * G])                     # [G, d]
    logits = (q @ K.T) / math.sqrt(d)                        # [G, T]
    mx = logits.max(dim=1, keepdim=True).values
    e = torch.exp(logits - mx)
    return ((e / e.sum(dim=1, keepdim=True)) @ V).numpy()


def sdpa_attention(w, b, h):
    L = int(w.seq_lens[b])
    page, G, d = w.page, w.G, w.d
    N = (L + page - 1) // page
    pp = w.page_table[b, :N].long()
    K = _f64(w.k_cache[pp, h]).reshape(N * page, d)[:L]
    V = _f64(w.v_cache[pp, h]).reshape(N * page, d)[:L]
    q = _f64(w.q[b, h * G:(h + 1) * G])
    o = torch.nn.functional.scaled_dot_product_attention(q[None, :, None, :].transpose(1, 1).reshape(1, G, 1, d),
                                                         K.expand(1, G, L, d), V.expand(1, G, L, d))
    return o.reshape(G, d).numpy()


def rand_w(seed, *, G=4, Hkv=2, d=16, page=4, lens=(37, 16, 5), dtype="f32", order="random", **kw):
    return make_custom(B=len(lens), Hq=G * Hkv, Hkv=Hkv, d=d, page=page, dtype=dtype, seq_lens=list(lens),
                       seed=seed, keys=kw.pop("keys", "recency"), order=order, **kw)


# ------------------------------------------------- attention arithmetic ----

@pytest.mark.parametrize("seed,dtype,G", [(0, "f32", 1), (1, "f32", 4), (2, "bf16", 4), (3, "bf16", 7), (4, "f32", 8)])
def test_eps0_is_full_attention(seed, dtype, G):
    """eps_m = eps_d = 0: nothing is ever stable, so the walk consumes every
    block and the output is plain softmax attention over the whole sequence."""
    w = rand_w(seed, G=G, dtype=dtype, lens=(37, 16, 5, 64), planted=3)
    r = oracle.run(w, eps_m=0.0, eps_d=0.0)
    N = w.n_blocks().numpy()
    assert (r.stop == N[:, None]).all()
    for b in range(w.B):
        for h in range(w.Hkv):
            ref = direct_attention(w, b, h)
            got = r.out[b, h * w.G:(h + 1) * w.G]
            assert np.abs(got - ref).max() <= 1e-12
            assert np.abs(got - sdpa_attention(w, b, h)).max() <= 1e-12


def test_single_block_cache():
    """A cache of one block: stop = 1 and out = softmax(q K^T / sqrt(d)) V."""
    w = rand_w(5, G=4, lens=(4, 3, 1), page=4)
    r = oracle.run(w)
    assert (r.stop == 1).all()
    for b in range(w.B):
        for h in range(w.Hkv):
            assert np.abs(r.out[b, h * w.G:(h + 1) * w.G] - direct_attention(w, b, h)).max() <= 1e-12


@pytest.mark.parametrize("seed,dtype", [(6, "f32"), (7, "bf16")])
def test_prefix_outputs_brute_force(seed, dtype):
    """Every prefix of the walk equals full softmax attention over exactly the
    tokens of the blocks walked so far (O(N^2) recomputation, N <= 16)."""
    w = rand_w(seed, G=2, d=8, page=3, lens=(40, 17, 3), dtype=dtype, planted=2)
    N = w.n_blocks().numpy()
    units, ss, refs = [], [], []
    for b in range(w.B):
        order = w.block_order[b, :N[b]].tolist()
        for h in range(w.Hkv):
            for s in range(1, N[b] + 1):
                units.append(b * w.Hkv + h)
                ss.append(s)
                refs.append(direct_attention(w, b, h, order[:s]))
    got = oracle.prefix_out(w, units, ss)
    assert np.abs(got - np.stack(refs)).max() <= 1e-12
    z = oracle.prefix_out(w, [0], [0])
    assert (z == 0).all()


def test_stats_and_stop_from_brute_force_prefixes():
    """The oracle's per-block statistics are those of consecutive brute-force
    prefixes, and its stop is where a direct reading of the rule stops on them."""
    w = rand_w(8, G=2, d=8, page=3, lens=(45, 30), planted=2, eps_m=0.05, eps_d=0.01, P=2, min_blocks=3)
    r = oracle.run(w, want_stats=True)
    N = w.n_blocks().numpy()
    for b in range(w.B):
        order = w.block_order[b, :N[b]].tolist()
        for h in range(w.Hkv):
            o = [direct_attention(w, b, h, order[:s]).ravel() for s in range(1, N[b] + 1)]
            c, stop = 0, None
            for j in range(N[b]):
                if j >= 1:
                    n1, n0 = np.linalg.norm(o[j]), np.linalg.norm(o[j - 1])
                    ds = abs(n1 - n0) / n0
                    dd = max(0.0, 1 - float(o[j] @ o[j - 1]) / (n1 * n0))
                    if j < r.stop[b, h]:      # the oracle walks no further than its stop
                        assert abs(r.ds[b, h, j] - ds) <= 1e-9 * max(ds, 1e-3)
                        assert abs(r.dd[b, h, j] - dd) <= 1e-9 * max(dd, 1e-3)
                    c = c + 1 if (ds < 0.05 and dd < 0.01) else 0
                if stop is None and c >= 2 and j + 1 >= 3:
                    stop = j + 1
            assert r.stop[b, h] == (stop if stop is not None else N[b])


@pytest.mark.parametrize("seed", [9, 10])
def test_permutation_invariance_at_eps0(seed):
    """Section 2.4: attention is invariant to the order blocks are folded in."""
    base = rand_w(seed, G=4, lens=(50, 23), order="sink_recency")
    r0 = oracle.run(base, eps_m=0.0, eps_d=0.0)
    for k in range(3):
        perm = torch.full_like(base.block_order, -1)
        for b in range(base.B):
            n = int(base.n_blocks()[b])
            perm[b, :n] = torch.randperm(n, generator=torch.Generator().manual_seed(100 * seed + k)).to(torch.int32)
        w = base.to("cpu")
        w.block_order = perm
        r = oracle.run(w, eps_m=0.0, eps_d=0.0)
        assert np.abs(r.out - r0.out).max() <= 1e-12


# --------------------------------------------------------- worked examples ----

def _tiny(keys, vals, L, page, order, scale, **par):
    """One sequence, one head, d = 2, identity page table; keys/values given."""
    n = (L + page - 1) // page
    T = n * page
    k = torch.zeros(n, 1, page, 2)
    v = torch.zeros(n, 1, page, 2)
    for t in range(T):
        k[t // page, 0, t % page] = torch.tensor(keys[t], dtype=torch.float32)
        v[t // page, 0, t % page] = torch.tensor(vals[t], dtype=torch.float32)
    w = make_custom(B=1, Hq=1, Hkv=1, d=2, page=page, dtype="f32", seq_lens=[L], seed=0, keys="noise",
                    page_table="identity", order=torch.tensor([order], dtype=torch.int32))
    w.q = torch.tensor([[[1.0, 0.0]]])
    w.k_cache, w.v_cache = k, v
    return oracle.run(w, scale=scale, want_stats=True, **par)


def test_worked_example_masked_tail():
    """Hand-derived.  q = (1,0), scale = ln 2, so a key (a,0) gets weight 2^a.
    Blocks of two tokens, L = 3: t0 k=(0,0) v=(1,0); t1 k=(1,0) v=(0,1);
    t2 k=(2,0) v=(1,1); t3 lies past L (its weight 2^9 must be ignored).
    Order [0,1]: o_0 = (1/3, 2/3), o_1 = (5/7, 6/7);
    d_scale = 3*sqrt(61)/(7*sqrt(5)) - 1, 1 - cos = 1 - 17/sqrt(305).
    Order [1,0]: o_0 = (1,1), o_1 = (5/7, 6/7);
    d_scale = 1 - sqrt(122)/14, 1 - cos = 1 - 11/sqrt(122)."""
    keys = [(0, 0), (1, 0), (2, 0), (9, 0)]
    vals = [(1, 0), (0, 1), (1, 1), (100, 100)]
    r = _tiny(keys, vals, 3, 2, [0, 1], math.log(2), eps_m=0.0, eps_d=0.0)
    assert r.stop[0, 0] == 2
    assert np.allclose(r.out[0, 0], [5 / 7, 6 / 7], rtol=0, atol=1e-14)
    assert math.isclose(r.ds[0, 0, 1], 3 * math.sqrt(61) / (7 * math.sqrt(5)) - 1, rel_tol=1e-12)
    assert math.isclose(r.dd[0, 0, 1], 1 - 17 / math.sqrt(305), rel_tol=1e-10)
    r = _tiny(keys, vals, 3, 2, [1, 0], math.log(2), eps_m=0.0, eps_d=0.0)
    assert np.allclose(r.out[0, 0], [5 / 7, 6 / 7], rtol=0, atol=1e-14)
    assert math.isclose(r.ds[0, 0, 1], 1 - math.sqrt(122) / 14, rel_tol=1e-12)
    assert math.isclose(r.dd[0, 0, 1], 1 - 11 / math.sqrt(122), rel_tol=1e-10)
    # thresholds between the two statistics of the [1,0] walk: scale passes, direction fails
    r = _tiny(keys, vals, 3, 2, [1, 0], math.log(2), eps_m=0.25, eps_d=0.004, P=1, min_blocks=1)
    assert r.stop[0, 0] == 2 and chr(r.flag[0, 0, 1]) == "F"
    r = _tiny(keys, vals, 3, 2, [1, 0], math.log(2), eps_m=0.25, eps_d=0.005, P=1, min_blocks=1)
    assert r.stop[0, 0] == 2 and chr(r.flag[0, 0, 1]) == "T"


def test_worked_example_patience():
    """Hand-derived.  q = 0 (all weights equal), one token per block, identity
    order: o_j is the running mean of v.  v = (2,0),(2,0),(2,3),(2,-1) gives
    o = (2,0),(2,0),(2,1),(2,1/2);
    j=1: d_scale = 0, 1-cos = 0;
    j=2: d_scale = (sqrt(5)-2)/2 ~ 0.1180, 1-cos = 1 - 2/sqrt(5) ~ 0.1056;
    j=3: d_scale = 1 - sqrt(85)/10 ~ 0.0780, 1-cos = 1 - 9/sqrt(85) ~ 0.0238."""
    keys = [(0, 0)] * 4
    vals = [(2, 0), (2, 0), (2, 3), (2, -1)]

    def run(**par):
        return _tiny(keys, vals, 4, 1, [0, 1, 2, 3], 0.0, **par)

    r = run(eps_m=0.0, eps_d=0.0)
    assert math.isclose(r.ds[0, 0, 2], (math.sqrt(5) - 2) / 2, rel_tol=1e-12)
    assert math.isclose(r.dd[0, 0, 2], 1 - 2 / math.sqrt(5), rel_tol=1e-12)
    assert math.isclose(r.ds[0, 0, 3], 1 - math.sqrt(85) / 10, rel_tol=1e-12)
    assert math.isclose(r.dd[0, 0, 3], 1 - 9 / math.sqrt(85), rel_tol=1e-12)
    assert abs(r.ds[0, 0, 1]) <= 1e-15 and abs(r.dd[0, 0, 1]) <= 1e-15
    assert run(eps_m=0.1, eps_d=0.05, P=1, min_blocks=1).stop[0, 0] == 2   # j=1 stable, P=1
    assert run(eps_m=0.1, eps_d=0.05, P=2, min_blocks=1).stop[0, 0] == 4   # j=2 resets the count
    assert run(eps_m=0.12, eps_d=0.11, P=2, min_blocks=1).stop[0, 0] == 3  # j=1,2 stable
    assert run(eps_m=0.12, eps_d=0.11, P=2, min_blocks=4).stop[0, 0] == 4  # min_blocks holds it
    assert run(eps_m=0.12, eps_d=0.10, P=2, min_blocks=1).stop[0, 0] == 4  # direction fails at j=2
    assert run(eps_m=0.11, eps_d=0.11, P=2, min_blocks=1).stop[0, 0] == 4  # scale fails at j=2


# ------------------------------------------------------------ stop rule ----

@pytest.mark.parametrize("P,minb", [(0, 0), (0, 3), (1, 1), (2, 2), (3, 1), (5, 2), (2, 9), (40, 1)])
def test_constant_values_closed_form(P, minb):
    """Every token of a (sequence, kv-head) carries the same value vector, so
    o_j = v for every j and both statistics vanish: the counter grows by one
    per block after the first, and the walk stops at min(N, max(min_blocks, P+1))
    (P = 0: min(N, max(min_blocks, 1))); the output is v."""
    w = rand_w(11, G=4, lens=(64, 23, 4, 1), page=4, value="constant", eps_m=1e-4, eps_d=1e-5, P=P, min_blocks=minb)
    r = oracle.run(w)
    N = w.n_blocks().numpy()
    for b in range(w.B):
        expect = min(N[b], max(minb, P + 1))
        assert (r.stop[b] == expect).all(), (b, r.stop[b], expect)
        for h in range(w.Hkv):
            pp = int(w.page_table[b, 0])
            v = _f64(w.v_cache[pp, h, 0]).numpy()
            assert np.abs(r.out[b, h * w.G:(h + 1) * w.G] - v[None]).max() <= 1e-12


def test_empty_sequences():
    w = rand_w(12, lens=(0, 5, 0))
    r = oracle.run(w)
    assert r.stop[0].tolist() == [0, 0] and r.stop[2].tolist() == [0, 0]
    assert (r.out[0] == 0).all() and (r.out[2] == 0).all()
    assert (r.stop[1] >= 1).all()


def test_sink_block_always_consumed():
    """Section 2.4: block 0 is always evaluated; the default order starts with it."""
    w = rand_w(13, lens=(64, 33, 1), value="constant", order="sink_recency", P=0, min_blocks=0, eps_m=1.0, eps_d=1.0)
    r = oracle.run(w)
    assert (r.stop == 1).all()
    assert (w.block_order[:, 0] == 0).all()
    bo = sink_recency_order(torch.tensor([5, 1, 0]), 6)
    assert bo.tolist() == [[0, 4, 3, 2, 1, -1], [0, -1, -1, -1, -1, -1], [-1] * 6]


def test_monotone_in_thresholds_and_patience():
    """Loosening a threshold can only make blocks stable (stop earlier);
    more patience or a larger min_blocks can only stop later; dropping either
    criterion (its threshold = +inf) stops no later than requiring both."""
    w = rand_w(14, G=4, d=16, page=2, lens=(120, 90), planted=4, planted_gain=6.0)
    def stop(**k):
        return oracle.run(w, **k).stop
    em = [1e-3, 3e-3, 1e-2, 3e-2, 1e-1]
    ed = [1e-4, 1e-3, 1e-2, 3e-2]
    base = dict(P=2, min_blocks=1)
    for i in range(len(em) - 1):
        assert (stop(eps_m=em[i + 1], eps_d=1e-2, **base) <= stop(eps_m=em[i], eps_d=1e-2, **base)).all()
    for i in range(len(ed) - 1):
        assert (stop(eps_m=3e-2, eps_d=ed[i + 1], **base) <= stop(eps_m=3e-2, eps_d=ed[i], **base)).all()
    for P in range(0, 4):
        assert (stop(eps_m=3e-2, eps_d=1e-2, P=P, min_blocks=1) <= stop(eps_m=3e-2, eps_d=1e-2, P=P + 1, min_blocks=1)).all()
    for mb in range(0, 6):
        assert (stop(eps_m=3e-2, eps_d=1e-2, P=2, min_blocks=mb) <= stop(eps_m=3e-2, eps_d=1e-2, P=2, min_blocks=mb + 1)).all()
    both = stop(eps_m=1e-2, eps_d=1e-3, **base)
    assert (stop(eps_m=1e-2, eps_d=float("inf"), **base) <= both).all()
    assert (stop(eps_m=float("inf"), eps_d=1e-3, **base) <= both).all()
    # something must actually stop early for this test to mean anything
    assert (both < w.n_blocks().numpy()[:, None]).any()


def test_value_scaling_invariance():
    """Scaling every value by c > 0 scales each o_j by c: both statistics are
    unchanged (stop unchanged) and the output scales by c."""
    w = rand_w(15, G=4, d=16, page=2, lens=(100, 64), planted=4, planted_gain=6.0, eps_m=1e-2, eps_d=1e-3, P=2)
    r = oracle.run(w, want_stats=True)
    w2 = w.to("cpu")
    w2.v_cache = w.v_cache * 4.0     # exact in binary floating point
    r2 = oracle.run(w2, want_stats=True)
    assert (r.stop == r2.stop).all()
    assert np.abs(r2.out - 4.0 * r.out).max() <= 1e-12
    m = ~np.isnan(r.ds)
    assert np.allclose(r.ds[m], r2.ds[m], rtol=1e-9, atol=1e-15)


def test_undecided_band_gives_both_stops():
    """Put eps_d exactly on a block's statistic: that block is flagged '?',
    and both the stop with it stable and the stop with it unstable are admissible."""
    w = rand_w(16, G=1, Hkv=1, d=8, page=2, lens=(60,), planted=0, eps_m=1.0, eps_d=1.0, P=1, min_blocks=1)
    r = oracle.run(w, eps_m=0.0, eps_d=0.0, want_stats=True)
    j = 5
    x = float(np.float32(r.dd[0, 0, j]))          # thresholds travel as binary32
    r2 = oracle.run(w, eps_m=float("inf"), eps_d=x, P=1, min_blocks=j + 1, want_stats=True)
    assert chr(r2.flag[0, 0, j]) == "?"
    assert r2.amb_count[0, 0] >= 1
    adm = r2.admissible[0]
    assert (j + 1) in adm and len(adm) >= 2 and r2.stop[0, 0] in adm


def test_rejects_bad_order():
    w = rand_w(17, lens=(20,), Hkv=1, G=1)
    w.block_order[0, 1] = w.block_order[0, 0]     # duplicate entry: not a permutation
    with pytest.raises(ValueError):
        oracle.run(w)
