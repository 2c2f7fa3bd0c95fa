"""Shared parity check: CUDA path against the CPU oracle.

Acceptance rule: for every (sequence, kv-head) unit the GPU's stop index must
be one the oracle admits (bit-exact when no block is undecided), and the GPU's
output must match the oracle's output after exactly that many blocks of the
walk, within max-abs 1e-5 for fp32 caches and 2e-3 for bf16 caches (fp32
accumulation).
"""
import numpy as np
import torch

import oracle

TOL = {torch.float32: 1e-5, torch.bfloat16: 2e-3}


def check(w_cpu, out_gpu, stop_gpu, *, units=None, scale=None, nthreads=0, tol=None):
    """w_cpu: the workload on the CPU.  out_gpu [B,Hq,d], stop_gpu [B,Hkv]
    (any device).  Returns a summary dict; raises AssertionError on mismatch."""
    out = out_gpu.detach().cpu().numpy().astype(np.float64)
    stop = stop_gpu.detach().cpu().numpy()
    r = oracle.run(w_cpu, scale=scale, want_out=False, nthreads=nthreads)
    B, Hkv, G = w_cpu.B, w_cpu.Hkv, w_cpu.G
    all_units = range(B * Hkv) if units is None else units
    bad = []
    for u in all_units:
        b, h = divmod(u, Hkv)
        if int(stop[b, h]) not in [int(x) for x in r.admissible[u]]:
            bad.append((b, h, int(stop[b, h]), [int(x) for x in r.admissible[u]], int(r.stop[b, h])))
    assert not bad, f"stop index outside the admissible set (b, h, gpu, admissible, canonical): {bad[:8]}"
    ul = list(all_units)
    ss = [int(stop[u // Hkv, u % Hkv]) for u in ul]
    ref = oracle.prefix_out(w_cpu, ul, ss, scale=scale, nthreads=nthreads)
    got = np.stack([out[u // Hkv, (u % Hkv) * G:(u % Hkv + 1) * G] for u in ul])
    err = float(np.abs(got - ref).max()) if len(ul) else 0.0
    t = TOL[w_cpu.k_cache.dtype] if tol is None else tol
    assert err <= t, f"max-abs output error {err:.3e} > {t:.1e}"
    N = w_cpu.n_blocks().numpy()
    tot_blocks = int(sum(N[u // Hkv] for u in ul))
    return dict(max_abs=err, ambiguous=int(r.amb_count.sum()), canonical_mismatch=int(
        sum(int(stop[u // Hkv, u % Hkv]) != int(r.stop[u // Hkv, u % Hkv]) for u in ul)),
        blocks_consumed=int(sum(ss)), blocks_total=tot_blocks)


def subset_sequences(w, seqs):
    """The same cache with only the listed sequences (all their kv heads)."""
    idx = torch.as_tensor(seqs, dtype=torch.long)
    v = w.to("cpu")
    v.q = w.q.detach().cpu()[idx]
    v.page_table = w.page_table.cpu()[idx]
    v.block_order = w.block_order.cpu()[idx]
    v.seq_lens = w.seq_lens.cpu()[idx]
    v.eps_m, v.eps_d = w.eps_m.cpu()[idx], w.eps_d.cpu()[idx]
    v.P, v.min_blocks = w.P.cpu()[idx], w.min_blocks.cpu()[idx]
    return v
