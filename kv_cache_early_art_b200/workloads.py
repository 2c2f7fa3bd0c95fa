"""Seeded synthetic decode-attention inputs.

This module builds the tensors that both the CUDA path and the CPU oracle
consume: queries, a paged K/V cache, the page table, the walk order, the
sequence lengths and the per-sequence ART parameters.  It holds none of the
method's arithmetic (no scores, no softmax, no statistics): only random draws,
the key construction the workloads prescribe, and the scatter of logical
tokens into physical pages.

Workloads (the long-context GQA decode shapes of the ART explainer's
evaluation, "4. Experimental Results": Mistral-7B / Llama-class models on long
inputs; LongBench itself is not available, these seeded tensors stand in for
it):

* ``tiny_fp32``     B=1, Hq=Hkv=4, d=64, L=1024, 16-token blocks, fp32,
                    contiguous cache, q,k,v ~ N(0,1), four planted tokens
                    k = 3*sqrt(d)*q_hat per head.
* ``llama8b_b8``    Llama-3-8B-shaped layer: Hq=32, Hkv=8, d=128, bf16,
                    B=8, L=8192, 64-token pages under a random page table,
                    power-law recency keys, v ~ N(0,1).
* ``llama8b_b32``   same distributions at B=32, L=32768.
* ``qwen7b_b4``     Qwen2.5-7B-shaped: Hq=28, Hkv=4, d=128, bf16, B=4,
                    L=131072, 16 planted heavy hitters per sequence
                    (k = 4*sqrt(d)*q_hat_grp) on top of recency keys.
* ``mistral7b_b128`` Mistral-7B-shaped: Hq=32, Hkv=8, d=128, bf16, B=128,
                    ragged L uniform in [1024, 16384], per-sequence patience
                    in {1,2,4} and eps_m in {1e-4, 1e-3} (eps_d = eps_m/10).

Draw order (fixed, so that the same seed always gives the same bits on a
given device):

1. ragged workloads only: sequence lengths, then per-sequence P and eps_m,
   from a CPU ``torch.Generator`` seeded with ``seed ^ 0x5EED``;
then, from one ``torch.Generator`` on the target device seeded with ``seed``:
2. q ~ N(0,1) of shape [B, Hq, d];
3. a permutation of the physical pages (random page tables only);
4. planted positions, per sequence (planted workloads only);
5. per sequence b: K noise [Hkv, L_b, d], then V [Hkv, L_b, d];
6. ``order="random"`` only: a permutation per sequence from a CPU generator
   seeded with ``seed * 7919 + b``.

Keys for recency workloads: k_t = noise_t + alpha_t * q_hat_grp with
alpha_t = 2 * (1 + age)^-0.5, age = L_b - 1 - t, and q_hat_grp the unit
vector along the sum of the group's (stored, i.e. already rounded) queries.
Planted tokens replace the whole key.  Values are drawn in fp32 and rounded
to the storage dtype by round-to-nearest-even.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field
from typing import Optional

import torch

__all__ = ["Workload", "CONFIGS", "make_workload", "make_custom", "sink_recency_order", "streaming_subset",
           "draft_queries", "token_view"]


@dataclass
class Workload:
    """Everything one ART decode-attention call needs, on one device."""

    name: str
    q: torch.Tensor            # [B, Hq, d]           dtype = cache dtype
    k_cache: torch.Tensor      # [num_pages, Hkv, page, d]
    v_cache: torch.Tensor      # [num_pages, Hkv, page, d]
    page_table: torch.Tensor   # [B, max_blocks] int32, -1 where unused
    block_order: torch.Tensor  # [B, max_blocks] int32, -1 where unused
    seq_lens: torch.Tensor     # [B] int32
    eps_m: torch.Tensor        # [B] float32
    eps_d: torch.Tensor        # [B] float32
    P: torch.Tensor            # [B] int32
    min_blocks: torch.Tensor   # [B] int32
    page: int
    meta: dict = field(default_factory=dict)

    @property
    def B(self) -> int:
        return self.q.shape[0]

    @property
    def Hq(self) -> int:
        return self.q.shape[1]

    @property
    def Hkv(self) -> int:
        return self.k_cache.shape[1]

    @property
    def d(self) -> int:
        return self.q.shape[2]

    @property
    def G(self) -> int:
        return self.Hq // self.Hkv

    @property
    def max_blocks(self) -> int:
        return self.page_table.shape[1]

    def n_blocks(self) -> torch.Tensor:
        """ceil(seq_len / page) per sequence (0 for empty sequences)."""
        s = self.seq_lens.to(torch.int64).clamp(min=0)
        return (s + self.page - 1) // self.page

    def to(self, device) -> "Workload":
        f = lambda t: t.to(device)
        return Workload(self.name, f(self.q), f(self.k_cache), f(self.v_cache), f(self.page_table),
                        f(self.block_order), f(self.seq_lens), f(self.eps_m), f(self.eps_d),
                        f(self.P), f(self.min_blocks), self.page, dict(self.meta))

    def uniform_params(self) -> Optional[tuple]:
        """(eps_m, eps_d, P, min_blocks) when every sequence shares them, else None."""
        vals = []
        for t in (self.eps_m, self.eps_d, self.P, self.min_blocks):
            u = torch.unique(t.cpu())
            if u.numel() != 1:
                return None
            vals.append(u.item())
        return tuple(vals)


# name -> parameters (see the module docstring for the prose form)
CONFIGS = {
    "tiny_fp32": dict(B=1, Hq=4, Hkv=4, d=64, L=1024, page=16, dtype="f32", keys="noise",
                      planted=4, planted_gain=3.0, planted_per="head", page_table="identity",
                      eps_m=1e-3, eps_d=1e-4, P=2, min_blocks=2),
    "llama8b_b8": dict(B=8, Hq=32, Hkv=8, d=128, L=8192, page=64, dtype="bf16", keys="recency",
                       planted=0, page_table="random", eps_m=5e-4, eps_d=5e-5, P=3, min_blocks=1),
    "llama8b_b32": dict(B=32, Hq=32, Hkv=8, d=128, L=32768, page=64, dtype="bf16", keys="recency",
                        planted=0, page_table="random", eps_m=5e-4, eps_d=5e-5, P=3, min_blocks=1),
    "qwen7b_b4": dict(B=4, Hq=28, Hkv=4, d=128, L=131072, page=64, dtype="bf16", keys="recency",
                      planted=16, planted_gain=4.0, planted_per="group", page_table="random",
                      eps_m=2e-4, eps_d=2e-5, P=4, min_blocks=4),
    "mistral7b_b128": dict(B=128, Hq=32, Hkv=8, d=128, L=(1024, 16384), page=64, dtype="bf16",
                           keys="recency", planted=0, page_table="random",
                           eps_m=(1e-4, 1e-3), eps_d="eps_m/10", P=(1, 2, 4), min_blocks=1),
}

_DT = {"f32": torch.float32, "bf16": torch.bfloat16}


def sink_recency_order(n_blocks: torch.Tensor, max_blocks: int) -> torch.Tensor:
    """Walk order [0, N-1, N-2, ..., 1] per sequence (sink block, then newest to
    oldest), -1 past N.  The ART explainer's "recency-first" traversal with the
    mandatory attention-sink block first (section 2.4)."""
    B = n_blocks.numel()
    out = torch.full((B, max_blocks), -1, dtype=torch.int32)
    for b in range(B):
        n = int(n_blocks[b])
        if n <= 0:
            continue
        out[b, 0] = 0
        if n > 1:
            out[b, 1:n] = torch.arange(n - 1, 0, -1, dtype=torch.int32)
    return out


def _unit(x: torch.Tensor) -> torch.Tensor:
    return x / x.norm(dim=-1, keepdim=True).clamp_min(1e-30)


def make_custom(*, B, Hq, Hkv, d, page, dtype="bf16", seq_lens, seed=0, keys="recency",
                planted=0, planted_gain=4.0, planted_per="group", page_table="random",
                order="sink_recency", eps_m=5e-4, eps_d=5e-5, P=3, min_blocks=1,
                value="normal", device="cpu", name="custom", spare_pages=0) -> Workload:
    """General seeded builder used by the named workloads and by the tests.

    ``seq_lens`` is a list of ints or a tensor.  ``eps_m``/``eps_d``/``P``/
    ``min_blocks`` are scalars or length-B sequences.  ``order`` is
    ``"sink_recency"``, ``"random"`` (a random permutation per sequence) or an
    explicit [B, max_blocks] tensor.  ``value="constant"`` gives every token of
    a (sequence, kv-head) the same value vector (a closed-form stop case).
    ``spare_pages`` adds never-referenced physical pages filled with noise.
    """
    assert Hq % Hkv == 0
    G = Hq // Hkv
    dev = torch.device(device)
    gen = torch.Generator(device=dev)
    gen.manual_seed(int(seed))
    sdt = _DT[dtype]

    seq_lens = torch.as_tensor(seq_lens, dtype=torch.int64).reshape(B)
    nblk = (seq_lens.clamp(min=0) + page - 1) // page
    max_blocks = max(1, int(nblk.max().item()))
    total_pages = int(nblk.sum().item()) + int(spare_pages)

    def per_seq(x, tdtype):
        t = torch.as_tensor(x, dtype=tdtype)
        return t.expand(B).clone() if t.dim() == 0 else t.reshape(B).clone()

    # 2. queries (stored dtype; the fp32 view of the stored values builds keys)
    q32 = torch.randn(B, Hq, d, generator=gen, device=dev)
    q = q32.to(sdt)
    qs = q.to(torch.float32)
    q_hat_head = _unit(qs)                                        # [B, Hq, d]
    q_hat_grp = _unit(qs.view(B, Hkv, G, d).sum(dim=2))           # [B, Hkv, d]

    # 3. page table
    pt = torch.full((B, max_blocks), -1, dtype=torch.int32)
    if page_table == "identity":
        perm = torch.arange(total_pages, dtype=torch.int64)
    elif page_table == "random":
        perm = torch.randperm(total_pages, generator=gen, device=dev).cpu()
    else:
        raise ValueError(page_table)
    off = 0
    for b in range(B):
        n = int(nblk[b])
        pt[b, :n] = perm[off:off + n].to(torch.int32)
        off += n

    # 4. planted positions (shared by all heads of a sequence)
    planted_pos = []
    for b in range(B):
        L = int(seq_lens[b])
        if planted > 0 and L > 0:
            k = min(planted, L)
            planted_pos.append(torch.randperm(L, generator=gen, device=dev)[:k].cpu())
        else:
            planted_pos.append(torch.zeros(0, dtype=torch.int64))

    k_cache = torch.zeros(total_pages, Hkv, page, d, dtype=sdt, device=dev)
    v_cache = torch.zeros(total_pages, Hkv, page, d, dtype=sdt, device=dev)

    # 5. keys and values, one sequence at a time
    for b in range(B):
        L = int(seq_lens[b])
        n = int(nblk[b])
        if L <= 0:
            continue
        kb = torch.randn(Hkv, L, d, generator=gen, device=dev)
        vb = torch.randn(Hkv, L, d, generator=gen, device=dev)
        if keys == "recency":
            age = (L - 1 - torch.arange(L, device=dev, dtype=torch.float32))
            alpha = 2.0 * (1.0 + age).pow(-0.5)                   # [L]
            kb = kb + alpha.view(1, L, 1) * q_hat_grp[b].view(Hkv, 1, d)
        elif keys != "noise":
            raise ValueError(keys)
        pos = planted_pos[b].to(dev)
        if pos.numel():
            if planted_per == "head":
                assert G == 1, "per-head planting needs Hq == Hkv"
                direc = q_hat_head[b]                              # [Hkv, d]
            else:
                direc = q_hat_grp[b]
            kb[:, pos, :] = (planted_gain * math.sqrt(d)) * direc.view(Hkv, 1, d)
        if value == "constant":
            vb = vb[:, :1, :].expand(Hkv, L, d).clone()
        elif value != "normal":
            raise ValueError(value)
        pad = n * page - L
        if pad:
            kb = torch.cat([kb, torch.zeros(Hkv, pad, d, device=dev)], dim=1)
            vb = torch.cat([vb, torch.zeros(Hkv, pad, d, device=dev)], dim=1)
        idx = pt[b, :n].to(torch.int64).to(dev)
        k_cache[idx] = kb.view(Hkv, n, page, d).permute(1, 0, 2, 3).to(sdt)
        v_cache[idx] = vb.view(Hkv, n, page, d).permute(1, 0, 2, 3).to(sdt)

    if spare_pages:
        used = torch.zeros(total_pages, dtype=torch.bool)
        for b in range(B):
            used[pt[b, :int(nblk[b])].to(torch.int64)] = True
        free = (~used).nonzero().flatten().to(dev)
        k_cache[free] = torch.randn(free.numel(), Hkv, page, d, generator=gen, device=dev).to(sdt)
        v_cache[free] = torch.randn(free.numel(), Hkv, page, d, generator=gen, device=dev).to(sdt)

    if isinstance(order, torch.Tensor):
        bo = order.to(torch.int32).cpu().clone()
    elif order == "sink_recency":
        bo = sink_recency_order(nblk, max_blocks)
    elif order == "random":
        bo = torch.full((B, max_blocks), -1, dtype=torch.int32)
        for b in range(B):
            n = int(nblk[b])
            if n:
                bo[b, :n] = torch.randperm(n, generator=torch.Generator().manual_seed(int(seed) * 7919 + b)).to(torch.int32)
    else:
        raise ValueError(order)

    eps_m_t = per_seq(eps_m, torch.float32)
    eps_d_t = per_seq(eps_d, torch.float32)
    P_t = per_seq(P, torch.int32)
    mb_t = per_seq(min_blocks, torch.int32)
    return Workload(name, q, k_cache, v_cache, pt.to(dev), bo.to(dev), seq_lens.to(torch.int32).to(dev),
                    eps_m_t.to(dev), eps_d_t.to(dev), P_t.to(dev), mb_t.to(dev), page,
                    dict(planted_pos=planted_pos, seed=seed, dtype=dtype))


def make_workload(name: str, seed: int = 0, device="cpu", seq_len: Optional[int] = None) -> Workload:
    """Build one of the named workloads in ``CONFIGS``.  seq_len replaces the
    length of a uniform-length workload (a smaller case of the same shape,
    e.g. for profiling); the workload is then named ``<name>_L<seq_len>``."""
    c = dict(CONFIGS[name])
    B = c["B"]
    if seq_len is not None:
        if isinstance(c["L"], tuple):
            raise ValueError(f"{name} has ragged lengths; seq_len applies to uniform-length workloads")
        c["L"] = int(seq_len)
        name = f"{name}_L{int(seq_len)}"
    if isinstance(c["L"], tuple):
        # ragged: lengths and per-sequence ART parameters come first in the draw order
        gen = torch.Generator().manual_seed(int(seed) ^ 0x5EED)
        lo, hi = c["L"]
        lens = torch.randint(lo, hi + 1, (B,), generator=gen)
        P = torch.tensor(c["P"])[torch.randint(0, len(c["P"]), (B,), generator=gen)]
        em = torch.tensor(c["eps_m"], dtype=torch.float32)[torch.randint(0, len(c["eps_m"]), (B,), generator=gen)]
        ed = em / 10.0
    else:
        lens = [c["L"]] * B
        P, em, ed = c["P"], c["eps_m"], c["eps_d"]
    w = make_custom(B=B, Hq=c["Hq"], Hkv=c["Hkv"], d=c["d"], page=c["page"], dtype=c["dtype"],
                    seq_lens=lens, seed=seed, keys=c["keys"], planted=c["planted"],
                    planted_gain=c.get("planted_gain", 4.0), planted_per=c.get("planted_per", "group"),
                    page_table=c["page_table"], eps_m=em, eps_d=ed, P=P,
                    min_blocks=c["min_blocks"], device=device, name=name)
    return w


def streaming_subset(w: Workload, window_blocks: int, sink_blocks: int = 1, name: str = None) -> Workload:
    """The same cache seen through a StreamingLLM-style pruning policy: per
    sequence only its first ``sink_blocks`` pages (attention sinks) and its
    last ``window_blocks`` pages are kept.  The kept pages are re-listed in a
    compacted page table (sinks first, then the window oldest to newest), so
    the pruned sequence is an ordinary paged sequence whose only partial page
    is its last; ``seq_lens`` shrink accordingly and the walk order becomes
    the default one of the compacted sequence.  K, V and q are shared with
    ``w`` (no copy).  This is how ART composes with a pruned cache (ART
    explainer, section 2.4: an orthogonal layer over the kept blocks)."""
    N = w.n_blocks().cpu()
    L = w.seq_lens.cpu().to(torch.int64)
    pt = w.page_table.cpu()
    B = w.B
    keep_n = torch.zeros(B, dtype=torch.int64)
    new_len = torch.zeros(B, dtype=torch.int64)
    rows = []
    for b in range(B):
        n, l = int(N[b]), int(L[b])
        if n <= sink_blocks + window_blocks:
            blocks = list(range(n))
        else:
            blocks = list(range(sink_blocks)) + list(range(n - window_blocks, n))
        rows.append(pt[b, blocks] if blocks else pt[b, :0])
        keep_n[b] = len(blocks)
        last = l - (n - 1) * w.page if n else 0          # tokens in the sequence's last page
        new_len[b] = (len(blocks) - 1) * w.page + last if blocks else 0
    mb = max(1, int(keep_n.max()))
    new_pt = torch.full((B, mb), -1, dtype=torch.int32)
    for b in range(B):
        new_pt[b, :int(keep_n[b])] = rows[b].to(torch.int32)
    dev = w.q.device
    order = sink_recency_order(keep_n, mb)
    return Workload(name or f"{w.name}_stream{window_blocks}", w.q, w.k_cache, w.v_cache, new_pt.to(dev),
                    order.to(dev), new_len.to(torch.int32).to(dev), w.eps_m, w.eps_d, w.P, w.min_blocks,
                    w.page, dict(w.meta, pruned=f"sinks {sink_blocks} + window {window_blocks} pages"))


def draft_queries(w: Workload, T: int, spread: float = 0.5, seed: int = 0) -> torch.Tensor:
    """Queries of T decode tokens per sequence, [B, T, Hq, d] in the cache's
    dtype: token 0 is w.q, token t > 0 is w.q + spread * N(0, 1) drawn in
    fp32 from a CPU generator seeded with seed * 131 + t (neighbouring draft
    tokens of one sequence ask similar questions), then rounded to the
    cache dtype."""
    q0 = w.q.detach().cpu().to(torch.float32)
    toks = [q0]
    for t in range(1, int(T)):
        g = torch.Generator().manual_seed(int(seed) * 131 + t)
        toks.append(q0 + float(spread) * torch.randn(q0.shape, generator=g, dtype=torch.float32))
    q = torch.stack(toks, dim=1).to(w.k_cache.dtype)
    return q.to(w.q.device)


def token_view(w: Workload, q_multi: torch.Tensor, t: int) -> Workload:
    """The single-query workload of token t: w with q = q_multi[:, t]."""
    v = w.to(w.q.device)
    v.q = q_multi[:, t].contiguous().to(w.q.device)
    return v
