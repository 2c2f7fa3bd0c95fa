"""Benchmark: ART decode attention on one B200 (or N independent replicas).

A step is one pass of the whole hot path over one decode batch: one launch
of the ART walk for every (sequence, kv-head) unit, which builds the default
walk order (sink block, then newest to oldest) on the fly in its producer.
The K/V cache is resident in HBM before timing starts; the L2 is flushed before every step,
outside the step's events (a 512 MiB write, then a 512 MiB read so that the
flush's dirty lines are not written back inside the step).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-cpu-baseline] [--no-e2e]
    python bench.py --table all      # every workload: ART, eps=0, ablations, importance order

Under torchrun each rank runs its own batch of the same shape (weak scaling,
no collective on the data path); rank 0 prints one JSON line.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

METRIC = "ART decode-attn queries/s; KV GB/s read & % of B200 HBM peak; % KV blocks skipped"
DEFAULT_WORKLOAD = "llama8b_b32"
WORKLOAD_TEXT = {
    "tiny_fp32": "tiny fp32: B=1, Hq=Hkv=4, d=64, L=1024, 16-token blocks, 4 planted tokens",
    "llama8b_b8": "Llama-3-8B-shaped GQA 32/8, d=128, bf16 paged KV, B=8, L=8192, 64-token pages, "
                  "power-law recency keys",
    "llama8b_b32": "Llama-3-8B-shaped GQA 32/8, d=128, bf16 paged KV, B=32, L=32768, 64-token pages",
    "qwen7b_b4": "Qwen2.5-7B-shaped GQA 28/4, d=128, bf16 paged KV, B=4, L=131072, 16 planted heavy hitters",
    "mistral7b_b128": "Mistral-7B-shaped GQA 32/8, d=128, bf16 paged KV, B=128, ragged L in [1024,16384]",
}
SPEC_HBM_GBS = 8000.0
L2_FLUSH_BYTES = 512 << 20


class L2Flush:
    """Evicts the K/V cache from L2 before a step, outside its events: a write
    of a 512 MiB buffer (4x the 126 MB L2), then a read of a second one, so
    that the step starts with L2 holding only clean lines of an unrelated
    buffer.  Without the read the write's dirty lines would be written back
    to HBM during the step and counted against it."""

    def __init__(self, torch, dev):
        self.torch = torch
        self.w = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.r = torch.ones(L2_FLUSH_BYTES // 4, dtype=torch.int32, device=dev)
        self.acc = torch.zeros((), dtype=torch.int64, device=dev)

    def __call__(self, i):
        self.w.fill_(i)
        self.torch.sum(self.r, dim=0, dtype=self.torch.int64, out=self.acc)


def measured_peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def kernel_source_hash():
    """Hash of what the walk kernel is built from -- its sources, the host
    header they include and the build script with its nvcc flags -- with
    comments and blank lines removed, so that a comment edit does not void an
    ncu record taken on the same code, while a change of code or flags does."""
    import re
    h = hashlib.sha256()
    for rel in ("kv_cache_early_art_b200/csrc/art_kernels.cuh", "kv_cache_early_art_b200/csrc/art_ptx.cuh",
                "kv_cache_early_art_b200/csrc/art_api.cu", "kv_cache_early_art_b200/csrc/art_host.h",
                "kv_cache_early_art_b200/csrc/art_walk.h", "kv_cache_early_art_b200/csrc/art_walk_dl.cuh", "kv_cache_early_art_b200/csrc/art_walk_gr.cuh", "kv_cache_early_art_b200/csrc/art_walk_f32.cu",
                "kv_cache_early_art_b200/csrc/art_walk_bf16.cu", "kv_cache_early_art_b200/csrc/art_walk_mma.cu",
                "kv_cache_early_art_b200/csrc/art_walk_multi.cu", "kv_cache_early_art_b200/build.py"):
        with open(os.path.join(ROOT, rel), encoding="utf-8") as f:
            src = f.read()
        if rel.endswith(".py"):
            src = re.sub(r'"""(?:.|\n)*?"""', "", src)
            src = re.sub(r"#[^\n]*", "", src)
        else:
            src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
            src = re.sub(r"//[^\n]*", "", src)
        src = "\n".join(line.rstrip() for line in src.splitlines() if line.strip())
        h.update(src.encode())
    return h.hexdigest()[:16]


def ncu_traffic(workload):
    """DRAM bytes per launch of the walk kernel from the committed ncu summary,
    only while it was taken on the current kernel sources."""
    path = os.path.join(ROOT, "profiles", f"art_walk_{workload}.json")
    try:
        with open(path) as f:
            rec = json.load(f)
        if rec.get("source_hash") == kernel_source_hash():
            return float(rec["dram_bytes_per_launch"])
    except Exception:
        pass
    return None


class ClockSampler:
    """nvidia-smi clock and throttle-reason samples during the timed region."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, device):
        import tempfile
        import torch
        props = torch.cuda.get_device_properties(device)
        uuid = getattr(props, "uuid", None)
        self.gpu = f"GPU-{uuid}" if uuid else str(device.index or 0)
        self.path = tempfile.mktemp(prefix="art_clocks_", suffix=".csv")
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(["nvidia-smi", "-i", self.gpu, f"--query-gpu={self.Q}",
                                          "--format=csv,noheader,nounits", "-lms", "100", "-f", self.path],
                                         stdout=subprocess.DEVNULL, stderr=subprocess.DEVNULL)
            time.sleep(0.3)
        except Exception:
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.send_signal(__import__("signal").SIGINT)
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            try:
                with open(self.path) as f:
                    self.lines = [l for l in f if l.strip()]
                os.unlink(self.path)
            except Exception:
                self.lines = []

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ("hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap")
        for l in self.lines:
            f = [x.strip() for x in l.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx = float(f[2])
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        sm.sort()
        return {"sm_mhz": sm[len(sm) // 2], "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def dist_env():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    return ws, rank, local


def replica_seed(rank: int) -> int:
    """Each replica decodes its own batch: same shape, different draws."""
    return 1000 * rank


def reduce_max(value: float, world: int, device=None) -> float:
    """Max over ranks of a host-side measurement (not a data-path collective)."""
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def reduce_sum(value: float, world: int, device=None) -> float:
    if world <= 1:
        return value
    import torch
    import torch.distributed as dist
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


# ---------------------------------------------------------------- oracle ----

def time_oracle(w_cpu, budget_s: float, ncores: int = 0):
    """The CPU oracle on a bounded sample of the batch: groups of sequences
    (enough kv-head units to give every thread one), cycling through the
    batch, until budget_s has passed (ncores threads; 0: every host core).
    Returns (queries/s, threads used, sequences timed, seconds)."""
    import oracle
    ncores = ncores or os.cpu_count() or 1
    per = max(1, -(-ncores // w_cpu.Hkv))           # sequences per call
    groups = [sequences(w_cpu, list(range(b, min(b + per, w_cpu.B)))) for b in range(0, w_cpu.B, per)]
    used = min(ncores, per * w_cpu.Hkv)
    done, i, t0 = 0, 0, time.perf_counter()
    while True:
        g = groups[i % len(groups)]
        oracle.run(g, want_out=True, nthreads=ncores)
        done += g.B
        i += 1
        el = time.perf_counter() - t0
        if el >= budget_s:
            break
    return done / el, used, done, el


def sequences(w, seqs):
    """The listed sequences of a CPU workload, sharing its caches."""
    v = w.to("cpu")
    sl = torch_index(seqs)
    v.q, v.page_table, v.block_order, v.seq_lens = w.q[sl], w.page_table[sl], w.block_order[sl], w.seq_lens[sl]
    v.eps_m, v.eps_d, v.P, v.min_blocks = w.eps_m[sl], w.eps_d[sl], w.P[sl], w.min_blocks[sl]
    return v


def torch_index(seqs):
    import torch
    return torch.as_tensor(seqs, dtype=torch.long)


def one_sequence(w, b):
    """Sequence b of a CPU workload, sharing its caches (the oracle's sample)."""
    return sequences(w, [b])


def run_reference(args):
    """The CPU oracle timed on the host cores; each step is a bounded sample of
    the workload: one sequence (one decode query, all its kv heads), cycling
    through the batch."""
    ws, rank, local = dist_env()
    if rank != 0:
        return 0
    from kv_cache_early_art_b200.workloads import make_workload
    w = make_workload(args.workload, seed=replica_seed(0), device="cpu")
    import oracle
    ncores = os.cpu_count() or 1
    samples = [one_sequence(w, b) for b in range(w.B)]
    for i in range(args.warmup):
        oracle.run(samples[i % w.B], nthreads=ncores)
    times = []
    for i in range(args.steps):
        t0 = time.perf_counter()
        oracle.run(samples[i % w.B], nthreads=ncores)
        times.append(time.perf_counter() - t0)
    ms = 1000.0 * sum(times) / len(times)
    value = 1.0 / (ms / 1000.0)
    sample = f"one {args.workload} sequence per step (1 query, its {w.Hkv} kv-head units), cycling the batch"
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": dict(config_for(args.workload, w, args.gpus),
                           l2="not applicable: the oracle runs on the host cores"),
            "cpu_baseline": {"value": value, "unit": "queries/s", "cores": ncores, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": value, "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)
    return 0


def config_for(name, w, gpus):
    p = w.uniform_params()
    cfg = {"workload": f"{name}: {WORKLOAD_TEXT.get(name, name)}", "B": w.B, "Hq": w.Hq, "Hkv": w.Hkv,
           "d": w.d, "page": w.page, "max_seq_len": int(w.seq_lens.max()),
           "params": ({"eps_m": p[0], "eps_d": p[1], "P": int(p[2]), "min_blocks": int(p[3])} if p else
                      "per-sequence"),
           "order": "sink block, then newest to oldest (built on the fly inside the walk)",
           "l2": "flushed before every step, outside the step events: 512 MiB write, then a 512 MiB read "
                 "so that no dirty line of the flush is written back inside the step",
           "parallelism": f"replicas x{gpus} (independent batches, no collective)"}
    return cfg


# ------------------------------------------------------------------ ours ----

def run_ours(args):
    import torch

    ws, rank, local = dist_env()
    if ws > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=__import__("datetime").timedelta(seconds=120))
    dev = torch.device("cuda", local if ws > 1 else 0)
    torch.cuda.set_device(dev)

    import kv_cache_early_art_b200 as art
    from kv_cache_early_art_b200.workloads import make_workload

    w = make_workload(args.workload, seed=replica_seed(rank), device=dev, seq_len=args.seq_len)
    wname = w.name
    B, Hkv, page, d = w.B, w.Hkv, w.page, w.d
    esize = w.k_cache.element_size()
    N = w.n_blocks().to(dev)
    full_blocks = int(N.sum().item()) * Hkv
    block_bytes = 2 * page * d * esize            # K and V of one page of one kv head
    uni = w.uniform_params()
    stream = torch.cuda.current_stream(dev)
    fetched = torch.zeros(B * Hkv, dtype=torch.int32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    T = args.multi                                # decode tokens per sequence sharing one walk
    if T > 1:
        from kv_cache_early_art_b200.workloads import draft_queries
        q_all = draft_queries(w, T, seed=0).to(dev)
        out = torch.empty(B, T, w.Hq, d, dtype=torch.float32, device=dev)
        stop = torch.empty(B, T, Hkv, dtype=torch.int32, device=dev)
        entry = art.art_decode_attention_multi
    else:
        q_all = w.q
        out = torch.empty(B, w.Hq, d, dtype=torch.float32, device=dev)
        stop = torch.empty(B, Hkv, dtype=torch.int32, device=dev)
        entry = art.art_decode_attention_ex

    def walked(st):
        """Blocks the walk consumed: per unit, the latest token's stop."""
        st = st.clamp(min=0)
        return int((st.amax(dim=1) if T > 1 else st).sum().item())
    flush = L2Flush(torch, dev)

    def step(eps_off=False, det_off=False):
        kw = dict(eps_m_per_seq=None if eps_off else w.eps_m, eps_d_per_seq=None if eps_off else w.eps_d,
                  P_per_seq=w.P, min_blocks_per_seq=w.min_blocks, blocks_fetched=fetched,
                  device_status=status, out=out, stop_block=stop)
        if det_off:
            kw["detector_off"] = 1
        return entry(q_all, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens,
                     eps_m=0.0, eps_d=0.0, want_info=True, **kw)

    def timed(n, eps_off=False, det_off=False):
        """n steps; per step: flush, then the walk between events.
        Returns per-step ms (twice: the whole step is the walk)."""
        ev = [[torch.cuda.Event(enable_timing=True) for _ in range(2)] for _ in range(n)]
        for i in range(n):
            flush(i)
            ev[i][0].record(stream)
            kw = dict(eps_m_per_seq=None if eps_off else w.eps_m, eps_d_per_seq=None if eps_off else w.eps_d,
                      P_per_seq=w.P, min_blocks_per_seq=w.min_blocks, blocks_fetched=fetched,
                      device_status=status, out=out, stop_block=stop)
            if det_off:
                kw["detector_off"] = 1
            entry(q_all, w.k_cache, w.v_cache, w.page_table, None, w.seq_lens, eps_m=0.0, eps_d=0.0, **kw)
            ev[i][1].record(stream)
        torch.cuda.synchronize(dev)
        ms = [e[0].elapsed_time(e[1]) for e in ev]
        return ms, ms

    _, _, info = step()
    for _ in range(max(args.warmup, 3)):
        step()
    torch.cuda.synchronize(dev)
    assert int(status.item()) == 0, f"device status {int(status.item())}"

    # ---- timed region (device time, max over ranks) ----
    if ws > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize(dev)
    with ClockSampler(dev) as clk:
        step_ms, walk_ms = timed(args.steps)
    torch.cuda.synchronize(dev)
    if ws > 1:
        torch.distributed.barrier()
    stops = stop.clone()
    art_out = out.clone()
    consumed = walked(stops)
    fetched_blocks = int(fetched.sum().item())
    assert int(status.item()) == 0
    ms = sum(step_ms) / len(step_ms)
    ms_walk = sum(walk_ms) / len(walk_ms)
    ms_max = reduce_max(ms, ws, dev)
    queries_all = reduce_sum(float(B * T), ws, dev)
    value = queries_all / (ms_max / 1000.0)

    # ---- termination disabled: the same kernel as full attention ----
    for _ in range(2):
        step(eps_off=True)
    f_step, f_walk = timed(max(3, args.steps // 4), eps_off=True)
    ms_full = sum(f_walk) / len(f_walk)
    full_consumed = walked(stop)
    det = detector_overhead(args, T, step, timed, out, stop, torch, dev)

    alg_bytes = consumed * block_bytes
    fetch_bytes = fetched_blocks * block_bytes
    peak, peak_kind = measured_peaks()
    achieved = alg_bytes / (ms_walk / 1000.0) / 1e9
    roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
            "traffic": ncu_traffic(wname if T == 1 else f"{wname}_shared{T}"),
            "peak_kind": peak_kind,
            "kernel": "art_walk_kernel (the whole step: the order is built inside it)" if T == 1 else
                      f"art_walk_kernel, {T} tokens per walk (the whole step)",
            "algorithmic_bytes_per_launch": alg_bytes}

    line = {"metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": ws, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_max, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": str(w.k_cache.dtype).replace("torch.", "").replace("bfloat16", "bf16"),
            "data": "synthetic", "config": dict(config_for(wname, w, ws), **(
                {"queries_per_sequence": T, "queries": "draft tokens sharing one walk: token 0 the workload's "
                 "query, token 1 that query plus 0.5 N(0,1); each token keeps its own ART decision"}
                if T > 1 else {})),
            "kv_gbs_fetched": fetch_bytes / (ms_walk / 1000.0) / 1e9,
            "kv_gbs_algorithmic": achieved,
            "hbm_frac_of_measured": fetch_bytes / (ms_walk / 1000.0) / 1e9 / peak,
            "hbm_frac_of_8tbs_spec": fetch_bytes / (ms_walk / 1000.0) / 1e9 / SPEC_HBM_GBS,
            "skip_frac_blocks": 1.0 - consumed / full_blocks,
            "skip_frac_bytes": 1.0 - fetched_blocks / full_blocks,   # the pages never read (speculation counted)
            "fetch_waste_blocks": fetched_blocks - consumed,
            "walk_ms": ms_walk,
            "full_attention": {"walk_ms": ms_full, "kv_gbs": full_consumed * block_bytes / (ms_full / 1000.0) / 1e9,
                               "queries_per_s": B * T / (ms_full / 1000.0),
                               "art_speedup": ms_full / ms_walk},
            "detector_overhead": det,
            "launch": info, "gpu_launches": args.steps,
            "roofline": roof, "clocks": clk.summary()}

    # ---- end to end through the public API: pinned host inputs in, results out ----
    if not args.no_e2e:
        # One pinned staging block per direction, as a caller would keep it:
        # q | page table | seq_lens go in with one copy, out | stop come back
        # with one.  The library takes views into the device blocks.
        def carve(parts, device=None, pin=False):
            offs, n = [], 0
            for t in parts:
                n = (n + 255) // 256 * 256
                offs.append(n)
                n += t.numel() * t.element_size()
            blk = torch.empty(n, dtype=torch.uint8, device=device, pin_memory=pin)
            views = [blk[o:o + t.numel() * t.element_size()].view(t.dtype).view(t.shape) for o, t in zip(offs, parts)]
            return blk, views
        ins = [q_all, w.page_table, w.seq_lens]
        in_h, (q_h, pt_h, sl_h) = carve(ins, pin=True)
        for hv, t in zip((q_h, pt_h, sl_h), ins):
            hv.copy_(t.cpu())
        in_d, (q_d, pt_d, sl_d) = carve(ins, device=dev)
        out_d, (out_v, stop_v) = carve([out, stop], device=dev)
        out_h, (out_hv, stop_hv) = carve([out, stop], pin=True)
        h2d = in_h.numel()
        d2h = out_h.numel()

        def e2e_step():
            in_d.copy_(in_h, non_blocking=True)
            entry(q_d, w.k_cache, w.v_cache, pt_d, None, sl_d, eps_m_per_seq=w.eps_m, eps_d_per_seq=w.eps_d,
                  P_per_seq=w.P, min_blocks_per_seq=w.min_blocks, out=out_v, stop_block=stop_v)
            out_h.copy_(out_d, non_blocking=True)

        for _ in range(3):
            e2e_step()
        torch.cuda.synchronize(dev)
        e_ms = []
        for i in range(args.steps):
            flush(i)
            a = torch.cuda.Event(enable_timing=True)
            b_ = torch.cuda.Event(enable_timing=True)
            a.record(stream)
            e2e_step()
            b_.record(stream)
            b_.synchronize()
            e_ms.append(a.elapsed_time(b_))
        # the staged path computed what the device-resident one did
        if not (torch.equal(out_hv, art_out.cpu()) and torch.equal(stop_hv, stops.cpu())):
            raise RuntimeError("end-to-end result differs from the device-resident walk")
        em = reduce_max(sum(e_ms) / len(e_ms), ws, dev)
        line["e2e"] = {"value": queries_all / (em / 1000.0), "unit": "queries/s", "h2d_bytes_per_step": h2d,
                       "d2h_bytes_per_step": d2h, "ms_per_step": em,
                       "note": "KV cache resident; per step q, page table and seq_lens in (one pinned block, one "
                               "copy), output and stops out (one copy)"}

    # ---- CPU oracle baseline (rank 0, N = 1) ----
    if rank == 0 and ws == 1 and not args.no_cpu_baseline:
        w_cpu = w.to("cpu")
        qps, cores, nseq, el = time_oracle(w_cpu, args.cpu_seconds)
        qps1, _, nseq1, el1 = time_oracle(w_cpu, args.cpu_seconds / 2, ncores=1)
        line["cpu_baseline"] = {"value": qps, "unit": "queries/s", "cores": cores, "kind": "oracle",
                                "sample": f"{nseq} {wname} sequences (decode queries, every kv head), "
                                          f"cycling through the batch, in {el:.1f} s",
                                "one_core": {"value": qps1, "sample": f"{nseq1} sequences in {el1:.1f} s"}}
    if ws > 1:
        torch.distributed.barrier()
        torch.distributed.destroy_process_group()
    if rank == 0:
        print(json.dumps(line), flush=True)
    return 0


def detector_overhead(args, T, step, timed, out, stop, torch, dev):
    """The ART explainer's section 4 ablation (detector cost with termination
    disabled): the walk at eps = 0, which forms every statistic and runs the
    patience rule but never stops, against the same walk built without the
    detector (detector_off), whose output must equal it bit for bit.  Rounds
    of the two alternate; each round's median step time, best round kept."""
    if T > 1:
        return None
    step(eps_off=True)
    ref_out, ref_stop = out.clone(), stop.clone()
    try:
        step(det_off=True)
    except Exception as e:           # not built for this shape
        return {"unavailable": str(e)}
    torch.cuda.synchronize(dev)
    identical = bool(torch.equal(out, ref_out) and torch.equal(stop, ref_stop))
    n = max(5, min(200, args.steps // 8))
    med = lambda xs: sorted(xs)[len(xs) // 2]
    eps0, off = [], []
    for _ in range(4):
        eps0.append(med(timed(n, eps_off=True)[1]))
        off.append(med(timed(n, det_off=True)[1]))
    a, b = min(eps0), min(off)
    return {"eps0_walk_ms": a, "detector_off_walk_ms": b, "overhead_frac": a / b - 1.0,
            "output_identical": identical, "rounds": 4, "steps_per_round": n,
            "note": "eps = 0 walk (statistics and patience formed, never stopping) against the walk built "
                    "without the detector; alternating rounds, median per round, best round"}


def run_table(args):
    """Every named workload (and two pruned-cache variants) with ART, the same
    kernel with termination disabled (eps = 0), and the ablations of the ART
    explainer's section 4 (scale only, direction only, no patience): walk time,
    blocks consumed and skipped, pages fetched, GB/s.  One JSON line per row,
    then a markdown table."""
    import torch

    import kv_cache_early_art_b200 as art
    from kv_cache_early_art_b200.workloads import CONFIGS, draft_queries, make_workload, streaming_subset

    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    flush = L2Flush(torch, dev)
    peak, _ = measured_peaks()
    inf = float("inf")
    rows = []

    def median_ms(fn):
        ts = []
        for i in range(args.table_reps):
            flush(i)
            a = torch.cuda.Event(enable_timing=True)
            b = torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            torch.cuda.synchronize(dev)
            ts.append(a.elapsed_time(b))
        ts.sort()
        return ts[len(ts) // 2]

    def measure(w, label, em, ed, P, importance=None):
        """importance = (summary, scores, order): the order is rebuilt from the
        page summaries inside the timed region, before the walk."""
        out = torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev)
        stop = torch.empty(w.B, w.Hkv, dtype=torch.int32, device=dev)
        fetched = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device=dev)
        status = torch.zeros(1, dtype=torch.int32, device=dev)
        kw = dict(eps_m_per_seq=em, eps_d_per_seq=ed, P_per_seq=P, min_blocks_per_seq=w.min_blocks,
                  blocks_fetched=fetched, device_status=status, out=out, stop_block=stop)
        order = w.block_order if importance is None else importance[2]

        def call():
            if importance is not None:
                art.art_build_order_importance(w.q, importance[0], w.page_table, w.seq_lens, w.page,
                                               block_scores=importance[1], block_order=importance[2],
                                               device_status=status)
            art.art_decode_attention_ex(w.q, w.k_cache, w.v_cache, w.page_table, order, w.seq_lens, **kw)

        call()
        ms = median_ms(call)
        assert int(status.item()) == 0
        N = w.n_blocks().to(dev)
        total = int(N.sum().item()) * w.Hkv
        used = int(stop.clamp(min=0).sum().item())
        bb = 2 * w.page * w.d * w.k_cache.element_size()
        row = {"workload": w.name, "variant": label, "ms": ms, "queries_per_s": w.B / (ms / 1e3),
               "blocks": total, "consumed": used, "skip_frac": 1.0 - used / max(total, 1),
               "fetched": int(fetched.sum().item()), "gbs": used * bb / (ms / 1e3) / 1e9,
               "hbm_frac": used * bb / (ms / 1e3) / 1e9 / peak}
        rows.append(row)
        print(json.dumps(row), flush=True)
        return row

    pairs = []

    def measure_pair(w):
        """Two decode tokens per sequence (the second the first plus noise):
        two separate single-query walks against one shared walk."""
        qm = draft_queries(w, 2, seed=0)
        kw = dict(eps_m_per_seq=w.eps_m, eps_d_per_seq=w.eps_d, P_per_seq=w.P, min_blocks_per_seq=w.min_blocks)
        sep = [(torch.empty(w.B, w.Hq, w.d, dtype=torch.float32, device=dev),
                torch.empty(w.B, w.Hkv, dtype=torch.int32, device=dev),
                torch.zeros(w.B * w.Hkv, dtype=torch.int32, device=dev)) for _ in range(2)]
        q_tok = [qm[:, t].contiguous() for t in range(2)]

        def separate():
            for t in range(2):
                art.art_decode_attention_ex(q_tok[t], w.k_cache, w.v_cache, w.page_table, w.block_order,
                                            w.seq_lens, out=sep[t][0], stop_block=sep[t][1],
                                            blocks_fetched=sep[t][2], **kw)
        out2 = torch.empty(w.B, 2, w.Hq, w.d, dtype=torch.float32, device=dev)
        stop2 = torch.empty(w.B, 2, w.Hkv, dtype=torch.int32, device=dev)
        fetched2 = torch.zeros(w.B * w.Hkv, dtype=torch.int32, device=dev)

        def shared():
            art.art_decode_attention_multi(qm, w.k_cache, w.v_cache, w.page_table, w.block_order, w.seq_lens,
                                           out=out2, stop_block=stop2, blocks_fetched=fetched2, **kw)
        separate()
        shared()
        ms_sep, ms_sh = median_ms(separate), median_ms(shared)
        bb = 2 * w.page * w.d * w.k_cache.element_size()
        f_sep = sum(int(x[2].sum().item()) for x in sep)
        f_sh = int(fetched2.sum().item())
        same = sum(int((stop2[:, t] != sep[t][1]).sum().item()) for t in range(2))
        row = {"workload": w.name, "ms_separate": ms_sep, "ms_shared": ms_sh, "queries": 2 * w.B,
               "consumed": int(stop2.clamp(min=0).sum().item()), "fetched_separate": f_sep, "fetched_shared": f_sh,
               "gbs_shared": f_sh * bb / (ms_sh / 1e3) / 1e9, "stop_differs": same}
        pairs.append(row)
        print(json.dumps(row), flush=True)

    names = list(CONFIGS) if args.table == "all" else args.table.split(",")
    for name in names:
        base = make_workload(name, device=dev)
        variants = [base]
        if name in ("llama8b_b32", "qwen7b_b4"):   # a StreamingLLM-style pruned cache: sink + last 64 pages
            variants.append(streaming_subset(base, window_blocks=64))
        for w in variants:
            B = w.B
            ones = torch.ones(B, dtype=torch.int32, device=dev)
            full = lambda v: torch.full((B,), v, dtype=torch.float32, device=dev)
            measure(w, "ART", w.eps_m, w.eps_d, w.P)
            measure(w, "full (eps=0)", full(0.0), full(0.0), w.P)
            measure(w, "scale only", w.eps_m, full(inf), w.P)
            measure(w, "direction only", full(inf), w.eps_d, w.P)
            measure(w, "no patience (P=1)", w.eps_m, w.eps_d, ones)
            # importance-first order: page summaries kept beside the cache (built
            # once, timed apart), the order rebuilt every step inside the timing
            summ = art.art_page_summary(w.k_cache, w.page_table, w.seq_lens, dtype=torch.bfloat16)
            sum_ms = median_ms(lambda: art.art_page_summary(w.k_cache, w.page_table, w.seq_lens, summ))
            bufs = (summ, torch.empty(B, w.max_blocks, dtype=torch.float32, device=dev),
                    torch.empty(B, w.max_blocks, dtype=torch.int32, device=dev))
            order_ms = median_ms(lambda: art.art_build_order_importance(
                w.q, summ, w.page_table, w.seq_lens, w.page, block_scores=bufs[1], block_order=bufs[2]))
            row = measure(w, "ART, importance order", w.eps_m, w.eps_d, w.P, importance=bufs)
            row.update(summary_ms=sum_ms, order_ms=order_ms)
            print(json.dumps({"workload": w.name, "summary_ms": sum_ms, "order_ms": order_ms}), flush=True)
            if w.d == 128 and 2 * w.G <= 8:      # two tokens fit one unit's eight rows
                measure_pair(w)
        del base, variants
        torch.cuda.empty_cache()
    print("| workload | variant | walk ms | queries/s | blocks consumed / total | skipped | pages fetched | GB/s | of HBM |")
    print("|---|---|---|---|---|---|---|---|---|")
    for r in rows:
        print(f"| {r['workload']} | {r['variant']} | {r['ms']:.4f} | {r['queries_per_s']:.0f} | "
              f"{r['consumed']} / {r['blocks']} | {100 * r['skip_frac']:.1f} % | {r['fetched']} | "
              f"{r['gbs']:.0f} | {100 * r['hbm_frac']:.1f} % |")
    print()
    print("| workload | page summaries (once per page fill) ms | importance order build ms (inside the row above) |")
    print("|---|---|---|")
    for r in rows:
        if "summary_ms" in r:
            print(f"| {r['workload']} | {r['summary_ms']:.4f} | {r['order_ms']:.4f} |")
    if pairs:
        print()
        print("| workload | two walks ms | one shared walk ms | speed-up | queries/s shared | pages fetched "
              "(two walks / shared) | shared GB/s | stops differing |")
        print("|---|---|---|---|---|---|---|---|")
        for r in pairs:
            print(f"| {r['workload']} | {r['ms_separate']:.4f} | {r['ms_shared']:.4f} | "
                  f"{r['ms_separate'] / r['ms_shared']:.2f}x | {r['queries'] / (r['ms_shared'] / 1e3):.0f} | "
                  f"{r['fetched_separate']} / {r['fetched_shared']} | {r['gbs_shared']:.0f} | {r['stop_differs']} |")
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=2000)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--seq-len", type=int, default=None,
                    help="replace a uniform-length workload's length (a smaller case of the same launch, "
                         "for profiling); the line then names <workload>_L<len>")
    ap.add_argument("--multi", type=int, default=1, choices=[1, 2],
                    help="decode tokens per sequence sharing one walk (2: art_decode_attention_multi)")
    ap.add_argument("--cpu-seconds", type=float, default=10.0)
    ap.add_argument("--table", default=None, help="'all' or comma-separated workloads: per-workload table")
    ap.add_argument("--table-reps", type=int, default=20)
    args = ap.parse_args(argv)
    if args.table:
        return run_table(args)
    if args.impl == "reference":
        return run_reference(args)
    return run_ours(args)


if __name__ == "__main__":
    sys.exit(main())
