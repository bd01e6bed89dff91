#!/usr/bin/env python
"""Benchmark of the two-level sparse-attention path on B200.

One step = one pass of the whole path (block pooling, block scoring + top-m,
token scoring + top-k, sparse attention) over one batch of synthetic input
already resident in HBM.  The default workload is the 64K-token prefill
(1 sequence, B=128, m=64, k=2048, 16 heads of 128); the metric is queries per
second, with the dominant (attention) kernel's fraction of its roofline.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl ours|reference]

Multi-GPU (torchrun, one rank per GPU): every rank runs its own independent
copy of the workload (a different seed); there is no collective on the data
path, so scaling is weak and the value is all ranks' queries over the slowest
rank's time.

Besides the device-resident step the line carries: `e2e` (the same metric
through the public API with the inputs in pinned host memory and O/LSE read
back: hisa_forward_host for prefill, hisa_forward_cached for decode),
`roofline` (the attention kernel against the bound of the kernel that ran:
the query-tile kernel's executed flops against the measured sustained bf16
rate; a gather kernel's gathered bytes against the measured L2 gather ceiling
(prefill) or the measured copy bandwidth (decode); the gathered bytes over
HBM as `effective_gbs`, and the DRAM traffic of the committed ncu record when
its source hash matches), `cpu_baseline`
(the oracle on the host cores, all cores and one), `clocks`, the flat-indexer
speedup and the needle recall of the probe query.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "hierarchical indexer+sparse-attn queries/s at 64K prefill; % of HBM roofline"
UNIT = "queries/s"
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 256 << 20


def _args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="prefill_64k")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-flat", action="store_true", help="skip the flat-indexer comparator")
    ap.add_argument("--no-clock", action="store_true", help="no clock sampling (and no padding steps), for profiling")
    ap.add_argument("--graph", choices=["auto", "on", "off"], default="auto",
                    help="replay each step from a CUDA graph (auto: for decode workloads)")
    ap.add_argument("--cpu-seconds", type=float, default=15.0, help="target CPU time of the oracle sample")
    ap.add_argument("--set", action="append", default=[], metavar="FIELD=VALUE",
                    help="override a workload field, e.g. --set n_q=32768 --set n_kv=32768")
    return ap.parse_args()


def workload(a, seed_offset=0):
    from synth.workloads import WORKLOADS

    w = WORKLOADS[a.workload]
    kw = {}
    for item in a.set:
        k, v = item.split("=", 1)
        kw[k] = int(v)
    if kw:
        w = w.with_(name=w.name + "+" + ",".join(f"{k}={v}" for k, v in kw.items()), **kw)
    return w.with_(seed=w.seed + seed_offset)


def workload_config(w) -> dict:
    """The workload's fields as the JSON line's `config` (both arms)."""
    return {"workload": w.name, "batch": w.batch, "n_q": w.n_q, "n_kv": w.n_kv, "d_idx": w.d_idx,
            "block": w.block, "top_m": w.top_m, "top_k": w.top_k, "n_heads": w.n_heads,
            "n_kv_heads": w.n_kv_heads, "d_head": w.d_head, "n_idx_heads": w.n_idx_heads, "needles": w.needles}


FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED = 1590.0, 1400.0


def _peaks():
    """(HBM GB/s, bf16 TFLOP/s burst, bf16 TFLOP/s sustained, "measured" | "fallback")."""
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            j = json.load(f)
        return float(j["hbm_gbs"]), float(j["bf16_tflops"]), float(j["bf16_tflops_sustained"]), "measured"
    except Exception:
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, FALLBACK_BF16_TFLOPS_SUSTAINED, "fallback"


class ClockSampler:
    """nvidia-smi clock / throttle sampling during the timed region."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int, enabled: bool = True):
        self.gpu = gpu_index
        self.enabled = enabled
        self.proc = None
        self.lines = []

    def __enter__(self):
        if not self.enabled:
            return self
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except Exception:
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], None, set()
        for ln in self.lines:
            parts = [x.strip() for x in ln.split(",")]
            if len(parts) < 9:
                continue
            try:
                sm.append(float(parts[1]))
                mx = float(parts[2])
            except ValueError:
                continue
            names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
            for name, val in zip(names, parts[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(value: float, device=None) -> float:
    """The largest of one float over all ranks (the job's time is the slowest rank's)."""
    import torch
    import torch.distributed as dist

    if not dist.is_available() or not dist.is_initialized() or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_value(queries_per_rank: int, world: int, max_ms: float) -> float:
    """Weak scaling: every rank runs its own copy, so the job processes world x the queries."""
    return queries_per_rank * world / (max_ms * 1e-3)


def closed_form_counts(w):
    """Per-query candidate counts and kept tokens from the closed forms of the path."""
    import numpy as np

    i = np.arange(w.n_q, dtype=np.int64)
    p = w.n_kv - w.n_q + i
    c = p // w.block
    s = np.minimum(w.top_m, c + 1)
    n_cand = np.where(s == c + 1, p + 1, (s - 1) * w.block + p % w.block + 1)
    k_eff = np.minimum(w.top_k, n_cand)
    return {"n_cand": int(n_cand.sum()) * w.batch, "k_eff": int(k_eff.sum()) * w.batch,
            "n_vis": int((c + 1).sum()) * w.batch}


def attention_bytes(w, counts):
    """Algorithmic bytes of one sparse-attention launch: every kept token's K and V rows of every
    KV head once per query (heads sharing a KV head share the rows), plus the query rows, output
    rows, LSE and index lists."""
    nq = w.batch * w.n_q
    gather = counts["k_eff"] * w.n_kv_heads * w.d_head * 2 * 2
    return gather + nq * w.n_heads * w.d_head * 2 * 2 + nq * w.n_heads * 4 + nq * w.top_k * 4


def qtile_flops(w):
    """Tensor-core flops of one query-tile attention launch: every (tile of 128 queries, visible tile of
    128 keys, head) runs S = Q Kᵀ and O += P V, 2 * 128^3 flops each (masked entries included)."""
    n_tiles = 0
    nqt = -(-w.n_q // 128)
    for qt in range(nqt):
        nr = min(128, w.n_q - 128 * qt)
        last = w.n_kv - w.n_q + 128 * qt + nr - 1
        n_tiles += last // 128 + 1
    return n_tiles * w.batch * w.n_heads * 2 * (2 * 128 ** 3), n_tiles * w.batch * w.n_heads


def indexer_bytes(w, counts):
    nq = w.batch * w.n_q
    hi = max(1, w.n_idx_heads)
    return (counts["n_cand"] * w.d_idx * 2            # token gather
            + w.batch * w.n_kv * w.d_idx * 2            # pooling read
            + nq * hi * w.d_idx * 2 + nq * (w.top_m + w.top_k) * 4)


def compulsory_bytes(w):
    """The floor of any schedule: every input read once (indexer keys and queries, head weights,
    Q, K, V) and every output written once (O, LSE); the index lists are intermediates."""
    nq = w.batch * w.n_q
    hi = max(1, w.n_idx_heads)
    return (w.batch * w.n_kv * w.d_idx * 2 + nq * hi * w.d_idx * 2 + (nq * hi * 4 if w.n_idx_heads else 0)
            + w.batch * w.n_kv * w.n_kv_heads * w.d_head * 2 * 2
            + nq * w.n_heads * w.d_head * 2 * 2 + nq * w.n_heads * 4)


def needle_recall(w, block_idx):
    """Fraction of the planted needle blocks among the probe query's kept blocks (the last query
    of each sequence: the query whose signs the needles follow), over all sequences."""
    from synth.workloads import needle_table

    if w.needles <= 0:
        return None
    sel = block_idx[:, w.n_q - 1].cpu().numpy()
    hits = total = 0
    for seq in range(w.batch):
        nb = set(needle_table(w, seq).tolist())
        hits += len(nb & set(sel[seq][sel[seq] >= 0].tolist()))
        total += len(nb)
    return hits / total if total else None


def l2_gather_peak(hs, dev, st, row_bytes=256, region_bytes=32 << 20, n_gathers=8 << 20):
    """Measured ceiling of the attention kernel's gathers (GB/s): hisa_gather_probe copying
    hashed 256-byte rows of a region into shared memory with the kernel's cp.async pattern and
    nothing else; a 32 MiB region (one head's K and V at 64K) stays in L2, a region of GiBs
    measures gathers from HBM.  The best of 5 event-timed
    launches at each of 2 and 3 CTAs (8 and 12 warps) per SM; returns (GB/s, CTAs per SM)."""
    import torch

    rows = torch.zeros(region_bytes, dtype=torch.uint8, device=dev)
    sink = torch.zeros(1, dtype=torch.int32, device=dev)
    best = (0.0, 0)
    for ctas in (2, 3):
        for _ in range(2):
            hs.hisa_gather_probe(rows, row_bytes, n_gathers, sink, ctas_per_sm=ctas, stream=st)
        ts = []
        for _ in range(5):
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            e0.record(st)
            hs.hisa_gather_probe(rows, row_bytes, n_gathers, sink, ctas_per_sm=ctas, stream=st)
            e1.record(st)
            e1.synchronize()
            ts.append(e0.elapsed_time(e1))
        best = max(best, (n_gathers * row_bytes / (min(ts) * 1e-3) / 1e9, ctas))
    return best


def _profile_record(kernel_file: str, summary_name: str, workload_name: str):
    """The committed ncu record of this kernel on this workload (DRAM bytes per launch, L2 hit
    rate), or None when there is none or the kernel changed since it was taken."""
    path = os.path.join(ROOT, "profiles", summary_name)
    src = os.path.join(ROOT, "hierarchical_sparse_attention_block_b200", "csrc", kernel_file)
    try:
        with open(path) as f:
            j = json.load(f)
        sha = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
        if j.get("source_sha256_16") != sha or j.get("workload") != workload_name:
            return None
        return j
    except Exception:
        return None


def run_ours(a, rank, world, local_rank):
    import numpy as np
    import torch

    import hierarchical_sparse_attention_block_b200 as hs
    import synth.device as sd
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(a, rank)
    p = hs.params_of(w)
    inp = sd.device_inputs(w, device=dev)
    wi = inp.get("w_idx")  # the indexer's head weights (multi-head indexer only)
    torch.cuda.synchronize()
    st = torch.cuda.Stream(device=dev)  # a side stream: CUDA graphs cannot be captured on the default one
    torch.cuda.set_stream(st)

    nq = w.batch * w.n_q
    bk = torch.empty((w.batch, w.n_blk, w.d_idx), dtype=torch.float32, device=dev)
    blk = torch.empty((w.batch, w.n_q, w.top_m), dtype=torch.int32, device=dev)
    tok = torch.empty((w.batch, w.n_q, w.top_k), dtype=torch.int32, device=dev)
    o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16, device=dev)
    lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32, device=dev)
    status = torch.zeros(1, dtype=torch.int32, device=dev)
    ws_topm = torch.empty(hs.hisa_block_topm_workspace_size(p), dtype=torch.uint8, device=dev)
    ws_tok = torch.empty(hs.hisa_token_topk_workspace_size(p)[1], dtype=torch.uint8, device=dev)
    n_attn_ws = hs.hisa_sparse_attn_workspace_size(p)
    ws_attn = torch.empty(max(n_attn_ws, 16), dtype=torch.uint8, device=dev)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=dev)

    stages = ["pool", "block_topm", "token_topk", "sparse_attn"]

    # Decode: the block keys of the cache persist across steps (pooled once at set-up, timed
    # separately); each step refreshes the newest block, which the new token changes.
    decode = w.n_q == 1
    pool_begin = w.n_blk - 1 if decode else 0
    pool_setup_ms = None
    if decode:
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        hs.hisa_block_pool(p, inp["k_idx"], bk, stream=st)
        e0.record(st)
        hs.hisa_block_pool(p, inp["k_idx"], bk, stream=st)
        e1.record(st)
        e1.synchronize()
        pool_setup_ms = e0.elapsed_time(e1)

    def step(ev):
        ev[0].record(st)
        hs.hisa_block_pool(p, inp["k_idx"], bk, pool_begin, -1, stream=st)
        ev[1].record(st)
        hs.hisa_block_topm(p, inp["q_idx"], bk, blk, None, status, ws_topm, stream=st, idx_weights=wi)
        ev[2].record(st)
        hs.hisa_token_topk(p, inp["q_idx"], inp["k_idx"], blk, tok, None, status, ws_tok, stream=st, idx_weights=wi)
        ev[3].record(st)
        hs.sparse_attn_fwd(p, inp["q"], inp["k"], inp["v"], tok, o, lse, status, ws_attn, stream=st)
        ev[4].record(st)

    def new_events():
        return [torch.cuda.Event(enable_timing=True) for _ in range(5)]

    for _ in range(a.warmup):
        flush.zero_()
        step(new_events())
    torch.cuda.synchronize()
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} after warm-up")

    # Decode steps are microseconds long: replay them from a CUDA graph, the whole step as one graph
    # (as a serving loop would) for the timed steps, and one graph per stage (the stage events
    # outside them) for the stage breakdown, in a separate pass.
    use_graph = a.graph == "on" or (a.graph == "auto" and decode)
    stage_step = None
    if use_graph:
        calls = [
            lambda: hs.hisa_block_pool(p, inp["k_idx"], bk, pool_begin, -1, stream=st),
            lambda: hs.hisa_block_topm(p, inp["q_idx"], bk, blk, None, status, ws_topm, stream=st, idx_weights=wi),
            lambda: hs.hisa_token_topk(p, inp["q_idx"], inp["k_idx"], blk, tok, None, status, ws_tok, stream=st,
                                       idx_weights=wi),
            lambda: hs.sparse_attn_fwd(p, inp["q"], inp["k"], inp["v"], tok, o, lse, status, ws_attn, stream=st),
        ]
        graphs = []
        for fn in calls:
            g = torch.cuda.CUDAGraph()
            with torch.cuda.graph(g, stream=st):
                fn()
            graphs.append(g)
        whole = torch.cuda.CUDAGraph()
        with torch.cuda.graph(whole, stream=st):
            for fn in calls:
                fn()
        torch.cuda.synchronize()

        def stage_step(ev):
            for j, g in enumerate(graphs):
                ev[j].record(st)
                g.replay()
            ev[4].record(st)

        def step(ev):  # noqa: F811
            ev[0].record(st)
            whole.replay()
            ev[4].record(st)

        for _ in range(a.warmup):
            step(new_events())
            stage_step(new_events())
        torch.cuda.synchronize()

    # the indexer alone and the flat comparator, for the speedup figure (outside the timed steps)
    comp = {}
    if world == 1 and not a.no_flat:
        flat_tok = torch.empty_like(tok)
        fmin, fpref = hs.hisa_flat_topk_workspace_size(p)
        ws_flat = torch.empty(fpref, dtype=torch.uint8, device=dev)
        for _ in range(2):
            hs.hisa_flat_topk(p, inp["q_idx"], inp["k_idx"], flat_tok, None, ws_flat, stream=st, idx_weights=wi)
        reps = max(2, min(a.steps, 5))
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        tt = []
        for _ in range(reps):
            flush.zero_()
            e0.record(st)
            hs.hisa_flat_topk(p, inp["q_idx"], inp["k_idx"], flat_tok, None, ws_flat, stream=st, idx_weights=wi)
            e1.record(st)
            e1.synchronize()
            tt.append(e0.elapsed_time(e1))
        comp["flat_indexer_ms"] = statistics.median(tt)
        del ws_flat, flat_tok

    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    evs = [new_events() for _ in range(a.steps)]
    g0, g1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clk = ClockSampler(local_rank if "CUDA_VISIBLE_DEVICES" not in os.environ else 0, enabled=not a.no_clock)
    with clk:
        # short timed regions (decode) are bracketed by extra untimed steps so the
        # sampler sees the GPU under this load
        t_pad = time.perf_counter()
        while not a.no_clock and time.perf_counter() - t_pad < 0.3:
            flush.zero_()
            step(new_events())
            torch.cuda.synchronize()
        g0.record(st)
        for s in range(a.steps):
            flush.zero_()
            step(evs[s])
        g1.record(st)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    torch.cuda.synchronize()
    stage_ms = {n: [] for n in stages}
    step_ms = [ev[0].elapsed_time(ev[4]) for ev in evs]
    sevs = evs
    if stage_step is not None:  # the stage breakdown of graph-replayed steps, in a pass of its own
        sevs = [new_events() for _ in range(a.steps)]
        for s in range(a.steps):
            flush.zero_()
            stage_step(sevs[s])
        torch.cuda.synchronize()
    for ev in sevs:
        for j, n in enumerate(stages):
            stage_ms[n].append(ev[j].elapsed_time(ev[j + 1]))
    ms = sum(step_ms) / len(step_ms)
    region_ms = g0.elapsed_time(g1)
    ms = max_over_ranks(ms, dev)
    if int(status.item()) != 0:
        raise RuntimeError(f"device status {int(status.item())} in the timed steps")

    counts = closed_form_counts(w)
    hbm_gbs, tf_burst, tf_sustained, peak_kind = _peaks()
    attn_ms = statistics.mean(stage_ms["sparse_attn"])
    a_bytes = attention_bytes(w, counts)
    eff_gbs = a_bytes / (attn_ms * 1e-3) / 1e9
    idx_ms = sum(statistics.mean(stage_ms[n]) for n in stages[:3])
    attn_kind = hs.hisa_sparse_attn_kernel(p, ws_attn.numel())

    # launches per step: pool, block score, top-m, 2 per token chunk, attention (query tile: masks,
    # V max, V to fp16, tiles; gather: one kernel, + merge when lists are split)
    per_q_keys = w.top_m * w.block * 4
    chunk = max(1, ws_tok.numel() // per_q_keys)
    n_chunks = math.ceil(nq / chunk)
    splits = 1 if n_attn_ws == 0 else 2
    attn_launches = 4 if attn_kind == hs.ATTN_QTILE else (1 if splits == 1 else 2)
    launches = 3 + 2 * n_chunks + attn_launches

    result = {
        "metric": METRIC, "value": job_value(nq, world, ms), "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
        "dtype": "bf16", "data": "synthetic (seeded SplitMix64; integer indexer q/k in [-4,4], unit-variance "
                                  "Irwin-Hall Q/K/V, planted needle blocks)",
        "config": {**workload_config(w), "parallelism": f"dp{world} (independent copies)",
                   "l2": f"flushed between steps ({L2_FLUSH_BYTES >> 20} MiB write)"},
        "roofline": None,
        "stages_ms": {n: statistics.mean(v) for n, v in stage_ms.items()},
        "pool_in_step": "newest block only (cache block keys persist)" if decode else "every block",
        "cuda_graph": "whole step as one graph (stage times from per-stage graphs, a separate pass)" if use_graph
                      else False,
        "pool_setup_ms": pool_setup_ms,
        "indexer_ms": idx_ms, "indexer_queries_per_s": nq / (idx_ms * 1e-3),
        "tokens_per_s": counts["k_eff"] / (ms * 1e-3),
        "end_to_end_hbm_roofline_frac_8tbs": ((a_bytes + indexer_bytes(w, counts)) / 8e12) / (ms * 1e-3),
        "compulsory_bytes": None if decode else compulsory_bytes(w),
        "compulsory_ms_at_8tbs": None if decode else compulsory_bytes(w) / 8e12 * 1e3,
        "needle_recall": needle_recall(w, blk),
        "region_ms_incl_l2_flush": region_ms,
        "gpu_launches": launches * a.steps,
        "clocks": clk.summary(),
    }
    # The dominant kernel's roofline, by the kernel that ran:
    #   query tile (prefill): tensor-bound; executed flops (masked entries included) over the stage time
    #     (which also holds the mask and V-conversion pre-passes) against the measured bf16 peak,
    #     sustained (the kernel runs inside a seconds-long loop of steps);
    #   gather, prefill: bound by the L2 -> SM gather rate (each head's K/V sits in L2 and serves many
    #     queries); algorithmic gather bytes against the measured gather ceiling of the same pattern;
    #   gather, decode: HBM-bound (no reuse); algorithmic bytes against the measured copy bandwidth.
    # The algorithmic bytes over the stage time, against HBM, are kept as effective_gbs: above the HBM
    # peak it is bandwidth the L2 (or tile reuse) supplies, not DRAM utilisation.
    rl = {"kernel": "sparse_attn_qtile" if attn_kind == hs.ATTN_QTILE else "sparse_attn", "peak_kind": peak_kind,
          "algorithmic_bytes_per_launch": a_bytes, "effective_gbs": eff_gbs,
          "effective_frac_of_hbm": eff_gbs / hbm_gbs, "traffic": None}
    if attn_kind == hs.ATTN_QTILE:
        fl, n_tile_heads = qtile_flops(w)
        tf = fl / (attn_ms * 1e-3) / 1e12
        rl.update({"bound": "tensor", "achieved": tf, "peak": tf_sustained, "unit": "TFLOP/s",
                   "frac": tf / tf_sustained, "frac_of_burst": tf / tf_burst,
                   "flops_per_launch": fl, "tile_heads_per_launch": n_tile_heads,
                   "selected_entry_frac": counts["k_eff"] * w.n_heads / (n_tile_heads * 128 * 128)})
        rec = _profile_record("sparse_attn_qtile.cu", f"sparse_attn_qtile_{w.name}.json", w.name)
    else:
        rec = _profile_record("sparse_attn.cu", f"sparse_attn_{w.name}.json", w.name)
        if decode:
            # decode gathers come from HBM with no reuse; the probe over a 4 GiB region (far larger than L2)
            # gives the gather ceiling of random 256-byte rows from DRAM
            pk, ctas = l2_gather_peak(hs, dev, st, region_bytes=4 << 30)
            rl.update({"bound": "hbm", "achieved": eff_gbs, "peak": hbm_gbs, "unit": "GB/s", "frac": eff_gbs / hbm_gbs,
                       "frac_of_nominal_8tbs": eff_gbs / 8000.0,
                       "hbm_gather": {"peak_gbs": pk, "frac": eff_gbs / pk,
                                      "probe": f"hisa_gather_probe: 16-byte cp.async gathers of hashed 256-byte rows "
                                               f"of a 4 GiB region (HBM) into shared memory, 4 stages, no arithmetic; "
                                               f"best of 8 and 12 warps per SM ({4 * ctas} here)"}})
        else:
            pk, ctas = l2_gather_peak(hs, dev, st)
            rl.update({"bound": "l2", "achieved": eff_gbs, "peak": pk, "unit": "GB/s", "frac": eff_gbs / pk,
                       "peak_kind": "measured in this run: hisa_gather_probe, 16-byte cp.async gathers of hashed "
                                    f"256-byte rows of a 32 MiB L2-resident region, best of 8 and 12 warps per SM "
                                    f"({4 * ctas} here)"})
    if rec is not None:
        # DRAM bytes of one launch from the committed ncu record of the same kernel source
        t = rec.get("dram_bytes_per_launch_full_workload")
        rl["traffic"] = t
        rl["dram_gbs"] = t / (attn_ms * 1e-3) / 1e9
        rl["dram_frac"] = t / (attn_ms * 1e-3) / 1e9 / hbm_gbs
        if rec.get("l2_hit_rate_pct") is not None:
            rl["l2_hit_rate_pct"] = rec["l2_hit_rate_pct"]
    result["roofline"] = rl
    if comp:
        result["flat_indexer_ms"] = comp["flat_indexer_ms"]
        result["speedup_vs_flat_indexer"] = comp["flat_indexer_ms"] / idx_ms

    if not a.no_e2e:
        result["e2e"] = run_e2e(a, hs, w, p, inp, dev, st, world)
    del inp
    torch.cuda.empty_cache()
    return result


def run_e2e(a, hs, w, p, inp, dev, st, world):
    """The same metric through the public API with host-resident inputs: every step copies its
    inputs from pinned host memory and reads the outputs back.  Prefill: every input is a step
    input and hisa_forward_host takes the host buffers, overlapping the copies with the work on
    a second stream.  Decode: the caches (k_idx, K, V) and their block keys stay resident on the
    device, as in a serving loop, the step inputs are the new queries (q_idx, Q), and
    hisa_forward_cached refreshes only the newest block."""
    import torch

    decode = w.n_q == 1
    names = ["q_idx", "q"] if decode else ["q_idx", "k_idx", "q", "k", "v"]
    if "w_idx" in inp:  # the indexer's head weights come with each step's queries
        names.append("w_idx")
    host = {k: inp[k].cpu().pin_memory() for k in names}
    h_o = torch.empty((w.batch, w.n_q, w.n_heads, w.d_head), dtype=torch.bfloat16).pin_memory()
    h_lse = torch.empty((w.batch, w.n_q, w.n_heads), dtype=torch.float32).pin_memory()
    h2d = sum(v.numel() * v.element_size() for v in host.values())
    d2h = h_o.numel() * 2 + h_lse.numel() * 4

    if decode:
        d_in = {k: (torch.empty_like(host[k], device=dev) if k in host else inp[k])
                for k in ["q_idx", "k_idx", "q", "k", "v"] + (["w_idx"] if "w_idx" in inp else [])}
        o = torch.empty(h_o.shape, dtype=h_o.dtype, device=dev)
        lse = torch.empty(h_lse.shape, dtype=h_lse.dtype, device=dev)
        ws = torch.empty(hs.hisa_forward_workspace_size(p), dtype=torch.uint8, device=dev)
        bk = torch.empty((w.batch, w.n_blk, w.d_idx), dtype=torch.float32, device=dev)
        hs.hisa_block_pool(p, d_in["k_idx"], bk, stream=st)  # pooled once; persists between steps

        def one():
            for k in host:
                d_in[k].copy_(host[k], non_blocking=True)
            hs.hisa_forward_cached(p, d_in["q_idx"], d_in["k_idx"], bk, w.n_blk - 1, d_in["q"], d_in["k"], d_in["v"],
                                   o, lse, None, None, None, ws, stream=st, idx_weights=d_in.get("w_idx"))
            h_o.copy_(o, non_blocking=True)
            h_lse.copy_(lse, non_blocking=True)
        api = "hisa_forward_cached (caches resident; queries copied in, O/LSE copied out)"
    else:
        ws = torch.empty(hs.hisa_forward_host_workspace_size(p), dtype=torch.uint8, device=dev)
        cs = torch.cuda.Stream(device=dev)

        def one():
            hs.hisa_forward_host(p, host["q_idx"], host["k_idx"], host["q"], host["k"], host["v"], h_o, h_lse, None,
                                 ws, stream=st, copy_stream=cs, idx_weights=host.get("w_idx"))
        api = "hisa_forward_host (host buffers; copies overlapped with the work on a second stream)"

    for _ in range(max(1, a.warmup)):
        one()
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    steps = max(1, min(a.steps, 5))
    e0.record(st)
    for _ in range(steps):
        one()
    e1.record(st)
    torch.cuda.synchronize()
    ms = max_over_ranks(e0.elapsed_time(e1) / steps, dev)
    del host, ws
    return {"value": job_value(w.batch * w.n_q, world, ms), "unit": UNIT, "ms_per_step": ms,
            "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps, "api": api}


def oracle_sample(w, seconds: float, device_inputs=None):
    """Time the CPU oracle (as it stands) on a position-stratified sample of queries, scaled to
    queries/s.  Inputs come from the seeded generator (device half, bit-identical to the host half)."""
    import numpy as np

    import oracle
    from synth.workloads import full_inputs

    O = oracle.Oracle()
    threads = O.threads()
    if device_inputs is not None:
        import torch

        inp = {k: (v.cpu().numpy() if v.dtype == torch.float32 else v.view(torch.int16).cpu().numpy().view(np.uint16))
               for k, v in device_inputs.items() if not k.startswith("_")}
    else:
        inp = full_inputs(w)
    t0 = time.perf_counter()
    bkeys = np.stack([O.block_pool(inp["k_idx"][s], w.block) for s in range(w.batch)])
    pool_s = time.perf_counter() - t0
    nq = w.batch * w.n_q
    done, elapsed, reps = 0, 0.0, 0
    rng = np.random.default_rng(0)
    if nq <= 8192:
        # small workloads: whole passes over every query
        while reps == 0 or elapsed < seconds:
            t0 = time.perf_counter()
            O.run(w, inp, block_keys=bkeys)
            elapsed += time.perf_counter() - t0
            done += nq
            reps += 1
        what = f"{reps} full pass(es) over all {nq} queries"
    else:
        n = 8
        while elapsed < seconds:
            ids = np.sort(rng.choice(nq, size=min(n, nq), replace=False)).astype(np.int64)
            t0 = time.perf_counter()
            O.run(w, inp, query_ids=ids, block_keys=bkeys)
            elapsed += time.perf_counter() - t0
            done += len(ids)
            n = min(n * 2, 4096)
        what = f"{done} query evaluations drawn uniformly over the {nq} positions"
    per_q = elapsed / done
    total_s = pool_s + per_q * nq
    # the same path on one core: a short sample of queries drawn the same way
    O.set_threads(1)
    try:
        ids = np.sort(rng.choice(nq, size=min(64, nq), replace=False)).astype(np.int64)
        t0 = time.perf_counter()
        O.run(w, inp, query_ids=ids, block_keys=bkeys)
        per_q1 = (time.perf_counter() - t0) / len(ids)
    finally:
        O.set_threads(threads)
    return {"value": nq / total_s, "unit": UNIT, "cores": threads, "kind": "oracle",
            "sample": f"{what}, full path (top-m, top-k, attention in fp64) plus pooling of every block; "
                      f"{elapsed + pool_s:.1f} s of CPU time, scaled to the whole workload",
            "single_core_value": 1.0 / per_q1, "single_core_sample": f"{len(ids)} queries on one thread "
                                                                     f"(pooling excluded)"}


def oracle_sample_rows(w, seconds: float):
    """The CPU oracle on whole sequences of a large workload (decode caches of tens of GiB):
    only the rows it touches are regenerated on the host (untimed); the oracle's own calls --
    pooling of every block, top-m, top-k and attention -- are timed."""
    import math as _m

    import numpy as np

    import oracle
    from synth.workloads import k_idx_rows, k_rows, q_idx_rows, q_rows, v_rows, w_idx_rows

    O = oracle.Oracle()
    timed, done_q, seqs = 0.0, 0, 0
    wall0 = time.perf_counter()
    for seq in range(w.batch):
        k_idx = k_idx_rows(w, seq, 0, w.n_kv)
        t0 = time.perf_counter()
        bk = O.block_pool(k_idx, w.block)
        timed += time.perf_counter() - t0
        for i in range(w.n_q):
            p = w.n_kv - w.n_q + i
            qi = q_idx_rows(w, seq, i, 1)[0]
            wi = w_idx_rows(w, seq, i, 1)[0] if w.n_idx_heads else None
            t0 = time.perf_counter()
            sel, _ = O.block_topm(qi, bk, w.block, p, w.top_m, w=wi)
            tok, _, _ = O.token_topk(qi, k_idx, w.block, p, sel, w.top_k, w=wi)
            timed += time.perf_counter() - t0
            valid = tok[tok >= 0]
            kk, vv = k_rows(w, seq, valid), v_rows(w, seq, valid)
            remap = np.full(w.top_k, -1, dtype=np.int32)
            remap[: len(valid)] = np.arange(len(valid), dtype=np.int32)
            qr = q_rows(w, seq, i, 1)[0]
            t0 = time.perf_counter()
            O.sparse_attn(qr, kk, vv, remap, 1.0 / _m.sqrt(w.d_head))
            timed += time.perf_counter() - t0
            done_q += 1
        seqs += 1
        if time.perf_counter() - wall0 > seconds:
            break
    return {"value": done_q / timed, "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{seqs} of {w.batch} sequences ({done_q} queries), full path including pooling of every "
                      f"block of each sampled sequence, single-threaded oracle calls; {timed:.2f} s of oracle time "
                      f"(host row regeneration excluded)"}


def main():
    a = _args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch

        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=300))

    if a.impl == "reference":
        if rank == 0:
            w = workload(a)
            budget = a.cpu_seconds * max(1, a.steps) / 10.0
            cpu = oracle_sample_rows(w, budget) if w.n_q == 1 else oracle_sample(w, budget)
            line = {"impl": "reference", "metric": METRIC, "value": cpu["value"], "unit": UNIT, "n_gpus": world,
                    "steps": a.steps, "warmup": a.warmup, "ms_per_step": 1e3 * w.batch * w.n_q / cpu["value"],
                    "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
                    "data": "synthetic", "config": {**workload_config(w), "parallelism": "host cores (oracle)"},
                    "cpu_baseline": {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")},
                    "e2e": {"value": cpu["value"], "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
            print(json.dumps(line), flush=True)
        if world > 1:
            import torch

            torch.distributed.destroy_process_group()
        return

    import torch

    res = run_ours(a, rank, world, local_rank)
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        import synth.device as sd

        w = workload(a)
        if w.n_q == 1:
            res["cpu_baseline"] = oracle_sample_rows(w, a.cpu_seconds)
        else:
            small = w.batch * w.n_q <= 8192
            dev_inp = None if small else sd.device_inputs(w, device=torch.device("cuda", local_rank))
            res["cpu_baseline"] = oracle_sample(w, a.cpu_seconds, dev_inp)
            del dev_inp
    if rank == 0:
        print(json.dumps(res), flush=True)
    if world > 1:
        torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
