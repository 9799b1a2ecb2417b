#!/usr/bin/env python
"""Benchmark of the MSA decode step (indexer -> max-pool -> top-16 -> sparse
attention) on B200, one process per GPU.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--impl reference]

Multi-GPU: launch with torch.distributed.run (one rank per GPU); the path
shards by sequence, so every rank decodes its own batch of the workload with
no data-path collective (weak scaling); the only collectives are the timing
barrier and the max-over-ranks of the measured time.

Prints one JSON line (rank 0).  `value` is whole-job decode queries/s (query
tokens of all ranks per second), device-timed with CUDA events; `roofline`
describes the kernel with the largest time share; `e2e` repeats the step
through the Python binding with host (pinned) query buffers copied in and the
output copied out inside the timed region, pipelined as a serving loop runs
(copies overlap other steps' decodes); `cpu_baseline` times the float64
oracle on a bounded sample of the same workload on the host cores.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "MSA decode queries/s and achieved HBM GB/s (% of B200 peak) at 128K ctx"
DEFAULT_WORKLOAD = "ctx128k_b64_t8"
SPEC_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


# ------------------------------------------------------------------ ranks --
def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def rank_seed_offset(rank: int) -> int:
    """Every rank decodes its own batch: same shapes, its own seed."""
    return 7919 * rank


def max_over_ranks(x: float, world: int) -> float:
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    dev = "cuda" if dist.get_backend() == "nccl" else "cpu"
    t = torch.tensor([x], dtype=torch.float64, device=dev)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


# ----------------------------------------------------------------- peaks --
def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return float(d.get("hbm_gbs", FALLBACK_HBM_GBS)), "measured"
    return FALLBACK_HBM_GBS, "fallback"


FALLBACK_BF16_TFLOPS = 1590.0


def measured_bf16_tflops():
    """Dense bf16 tensor throughput (burst) from the generated file, else
    the pool's earlier measurement; the FP8 figure is twice it (the nominal
    FP8 / bf16 ratio of the part)."""
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        if "bf16_tflops" in d:
            return float(d["bf16_tflops"]), "measured"
    return FALLBACK_BF16_TFLOPS, "fallback"


def source_sha(files) -> str:
    h = hashlib.sha1()
    for f in files:
        h.update(open(os.path.join(ROOT, f), "rb").read())
    return h.hexdigest()[:12]


KERNEL_SOURCES = {
    "indexer": ["block_sparse_attention_decode_b200/csrc/msa_indexer.cu",
                "block_sparse_attention_decode_b200/csrc/msa_device.cuh"],
    "attention": ["block_sparse_attention_decode_b200/csrc/msa_attn.cu",
                  "block_sparse_attention_decode_b200/csrc/msa_device.cuh"],
    "topk": ["block_sparse_attention_decode_b200/csrc/msa_topk.cu"],
    "indexer_exact": ["block_sparse_attention_decode_b200/csrc/msa_indexer.cu",
                      "block_sparse_attention_decode_b200/csrc/msa_device.cuh"],
}


L2_BYTES = 126 * 1000 * 1000


def l2_notes(cache_bytes: int):
    """How the timed regions treat L2 for a cache of cache_bytes: the note of
    the device-timed steps and the note of the end-to-end loop."""
    gb = cache_bytes / 1e9
    if cache_bytes > L2_BYTES:
        return ("256 MiB written before each timed step (outside the events); "
                "inputs %.1f GB > 126 MB L2" % gb, "no L2 flush (inputs > L2)")
    return ("256 MiB written before each timed step (outside the events); inputs %.3f GB "
            "fit in the 126 MB L2, so the flush is what sends them back to HBM" % gb,
            "no L2 flush: the inputs (%.3f GB) fit in L2 and stay there from step to step" % gb)


def dram_traffic(kernel: str, workload: str):
    """Per-launch DRAM bytes from the committed ncu summary, or None when the
    kernel source changed since the counters were taken."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p)).get(kernel, {})
    if d.get("workload") != workload or d.get("source_sha") != source_sha(KERNEL_SOURCES[kernel]):
        return None
    return d.get("bytes_per_launch")


# ---------------------------------------------------------------- clocks --
def smi_index(local_rank: int) -> str:
    vis = os.environ.get("CUDA_VISIBLE_DEVICES")
    if vis:
        ids = [x.strip() for x in vis.split(",") if x.strip()]
        if local_rank < len(ids):
            return ids[local_rank]
    return str(local_rank)


class ClockSampler:
    """nvidia-smi clocks/throttle reasons sampled while the timed region runs."""
    Q = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
         "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
         "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), "--query-gpu=" + self.Q,
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.t = threading.Thread(target=self._read, daemon=True)
            self.t.start()
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append((time.time(), line.strip()))

    def mark(self, which: str):
        setattr(self, which, time.time())

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        t0, t1 = getattr(self, "start", 0.0), getattr(self, "stop", float("inf"))
        for ts, ln in self.lines:
            if not (t0 <= ts <= t1 + 0.15):
                continue
            f = [x.strip() for x in ln.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx), "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ byte model --
def algorithmic_bytes(w, sel):
    """Bytes the traffic model of the method implies for one step: the full
    index-key scan, the selected K/V only (each distinct block of a (sequence,
    group) once, over the union of its query tokens' selections, counting only
    the visible tokens of a partial block), the queries and the output."""
    import torch
    lens = w.seq_lens.long()
    idx_per_tok = 128 if w.idx_fp8 else 72
    idx_bytes = int(lens.sum().item()) * idx_per_tok
    B, T = w.batch, w.q_tokens
    s = sel.long()                                        # [B][T][4][16]
    mp = w.max_pages
    mark = torch.zeros(B, 4, mp + 1, dtype=torch.bool, device=s.device)
    flat = torch.where(s >= 0, s, torch.full_like(s, mp))  # -1 -> dummy column
    mark.scatter_(2, flat.permute(0, 2, 1, 3).reshape(B, 4, T * 16), True)
    mark = mark[:, :, :mp]
    blk = torch.arange(mp, device=s.device)
    valid_tok = (lens.view(B, 1) - blk.view(1, mp) * 128).clamp(0, 128)   # tokens in block
    kv_tokens = int((mark.to(torch.int64) * valid_tok.view(B, 1, mp)).sum().item())
    kv_bytes = kv_tokens * 144
    q_bytes = B * T * (64 * 128 + 4 * 128)
    out_bytes = B * T * 64 * 128 * 2
    return {"index_scan": idx_bytes, "kv_selected": kv_bytes, "queries": q_bytes,
            "output": out_bytes, "total": idx_bytes + kv_bytes + q_bytes + out_bytes,
            "kv_tokens": kv_tokens}


# --------------------------------------------------------- CPU baseline --
def cpu_sample_workload(name: str, seed_offset: int = 0, nseq: int = 1):
    """nseq sequences with the shapes of `name` (the longest context of the
    workload, all of its query tokens), generated on the host: a bounded
    sample of the workload."""
    from block_sparse_attention_decode_b200 import synth
    kw = dict(synth.WORKLOADS[name])
    if kw["seq_lens"] is None:
        kw["seq_lens"] = synth.ragged_lengths(kw["batch"], 2048, 262144, kw["seed"])
    L = max(kw["seq_lens"])
    kw.update(batch=nseq, seq_lens=[L] * nseq, seed=kw["seed"] + 100 + seed_offset)
    return synth.make_workload(name + "_cpu_sample", device="cpu", **kw)


def oracle_step(w, rows, threads):
    """The float64 oracle's whole path (index scan, top-16, attention) for the
    (sequence, token) rows of w on `threads` host threads; seconds."""
    import numpy as np
    import oracle
    oracle.set_threads(threads)
    n = lambda t: None if t is None else t.numpy()
    c = oracle.Cache(idx_data=n(w.idx_data), idx_scale=n(w.idx_scale), k_data=n(w.k_data),
                     k_scale=n(w.k_scale), v_data=n(w.v_data), v_scale=n(w.v_scale),
                     s_idx=w.s_idx, s_k=w.s_k, s_v=w.s_v, page_table=n(w.page_table),
                     max_pages=w.max_pages, seq_lens=n(w.seq_lens), q_tokens=w.q_tokens)
    t0 = time.perf_counter()
    oracle.decode(c, np.ascontiguousarray(n(w.qi)), w.s_qi, np.ascontiguousarray(n(w.q)), w.s_q,
                  w.softmax_scale, list(rows))
    return time.perf_counter() - t0


def host_threads() -> int:
    """Threads both oracle arms use: every host core."""
    return max(1, os.cpu_count() or 1)


def cpu_baseline(name: str, budget_s: float = 20.0):
    import math
    from block_sparse_attention_decode_b200 import synth
    threads = host_threads()
    T = synth.WORKLOADS[name]["q_tokens"]
    nseq = max(1, math.ceil(threads / T))          # enough (sequence, token) rows for every thread
    w = cpu_sample_workload(name, nseq=nseq)
    rows = [(b, t) for b in range(nseq) for t in range(T)]
    dt = oracle_step(w, rows, threads)
    reps = 1
    while dt * (reps + 1) / reps < budget_s and reps < 3:
        dt += oracle_step(w, rows, threads)
        reps += 1
    qps = reps * len(rows) / dt
    return {"value": qps, "unit": "queries/s", "cores": threads, "kind": "oracle",
            "sample": "%d x (%d sequences of %d tokens, all %d query tokens of each: full index "
                      "scan, top-16, attention) of %s, float64 C oracle on %d host threads"
                      % (reps, nseq, int(w.seq_lens[0]), T, name, threads)}


# --------------------------------------------------------- sub-records --
def timed(fn, steps, flush, stream, mean=False):
    """Median (or mean) CUDA-event time (ms) of fn over `steps` runs, L2
    flushed before each (outside the events), after 3 untimed runs."""
    import torch
    for _ in range(3):
        fn()
    ts = []
    for _ in range(steps):
        flush.fill_(1)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(stream)
        fn()
        e1.record(stream)
        torch.cuda.synchronize()
        ts.append(e0.elapsed_time(e1))
    return statistics.mean(ts) if mean else statistics.median(ts)


def prefill_record(steps, flush, stream):
    """Chunked prefill (1 sequence, 65,536 cached + 2,048 new tokens, every
    new token a query with its own top-16 over its causal prefix): step time,
    tokens/s and the two contractions' FLOP/s against the FP8 dense peak
    (2 x the measured bf16 burst)."""
    import torch
    import block_sparse_attention_decode_b200 as msa
    from block_sparse_attention_decode_b200 import synth
    name = "prefill_67584_t2048"
    w = synth.make_workload(name, device="cuda", **dict(synth.WORKLOADS[name]))
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    B, T = w.batch, w.q_tokens
    out = torch.empty(B, T, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, T, 4, 16, dtype=torch.int32, device="cuda")
    bs = torch.empty(B, T, 4, w.max_pages, device="cuda")
    step = lambda: msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws, stream)
    ms = timed(step, steps, flush, stream)
    per = {
        "indexer": timed(lambda: msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, None, bs, ws, stream), steps, flush, stream),
        "topk": timed(lambda: msa.msa_block_maxpool_topk(bs, False, seqs, sel, ws, stream), steps, flush, stream),
        "attention": timed(lambda: msa.msa_sparse_attn_decode(cache, seqs, w.q, w.s_q, sel, w.softmax_scale, out, ws, stream),
                           steps, flush, stream),
    }
    st, detail = msa.msa_get_last_error(ws, stream)
    if st != msa.MSA_OK:
        raise RuntimeError("device error %d (%d) in the prefill record" % (st, detail))
    L = int(w.seq_lens[0])
    pos = torch.arange(L - T, L, dtype=torch.float64)
    # indexer: every index query (4 per token) against every visible key, 128-dim dot products
    idx_flop = float(4 * 2 * 128 * (pos + 1).sum())
    # attention: 16 heads per (token, group), QK and PV over the visible keys of the selection
    s = sel[0].long().cpu()                                   # [T][4][16]
    blk_keys = (torch.clamp((pos.view(T, 1, 1) + 1) - s.double() * 128, 0, 128) * (s >= 0))
    att_flop = float(blk_keys.sum() * 16 * 128 * 2 * 2)
    bf16, src = measured_bf16_tflops()
    fp8 = 2 * bf16
    rec = {"workload": name, "ms_per_step": ms, "tokens_per_s": T / (ms * 1e-3), "kernel_ms": per,
           "fp8_peak_tflops": fp8, "peak_note": "2 x the %s dense bf16 burst (nominal FP8/bf16 ratio)" % src}
    for k, f in (("indexer", idx_flop), ("attention", att_flop)):
        tf = f / (per[k] * 1e-3) / 1e12
        rec[k] = {"gflop": f / 1e9, "tflops": tf, "frac_of_fp8_peak": tf / fp8}
    del w, cache, out, sel, bs, ws
    torch.cuda.empty_cache()
    return rec


def shared_prefix_record(steps, flush, stream):
    """Shared-prefix decode ([post, "AMD GPU support", "NVFP4 MSA kernel"]):
    64 sequences of 131,072 tokens whose first 65,536 tokens (512 blocks) are
    the same cached pages, 8 query tokens each.  The grouped step reads and
    decodes each shared page once per tile of 128 of the group's index
    queries, the plain step once per sequence; both timed, bytes counting each
    shared page once."""
    import torch
    import block_sparse_attention_decode_b200 as msa
    from block_sparse_attention_decode_b200 import synth
    B, L, T, pre = 64, 131072, 8, 512
    w = synth.make_workload("prefix64k_b64_t8", B, [L] * B, T, paged=True, seed=1006, device="cuda",
                            prefix_groups=[(B, pre)])
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    groups = msa.PrefixGroups.of([(B, pre)])
    ws = msa.alloc_workspace(seqs)
    out = torch.empty(B, T, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, T, 4, 16, dtype=torch.int32, device="cuda")
    bs = torch.empty(B, T, 4, w.max_pages, device="cuda")
    ms_g = timed(lambda: msa.msa_decode_grouped(cache, seqs, groups, w.qi, w.s_qi, w.q, w.s_q,
                                                w.softmax_scale, out, sel, ws, stream), steps, flush, stream)
    ms_u = timed(lambda: msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel,
                                        ws, stream), steps, flush, stream)
    idx_g = timed(lambda: msa.msa_indexer_score_grouped(cache, seqs, groups, w.qi, w.s_qi, None, bs, ws, stream),
                  steps, flush, stream)
    idx_u = timed(lambda: msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, None, bs, ws, stream), steps, flush, stream)
    st, detail = msa.msa_get_last_error(ws, stream)
    if st != msa.MSA_OK:
        raise RuntimeError("device error %d (%d) in the shared-prefix record" % (st, detail))
    by = algorithmic_bytes(w, sel)
    idx_unique = w.num_pages * 128 * 72          # every distinct index page once
    total = by["total"] - by["index_scan"] + idx_unique
    peak, _ = measured_peaks()
    rec = {"workload": "prefix64k_b64_t8: 64 x 131,072 tokens, the first 65,536 shared, 8 query tokens",
           "grouped_ms": ms_g, "plain_ms": ms_u, "indexer_grouped_ms": idx_g, "indexer_plain_ms": idx_u,
           "queries_per_s": B * T / (ms_g * 1e-3), "algorithmic_bytes": total,
           "index_bytes_distinct_pages": idx_unique,
           "achieved_gbs": total / (ms_g * 1e-3) / 1e9, "frac_of_measured": total / (ms_g * 1e-3) / 1e9 / peak}
    del w, cache, out, sel, bs, ws
    torch.cuda.empty_cache()
    return rec


# ------------------------------------------------------------- GPU arm ----
def run_gpu(args, rank, world, local_rank):
    import torch
    import block_sparse_attention_decode_b200 as msa
    from block_sparse_attention_decode_b200 import build as msa_build
    from block_sparse_attention_decode_b200 import synth

    torch.cuda.set_device(local_rank)
    if rank == 0 or not os.path.exists(msa.LIB_PATH):
        msa_build.build()
    barrier(world)
    msa.load()
    name = args.workload
    kw = dict(synth.WORKLOADS[name])
    if kw["seq_lens"] is None:
        kw["seq_lens"] = synth.ragged_lengths(kw["batch"], 2048, 262144, kw["seed"])
    if args.batch:
        kw["seq_lens"] = (list(kw["seq_lens"]) * args.batch)[: args.batch]
        kw["batch"] = args.batch
    kw["seed"] += rank_seed_offset(rank)
    w = synth.make_workload(name, device="cuda", **kw)
    cache, seqs = msa.cache_of(w), msa.seqs_of(w)
    ws = msa.alloc_workspace(seqs)
    B, T = w.batch, w.q_tokens
    out = torch.empty(B, T, 64, 128, dtype=torch.bfloat16, device="cuda")
    sel = torch.empty(B, T, 4, 16, dtype=torch.int32, device="cuda")
    bscores = torch.empty(B, T, 4, w.max_pages, dtype=torch.float32, device="cuda")
    flush = torch.empty(256 * 1024 * 1024, dtype=torch.uint8, device="cuda")   # > 126 MB L2
    stream = torch.cuda.current_stream()

    def step():
        msa.msa_decode(cache, seqs, w.qi, w.s_qi, w.q, w.s_q, w.softmax_scale, out, sel, ws, stream)

    clk = ClockSampler(smi_index(local_rank)).__enter__()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    st, detail = msa.msa_get_last_error(ws)
    if st != msa.MSA_OK:
        raise RuntimeError("device error %d (%d) during warm-up" % (st, detail))

    # ---- timed region: K steps, L2 flushed before each (outside the events)
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
           for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    clk.mark("start")
    t_wall = time.perf_counter()
    for e0, e1 in evs:
        flush.fill_(1)
        e0.record(stream)
        step()
        e1.record(stream)
    torch.cuda.synchronize()
    t_wall = time.perf_counter() - t_wall
    barrier(world)
    ms = sum(e0.elapsed_time(e1) for e0, e1 in evs) / args.steps
    ms_max = max_over_ranks(ms, world)

    # ---- per-kernel times: each stage entry point timed on its own (L2
    # flushed before each launch, outside the events), so that no kernel's
    # time includes a neighbour's tail overlapped by programmatic launch
    names = ("indexer", "topk", "attention")
    per = {
        "indexer": timed(lambda: msa.msa_indexer_score(cache, seqs, w.qi, w.s_qi, None, bscores, ws, stream),
                         args.steps, flush, stream, mean=True),
        "topk": timed(lambda: msa.msa_block_maxpool_topk(bscores, False, seqs, sel, ws, stream),
                      args.steps, flush, stream, mean=True),
        "attention": timed(lambda: msa.msa_sparse_attn_decode(cache, seqs, w.q, w.s_q, sel, w.softmax_scale,
                                                              out, ws, stream), args.steps, flush, stream, mean=True),
    }
    st, detail = msa.msa_get_last_error(ws)
    if st != msa.MSA_OK:
        raise RuntimeError("device error %d (%d) during timing" % (st, detail))

    bytes_ = algorithmic_bytes(w, sel)
    kernel_bytes = {"indexer": bytes_["index_scan"] + B * T * 512 + B * T * 4 * w.max_pages * 4,
                    "topk": B * T * 4 * w.max_pages * 4 + B * T * 4 * 16 * 4,
                    "attention": bytes_["kv_selected"] + B * T * 64 * 128 * 3 + B * T * 4 * 16 * 4}
    dom = max(names, key=lambda k: per[k])
    peak, peak_src = measured_peaks()
    achieved = kernel_bytes[dom] / (per[dom] * 1e-3) / 1e9
    traffic = dram_traffic(dom, name)

    # ---- the exact index-score variant (MSA_IDX_NVFP4_EXACT: the same NVFP4
    # index keys scored at their exact value with FP16 MMA), timed like the
    # indexer above on the same cache
    idx_exact = None
    if not w.idx_fp8:
        cache_x = msa.Cache(w.idx_data, w.idx_scale, w.k_data, w.k_scale, w.v_data, w.v_scale,
                            w.s_idx, w.s_k, w.s_v, idx_exact=True)
        for _ in range(3):
            msa.msa_indexer_score(cache_x, seqs, w.qi, w.s_qi, None, bscores, ws, stream)
        evx = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
               for _ in range(args.steps)]
        for e0, e1 in evx:
            flush.fill_(1)
            e0.record(stream)
            msa.msa_indexer_score(cache_x, seqs, w.qi, w.s_qi, None, bscores, ws, stream)
            e1.record(stream)
        torch.cuda.synchronize()
        st, detail = msa.msa_get_last_error(ws)
        if st != msa.MSA_OK:
            raise RuntimeError("device error %d (%d) in the exact indexer" % (st, detail))
        x_ms = sum(a.elapsed_time(b) for a, b in evx) / args.steps
        x_gbs = kernel_bytes["indexer"] / (x_ms * 1e-3) / 1e9
        idx_exact = {"ms": x_ms, "achieved_gbs": x_gbs, "frac": x_gbs / peak,
                     "bytes_per_launch": kernel_bytes["indexer"],
                     "traffic": dram_traffic("indexer_exact", name),
                     "note": "NVFP4 index keys decoded exactly to FP16 and scored with FP16 "
                             "MMA (no E4M3 re-rounding); not part of the timed step"}

    # ---- the step before the path: writing the step's B*T new tokens into
    # the cache (their K, V and index key, from bf16), timed on its own into
    # a scratch copy of the pages it writes so the benchmark cache is unchanged
    g_ins = torch.Generator(device=w.k_data.device).manual_seed(12345)
    k_new = torch.randn(B, T, 4, 128, generator=g_ins, device=w.k_data.device).to(torch.bfloat16)
    v_new = torch.randn(B, T, 4, 128, generator=g_ins, device=w.k_data.device).to(torch.bfloat16)
    i_new = torch.randn(B, T, 128, generator=g_ins, device=w.k_data.device).to(torch.bfloat16)
    ins_cache = msa.Cache(w.idx_data.clone(), None if w.idx_scale is None else w.idx_scale.clone(),
                          w.k_data.clone(), w.k_scale.clone(), w.v_data.clone(), w.v_scale.clone(),
                          w.s_idx, w.s_k, w.s_v)
    for _ in range(3):
        msa.msa_kv_insert(ins_cache, seqs, k_new, v_new, i_new, ws, stream)
    ins_ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(20)]
    for e0, e1 in ins_ev:
        flush.fill_(1)
        e0.record(stream)
        msa.msa_kv_insert(ins_cache, seqs, k_new, v_new, i_new, ws, stream)
        e1.record(stream)
    torch.cuda.synchronize()
    ins_ms = statistics.median(a.elapsed_time(b) for a, b in ins_ev)
    ins_bytes = B * T * (2 * 4 * 128 * 2 + 128 * 2 + 2 * 4 * 72 + (128 if w.idx_fp8 else 72))
    del ins_cache

    # ---- end to end through the binding: host queries in, output out.
    # Steps run as a serving loop runs them: step i+1's queries are copied
    # in (copy stream) and step i's output copied out (another copy stream)
    # while a decode runs; inputs and outputs are double-buffered on the
    # device and every step's copies lie inside the timed region.  The
    # cache (5.4 GB) exceeds L2, so this loop writes no flush buffer.
    h_qi = w.qi.cpu().pin_memory()
    h_q = w.q.cpu().pin_memory()
    h_lens = w.seq_lens.cpu().pin_memory()
    h_out = [torch.empty(out.shape, dtype=out.dtype).pin_memory() for _ in range(2)]
    d_qi = [torch.empty_like(w.qi) for _ in range(2)]
    d_q = [torch.empty_like(w.q) for _ in range(2)]
    d_lens = [torch.empty_like(w.seq_lens) for _ in range(2)]
    d_out = [out, torch.empty_like(out)]
    seqs_e2e = [msa.Seqs(d_lens[j], T, w.max_pages, w.page_table) for j in range(2)]
    s_in, s_out = torch.cuda.Stream(), torch.cuda.Stream()

    def run_e2e(nsteps):
        ev_in = [torch.cuda.Event() for _ in range(nsteps)]
        ev_dec = [torch.cuda.Event() for _ in range(nsteps)]
        ev_out = [torch.cuda.Event() for _ in range(nsteps)]
        t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        t0.record(stream)
        s_in.wait_stream(stream)
        s_out.wait_stream(stream)
        for i in range(nsteps):
            j = i & 1
            with torch.cuda.stream(s_in):
                if i >= 2:
                    s_in.wait_event(ev_dec[i - 2])      # decode i-2 has read buffers j
                d_qi[j].copy_(h_qi, non_blocking=True)
                d_q[j].copy_(h_q, non_blocking=True)
                d_lens[j].copy_(h_lens, non_blocking=True)
                ev_in[i].record(s_in)
            stream.wait_event(ev_in[i])
            if i >= 2:
                stream.wait_event(ev_out[i - 2])        # output j of step i-2 copied out
            msa.msa_decode(cache, seqs_e2e[j], d_qi[j], w.s_qi, d_q[j], w.s_q, w.softmax_scale,
                           d_out[j], None, ws, stream)
            ev_dec[i].record(stream)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev_dec[i])
                h_out[j].copy_(d_out[j], non_blocking=True)
                ev_out[i].record(s_out)
        stream.wait_event(ev_out[nsteps - 1])
        t1.record(stream)
        return t0, t1

    run_e2e(2)
    torch.cuda.synchronize()
    barrier(world)
    t0, t1 = run_e2e(args.steps)
    torch.cuda.synchronize()
    clk.mark("stop")
    clk.__exit__(None, None, None)
    clocks = clk.summary()
    ms_e2e = max_over_ranks(t0.elapsed_time(t1) / args.steps, world)
    h2d = h_qi.numel() + h_q.numel() + h_lens.numel() * 4
    d2h = h_out[0].numel() * 2

    # sub-records on other workloads (not part of the step): chunked prefill
    # and a batch sharing a cached prefix
    extra = {}
    if rank == 0 and not args.no_extra:
        extra["prefill"] = prefill_record(10, flush, stream)
        extra["shared_prefix"] = shared_prefix_record(10, flush, stream)

    cache_bytes = (w.idx_data.numel() + 2 * (w.k_data.numel() + w.k_scale.numel())
                   + (w.idx_scale.numel() if w.idx_scale is not None else 0))
    l2_note, e2e_l2_note = l2_notes(cache_bytes)
    result = None
    if rank == 0:
        q_total = B * T * world
        value = q_total / (ms_max * 1e-3)
        gbs = bytes_["total"] / (ms * 1e-3) / 1e9
        result = {
            "metric": METRIC, "value": value, "unit": "queries/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_max,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None,
            "dtype": "fp8_e4m3", "data": "synthetic",
            "config": {"workload": name if not args.batch else "%s (batch %d)" % (name, B), "batch_per_gpu": B, "context": int(w.seq_lens.max()),
                       "q_tokens": T, "index_keys": "fp8" if w.idx_fp8 else "nvfp4",
                       "kv_cache": "nvfp4, 128-token pages" + (", shuffled page table"
                                                                 if w.page_table is not None else ""),
                       "global_batch": B * world, "parallelism": "dp%d" % world,
                       "l2": l2_note},
            "hbm": {"algorithmic_bytes_per_step": bytes_["total"], "achieved_gbs": gbs,
                    "frac_of_measured": gbs / peak, "frac_of_spec_8000": gbs / SPEC_HBM_GBS,
                    "peak_source": peak_src, "bytes": bytes_},
            "roofline": {"kernel": dom, "bound": "hbm", "achieved": achieved, "peak": peak,
                         "unit": "GB/s", "frac": achieved / peak, "traffic": traffic,
                         "algorithmic_bytes_per_launch": kernel_bytes[dom],
                         "peak_source": peak_src},
            "kernel_ms": per,
            "indexer_exact": idx_exact,
            "kv_insert": {"ms": ins_ms, "tokens": B * T, "bytes": ins_bytes,
                          "gbs": ins_bytes / (ins_ms * 1e-3) / 1e9,
                          "note": "writing the step's new tokens into the cache (not part of the "
                                  "step): bf16 K, V and index key in, NVFP4 codes and scales out"},
            "gpu_launches": 3 * args.steps,
            "clocks": {"sm_mhz": clocks["sm_mhz"], "sm_max_mhz": clocks["sm_max_mhz"],
                       "reasons": clocks["reasons"], "samples": clocks["samples"]},
            "e2e": {"value": q_total / (ms_e2e * 1e-3), "unit": "queries/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": ms_e2e,
                    "mode": "pipelined: each step's queries copied in and output copied out on "
                            "copy streams, overlapping other steps' decodes; " + e2e_l2_note},
            "wall_s_timed_region": t_wall,
        }
        result.update(extra)
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD)
    ap.add_argument("--batch", type=int, default=0,
                    help="override the workload's batch (smaller cases for profiling)")
    ap.add_argument("--impl", default="native", choices=["native", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-extra", action="store_true",
                    help="skip the prefill and shared-prefix sub-records")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    rank, world, local_rank = rank_info()

    if args.impl == "reference":
        # The reference arm is the float64 oracle on the host cores, rank 0 only.
        if rank != 0:
            return 0
        w = cpu_sample_workload(args.workload)
        threads = host_threads()
        # K steps of T queries each (every query token of the sampled sequence:
        # full index scan, top-16, attention), evaluated together on all host
        # cores, so that even a few steps give every core rows; the W warm-up
        # steps likewise.
        T = w.q_tokens
        oracle_step(w, [(0, k % T) for k in range(args.warmup * T)], threads)
        t = oracle_step(w, [(0, k % T) for k in range(args.steps * T)], threads)
        qps = args.steps * T / t
        sample = ("per step: the %d query tokens of 1 sequence of %d tokens (shapes of %s): "
                  "full index scan, top-16 and attention in the float64 C oracle; the %d steps "
                  "run together on %d host threads" % (T, int(w.seq_lens[0]), args.workload,
                                                       args.steps, threads))
        print(json.dumps({
            "impl": "reference", "metric": METRIC, "value": qps, "unit": "queries/s",
            "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": 1e3 * t / args.steps, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "sample": sample},
            "cpu_baseline": {"value": qps, "unit": "queries/s", "cores": threads, "kind": "oracle",
                             "sample": sample},
            "e2e": {"value": qps, "unit": "queries/s", "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
        }), flush=True)
        return 0

    if world > 1:
        import datetime
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        res = run_gpu(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.barrier()
            dist.destroy_process_group()
    if rank == 0:
        if not args.no_cpu_baseline and world == 1:
            res["cpu_baseline"] = cpu_baseline(args.workload)
        print(json.dumps(res), flush=True)
    return 0


if __name__ == "__main__":
    sys.exit(main())
