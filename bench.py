"""Benchmark: one step of paged KV-cache attention on a synthetic in-flight batch.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl pkv|reference]

A step is the whole hot path for one layer of one iteration: kv_append of the
step's new tokens, host planning of the launch, and paged_attention (persistent
attention kernel plus the merge of split key ranges).  The default workload is
the Llama-3-8B-shaped decode batch (64 sequences, lengths U[512, 4096], 32/8
heads, head_dim 128, block 64, bf16 KV).  The pool (~755 MB) is larger than L2
and L2 is also flushed (a 512 MB read) before every timed step.

Prints ONE JSON line (rank 0).  Under torchrun every rank runs an independent
replica on its own GPU (the path has no exchange step); time is the max over
ranks.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import re
import statistics
import subprocess
import sys
import tempfile
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "paged decode-attention KV GB/s & % of B200 HBM peak; decode tokens/s"
NOMINAL_HBM_GBS = 8000.0
FALLBACK_HBM_GBS = 6650.0


def peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


def elem_bytes(dtype: str) -> int:
    return {"f32": 4, "bf16": 2, "f16": 2, "e4m3": 1}[dtype]


def algorithmic_bytes(w, plan_info=None) -> dict:
    """Bytes one step must move: distinct K/V bytes read, q, out, tables, scales, partials, appended rows."""
    from paged_kv_attention_block_b200.workloads import kv_row_bytes

    row = w.num_kv_heads * kv_row_bytes(w.kv_dtype, w.head_dim)  # one token of one layer, K or V (NVFP4: + block scales)
    kv = sum(tokens for _, tokens in w.distinct_kv_blocks()) * row * 2
    qb = elem_bytes(w.q_dtype)
    q = w.total_q * w.num_q_heads * w.head_dim * qb
    out = q
    tables = sum((int(L) + w.block_size - 1) // w.block_size for L in w.seq_lens) * 4 + w.num_seqs * 8
    scales = 2 * w.num_kv_heads * 4 if w.kv_dtype in ("e4m3", "nvfp4") else 0
    parts = 0
    if plan_info:
        parts = plan_info["num_partial_rows"] * (w.head_dim + 1) * 4 * 2
    new_rows = w.total_q * w.num_kv_heads * 2  # (token, head) rows of K and V
    append = new_rows * (w.head_dim * elem_bytes(w.kv_in_dtype) + kv_row_bytes(w.kv_dtype, w.head_dim))
    attn = kv + q + out + tables + scales + parts
    # The attention kernels alone: everything but the merge's read of the partials and its output.
    kernels = kv + q + out + tables + scales + parts // 2
    return {"kv": kv, "attention": attn, "kernels": kernels, "append": append, "step": attn + append}


def prefill_flops(w) -> float:
    """4 d Hq per causal-valid (query, key) pair of the prefill chunks (q_len > 1)."""
    pairs = 0
    for L, ql in zip(w.seq_lens.astype(np.int64), w.q_lens.astype(np.int64)):
        if ql > 1:
            pairs += ql * (L - ql) + ql * (ql + 1) // 2 if w.causal else ql * L
    return 4.0 * w.head_dim * w.num_q_heads * float(pairs)


def bf16_peak_tflops():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            return float(json.load(f)["bf16_tflops"]), "measured"
    return 1590.0, "fallback"


def decode_rows(w) -> int:
    return int((w.q_lens == 1).sum())


class ClockSampler:
    """nvidia-smi samples during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        # The raw samples go to $PKV_BENCH_OUT (default: the system temp directory).
        out = os.environ.get("PKV_BENCH_OUT") or tempfile.gettempdir()
        self.path = os.path.join(out, f"pkv_clocks_rank{index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.QUERY}",
                                          "--format=csv,noheader,nounits", "-lms", "100"], stdout=self.f,
                                         stderr=subprocess.DEVNULL)
            t0 = time.time()  # start timing only once sampling has begun
            while time.time() - t0 < 10 and os.path.getsize(self.path) == 0 and self.proc.poll() is None:
                time.sleep(0.05)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in open(self.path):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            try:
                sm.append(float(f[1]))
                smax.append(float(f[2]))
            except ValueError:
                continue
            for n, v in zip(names, f[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


# The sources the decode-tile attention kernel (the roofline kernel of the default workload) is
# built from: a traffic figure is reported only for the sources it was taken on.
TRAFFIC_SOURCES = ("attn_tma.cu", "attn_tile.cuh", "attn_args.h", "common.cuh", "internal.h", "plan_format.h")


def _code_only(src: str) -> str:
    """C/C++ source without comments, blank lines or runs of spaces: a comment edit does not change
    the kernel."""
    src = re.sub(r"/\*.*?\*/", " ", src, flags=re.S)
    src = re.sub(r"//[^\n]*", "", src)
    return "\n".join(" ".join(line.split()) for line in src.splitlines() if line.strip())


def read_stream_gbs(buf, reps: int = 10):
    """A plain read-only HBM stream as the practical ceiling: the library's pkv_stream_read over
    ``buf`` (larger than L2), in both its forms (16-byte loads from every thread; 1-D bulk copies
    into a shared-memory ring, as the attention kernels' producers issue them), CUDA events around
    each pass, the median pass of each form.  None if it cannot be taken."""
    import torch
    from paged_kv_attention_block_b200 import api

    try:
        sink = torch.zeros(1, dtype=torch.int32, device=buf.device)
        status = torch.zeros(1, dtype=torch.int32, device=buf.device)
        res = {}
        for mode, name in ((0, "loads"), (1, "bulk")):
            times = []
            for _ in range(reps + 2):
                s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                s.record()
                api.stream_read(buf, sink, mode=mode, status=status)
                e.record()
                e.synchronize()
                times.append(s.elapsed_time(e))
            res[name] = buf.numel() * buf.element_size() / (statistics.median(times[2:]) * 1e-3) / 1e9
        if int(status.item()) != 0:
            return None
        return res
    except Exception:  # noqa: BLE001 - a missing ceiling must not cost the benchmark line
        return None


def kernel_source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "paged_kv_attention_block_b200", "csrc")
    for name in TRAFFIC_SOURCES:
        with open(os.path.join(csrc, name), encoding="utf-8") as f:
            h.update(name.encode() + _code_only(f.read()).encode())
    with open(os.path.join(ROOT, "include", "pkv.h"), encoding="utf-8") as f:
        h.update(_code_only(f.read()).encode())
    return h.hexdigest()[:16]


def traffic_for(config: str):
    """ncu DRAM bytes per attention launch, if captured on the current kernel source."""
    p = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(p):
        return None
    with open(p) as f:
        d = json.load(f)
    e = d.get(config)
    if not e or e.get("kernel_source") != kernel_source_hash():
        return None
    return e.get("dram_bytes_per_launch")


# ---------------------------------------------------------------------------
# CPU oracle (the reference arm and the cpu_baseline figure)
# ---------------------------------------------------------------------------

def _sample_seqs(w, max_seqs: int | None, max_work: float | None) -> list:
    """The sequences an oracle sample covers: of the first ``max_seqs`` (default all), in batch order,
    each one that keeps the (query row x key x query head) work of one step within ``max_work``
    (the lightest one alone if none does)."""
    n = w.num_seqs if max_seqs is None else min(max_seqs, w.num_seqs)
    seqs, work = [], 0.0
    cost = [float(w.q_lens[s]) * float(w.seq_lens[s]) * w.num_q_heads for s in range(n)]
    for s in range(n):
        if w.q_lens[s] == 0 or (max_work is not None and work + cost[s] > max_work):
            continue
        seqs.append(s)
        work += cost[s]
    if not seqs:  # nothing fits: the lightest scheduled sequence alone
        seqs = [min((s for s in range(n) if w.q_lens[s] > 0), key=lambda s: cost[s])]
    return seqs


def _oracle_worker(job):
    """One process of the oracle sample: rebuild the workload from its seed, append the history of
    this worker's sequences into a pool of its own, wait for the others, then time whole steps."""
    name, kwargs, seqs, budget_s, barrier = job
    import oracle.pkv_oracle as O
    from paged_kv_attention_block_b200 import workloads as W

    w = W.NAMED[name](**kwargs)
    pool = O.new_pool(w.num_blocks, w.num_layers, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype,
                      w.k_scale, w.v_scale)
    k, v, cu, sp = w.packed_kv("history", seqs)
    O.kv_append(pool, w.layer, k, v, w.kv_in_dtype, cu, sp, w.block_tables[seqs])
    q = O.decode_bits(w.q, w.q_dtype) if w.q_dtype != "f32" else w.q.astype(np.float64)
    kn, vn, cun, spn = w.packed_kv("new", seqs)
    if barrier is not None:
        barrier.wait()
    steps, t_wall = 0, 0.0
    while t_wall < budget_s or steps == 0:
        w0 = time.perf_counter()
        O.kv_append(pool, w.layer, kn, vn, w.kv_in_dtype, cun, spn, w.block_tables[seqs])
        O.paged_attention(pool, w.layer, q, w.cu_q_lens, w.seq_lens, w.block_tables, w.num_q_heads,
                          w.softmax_scale, w.causal, seqs=seqs, window=w.window)
        t_wall += time.perf_counter() - w0
        steps += 1
    return steps, t_wall


def oracle_sample(w, budget_s: float = 10.0, max_seqs: int | None = None, max_work: float | None = None,
                  procs: int | None = None, kwargs: dict | None = None):
    """Time the oracle on whole steps (kv_append + attention) of a sample of the batch's sequences
    for about ``budget_s`` seconds, on ``procs`` processes (default: every core this process may
    use, capped at the sampled sequences).  Each process (spawned, so none inherits a CUDA
    context) rebuilds the workload from its seed (``kwargs``: the workload builder's arguments),
    takes a share of the sequences (heaviest to the lightest share) and, after a common start,
    runs whole steps of the oracle on it with one BLAS thread.  Throughput = the sample's bytes per
    step summed over the shares' step rates."""
    import multiprocessing as mp

    procs = procs or len(os.sched_getaffinity(0))
    seqs = _sample_seqs(w, max_seqs, max_work)
    procs = max(1, min(procs, len(seqs)))
    shares, load = [[] for _ in range(procs)], [0.0] * procs
    for s in sorted(seqs, key=lambda s: -float(w.q_lens[s]) * float(w.seq_lens[s])):
        i = load.index(min(load))
        shares[i].append(s)
        load[i] += float(w.q_lens[s]) * float(w.seq_lens[s])
    shares = [sorted(sh) for sh in shares if sh]
    ctx = mp.get_context("spawn")
    env = {k: os.environ.get(k) for k in ("OMP_NUM_THREADS", "OPENBLAS_NUM_THREADS", "MKL_NUM_THREADS")}
    for k in env:
        os.environ[k] = "1"  # inherited by the spawned workers: one BLAS thread each
    try:
        with ctx.Manager() as mgr:
            barrier = mgr.Barrier(len(shares))
            with ctx.Pool(len(shares)) as pool:
                res = pool.map(_oracle_worker, [(w.name, kwargs or {}, sh, budget_s, barrier) for sh in shares])
    finally:
        for k, v in env.items():
            if v is None:
                os.environ.pop(k, None)
            else:
                os.environ[k] = v

    def sub_of(ss):
        sub = type(w)(**{**w.__dict__})
        sub.seq_lens, sub.q_lens = w.seq_lens[ss], w.q_lens[ss]
        sub.block_tables = w.block_tables[ss]
        return sub

    rate = sum(algorithmic_bytes(sub_of(sh))["step"] * n / t for sh, (n, t) in zip(shares, res))
    tok = sum(decode_rows(sub_of(sh)) * n / t for sh, (n, t) in zip(shares, res))
    steps = min(n for n, _ in res)
    wall = max(t for _, t in res)
    return {
        "value": rate / 1e9,
        "unit": "GB/s",
        "cores": len(shares),
        "kind": "oracle",
        "sample": f"{len(seqs)} of {w.num_seqs} sequences of {w.name}, whole steps (kv_append + attention, "
                  f"float64 numpy) on {len(shares)} processes of one thread, >= {steps} steps each, {wall:.1f} s",
        "ms_per_step": algorithmic_bytes(sub_of(seqs))["step"] / rate * 1e3,
        "decode_tok_s": tok,
    }


def run_reference(args, rank: int, world: int):
    if rank != 0:
        return
    from paged_kv_attention_block_b200 import workloads as W

    w = W.NAMED[args.config]()
    per_step = []
    base = None
    for i in range(args.warmup + args.steps):
        r = oracle_sample(w, budget_s=args.ref_budget, max_seqs=args.ref_seqs)
        if i >= args.warmup:
            per_step.append(r["ms_per_step"])
            base = r
    ms = float(np.mean(per_step))
    line = {
        "impl": "reference", "metric": METRIC, "value": base["value"], "unit": "GB/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
        "config": {"workload": w.name, "sample": base["sample"]},
        "cpu_baseline": {k: base[k] for k in ("value", "unit", "cores", "kind", "sample")},
        "e2e": {"value": base["value"], "unit": "GB/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "decode_tok_s": base["decode_tok_s"],
    }
    print(json.dumps(line), flush=True)


# ---------------------------------------------------------------------------
# The CUDA path
# ---------------------------------------------------------------------------

def max_over_ranks(values, device=None):
    """Element-wise max of per-rank values (device time: the slowest replica sets the step time)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor(values, dtype=torch.float64, device=device)
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return [float(x) for x in t.cpu()]


# Workloads measured after the headline one (one GPU only), with the oracle's work per sample step.
SECONDARY = ("longctx_fp8", "mixed_bf16", "prefix_reuse_bf16", "llama3_8b_decode_nvfp4")
ORACLE_WORK = {"llama3_8b_decode_bf16": None, "longctx_fp8": 2 * 131072 * 32, "mixed_bf16": 8e6,
               "prefix_reuse_bf16": 6e6, "llama3_8b_decode_nvfp4": None}
BAR_FRAC_OF_NOMINAL = 0.70  # the stated bar: decode attention at >= 70 % of a nominal 8 TB/s


def measure(w, args, dev, world, plan_opts, steps):
    """Time one workload on this rank's GPU: the device step (kv_append + plan upload + attention
    kernels + merge, one CUDA graph per step, L2 flushed before each), the attention call and its
    kernels alone (split graphs with kernel events), the prefill chunks alone, and the step end to
    end through GraphStep.  Returns raw times and the plan; the caller formats the line."""
    import torch
    import torch.distributed as dist

    from paged_kv_attention_block_b200 import api, runner

    dw = runner.DeviceWorkload(w, device=dev)
    plan_kw = dict(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                   block_size=w.block_size, kv_dtype=w.kv_dtype, causal=w.causal, block_tables=w.block_tables,
                   **({"window": w.window} if w.window else {}), **plan_opts)
    plan = api.plan_attention(w.cu_q_lens, w.seq_lens, **plan_kw)
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device=dev)
    out = torch.empty_like(dw.q)
    # L2 is flushed before each step by reading a 512 MB buffer: the KV leaves L2 and the lines
    # left behind are clean, so no write-back of the flush lands in the timed region.
    flush = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    stream = torch.cuda.Stream(dev)
    # Events recorded by the library right before and after the attention kernels (inside the
    # graphs): the dominant kernels' own duration, read back one step at a time after the timed run.
    kev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    with torch.cuda.stream(stream):
        for e in kev:
            e.record(stream)  # creates the CUDA events

    # The GPU side of a step runs from CUDA graphs: one for kv_append and one attention graph per
    # page-locked plan buffer (double-buffered), so the events below time GPU work only.  The host
    # plans every step into the buffer whose previous upload has completed.
    planner = api.Planner(w.cu_q_lens, w.seq_lens, **plan_kw)
    bufs = [planner.plan() for _ in range(2)]
    with torch.cuda.stream(stream):
        for _ in range(3):  # eager warm-up: occupancy queries, tensor-map encoder lookup
            dw.append_new()
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, bufs[0], w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status)
    torch.cuda.synchronize(dev)
    # The timed steps replay one graph per step (kv_append then paged_attention), one graph per
    # plan buffer.  A second set holds the paged_attention call alone (plan staging, kernels,
    # merge), timed back to back like the steps; a third the same call with events recorded by
    # the library around the attention kernels, replayed one at a time for the kernel-only time
    # (event record nodes inside the timed graphs would add latency).
    g_step = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            dw.append_new()
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, b, w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status)
        g_step.append(g)
    g_attn = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, b, w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status)
        g_attn.append(g)
    g_attn_ev = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, b, w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status, kernel_events=kev)
        g_attn_ev.append(g)
    done = [None, None]
    host_plan_s = 0.0

    def step(i, evs=None, split=None):
        """One step; `evs` = (start, -, end) events; split: "attn" the attention call alone (no
        append), "attn_ev" the same with kernel events, instead of the one-graph step."""
        nonlocal host_plan_s
        slot = i % 2
        if done[slot] is not None:
            done[slot].synchronize()  # the upload that read this buffer has run
        t0 = time.perf_counter()
        planner.plan_into(bufs[slot].buffer)
        host_plan_s += time.perf_counter() - t0
        with torch.cuda.stream(stream):
            flush.sum()
            if evs:
                evs[0].record(stream)
            if split == "attn":
                g_attn[slot].replay()
            elif split == "attn_ev":
                g_attn_ev[slot].replay()
            else:
                g_step[slot].replay()
            if evs:
                evs[2].record(stream)
            e = torch.cuda.Event()
            e.record(stream)
            done[slot] = e

    for i in range(max(3, args.warmup)):
        step(i)
    torch.cuda.synchronize(dev)
    if world > 1:
        dist.barrier()
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(steps)]
    nsplit = min(steps, 300)
    ev_split = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(nsplit)]
    host_plan_s = 0.0
    with ClockSampler(dev.index or 0) as clocks:
        torch.cuda.synchronize(dev)
        for i in range(steps):
            step(i, ev[i])
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    host_plan_us = host_plan_s / steps * 1e6
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    ms = float(np.mean(step_ms))
    # The attention call alone, back to back like the steps; then the attention kernels' own
    # duration from the graphs with kernel events, one at a time, each read back after it ran.
    for i in range(nsplit):
        step(i, ev_split[i], split="attn")
    torch.cuda.synchronize(dev)
    attn = float(np.mean([a_.elapsed_time(c) for a_, _, c in ev_split]))
    kern_ms = []
    for i in range(nsplit):
        step(i, split="attn_ev")
        torch.cuda.synchronize(dev)
        kern_ms.append(kev[0].elapsed_time(kev[1]))
    kern = float(np.mean(kern_ms))
    ms, attn, kern = max_over_ranks([ms, attn, kern], dev)
    assert int(dw.status.item()) == 0, "device status set during the benchmark"
    # Planning through the general binding call (request and host arrays built per call), for
    # comparison with host_plan_us (one library call through a reusable Planner).
    t0 = time.perf_counter()
    for _ in range(200):
        api.plan_attention(w.cu_q_lens, w.seq_lens, buffer=bufs[0].buffer, **plan_kw)
    plan_call_us = (time.perf_counter() - t0) / 200 * 1e6
    del g_step, g_attn, g_attn_ev
    read_ceiling = read_stream_gbs(flush)
    del flush
    e2e = run_e2e(args, w, dw, plan_opts, dev, api, steps)
    e2e["ms"] = max_over_ranks([e2e["ms"]], dev)[0]
    prefill = run_prefill_only(w, dev, api, runner, plan_kw) if prefill_flops(w) > 0 else None
    del dw, ws, out
    torch.cuda.synchronize(dev)
    torch.cuda.empty_cache()
    return {"ms": ms, "attn": attn, "kern": kern, "host_plan_us": host_plan_us, "plan_call_us": plan_call_us,
            "plan": plan.info, "e2e": e2e, "prefill": prefill, "clocks": clocks.summary(),
            "read_ceiling": read_ceiling}


def summarise(w, r, world, peak, peak_kind):
    """Rates, roofline and the stated bar for one measured workload."""
    b = algorithmic_bytes(w, r["plan"])
    value = b["step"] * world / (r["ms"] * 1e-3) / 1e9
    achieved = b["kernels"] / (r["kern"] * 1e-3) / 1e9
    n_tc = r["plan"]["num_tc_items"]
    kernels = " + ".join(k for k, on in (("attn_tma_kernel", r["plan"]["num_items"] > n_tc),
                                          ("attn_tc_kernel", n_tc > 0)) if on)
    bar_gbs = BAR_FRAC_OF_NOMINAL * NOMINAL_HBM_GBS
    attn_gbs = b["attention"] / (r["attn"] * 1e-3) / 1e9
    return {
        "value": value, "ms_per_step": r["ms"], "attention_ms": r["attn"], "attention_kernels_ms": r["kern"],
        "decode_tok_s": decode_rows(w) * world / (r["ms"] * 1e-3),
        "step_bytes": b["step"], "kv_bytes": b["kv"],
        "hbm_frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS, "hbm_frac_of_measured": value / world / peak,
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                     "frac_of_nominal_8tbs": achieved / NOMINAL_HBM_GBS, "traffic": traffic_for(w.name),
                     "peak_source": peak_kind, "kernel": kernels,
                     "timed": "kernel-only CUDA events around the attention kernels, L2 flushed before each of "
                              "up to 300 steps"},
        # The stated bar (70 % of a nominal 8 TB/s on algorithmic bytes) for the attention kernels
        # alone, for the whole paged_attention call (plan upload + kernels + merge) and for the step
        # (kv_append included).
        "bar_70pct_of_nominal": {"gbs": bar_gbs, "kernels_us": b["kernels"] / bar_gbs / 1e3,
                                 "kernels_met": achieved >= bar_gbs, "attention_call_gbs": attn_gbs,
                                 "attention_call_met": attn_gbs >= bar_gbs, "step_met": value / world >= bar_gbs},
        "host_plan_us": r["host_plan_us"], "plan_attention_call_us": r["plan_call_us"],
        "e2e": {"value": b["step"] * world / (r["e2e"]["ms"] * 1e-3) / 1e9, "unit": "GB/s",
                "h2d_bytes_per_step": r["e2e"]["h2d"], "d2h_bytes_per_step": r["e2e"]["d2h"],
                "ms_per_step": r["e2e"]["ms"]},
        "clocks": r["clocks"],
        "plan": {k: r["plan"][k] for k in ("num_items", "num_tc_items", "num_reduce", "num_partial_rows",
                                           "num_groups", "num_ctas", "tc_num_ctas", "side_by_side",
                                           "heads_per_item")},
        # kv_append, the plan staging kernel (the plans are page-locked), the attention kernels present
        # in the plan, the merge when the plan has one.
        "launches_per_step": 2 + (r["plan"]["num_items"] > n_tc) + (n_tc > 0) + (r["plan"]["num_reduce"] > 0),
    }


def workload_config(w, world):
    return {"workload": w.name, "batch": w.num_seqs, "kv_tokens": int(w.seq_lens.sum()),
            "q_tokens": w.total_q, "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads,
            "head_dim": w.head_dim, "block_size": w.block_size, "kv_dtype": w.kv_dtype,
            "l2": "flushed before every step by reading a 512 MB buffer; pool larger than L2",
            "parallelism": f"replicas{world}"}


def run_pkv(args, rank: int, world: int, local_rank: int):
    import torch

    from paged_kv_attention_block_b200 import build

    build.build()
    from paged_kv_attention_block_b200 import workloads as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    builder = W.NAMED[args.config]
    w = builder(seed=builder.__defaults__[0] + 1000 * rank) if rank else builder()
    plan_opts = {"kv_split": args.kv_split} if args.kv_split else {}
    if args.num_ctas:
        plan_opts["num_ctas"] = args.num_ctas
    if args.tc_num_ctas:
        plan_opts["tc_num_ctas"] = args.tc_num_ctas
    if args.heads_per_item:
        plan_opts["heads_per_item"] = args.heads_per_item
    peak, peak_kind = peaks()
    r = measure(w, args, dev, world, plan_opts, args.steps)
    head = summarise(w, r, world, peak, peak_kind)
    # The other configurations, each measured the same way (one GPU; the scaling runs time the
    # headline workload only).  Each pool is freed before the next is staged.
    extra = {}
    names = [] if world > 1 or args.workloads == "none" else \
        [n for n in (SECONDARY if args.workloads == "all" else args.workloads.split(",")) if n != w.name]
    for name in names:
        w2 = W.NAMED[name]()
        r2 = measure(w2, args, dev, world, {}, min(args.steps, 500))
        extra[name] = {"config": workload_config(w2, world), **summarise(w2, r2, world, peak, peak_kind)}
        if r2["prefill"] is not None:
            extra[name]["prefill"] = r2["prefill"]
        extra[name]["_w"] = w2
    if rank != 0:
        return
    cpu = None
    if world == 1 and not args.no_cpu:
        cpu = oracle_sample(w, budget_s=args.ref_budget, max_seqs=args.ref_seqs, max_work=ORACLE_WORK.get(w.name))
        for name, e in extra.items():
            c = oracle_sample(e["_w"], budget_s=args.ref_budget / 2, max_work=ORACLE_WORK.get(name))
            e["cpu_baseline"] = {k: c[k] for k in ("value", "unit", "cores", "kind", "sample")}
    for e in extra.values():
        e.pop("_w").release()
    rc = r["read_ceiling"]
    line = {
        "metric": METRIC, "value": head["value"], "unit": "GB/s", "n_gpus": world, "steps": args.steps,
        "warmup": max(3, args.warmup), "ms_per_step": head["ms_per_step"], "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
        "config": workload_config(w, world),
        **{k: head[k] for k in ("decode_tok_s", "hbm_frac_of_nominal_8tbs", "hbm_frac_of_measured")},
        "read_stream_ceiling": None if rc is None else {
            "value": max(rc.values()), "unit": "GB/s", "loads": rc["loads"], "bulk": rc["bulk"],
            "kernels_frac": head["roofline"]["achieved"] / max(rc.values()),
            "how": "pkv_stream_read over a 512 MB buffer (16-byte loads from every thread; 1-D bulk copies into a "
                   "shared-memory ring), CUDA events, median of 10 passes each; value = the faster form"},
        **{k: head[k] for k in ("step_bytes", "kv_bytes", "attention_ms", "attention_kernels_ms", "host_plan_us",
                                "plan_attention_call_us", "roofline", "bar_70pct_of_nominal")},
        "cpu_baseline": None if cpu is None else {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")},
        "e2e": head["e2e"],
        "gpu_launches": head["launches_per_step"] * args.steps,
        "clocks": head["clocks"],
        "plan": head["plan"],
    }
    if r["prefill"] is not None:
        line["prefill"] = r["prefill"]
    if extra:
        line["workloads"] = extra
    print(json.dumps(line), flush=True)


def run_prefill_only(w, dev, api, runner, plan_kw, steps: int = 100):
    """The prefill chunks of the batch alone (same lengths, same cached prefixes): tensor TFLOP/s
    of the tcgen05 kernel, from kernel-only events, L2 flushed before each launch."""
    import torch
    from paged_kv_attention_block_b200 import workloads as W

    idx = [i for i in range(w.num_seqs) if int(w.q_lens[i]) > 1]
    sub = W.build(w.name + "_prefill_only", seed=7, kv_dtype=w.kv_dtype, num_q_heads=w.num_q_heads,
                  num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=w.block_size,
                  seq_lens=w.seq_lens[idx], q_lens=w.q_lens[idx], causal=w.causal)
    dw = runner.DeviceWorkload(sub, device=dev)
    dw.append_new()
    kw = {k: v for k, v in plan_kw.items() if k != "block_tables"}
    plan = api.plan_attention(sub.cu_q_lens, sub.seq_lens, **{**kw, "block_tables": sub.block_tables})
    out = torch.empty_like(dw.q)
    ws = torch.empty(max(plan.workspace_bytes, 256), dtype=torch.uint8, device=dev)
    flush = torch.ones(128 << 20, dtype=torch.float32, device=dev)
    kev = (torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
    for e in kev:
        e.record()
    times = []
    for i in range(steps + 3):
        flush.sum()
        api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, plan, sub.softmax_scale, sub.causal,
                            out=out, workspace=ws, status=dw.status, kernel_events=kev)
        torch.cuda.synchronize(dev)
        if i >= 3:
            times.append(kev[0].elapsed_time(kev[1]))
    assert int(dw.status.item()) == 0
    us = float(np.mean(times)) * 1e3
    flops = prefill_flops(sub)
    peak, kind = bf16_peak_tflops()
    tflops = flops / (us * 1e-6) / 1e12
    return {"workload": f"the {len(idx)} prefill chunks of {w.name} alone", "flops": flops, "us": us,
            "tflops": tflops, "peak_tflops": peak, "peak_source": kind, "frac": tflops / peak,
            "kernel": "attn_tc_kernel" if plan.info["num_tc_items"] else "attn_tma_kernel"}


def run_e2e(args, w, dw, plan_opts, dev, api, steps):
    """The step end to end through the public API as a serving loop runs it (api.GraphStep):
    every step plans on the host, copies its packed inputs (q, new K/V, lengths, positions,
    tables) and its plan from page-locked host memory, appends, runs attention and copies the
    output back to page-locked host memory: three graph replays per step (copy in, kernels, copy
    out) on three streams, two buffer slots, so copies overlap the neighbouring steps' kernels and
    the host plans step i+1 while the GPU runs step i.  Time = events from before the first input
    copy to after the last output copy of n back-to-back steps, divided by n."""
    import torch

    names = {"q": dw.q, "k_new": dw.k_new, "v_new": dw.v_new, "cu_q": dw.cu_q, "seq_lens": dw.seq_lens,
             "start_pos": dw.start_pos, "block_tables": dw.block_tables}
    kw = dict(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim, block_size=w.block_size,
              kv_dtype=w.kv_dtype, causal=w.causal, **({"window": w.window} if w.window else {}), **plan_opts)
    gs = api.GraphStep(dw.cache, names, kw, w.softmax_scale, w.causal, stream=torch.cuda.Stream(dev))
    for views in gs.host:
        for k, v in names.items():
            views[k].copy_(v.cpu())
    for _ in range(4):
        gs.wait(gs.run())
    n = max(2, min(steps, 500))
    torch.cuda.synchronize(dev)
    s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    s.record(gs.copy_in_stream)  # before the first input copy
    slot = None
    for _ in range(n):
        slot = gs.run()
    e.record(gs.copy_out_stream)  # after the last output copy
    out = gs.wait(slot)
    e.synchronize()
    assert torch.isfinite(out.float()).all(), "non-finite output in the end-to-end loop"
    plan_bytes = gs._plans[0].info["plan_bytes"]
    return {"ms": s.elapsed_time(e) / n, "h2d": int(gs.h2d_bytes + plan_bytes), "d2h": int(gs.d2h_bytes)}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=3000)
    ap.add_argument("--warmup", type=int, default=20)
    ap.add_argument("--impl", choices=["pkv", "reference"], default="pkv")
    ap.add_argument("--config", default="llama3_8b_decode_bf16")
    ap.add_argument("--kv-split", type=int, default=0)
    ap.add_argument("--num-ctas", type=int, default=0, help="decode-tile kernel CTAs (0: all that fit)")
    ap.add_argument("--tc-num-ctas", type=int, default=0,
                    help="> 0: the tcgen05 kernel side by side on this many CTAs (needs --num-ctas); < 0: never")
    ap.add_argument("--heads-per-item", type=int, default=0,
                    help="KV heads per decode-sized work item: 1 or 4 (0: the planner decides)")
    ap.add_argument("--ref-budget", type=float, default=10.0, help="seconds of oracle work per reference sample")
    ap.add_argument("--ref-seqs", type=int, default=None, help="sequences in the oracle sample (default all)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline oracle timing")
    ap.add_argument("--workloads", default="all",
                    help="other workloads measured after the headline one (one GPU): all, none or a comma list")
    args = ap.parse_args()
    rank = int(os.environ.get("RANK", 0))
    world = int(os.environ.get("WORLD_SIZE", 1))
    local_rank = int(os.environ.get("LOCAL_RANK", 0))
    if args.impl == "reference":
        run_reference(args, rank, world)
        return
    if world > 1:
        import datetime

        import torch.distributed as dist

        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120))
    try:
        run_pkv(args, rank, world, local_rank)
    finally:
        if world > 1:
            import torch.distributed as dist

            dist.destroy_process_group()


if __name__ == "__main__":
    main()
