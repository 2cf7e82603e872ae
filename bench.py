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
    """A plain read-only stream as the practical HBM ceiling: torch's sum over ``buf`` (larger
    than L2), CUDA events around each pass, the median pass.  None if it cannot be taken."""
    import torch

    try:
        times = []
        for _ in range(reps + 2):
            s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            s.record()
            buf.sum()
            e.record()
            e.synchronize()
            times.append(s.elapsed_time(e))
        ms = statistics.median(times[2:])
        return buf.numel() * buf.element_size() / (ms * 1e-3) / 1e9
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

def oracle_sample(w, budget_s: float = 10.0, max_seqs: int | None = None):
    """Time the oracle on whole-batch steps (or a prefix of sequences) for about budget_s seconds."""
    import oracle.pkv_oracle as O

    seqs = list(range(w.num_seqs if max_seqs is None else min(max_seqs, w.num_seqs)))
    pool = O.new_pool(w.num_blocks, w.num_layers, w.num_kv_heads, w.block_size, w.head_dim, w.kv_dtype,
                      w.k_scale, w.v_scale)
    k, v, cu, sp = w.packed_kv("history", seqs)
    O.kv_append(pool, w.layer, k, v, w.kv_in_dtype, cu, sp, w.block_tables[seqs])
    q = O.decode_bits(w.q, w.q_dtype) if w.q_dtype != "f32" else w.q.astype(np.float64)
    kn, vn, cun, spn = w.packed_kv("new", seqs)
    steps, t_wall, t_cpu = 0, 0.0, 0.0
    while t_wall < budget_s or steps == 0:
        c0, w0 = time.process_time(), time.perf_counter()
        O.kv_append(pool, w.layer, kn, vn, w.kv_in_dtype, cun, spn, w.block_tables[seqs])
        O.paged_attention(pool, w.layer, q, w.cu_q_lens, w.seq_lens, w.block_tables, w.num_q_heads,
                          w.softmax_scale, w.causal, seqs=seqs)
        t_wall += time.perf_counter() - w0
        t_cpu += time.process_time() - c0
        steps += 1
    # Bytes of the sampled sequences only.
    sub = type(w)(**{**w.__dict__})
    sub.seq_lens, sub.q_lens = w.seq_lens[seqs], w.q_lens[seqs]
    sub.block_tables = w.block_tables[seqs]
    b = algorithmic_bytes(sub)
    per_step = t_wall / steps
    return {
        "value": b["step"] / per_step / 1e9,
        "unit": "GB/s",
        "cores": max(1, round(t_cpu / t_wall)),
        "kind": "oracle",
        "sample": f"{len(seqs)} of {w.num_seqs} sequences of {w.name}, {steps} whole steps "
                  f"(kv_append + attention, float64 numpy), {t_wall:.1f} s",
        "ms_per_step": per_step * 1e3,
        "decode_tok_s": decode_rows(sub) / per_step,
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


def run_pkv(args, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist

    from paged_kv_attention_block_b200 import build

    build.build()
    from paged_kv_attention_block_b200 import api, runner, workloads as W

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    builder = W.NAMED[args.config]
    w = builder(seed=builder.__defaults__[0] + 1000 * rank) if rank else builder()
    dw = runner.DeviceWorkload(w, device=dev)
    plan_opts = {}
    if args.kv_split:
        plan_opts["kv_split"] = args.kv_split
    plan_kw = dict(num_q_heads=w.num_q_heads, num_kv_heads=w.num_kv_heads, head_dim=w.head_dim,
                   block_size=w.block_size, kv_dtype=w.kv_dtype, causal=w.causal, block_tables=w.block_tables,
                   **plan_opts)
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
    bufs = [api.plan_attention(w.cu_q_lens, w.seq_lens, **plan_kw) for _ in range(2)]
    with torch.cuda.stream(stream):
        for _ in range(3):  # eager warm-up: occupancy queries, tensor-map encoder lookup
            dw.append_new()
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, bufs[0], w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status)
    torch.cuda.synchronize(dev)
    # The timed steps replay one graph per step (kv_append then paged_attention), one graph per
    # plan buffer.  A second set splits the step into an append graph and an attention graph
    # whose library call also records events around the attention kernels: the per-phase and
    # kernel-only times come from replaying those one step at a time after the timed run (event
    # record nodes inside the timed graphs would add latency to the step).
    g_step = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            dw.append_new()
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, b, w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status)
        g_step.append(g)
    g_append = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g_append, stream=stream):
        dw.append_new()
    g_attn_ev = []
    for b in bufs:
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            api.paged_attention(dw.cache, dw.q, dw.cu_q, dw.seq_lens, dw.block_tables, b, w.softmax_scale,
                                w.causal, out=out, workspace=ws, status=dw.status, kernel_events=kev)
        g_attn_ev.append(g)
    done = [None, None]
    host_plan_s = 0.0

    def step(i, evs=None, split=False):
        """One step; `evs` = (start, after append, end) events; split: the append and attention
        graphs (the latter with kernel events) instead of the one-graph step."""
        nonlocal host_plan_s
        slot = i % 2
        if done[slot] is not None:
            done[slot].synchronize()  # the upload that read this buffer has run
        t0 = time.perf_counter()
        api.plan_attention(w.cu_q_lens, w.seq_lens, buffer=bufs[slot].buffer, **plan_kw)
        host_plan_s += time.perf_counter() - t0
        with torch.cuda.stream(stream):
            flush.sum()
            if evs:
                evs[0].record(stream)
            if split:
                g_append.replay()
                if evs:
                    evs[1].record(stream)
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
    ev = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(args.steps)]
    nsplit = min(args.steps, 300)
    ev_split = [tuple(torch.cuda.Event(enable_timing=True) for _ in range(3)) for _ in range(nsplit)]
    host_plan_s = 0.0
    with ClockSampler(local_rank) as clocks:
        torch.cuda.synchronize(dev)
        for i in range(args.steps):
            step(i, ev[i])
        torch.cuda.synchronize(dev)
        if world > 1:
            dist.barrier()
    step_ms = [a.elapsed_time(c) for a, _, c in ev]
    ms = float(np.mean(step_ms))
    # Per phase and the attention kernels' own duration: the same steps from the split graphs,
    # one at a time, each read back after it ran.
    kern_ms = []
    for i in range(nsplit):
        step(i, ev_split[i], split=True)
        torch.cuda.synchronize(dev)
        kern_ms.append(kev[0].elapsed_time(kev[1]))
    attn = float(np.mean([b.elapsed_time(c) for _, b, c in ev_split]))
    kern = float(np.mean(kern_ms))
    ms, attn, kern = max_over_ranks([ms, attn, kern], dev)
    assert int(dw.status.item()) == 0, "device status set during the benchmark"
    del g_step, g_append, g_attn_ev
    prefill = run_prefill_only(w, dev, api, runner, plan_kw) if rank == 0 and prefill_flops(w) > 0 else None

    b = algorithmic_bytes(w, plan.info)
    value = b["step"] * world / (ms * 1e-3) / 1e9
    achieved = b["kernels"] / (kern * 1e-3) / 1e9
    peak, peak_kind = peaks()

    read_ceiling = read_stream_gbs(flush)

    # End to end through the public API from pinned host buffers.
    e2e = run_e2e(args, w, dw, plan_opts, dev, torch.cuda.current_stream(dev), api)
    e2e["ms"] = max_over_ranks([e2e["ms"]], dev)[0]

    n_tc = plan.info["num_tc_items"]
    launches_per_step = (1 + (plan.info["num_items"] > n_tc) + (n_tc > 0) + (plan.info["num_reduce"] > 0))
    kernels = " + ".join(k for k, on in (("attn_tma_kernel", plan.info["num_items"] > n_tc),
                                          ("attn_tc_kernel", n_tc > 0)) if on)
    if rank == 0:
        cpu = oracle_sample(w, budget_s=args.ref_budget, max_seqs=args.ref_seqs) if world == 1 and not args.no_cpu else None
        line = {
            "metric": METRIC, "value": value, "unit": "GB/s", "n_gpus": world, "steps": args.steps,
            "warmup": max(3, args.warmup), "ms_per_step": ms, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": w.kv_dtype, "data": "synthetic",
            "config": {"workload": w.name, "batch": w.num_seqs, "kv_tokens": int(w.seq_lens.sum()),
                       "num_q_heads": w.num_q_heads, "num_kv_heads": w.num_kv_heads, "head_dim": w.head_dim,
                       "block_size": w.block_size,
                       "l2": "flushed before every step by reading a 512 MB buffer; pool larger than L2",
                       "parallelism": f"replicas{world}"},
            "decode_tok_s": decode_rows(w) * world / (ms * 1e-3),
            "hbm_frac_of_nominal_8tbs": value / world / NOMINAL_HBM_GBS,
            "hbm_frac_of_measured": value / world / peak,
            "read_stream_ceiling": None if read_ceiling is None else {
                "value": read_ceiling, "unit": "GB/s", "kernels_frac": achieved / read_ceiling,
                "how": "torch sum over a 512 MB float32 buffer, CUDA events, median of 10 passes"},
            "step_bytes": b["step"], "kv_bytes": b["kv"],
            "attention_ms": attn, "attention_kernels_ms": kern, "host_plan_us": host_plan_s / args.steps * 1e6,
            "roofline": {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                         "frac": achieved / peak, "traffic": traffic_for(w.name), "peak_source": peak_kind,
                         "kernel": kernels, "timed": "kernel-only CUDA events around the attention kernels, "
                                                     "L2 flushed before each of up to 300 steps"},
            "cpu_baseline": None if cpu is None else {k: cpu[k] for k in ("value", "unit", "cores", "kind", "sample")},
            "e2e": {"value": b["step"] * world / (e2e["ms"] * 1e-3) / 1e9, "unit": "GB/s",
                    "h2d_bytes_per_step": e2e["h2d"], "d2h_bytes_per_step": e2e["d2h"], "ms_per_step": e2e["ms"]},
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clocks.summary(),
            "plan": {k: plan.info[k] for k in ("num_items", "num_tc_items", "num_reduce", "num_partial_rows",
                                               "num_groups", "num_ctas")},
        }
        if prefill is not None:
            line["prefill"] = prefill
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


def run_e2e(args, w, dw, plan_opts, dev, stream, api):
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
              kv_dtype=w.kv_dtype, causal=w.causal, **plan_opts)
    gs = api.GraphStep(dw.cache, names, kw, w.softmax_scale, w.causal, stream=torch.cuda.Stream(dev))
    for views in gs.host:
        for k, v in names.items():
            views[k].copy_(v.cpu())
    for _ in range(4):
        gs.wait(gs.run())
    n = max(2, min(args.steps, 500))
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
    ap.add_argument("--ref-budget", type=float, default=10.0, help="seconds of oracle work per reference sample")
    ap.add_argument("--ref-seqs", type=int, default=None, help="sequences in the oracle sample (default all)")
    ap.add_argument("--no-cpu", action="store_true", help="skip the cpu_baseline oracle timing")
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
