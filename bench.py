"""Benchmark of the DSA hot path on B200.

One step = one pass of the whole path over one batch of synthetic input:
lightning-indexer scores -> per-query top-k -> sparse MLA over the selected
latent rows.  Default workload: DSA decode, 32 sequences of 32,768 cached
tokens, one new query each, top-2048, 128 MLA heads (576/512), bf16.  A
second line of measurement on the 16,384-token causal prefill workload is
reported under "prefill" in the same JSON line.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

Multi-GPU (launched by torchrun, one process per GPU): every rank runs its
own independent batch (replicas, weak scaling, no collective on the data
path); the step time is the max over ranks.

Timing: the step is captured in a CUDA graph and each replay is bracketed by
CUDA events on the launching stream.  Decode: the inputs exceed L2 (268 MB of
indexer keys, 1.2 GB of latent cache), so nothing is flushed between replays
(a written flush would leave dirty lines whose write-back lands in the next
step).  Prefill: a 256 MB buffer is written between replays (its 1 GB score
matrix also evicts L2 every step).  Per-kernel times come from graphs holding
one library call each.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import math
import os
import re
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

INDEXER_SRC = "indexer_tc.cu"     # source of the kernel that runs the bf16 indexer
METRIC = "DSA decode queries/s @32K ctx & prefill tok/s; fraction of HBM/tensor roofline"


# ------------------------------------------------------------------ ranks ----

def dist_env():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def init_dist(backend: str):
    import datetime
    import torch.distributed as dist
    rank, world, _ = dist_env()
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend=backend, timeout=datetime.timedelta(seconds=120))
    return rank, world


def max_over_ranks(x: float, device=None) -> float:
    """Max of a per-rank float over all ranks (identity when not distributed)."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device=None):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized() and dist.get_world_size() > 1:
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


# ------------------------------------------------------------ roofline ----

def measured_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return {"hbm_gbs": d["hbm_gbs"], "bf16_tflops": d["bf16_tflops"],
                "bf16_tflops_sustained": d.get("bf16_tflops_sustained", d["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def indexer_bytes(wl) -> int:
    """Algorithmic bytes of one indexer launch: every visible key row read
    once, the queries and weights read once, the visible scores written."""
    key_b = {"bf16": 2, "fp32": 4, "fp8": 1, "fp4": 0.5}[wl.idx_key_dtype]
    scale_b = 4 if wl.idx_key_dtype in ("fp8", "fp4") else 0
    q_b = 2 if wl.dtype == "bf16" else 4
    if wl.mode == "decode":
        vis = wl.ctx * wl.rows          # one query per cache in these workloads
        keys = wl.batch * wl.ctx
    else:
        vis = wl.rows * (wl.rows + 1) // 2
        keys = wl.ctx
    return int(keys * wl.idx_dim * key_b + keys * scale_b + wl.rows * wl.idx_heads * (wl.idx_dim * q_b + 4) + vis * 4)


def indexer_flops(wl) -> int:
    vis = wl.ctx * wl.rows if wl.mode == "decode" else wl.rows * (wl.rows + 1) // 2
    return 2 * vis * wl.idx_heads * wl.idx_dim


def mla_flops(wl) -> int:
    sel = wl.rows * wl.topk if wl.mode == "decode" else sum(min(t + 1, wl.topk) for t in range(wl.rows))
    return 2 * sel * wl.heads * (wl.d_qk + wl.d_v)


def mla_bytes(wl) -> int:
    sel = wl.rows * wl.topk if wl.mode == "decode" else sum(min(t + 1, wl.topk) for t in range(wl.rows))
    e = 2 if wl.dtype == "bf16" else 4
    return sel * wl.d_qk * e + wl.rows * wl.heads * (wl.d_qk + wl.d_v) * e + wl.rows * wl.topk * 4


def profiled_traffic(kernel: str, workload: str, source_file: str):
    """DRAM bytes per launch from a committed ncu summary, if the summary was
    taken on the current source of the kernel (same sha256 prefix)."""
    path = os.path.join(ROOT, "profiles", f"{kernel}__{workload}.md")
    if not os.path.exists(path) or not os.path.exists(source_file):
        return None
    txt = open(path).read()
    m = re.search(r"traffic_bytes_per_launch:\s*([0-9.eE+]+)", txt)
    h = re.search(r"kernel_source_sha256:\s*([0-9a-f]+)", txt)
    if not m or not h:
        return None
    cur = hashlib.sha256(open(source_file, "rb").read()).hexdigest()
    if not cur.startswith(h.group(1)):
        return None
    return float(m.group(1))


# --------------------------------------------------------------- clocks ----

class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons while running."""
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "200"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                out, _ = self.proc.communicate(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                out, _ = self.proc.communicate()
            self.lines = [l for l in out.splitlines() if l.strip()]

    def summary(self):
        if not self.lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"], "samples": 0}
        sm, smax, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for l in self.lines:
            p = [x.strip() for x in l.split(",")]
            if len(p) < 9:
                continue
            try:
                sm.append(float(p[1]))
                smax = float(p[2])
            except ValueError:
                continue
            for n, v in zip(names, p[5:9]):
                if v.lower() == "active":
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": smax, "reasons": sorted(reasons),
                "samples": len(sm)}


# ------------------------------------------------------------ our arm ----

def pool_caches(dsa, wl, inp):
    """CSA workloads: pool the raw caches m:1 (csa_compress) into block caches."""
    if wl.compress_m > 1:
        inp["k_idx"] = dsa.csa_compress(inp["k_idx"], wl.compress_m)
        inp["kv"] = dsa.csa_compress(inp["kv"], wl.compress_m)
    return inp


class DecodeStep:
    """Preallocated buffers and the three library calls of one step."""

    def __init__(self, dsa, wl, inp, device):
        import torch
        pool_caches(dsa, wl, inp)
        self.dsa, self.wl, self.inp = dsa, wl, inp
        self.logits = torch.empty((wl.rows, wl.ctx), dtype=torch.float32, device=device)
        self.idx = torch.empty((wl.rows, wl.topk), dtype=torch.int32, device=device)
        self.out = torch.empty((wl.rows, wl.heads, wl.d_v), dtype=inp["q"].dtype, device=device)
        self.lse = torch.empty((wl.rows, wl.heads), dtype=torch.float32, device=device)
        n = dsa.topk_workspace_size(wl.rows, wl.ctx, wl.topk)
        self.topk_ws = torch.empty(max(n, 1), dtype=torch.uint8, device=device) if n else None
        n = dsa.sparse_mla_workspace_size(wl.rows, wl.topk, wl.heads, wl.d_qk, wl.d_v, inp["q"].dtype)
        self.mla_ws = torch.empty(max(n, 1), dtype=torch.uint8, device=device) if n else None

    def run_one(self, name):
        d, wl, i = self.dsa, self.wl, self.inp
        if name == "dsa_indexer_logits":
            d.indexer_logits(i["q_idx"], i["w"], i["k_idx"], i["row_batch"], i["row_pos"],
                             k_scale=i.get("k_scale"), out=self.logits)
        elif name == "dsa_topk":
            d.topk(self.logits, i["row_pos"], wl.topk, ctx_len=wl.ctx, out=self.idx, workspace=self.topk_ws)
        else:
            d.sparse_mla(i["q"], i["kv"], self.idx, i["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                         page_table=i.get("page_table"), out=self.out, lse=self.lse, workspace=self.mla_ws)

    def run(self):
        for name in ("dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla"):
            self.run_one(name)


def _graph(fn):
    """Capture fn() (library calls on the current stream) into a CUDA graph."""
    import torch
    s = torch.cuda.Stream()
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        fn()                                  # warm (kernel attributes, tensor maps) outside capture
    torch.cuda.current_stream().wait_stream(s)
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        fn()
    torch.cuda.synchronize()
    return g


def replay_stats(ms_list):
    """Summary of per-replay device times (ms): the median is the headline
    figure; mean, min, p90 and max show whether a slow replay is an outlier
    or a steady slowdown."""
    s = sorted(ms_list)
    n = len(s)
    return {"median": statistics.median(s), "mean": statistics.mean(s), "min": s[0],
            "p90": s[min(n - 1, int(math.ceil(0.9 * n)) - 1)], "max": s[-1], "n": n}


def stats_json(st, nd=4):
    return {k: (round(v, nd) if k != "n" else v) for k, v in st.items()}


def time_graph(g, steps, device, flush=None, flush_read=None):
    """Replay `g` `steps` times, each bracketed by CUDA events on the current
    stream; with `flush` (a buffer larger than L2) it is written before each
    replay, outside the events.  Returns replay_stats() of the per-replay
    device times in ms.  Without `flush` the inputs themselves must exceed
    L2: a written flush leaves L2 full of dirty lines whose write-back would
    then be charged to the next replay.  `flush_read` (a buffer larger than
    L2) is instead read before each replay, which evicts L2 without dirtying
    it."""
    import torch
    evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(steps)]
    barrier(device)
    torch.cuda.synchronize(device)
    sink = torch.empty((), dtype=torch.float32, device=device)
    for a, b in evs:
        if flush is not None:
            flush.zero_()
        if flush_read is not None:
            torch.sum(flush_read, dim=0, out=sink)
        a.record()
        g.replay()
        b.record()
    torch.cuda.synchronize(device)
    barrier(device)
    return replay_stats([a.elapsed_time(b) for a, b in evs])


def time_steps(step, steps, warmup, device, flush=None, soak_s=0.0):
    """The step (indexer -> top-k -> sparse MLA) is captured once into a CUDA
    graph and replayed: timings are device time, free of host launch gaps.
    Per-kernel times come from graphs holding one library call each.
    Returns (replay_stats of the step in ms, {kernel: median ms}, library
    kernel launches in the timed steps)."""
    import torch
    dsa = step.dsa
    n0 = dsa.launch_count()
    g_step = _graph(step.run)
    per_step = (dsa.launch_count() - n0) // 2          # launches recorded by the warm run + the capture
    for _ in range(warmup):
        g_step.replay()
    torch.cuda.synchronize(device)
    if soak_s > 0:                      # same step, back to back, so the clock sampler sees it under load
        t_end = time.perf_counter() + soak_s
        while time.perf_counter() < t_end:
            for _ in range(50):
                g_step.replay()
            torch.cuda.synchronize(device)
    st = time_graph(g_step, steps, device, flush)
    kern = {}
    for name in ("dsa_indexer_logits", "dsa_topk", "dsa_sparse_mla"):
        g = _graph(lambda n=name: step.run_one(n))
        g.replay()
        kern[name] = time_graph(g, max(3, steps // 2), device, flush)["median"]
        del g
    return st, kern, per_step * steps


def e2e_decode(dsa, wl, inp, step, steps, device):
    """Same metric through the public API with host buffers.  Every step
    copies its new inputs from pinned host memory (the queries and head
    weights, and the new token's indexer-key and latent rows appended to each
    cache), runs the path, and reads the attention output and lse back.

    Steps are pipelined the way a serving loop runs them: two slots of
    per-step device buffers; the input copies run on one stream and the
    readback on another, each ordered against the compute stream by events,
    so step i+1's copies and step i's readback overlap step i's compute.  The
    compute part of a step is the cache-row appends and the three library
    calls, and each stream's part of a step (the input copies, the compute, the
    readback) is one CUDA graph per slot, so the host only replays three
    graphs and orders them with events.  The timed region runs from the first
    input copy to the last readback."""
    import torch
    g = torch.Generator().manual_seed(1234)
    last = wl.ctx - 1
    slots = []
    for s_ in range(2):
        sin = dict(inp)
        for name in ("q_idx", "w", "q"):
            sin[name] = torch.empty_like(inp[name])
            sin[name].copy_(inp[name])
        st = DecodeStep(dsa, wl, sin, device)
        host = {name: inp[name].cpu().pin_memory() for name in ("q_idx", "w", "q")}
        host["new_k"] = (torch.randn((wl.batch, wl.idx_dim), generator=g) / math.sqrt(wl.idx_dim)).to(
            inp["k_idx"].dtype).pin_memory()
        host["new_kv"] = (torch.randn((wl.batch, wl.d_qk), generator=g) / math.sqrt(wl.d_qk)).to(
            inp["kv"].dtype).pin_memory()
        out_h = torch.empty(st.out.shape, dtype=st.out.dtype).pin_memory()
        lse_h = torch.empty(st.lse.shape, dtype=torch.float32).pin_memory()
        # the new rows land in device staging buffers with the other inputs
        # (host copies stay on the input stream's copy engine); the step's
        # graph appends them to the caches with device-side copies
        stage = {"new_k": host["new_k"].to(device), "new_kv": host["new_kv"].to(device)}

        def compute(st=st, stage=stage):
            inp["k_idx"][:, last].copy_(stage["new_k"])
            if "page_table" not in inp:
                inp["kv"][:, last].copy_(stage["new_kv"])
            st.run()

        def copy_in(st=st, host=host, stage=stage):
            for name in ("new_k", "new_kv"):
                stage[name].copy_(host[name], non_blocking=True)
            for name in ("q_idx", "w", "q"):
                st.inp[name].copy_(host[name], non_blocking=True)

        def copy_out(st=st, out_h=out_h, lse_h=lse_h):
            out_h.copy_(st.out, non_blocking=True)
            lse_h.copy_(st.lse, non_blocking=True)

        slots.append({"st": st, "host": host, "stage": stage, "out_h": out_h, "lse_h": lse_h,
                      "graph": _graph(compute), "g_in": _graph(copy_in), "g_out": _graph(copy_out)})
    h2d = sum(slots[0]["host"][n].numel() * slots[0]["host"][n].element_size() for n in slots[0]["host"])
    h2d -= 0 if "page_table" not in inp else slots[0]["host"]["new_kv"].numel() * 2
    d2h = slots[0]["out_h"].numel() * slots[0]["out_h"].element_size() + slots[0]["lse_h"].numel() * 4

    s_in, s_comp, s_out = torch.cuda.Stream(), torch.cuda.Stream(), torch.cuda.Stream()
    ev = {k: [torch.cuda.Event() for _ in range(2)] for k in ("in", "comp", "out")}

    def one(i):
        sl = slots[i & 1]
        e_in, e_comp, e_out = ev["in"][i & 1], ev["comp"][i & 1], ev["out"][i & 1]
        with torch.cuda.stream(s_in):
            s_in.wait_event(e_comp)                 # the slot's inputs are no longer read
            sl["g_in"].replay()
            e_in.record(s_in)
        s_comp.wait_event(e_in)
        s_comp.wait_event(e_out)                    # the slot's outputs have been read back
        with torch.cuda.stream(s_comp):
            sl["graph"].replay()
            e_comp.record(s_comp)
        with torch.cuda.stream(s_out):
            s_out.wait_event(e_comp)
            sl["g_out"].replay()
            e_out.record(s_out)

    for i in range(4):
        one(i)
    torch.cuda.synchronize(device)
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record(s_in)
    for i in range(steps):
        one(i)
    s_out.wait_event(ev["out"][(steps - 1) & 1])
    b.record(s_out)
    torch.cuda.synchronize(device)
    ms = a.elapsed_time(b) / steps
    return ms, h2d, d2h


def cpu_baseline_decode(wl, inp, budget_s: float = 12.0):
    """The oracle, as it stands, on a bounded sample of the same workload:
    whole query rows (index scores over all keys, top-k, attention), cycling
    over the batch, until the time budget is used.  Returns (queries/s, rows
    done, threads, seconds)."""
    import numpy as np
    import oracle
    import torch
    done, t_used = 0, 0.0
    host = {}                                        # host copies per query row (taken outside the timing)
    for rr in range(1 << 20):
        r = rr % wl.rows
        if r not in host:
            b = int(inp["row_batch"][r])
            ks = inp["k_scale"][b:b + 1].cpu() if "k_scale" in inp else None
            if "page_table" in inp:
                kv = inp["kv"].index_select(0, inp["page_table"][b].long()).cpu()
                table = torch.arange(kv.shape[0], dtype=torch.int32).view(1, -1)
            else:
                kv = inp["kv"][b:b + 1].cpu()
                table = None
            host[r] = (inp["q_idx"][r:r + 1].cpu(), inp["w"][r:r + 1].cpu(), inp["k_idx"][b:b + 1].cpu(), ks,
                       inp["row_pos"][r:r + 1].cpu(), kv, table, inp["q"][r:r + 1].cpu())
            if len(host) > 8:                        # bound host memory: keep a few rows
                host.pop(next(iter(host)))
        q_idx, w, kb, ks, rp, kv, table, q = host[r]
        rb0 = torch.zeros(1, dtype=torch.int32)
        t0 = time.perf_counter()
        scores = oracle.index_scores(q_idx, w, kb, rb0, rp, k_scale=ks)
        idx = oracle.topk(scores, rp, wl.topk)
        oracle.sparse_mla(q, kv, idx, rb0, wl.softmax_scale, wl.d_v, wl.ctx, page_table=table)
        t_used += time.perf_counter() - t0
        done += 1
        if t_used >= budget_s:
            break
    return done / t_used, done, oracle.max_threads(), t_used


def _oracle_rows(fn, n_rows: int, budget_s: float):
    """Call fn(r) for r = 0, 1, ... (cycling over n_rows) until budget_s of
    CPU time is used; returns (calls/s, calls, seconds)."""
    done, t_used = 0, 0.0
    while t_used < budget_s:
        t0 = time.perf_counter()
        fn(done % n_rows)
        t_used += time.perf_counter() - t0
        done += 1
    return done / t_used, done, t_used


def run_kernel_only(args):
    """One kernel of the step, alone, on the workload's real inputs (the step
    runs once first so that top-k indices exist).  Used for profiler captures
    of a single kernel; prints its mean event time."""
    import torch
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    import sparse_attention_logits_b200 as dsa
    import workloads
    if args.kernel_only == "prepare":
        return run_prepare_only(dsa, workloads, device, args)
    wl = workloads.BY_NAME[args.workload]
    if args.prefill_tokens and wl.mode == "prefill":
        # a shorter prompt of the same prefill workload (profiler captures
        # that collect more than kernel durations stay a few GB in size)
        wl = wl.with_(name=f"{wl.name}_T{args.prefill_tokens}", rows=args.prefill_tokens, ctx=args.prefill_tokens)
    inp = workloads.generate(wl, device=device, seed=0)
    step = DecodeStep(dsa, wl, inp, device)
    step.run()
    i = inp
    launch = {
        "indexer": lambda: dsa.indexer_logits(i["q_idx"], i["w"], i["k_idx"], i["row_batch"], i["row_pos"],
                                              k_scale=i.get("k_scale"), out=step.logits),
        "topk": lambda: dsa.topk(step.logits, i["row_pos"], wl.topk, ctx_len=wl.ctx, out=step.idx,
                                 workspace=step.topk_ws),
        "mla": lambda: dsa.sparse_mla(i["q"], i["kv"], step.idx, i["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx,
                                      page_table=i.get("page_table"), out=step.out, lse=step.lse,
                                      workspace=step.mla_ws),
    }[args.kernel_only]
    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    a.record()
    for _ in range(args.steps):
        launch()
    b.record()
    torch.cuda.synchronize()
    dsa.get_device_error(device)
    host_ms = a.elapsed_time(b) / args.steps
    g = _graph(launch)
    dev = time_graph(g, args.steps, device)
    print(json.dumps({"kernel": args.kernel_only, "workload": wl.name, "ms": dev["median"],
                      "ms_stats": stats_json(dev), "ms_stream_launches": host_ms}))


def run_prepare_only(dsa, workloads, device, args):
    """dsa_indexer_prepare alone on `--prep-tokens` tokens (V3-class sizes,
    fp8 key cache of 64K rows, about 0.1 GB on the device): for profiler
    captures.  Prints the mean event time of one call."""
    import torch
    T = args.prep_tokens
    shape = workloads.PrepareShape(T, PREP_D_C, PREP_D_MODEL, max_pos=4096, cache_rows=max(T, 65536))
    inp = {k: v.to(device) for k, v in workloads.make_prepare_inputs(shape, seed=0, skip=0.0).items()}
    cache = torch.zeros((shape.cache_rows, 128), dtype=torch.uint8, device=device)
    scale = torch.ones(shape.cache_rows, dtype=torch.float32, device=device)
    q_out = torch.empty((T, 64, 128), dtype=torch.bfloat16, device=device)
    w_out = torch.empty((T, 64), dtype=torch.float32, device=device)
    ws = torch.empty(max(dsa.indexer_prepare_workspace_size(T, 64, PREP_D_C, PREP_D_MODEL), 1), dtype=torch.uint8,
                     device=device)

    def launch():
        dsa.indexer_prepare(inp["c_q"], inp["gamma"], inp["wq_b"], inp["h"], inp["wk"], inp["w_proj"], inp["pos"],
                            inp["slot"], cache, scale, inp["rope_cos"], inp["rope_sin"], q_out=q_out, w_out=w_out,
                            workspace=ws)

    for _ in range(args.warmup):
        launch()
    torch.cuda.synchronize()
    dsa.get_device_error(device)
    g = _graph(launch)
    evict = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    dev = time_graph(g, args.steps, device, flush_read=evict)
    print(json.dumps({"kernel": "prepare", "tokens": T, "ms": dev["median"], "ms_stats": stats_json(dev)}))


def run_ours(args):
    import torch
    rank, world = init_dist("nccl")
    _, _, local = dist_env()
    device = torch.device("cuda", local)
    torch.cuda.set_device(device)
    import sparse_attention_logits_b200 as dsa
    import workloads

    wl = workloads.BY_NAME[args.workload]
    inp = workloads.generate(wl, device=device, seed=rank)
    step = DecodeStep(dsa, wl, inp, device)
    peaks = measured_peaks()

    with ClockSampler(device.index if "CUDA_VISIBLE_DEVICES" not in os.environ else local) as clk:
        st, kern, launches = time_steps(step, args.steps, args.warmup, device, soak_s=1.5)
    dsa.get_device_error(device)
    ms_max = max_over_ranks(st["median"], device)
    value = wl.rows * world / (ms_max / 1e3)

    ib = indexer_bytes(wl)
    ach = ib / (kern["dsa_indexer_logits"] / 1e3) / 1e9
    traffic = profiled_traffic("dsa_indexer_logits", wl.name, os.path.join(ROOT, "sparse_attention_logits_b200",
                                                                            "csrc", INDEXER_SRC))
    roof = {"kernel": "dsa_indexer_logits", "bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
            "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4), "traffic": traffic,
            "algorithmic_bytes": ib, "peak_source": peaks["source"]}

    e2e_ms, h2d, d2h = e2e_decode(dsa, wl, inp, step, max(3, args.steps // 2), device)
    e2e_ms = max_over_ranks(e2e_ms, device)

    result = {
        "metric": METRIC, "value": round(value, 1), "unit": "queries/s", "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms_max, 4), "ms_stats": stats_json(st),
        "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "ctx": wl.ctx, "topk": wl.topk,
                   "indexer": f"{wl.idx_heads}x{wl.idx_dim}", "mla": f"{wl.heads}h {wl.d_qk}/{wl.d_v}",
                   "parallelism": f"replicas{world}",
                   "launch": "CUDA graph of the step (device time, median of the timed replays)",
                   "l2": "inputs larger than L2 (keys 268 MB, latent cache 1.2 GB); no flush between steps"},
        "roofline": roof,
        "kernels_ms": {k: round(v, 4) for k, v in kern.items()},
        "gpu_launches": launches,
        "e2e": {"value": round(wl.rows * world / (e2e_ms / 1e3), 1), "unit": "queries/s",
                "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "clocks": clk.summary(),
    }
    if args.prefill:
        result["prefill"] = run_prefill(dsa, workloads, device, peaks, args)
    if args.tiny:
        result["tiny_prefill"] = run_tiny(dsa, workloads, device, peaks, args)
    if args.compress:
        result["csa_compress"] = run_compress(dsa, workloads, device, peaks, args)
    if args.others:
        result["other_decodes"] = run_other_decodes(dsa, workloads, device, peaks, args)
    if args.v4:
        result["v4_variants"] = run_v4_variants(dsa, workloads, device, peaks, args)
    if args.prepare:
        result["indexer_prepare"] = run_prepare(dsa, workloads, device, peaks, args)
    if world == 1 and rank == 0 and args.cpu_baseline:
        qps, n, cores, secs = cpu_baseline_decode(wl, inp)
        result["cpu_baseline"] = {"value": round(qps, 4), "unit": "queries/s", "cores": cores, "kind": "oracle",
                                  "sample": f"{n} whole query rows of {wl.name} ({secs:.1f} s of CPU work)"}
    if rank == 0:
        print(json.dumps(result), flush=True)
    _finish()


def run_prefill(dsa, workloads, device, peaks, args):
    import torch
    rank, world, _ = dist_env()
    wl = workloads.PREFILL_16K
    inp = workloads.generate(wl, device=device, seed=100 + rank)
    step = DecodeStep(dsa, wl, inp, device)
    flush = torch.empty(256 * 1024 * 1024 // 4, dtype=torch.float32, device=device)
    steps = max(2, args.steps // 4)
    st, kern, launches = time_steps(step, steps, max(3, args.warmup // 2), device, flush)
    ms_max = max_over_ranks(st["median"], device)
    fl_i, fl_m = indexer_flops(wl), mla_flops(wl)
    pk = peaks["bf16_tflops"]
    mla_t = fl_m / (kern["dsa_sparse_mla"] / 1e3) / 1e12
    idx_t = fl_i / (kern["dsa_indexer_logits"] / 1e3) / 1e12
    cpu = None
    if rank == 0 and world == 1 and args.cpu_baseline:
        cpu = cpu_baseline_prefill(wl, inp)
    del inp, step, flush
    torch.cuda.empty_cache()
    res = {"workload": wl.name, "value": round(wl.rows * world / (ms_max / 1e3), 1), "unit": "tokens/s",
            "ms_per_step": round(ms_max, 3), "ms_stats": stats_json(st, 3), "steps": steps,
            "kernels_ms": {k: round(v, 3) for k, v in kern.items()},
            "roofline": {"kernel": "dsa_sparse_mla", "bound": "tensor", "achieved": round(mla_t, 1), "peak": pk,
                         "unit": "TFLOP/s", "frac": round(mla_t / pk, 4), "traffic": None,
                         "algorithmic_flops": fl_m},
            "indexer_roofline": {"bound": "tensor", "achieved": round(idx_t, 1), "peak": pk, "unit": "TFLOP/s",
                                 "frac": round(idx_t / pk, 4), "algorithmic_flops": fl_i}}
    if cpu is not None:
        res["cpu_baseline"] = cpu
    return res


def prefill_sample_rows(n_tokens: int, n: int = 256, seed: int = 7):
    """Seeded sample of prefill query rows for the oracle baseline: the
    keep-all boundary (0, k-1, k) and the last token, plus rows drawn
    uniformly without replacement from the rest."""
    import torch
    fixed = [0, 2047, 2048, n_tokens - 1]
    g = torch.Generator().manual_seed(seed)
    rest = [int(x) for x in torch.randperm(n_tokens, generator=g) if int(x) not in fixed]
    return sorted(fixed + rest[:n - len(fixed)])


def cpu_baseline_prefill(wl, inp):
    """The oracle, as it stands, on a seeded sample of 256 query rows of the
    16K-token prefill (index scores over each row's visible prefix, top-k,
    attention over the selected rows), in one call per stage so that its
    OpenMP loop over rows uses every core.  Throughput is the sample's rows
    over its time: an extrapolation to the whole prefill, labelled as such."""
    import oracle
    import torch
    rows = prefill_sample_rows(wl.rows)
    ids = torch.tensor(rows, dtype=torch.long, device=inp["q"].device)
    # host copies of the sampled rows' queries and of the shared caches (outside the timing)
    q_idx, w, q = inp["q_idx"][ids].cpu(), inp["w"][ids].cpu(), inp["q"][ids].cpu()
    rb, rp = inp["row_batch"][ids].cpu(), inp["row_pos"][ids].cpu()
    k_idx, kv = inp["k_idx"].cpu(), inp["kv"].cpu()
    t0 = time.perf_counter()
    scores = oracle.index_scores(q_idx, w, k_idx, rb, rp)
    sel = oracle.topk(scores, rp, wl.topk)
    oracle.sparse_mla(q, kv, sel, rb, wl.softmax_scale, wl.d_v, wl.ctx)
    secs = time.perf_counter() - t0
    return {"value": round(len(rows) / secs, 3), "unit": "tokens/s", "cores": oracle.max_threads(), "kind": "oracle",
            "sample": (f"{len(rows)} seeded query rows of {wl.name} (positions 0, 2047, 2048, {wl.rows - 1} and "
                       f"{len(rows) - 4} uniform others), {secs:.1f} s of CPU work; tokens/s extrapolated from the "
                       f"sample's mean time per row")}


def run_other_decodes(dsa, workloads, device, peaks, args):
    """The two other decode workloads, each a whole step (indexer -> top-k ->
    sparse MLA) in a CUDA graph, timed like the main step, against the HBM
    roofline of its algorithmic bytes: CSA decode over 4 x 262,144 pooled
    entries of 1,048,576-token caches (pooling is per 4 new tokens, outside
    the step), and decode over 64 x 131,072 keys with fp8 indexer keys and a
    paged latent cache, and the same with fp4 (e2m1) indexer keys."""
    import torch
    rank, world, _ = dist_env()
    res = {}
    fp4 = workloads.DECODE_128K_FP8_PAGED.with_(name="dsa_decode_fp4idx_paged64_B64_L131072_k2048",
                                                idx_key_dtype="fp4")
    for wl in (workloads.CSA_DECODE_1M, workloads.DECODE_128K_FP8_PAGED, fp4):
        inp = workloads.generate(wl, device=device, seed=300 + rank)
        step = DecodeStep(dsa, wl, inp, device)
        st, kern, _ = time_steps(step, max(5, args.steps // 2), 3, device, soak_s=0.5)
        ms = max_over_ranks(st["median"], device)
        b = indexer_bytes(wl) + mla_bytes(wl)
        if wl.page_size:
            b += wl.batch * (wl.ctx // wl.page_size) * 4          # the page table
        ach = b / (ms / 1e3) / 1e9
        res[wl.name] = {"value": round(wl.rows * world / (ms / 1e3), 1), "unit": "queries/s",
                        "ms_per_step": round(ms, 4), "ms_stats": stats_json(st),
                        "kernels_ms": {k: round(v, 4) for k, v in kern.items()},
                        "roofline": {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"],
                                     "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                                     "algorithmic_bytes": b},
                        "l2": "inputs larger than L2; no flush between steps"}
        del inp, step
        torch.cuda.empty_cache()
    return res


def run_compress(dsa, workloads, device, peaks, args):
    """CSA token compression (csa_compress, m = 4) of the raw caches of the
    1M-token CSA decode: the 4 x 1,048,576 x 576 latent cache and the
    4 x 1,048,576 x 128 indexer key cache, both bf16, pooled into 262,144
    entries per sequence.  One graph holds the two calls; the raw caches
    (5.9 GB) exceed L2, so nothing is flushed between replays.  Roofline:
    every raw row read once and every pooled row written once (7.38 GB) over
    the event time, against the measured HBM copy bandwidth."""
    import torch
    rank, world, _ = dist_env()
    wl = workloads.CSA_DECODE_1M
    inp = workloads.generate(wl, device=device, seed=400 + rank)
    raw_k, raw_kv = inp["k_idx"], inp["kv"]
    del inp
    m = wl.compress_m
    out_k = torch.empty((wl.batch, wl.ctx, wl.idx_dim), dtype=raw_k.dtype, device=device)
    out_kv = torch.empty((wl.batch, wl.ctx, wl.d_qk), dtype=raw_kv.dtype, device=device)

    def call():
        dsa.csa_compress(raw_kv, m, out=out_kv)
        dsa.csa_compress(raw_k, m, out=out_k)

    n0 = dsa.launch_count()
    g = _graph(call)
    launches = (dsa.launch_count() - n0) // 2
    for _ in range(3):
        g.replay()
    st = time_graph(g, max(5, args.steps // 2), device)
    ms = max_over_ranks(st["median"], device)
    dsa.get_device_error(device)
    del g
    moved = (raw_k.numel() + raw_kv.numel()) * raw_k.element_size() + \
        (out_k.numel() + out_kv.numel()) * out_k.element_size()
    ach = moved / (ms / 1e3) / 1e9
    raw_tokens = wl.batch * wl.raw_ctx
    res = {"workload": f"csa_compress_bf16_B{wl.batch}_L{wl.raw_ctx}_m{m}_d{wl.d_qk}+d{wl.idx_dim}",
           "value": round(raw_tokens * world / (ms / 1e3), 1), "unit": "raw tokens/s",
           "ms_per_step": round(ms, 4), "ms_stats": stats_json(st), "gpu_launches": launches,
           "roofline": {"kernel": "csa_compress", "bound": "hbm", "achieved": round(ach, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": round(ach / peaks["hbm_gbs"], 4),
                        "algorithmic_bytes": moved},
           "l2": "raw caches (5.9 GB) larger than L2; no flush between replays"}
    if rank == 0 and world == 1 and args.cpu_baseline:
        import oracle
        n_raw = 65536                                # raw rows of each cache in the sample (sequence 0)
        kv_h, k_h = raw_kv[:1, :n_raw].cpu(), raw_k[:1, :n_raw].cpu()

        def pool(_):
            oracle.csa_compress(kv_h, m)
            oracle.csa_compress(k_h, m)
        v, n, secs = _oracle_rows(pool, 1, 3.0)
        res["cpu_baseline"] = {"value": round(v * n_raw, 1), "unit": "raw tokens/s", "cores": oracle.max_threads(),
                               "kind": "oracle",
                               "sample": f"{n} poolings of {n_raw} raw rows of both caches ({secs:.1f} s of CPU work)"}
    del raw_k, raw_kv, out_k, out_kv
    torch.cuda.empty_cache()
    return res


def run_tiny(dsa, workloads, device, peaks, args):
    """The tiny fp32 causal prefill (256 tokens, top-64, 4 x 32 indexer, 8 MQA
    heads over a 64-d latent): the whole path as one graph.  It moves about
    0.3 MB and is bound by launch and synchronisation latency, so it is
    reported as microseconds per step; its inputs stay in L2."""
    import oracle
    import torch
    rank, world, _ = dist_env()
    wl = workloads.TINY_PREFILL_FP32
    inp = workloads.generate(wl, device=device, seed=500 + rank)
    step = DecodeStep(dsa, wl, inp, device)
    st, kern, launches = time_steps(step, max(20, args.steps), 3, device)
    us = max_over_ranks(st["median"], device) * 1e3
    res = {"workload": wl.name, "us_per_step": round(us, 2), "value": round(wl.rows * world / (us / 1e6), 1),
           "unit": "tokens/s", "ms_stats": stats_json(st, 5),
           "kernels_us": {k: round(v * 1e3, 2) for k, v in kern.items()}, "gpu_launches": launches,
           "l2": "inputs (0.3 MB) stay in L2: latency-bound"}
    if rank == 0 and world == 1 and args.cpu_baseline:
        h = {k: v.cpu() for k, v in inp.items()}

        def whole(_):
            sc = oracle.index_scores(h["q_idx"], h["w"], h["k_idx"], h["row_batch"], h["row_pos"])
            sel = oracle.topk(sc, h["row_pos"], wl.topk)
            oracle.sparse_mla(h["q"], h["kv"], sel, h["row_batch"], wl.softmax_scale, wl.d_v, wl.ctx)
        v, n, secs = _oracle_rows(whole, 1, 2.0)
        res["cpu_baseline"] = {"value": round(v * wl.rows, 1), "unit": "tokens/s", "cores": oracle.max_threads(),
                               "kind": "oracle", "sample": f"{n} whole steps ({secs:.1f} s of CPU work)"}
    del inp, step
    torch.cuda.empty_cache()
    return res


V4_WINDOW = 128       # raw rows in the CSA window (the pages give no size)
V4_SINK = 4           # raw rows in the CSA attention sink: the sequence's first rows (the pages give no size)
HCA_M = 128           # HCA pooling factor m'


def run_v4_variants(dsa, workloads, device, peaks, args):
    """DeepSeek-V4's two compressed-attention variants at the 1M-token CSA
    shapes (4 sequences of 1,048,576 raw tokens, one new query each):

    csa_step: pooled indexer keys -> top-1024 pooled entries -> CSA core
      attention over those entries plus a window of the last 128 raw rows
      and a sink of the first 4 raw rows.
      The pooling itself (csa_compress) runs once per 4 new tokens in a real
      cache and is not part of the step.
    hca: dense attention of each query over all 8,192 entries of the 128:1
      pooled latent cache (pooling again outside the step).
    Each is captured in a CUDA graph and timed like the main step; the
    roofline is HBM bytes (what must be read once) over the event time."""
    import torch
    rank, world, _ = dist_env()
    wl = workloads.CSA_DECODE_1M
    inp = workloads.generate(wl, device=device, seed=200 + rank)
    raw_kv = inp["kv"]
    k_c = dsa.csa_compress(inp["k_idx"], wl.compress_m)
    kv_c = dsa.csa_compress(raw_kv, wl.compress_m)
    del inp["k_idx"]
    rows, ctx = wl.rows, wl.ctx
    logits = torch.empty((rows, ctx), dtype=torch.float32, device=device)
    idx = torch.empty((rows, wl.topk), dtype=torch.int32, device=device)
    n = dsa.topk_workspace_size(rows, ctx, wl.topk)
    tws = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
    n = dsa.sparse_mla_workspace_size(rows, wl.topk + V4_WINDOW + V4_SINK, wl.heads, wl.d_qk, wl.d_v, torch.bfloat16)
    mws = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
    out = torch.empty((rows, wl.heads, wl.d_v), dtype=torch.bfloat16, device=device)
    lse = torch.empty((rows, wl.heads), dtype=torch.float32, device=device)
    win_pos = torch.full((rows,), wl.raw_ctx - 1, dtype=torch.int32, device=device)

    class Csa:
        def run_one(self, name):
            if name == "dsa_indexer_logits":
                dsa.indexer_logits(inp["q_idx"], inp["w"], k_c, inp["row_batch"], inp["row_pos"], out=logits)
            elif name == "dsa_topk":
                dsa.topk(logits, inp["row_pos"], wl.topk, ctx_len=ctx, out=idx, workspace=tws)
            else:
                dsa.csa_core_attention(inp["q"], kv_c, idx, inp["row_batch"], wl.softmax_scale, wl.d_v, ctx, raw_kv,
                                       win_pos, V4_WINDOW, out=out, lse=lse, workspace=mws, n_sink=V4_SINK)

        def run(self):
            for nm in ("dsa_indexer_logits", "dsa_topk", "csa_core_attention"):
                self.run_one(nm)

    st = Csa()
    st.dsa = dsa
    g = _graph(st.run)
    for _ in range(3):
        g.replay()
    steps = max(5, args.steps)
    st_step = time_graph(g, steps, device)
    ms = max_over_ranks(st_step["median"], device)
    del g
    # alone, the gathered rows (5 MB) would stay in L2 between replays: read
    # a 256 MB buffer before each one
    evict = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    ga = _graph(lambda: st.run_one("csa_core_attention"))
    ga.replay()
    ms_attn = time_graph(ga, steps, device, flush_read=evict)["median"]
    del ga
    sel_rows = rows * (wl.topk + V4_WINDOW + V4_SINK)
    step_bytes = (indexer_bytes(wl) + sel_rows * wl.d_qk * 2 + rows * wl.heads * (wl.d_qk + wl.d_v) * 2)
    attn_bytes = sel_rows * wl.d_qk * 2 + rows * wl.heads * (wl.d_qk + wl.d_v) * 2
    csa = {"workload": f"{wl.name}+window{V4_WINDOW}+sink{V4_SINK}", "value": round(rows * world / (ms / 1e3), 1),
           "unit": "queries/s", "ms_per_step": round(ms, 4), "ms_stats": stats_json(st_step),
           "core_attention_ms": round(ms_attn, 4),
           "roofline": {"bound": "hbm", "achieved": round(step_bytes / (ms / 1e3) / 1e9, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(step_bytes / (ms / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                        "algorithmic_bytes": step_bytes},
           "core_attention_bytes": attn_bytes,
           "l2": "step: pooled keys (268 MB) exceed L2, no flush; core attention alone: 256 MB read between replays"}
    if rank == 0 and world == 1 and args.cpu_baseline:
        import oracle
        # host copy of the raw rows the step reads: the sink rows, then the window's rows
        win_rows = torch.cat([raw_kv[:, :V4_SINK], raw_kv[:, wl.raw_ctx - V4_WINDOW:]], dim=1).cpu()
        keys_h, kvc_h = k_c.cpu(), kv_c.cpu()
        rb0 = torch.zeros(1, dtype=torch.int32)

        def csa_row(r):
            b = int(inp["row_batch"][r])
            rp = inp["row_pos"][r:r + 1].cpu()
            sc = oracle.index_scores(inp["q_idx"][r:r + 1].cpu(), inp["w"][r:r + 1].cpu(), keys_h[b:b + 1], rb0, rp)
            sel = oracle.topk(sc, rp, wl.topk)
            oracle.csa_core_attention(inp["q"][r:r + 1].cpu(), kvc_h[b:b + 1], sel, rb0, wl.softmax_scale, wl.d_v,
                                      ctx, win_rows[b:b + 1], torch.tensor([V4_SINK + V4_WINDOW - 1], dtype=torch.int32),
                                      V4_WINDOW, n_sink=V4_SINK)
        v, n, secs = _oracle_rows(csa_row, rows, 6.0)
        csa["cpu_baseline"] = {"value": round(v, 4), "unit": "queries/s", "cores": oracle.max_threads(),
                               "kind": "oracle", "sample": f"{n} whole query rows ({secs:.1f} s of CPU work)"}
        del win_rows, keys_h, kvc_h
    del logits, idx, tws, k_c, kv_c
    # HCA over the 128:1 pooled cache
    kv_h = dsa.csa_compress(raw_kv, HCA_M)
    del raw_kv, inp["kv"]
    torch.cuda.empty_cache()
    L_h = kv_h.shape[1]
    last = torch.full((rows,), L_h - 1, dtype=torch.int32, device=device)
    n = dsa.sparse_mla_workspace_size(rows, L_h, wl.heads, wl.d_qk, wl.d_v, torch.bfloat16)
    hws = torch.empty(max(n, 1), dtype=torch.uint8, device=device)
    gh = _graph(lambda: dsa.hca_attention(inp["q"], kv_h, inp["row_batch"], last, wl.softmax_scale, wl.d_v,
                                          out=out, lse=lse, workspace=hws))
    for _ in range(3):
        gh.replay()
    st_h = time_graph(gh, steps, device, flush_read=evict)
    ms_h = max_over_ranks(st_h["median"], device)
    del gh
    h_bytes = rows * L_h * wl.d_qk * 2 + rows * wl.heads * (wl.d_qk + wl.d_v) * 2
    hca = {"workload": f"hca_decode_bf16_B4_L1048576_m{HCA_M}", "value": round(rows * world / (ms_h / 1e3), 1),
           "unit": "queries/s", "ms_per_step": round(ms_h, 4), "ms_stats": stats_json(st_h),
           "roofline": {"bound": "hbm", "achieved": round(h_bytes / (ms_h / 1e3) / 1e9, 1),
                        "peak": peaks["hbm_gbs"], "unit": "GB/s",
                        "frac": round(h_bytes / (ms_h / 1e3) / 1e9 / peaks["hbm_gbs"], 4),
                        "algorithmic_bytes": h_bytes},
           "l2": "256 MB buffer read between replays (the 38 MB pooled cache would stay in L2)"}
    if rank == 0 and world == 1 and args.cpu_baseline:
        import oracle
        kvh_h = kv_h.cpu()

        def hca_row(r):
            oracle.hca_attention(inp["q"][r:r + 1].cpu(), kvh_h[int(inp["row_batch"][r]):][:1],
                                 torch.zeros(1, dtype=torch.int32), last[r:r + 1].cpu(), wl.softmax_scale, wl.d_v)
        v, n, secs = _oracle_rows(hca_row, rows, 4.0)
        hca["cpu_baseline"] = {"value": round(v, 4), "unit": "queries/s", "cores": oracle.max_threads(),
                               "kind": "oracle", "sample": f"{n} whole query rows ({secs:.1f} s of CPU work)"}
        del kvh_h
    del kv_h, inp, out, lse, hws, evict
    torch.cuda.empty_cache()
    return {"csa_core_attention_decode": csa, "hca_decode": hca}


PREP_D_C, PREP_D_MODEL = 1536, 7168      # query latent and hidden size of a V3-class model


def run_prepare(dsa, workloads, device, peaks, args):
    """The step before the path: the indexer's queries, head weights and keys
    from the query latent and the hidden states (one dsa_indexer_prepare
    call: three projections, RMSNorm, rotary encoding, the key-cache write).

    decode: 64 new tokens (one per sequence of the 128K fp8-key decode), keys
      appended to the 64 x 131072-row fp8 cache.  Memory-bound: the roofline
      is the bytes that must cross HBM once (weights, activations, outputs)
      over the event time, with a 256 MB buffer read between replays (the
      30 MB of weights would otherwise stay in L2).
    prefill: 16384 tokens of one sequence (bf16 key cache), against the bf16
      tensor peak."""
    import torch
    rank, world, _ = dist_env()
    H, D, d_rope = 64, 128, 64
    evict = torch.ones(64 * 1024 * 1024, dtype=torch.float32, device=device)
    out = {}
    for name, T, fmt, rows_cache, max_pos in (
            (f"indexer_prepare_decode_T64_dc{PREP_D_C}_d{PREP_D_MODEL}_fp8cache", 64, "fp8", 64 * 131072, 131072),
            (f"indexer_prepare_prefill_T16384_dc{PREP_D_C}_d{PREP_D_MODEL}_bf16cache", 16384, "bf16", 16384, 16384)):
        shape = workloads.PrepareShape(T, PREP_D_C, PREP_D_MODEL, n_heads=H, head_dim=D, d_rope=d_rope,
                                       max_pos=max_pos, cache_rows=rows_cache)
        host_inp = workloads.make_prepare_inputs(shape, seed=300 + rank, skip=0.0)
        inp = {k: v.to(device) for k, v in host_inp.items()}
        if fmt == "fp8":
            cache = torch.zeros((rows_cache, D), dtype=torch.uint8, device=device)
            scale = torch.ones(rows_cache, dtype=torch.float32, device=device)
            seq = torch.arange(T, device=device, dtype=torch.int64)
            inp["pos"] = torch.full((T,), max_pos - 1, dtype=torch.int32, device=device)
            inp["slot"] = seq * 131072 + (max_pos - 1)         # each sequence's newest position
        else:
            cache = torch.zeros((rows_cache, D), dtype=torch.bfloat16, device=device)
            scale = None
            inp["pos"] = torch.arange(T, dtype=torch.int32, device=device)
            inp["slot"] = torch.arange(T, dtype=torch.int64, device=device)
        q_out = torch.empty((T, H, D), dtype=torch.bfloat16, device=device)
        w_out = torch.empty((T, H), dtype=torch.float32, device=device)
        ws = torch.empty(max(dsa.indexer_prepare_workspace_size(T, H, PREP_D_C, PREP_D_MODEL), 1), dtype=torch.uint8,
                         device=device)

        def call():
            dsa.indexer_prepare(inp["c_q"], inp["gamma"], inp["wq_b"], inp["h"], inp["wk"], inp["w_proj"],
                                inp["pos"], inp["slot"], cache, scale, inp["rope_cos"], inp["rope_sin"],
                                q_out=q_out, w_out=w_out, workspace=ws)

        n0 = dsa.launch_count()
        g = _graph(call)
        launches = (dsa.launch_count() - n0) // 2
        for _ in range(3):
            g.replay()
        steps = max(5, args.steps)
        st = time_graph(g, steps, device, flush_read=evict)
        ms = max_over_ranks(st["median"], device)
        del g
        dsa.get_device_error(device)
        w_bytes = (H * D * PREP_D_C + D * PREP_D_MODEL + H * PREP_D_MODEL) * 2 + PREP_D_C * 4
        a_bytes = T * (PREP_D_C + PREP_D_MODEL) * 2 + T * (4 + 8)
        o_bytes = T * H * D * 2 + T * H * 4 + T * (D + 4 if fmt == "fp8" else 2 * D)
        hbm = w_bytes + a_bytes + o_bytes
        flops = 2 * T * (H * D * PREP_D_C + (D + H) * PREP_D_MODEL)
        rec = {"workload": name, "value": round(T * world / (ms / 1e3), 1), "unit": "tokens/s",
               "ms_per_call": round(ms, 4), "ms_stats": stats_json(st), "gpu_launches": launches,
               "l2": "256 MB buffer read between replays"}
        if T <= 128:
            ach = hbm / (ms / 1e3) / 1e9
            rec["roofline"] = {"bound": "hbm", "achieved": round(ach, 1), "peak": peaks["hbm_gbs"], "unit": "GB/s",
                               "frac": round(ach / peaks["hbm_gbs"], 4), "algorithmic_bytes": hbm}
        else:
            ach = flops / (ms / 1e3) / 1e12
            rec["roofline"] = {"bound": "tensor", "achieved": round(ach, 1), "peak": peaks["bf16_tflops"],
                               "unit": "TFLOP/s", "frac": round(ach / peaks["bf16_tflops"], 4),
                               "algorithmic_flops": flops}
        if T <= 128 and rank == 0 and world == 1 and args.cpu_baseline:
            import oracle
            pos_h = inp["pos"].cpu().numpy()
            fmt = oracle.FP8 if scale is not None else oracle.BF16

            def prep_call(_):
                _, _, k64 = oracle.indexer_prepare(host_inp["c_q"], host_inp["gamma"], 1e-6, host_inp["wq_b"],
                                                   host_inp["h"], host_inp["wk"], host_inp["w_proj"],
                                                   host_inp["rope_cos"], host_inp["rope_sin"], pos_h, H, d_rope)
                oracle.key_rows_f32(k64.astype("float32"), pos_h, host_inp["rope_cos"], host_inp["rope_sin"], 0,
                                    fmt)
            v, n, secs = _oracle_rows(prep_call, 1, 3.0)
            rec["cpu_baseline"] = {"value": round(v * T, 2), "unit": "tokens/s", "cores": oracle.max_threads(),
                                   "kind": "oracle",
                                   "sample": f"{n} whole {T}-token calls ({secs:.1f} s of CPU work)"}
        out["decode" if T <= 128 else "prefill"] = rec
        del inp, cache, scale, q_out, w_out, ws
        torch.cuda.empty_cache()
    del evict
    torch.cuda.empty_cache()
    return out


def _finish():
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        dist.destroy_process_group()


# ------------------------------------------------------- reference arm ----

def run_reference(args):
    """The oracle (plain C, fp64) timed on the host cores on a bounded sample
    of the same workload: each step = whole query rows until ~budget s."""
    rank, world, _ = dist_env()
    if rank != 0:
        return
    import torch
    import workloads
    wl = workloads.BY_NAME[args.workload]
    # inputs drawn on the host: only the rows the sample touches are needed,
    # but the caches are drawn whole so the sample sees the same workload
    inp = workloads.generate(wl, device="cpu", seed=0)
    budget = max(2.0, 120.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        cpu_baseline_decode(wl, inp, budget_s=budget / 4)
    vals, secs, rows_done = [], 0.0, 0
    for _ in range(args.steps):
        qps, n, cores, s = cpu_baseline_decode(wl, inp, budget_s=budget)
        vals.append(qps)
        secs += s
        rows_done += n
    value = rows_done / secs
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": round(value, 4), "unit": "queries/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(1e3 * secs / args.steps, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": wl.name, "batch": wl.batch, "ctx": wl.ctx, "topk": wl.topk,
                   "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 4), "unit": "queries/s", "cores": cores, "kind": "oracle",
                         "sample": f"{rows_done} whole query rows over {args.steps} steps"},
        "e2e": {"value": round(value, 4), "unit": "queries/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="dsa_decode_bf16_B32_L32768_k2048")
    ap.add_argument("--no-prefill", dest="prefill", action="store_false")
    ap.add_argument("--no-v4", dest="v4", action="store_false")
    ap.add_argument("--no-prepare", dest="prepare", action="store_false")
    ap.add_argument("--no-other-decodes", dest="others", action="store_false")
    ap.add_argument("--no-compress", dest="compress", action="store_false")
    ap.add_argument("--no-tiny", dest="tiny", action="store_false")
    ap.add_argument("--no-cpu-baseline", dest="cpu_baseline", action="store_false")
    ap.add_argument("--prep-tokens", type=int, default=64, help="tokens of --kernel-only prepare")
    ap.add_argument("--prefill-tokens", type=int, default=0,
                    help="--kernel-only on the prefill workload: use a prompt of this many tokens")
    ap.add_argument("--kernel-only", choices=["indexer", "topk", "mla", "prepare"], default=None,
                    help="time one kernel of the step alone (for profiler captures)")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.kernel_only:
        run_kernel_only(args)
    elif args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
