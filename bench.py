"""Benchmark of the NVFP4 KV-cache hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload rollout] [--impl ours|reference]

One step of the default workload is the long-rollout step t = 39 of a 30-layer, 12-head video
DiT: for every layer, quantise the new 3-frame chunk's K/V (4680 tokens) into chunk slot 39 of
that layer's 40-slot NVFP4 cache and run the chunk's 4680 queries against the 1 sink + 7 window
chunks (37440 keys).  The single-layer workloads (1.3B-class, 5B-class, few-step decode) are
timed in the same run and reported as sub-records of the JSON line (``workloads``).

Prints one JSON line (rank 0).  ``value`` is attention TFLOP/s over the whole step (quantise +
attention, inputs resident in HBM); ``roofline`` reports the attention call against the measured
bf16 tensor peak, ``quantize`` the quantiser against measured HBM bandwidth, ``footprint`` the
resident NVFP4 cache against a bf16 cache of the same shape (both allocated), ``e2e`` the same
metric through the public API with the step's inputs copied from pinned host memory and its
outputs copied back inside the timed region, ``cpu_baseline`` the CPU oracle on a bounded sample.
With N > 1 (one process per GPU under torchrun) every rank runs its own replica of the workload:
the path has no exchange step, so there is no collective in the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import platform
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4-KV chunk attention TFLOP/s and KV-quantize GB/s on 1 B200 (% roofline)"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
SUB_WORKLOADS = ("1.3b", "5b", "fewstep")


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def cpu_model() -> str:
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return platform.processor() or "unknown"


def work(w):
    """Algorithmic FLOPs and bytes of one layer: one attention call and one quantise call."""
    d = w.head_dim
    lk = w.visible_tokens
    attn_flops = 4.0 * w.batch * w.heads * w.q_tokens * lk * d
    per_key = d // 2 + d // 16  # code + scale bytes per token, head and tensor
    attn_bytes = (w.batch * w.q_tokens * w.heads * d * 2            # Q bf16
                  + w.batch * w.q_tokens * w.heads * d * 4          # O fp32
                  + 2 * w.batch * w.heads * lk * per_key            # K and V codes + scales
                  + 2 * w.batch * w.heads * len(w.visible_chunks) * 4)  # FP32 scales
    n = w.batch * w.chunk_tokens * w.heads
    quant_bytes = 2 * (n * d * 2 + n * per_key + w.batch * w.heads * 4)
    return attn_flops, attn_bytes, quant_bytes


class ClockSampler:
    """nvidia-smi clock / throttle sampling while the timed region runs."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.proc = None
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            time.sleep(0.3)
        except OSError:
            self.proc = None

    def stop(self):
        if self.proc is None:
            return None
        time.sleep(0.2)
        self.proc.terminate()
        try:
            out, _ = self.proc.communicate(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
            out, _ = self.proc.communicate()
        sm, smax, power, reasons = [], [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
                power.append(float(parts[2]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "power_w_max": max(power) if power else None, "samples": len(sm)}


def oracle_sample(w, budget_s: float):
    """Time the CPU oracle on a bounded sample of one layer of the workload (one head: quantise the
    visible chunks, then attention rows until the budget is spent).  Returns the measured sample
    (its FLOPs and seconds) and the per-step time extrapolated to the whole workload."""
    import oracle
    from nvfp4_quantised_kv_b200 import synthetic
    oc = oracle.Cache(1, 1, w.head_dim, w.chunk_tokens, w.capacity)
    k, v = synthetic.chunk_kv(w, w.q_chunk)
    k1, v1 = np.ascontiguousarray(k[:1, :, :1]), np.ascontiguousarray(v[:1, :, :1])
    t0 = time.perf_counter()
    for slot in w.visible_chunks:
        oc.append(slot, k1, v1)
    t_quant_head = (time.perf_counter() - t0) / len(w.visible_chunks)
    q = np.ascontiguousarray(synthetic.queries(w)[:1, :, :1])
    rows_done, t_rows = 0, 0.0
    n = 8
    while t_rows < budget_s and rows_done < w.q_tokens:
        rows = np.array([(0, 0, (rows_done + i) % w.q_tokens) for i in range(n)], np.int32)
        t0 = time.perf_counter()
        oracle.attention_rows(q, oc, w.q_chunk, w.n_sink, w.window, rows)
        t_rows += time.perf_counter() - t0
        rows_done += n
        n = min(2 * n, 256)
    t_row = t_rows / rows_done
    step_s = w.layers * (t_quant_head * w.batch * w.heads
                         + t_row * w.batch * w.heads * w.q_tokens * w.attn_calls)
    sample_flops = 4.0 * rows_done * w.visible_tokens * w.head_dim
    sample = (f"oracle on 1 core of {cpu_model()}: quantise 1 head of {len(w.visible_chunks)} chunks x "
              f"{w.chunk_tokens} tokens, attention of {rows_done} query rows x {w.visible_tokens} keys of "
              f"1 head; extrapolated to {w.layers} layer(s) x {w.batch * w.heads} heads x {w.q_tokens} rows"
              f" x {w.attn_calls} call(s)")
    return {"step_s_extrapolated": step_s, "sample": sample, "sample_flops": sample_flops,
            "sample_attn_s": t_rows, "sample_s": t_quant_head * len(w.visible_chunks) + t_rows}


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands, on a bounded sample of the workload per
    step.  The line reports what was timed: the sample's attention FLOPs over its time."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    for _ in range(args.warmup):
        oracle_sample(w, args.ref_budget / 4)
    recs = [oracle_sample(w, args.ref_budget) for _ in range(args.steps)]
    flops = sum(r["sample_flops"] for r in recs)
    attn_s = sum(r["sample_attn_s"] for r in recs)
    value = flops / attn_s / 1e12
    ms_per_step = 1e3 * statistics.mean(r["sample_s"] for r in recs)
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "extrapolated_ms_per_full_step": 1e3 * statistics.median(r["step_s_extrapolated"] for r in recs),
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": recs[-1]["sample"] + " (each step times one such sample)"},
            "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line), flush=True)


def max_over_ranks(values, device):
    """Element-wise max of per-rank timings over all ranks (identity on one process): a
    multi-GPU number is the slowest rank's."""
    import torch
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return list(values)
    t = torch.tensor(list(values), device=device, dtype=torch.float64)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.tolist()


def whole_job_rate(units_per_rank, world, ms_per_step):
    """Whole-job throughput: the units all ranks processed per second of the slowest rank."""
    return units_per_rank * world / (ms_per_step * 1e-3)


def replica_seed(seed, rotation, rank):
    """Seed of one rotating input set of one rank: every replica draws its own inputs."""
    return seed + 1000 * rotation + 7919 * rank


def n_sets(w):
    """Input sets cycled between steps so consecutive steps touch disjoint memory (> L2): four
    rotating sets for one layer; the 30-layer step already touches ~3 GB."""
    return 1 if w.layers > 1 else 4


def config_of(w):
    return {"workload": w.name, "layers": w.layers, "batch": w.batch, "heads": w.heads,
            "head_dim": w.head_dim, "chunk_tokens": w.chunk_tokens, "q_tokens": w.q_tokens,
            "visible_keys": w.visible_tokens, "resident_chunks": w.capacity, "n_sink": w.n_sink,
            "window": w.window, "attention_calls_per_step": w.attn_calls,
            "l2": ("one step touches every layer's cache and inputs (~3.3 GB, far above L2)" if w.layers > 1 else
                   f"{n_sets(w)} rotating input/cache/output sets per GPU, each larger than a third of L2; "
                   "consecutive steps touch disjoint memory"),
            "parallelism": "replicas"}


class Runner:
    """Caches, inputs and outputs of one workload on one GPU, and its timed step."""

    def __init__(self, w, dev, rank, ws, recipe=False):
        import torch
        import nvfp4_quantised_kv_b200 as nk
        from nvfp4_quantised_kv_b200 import synthetic
        self.w, self.dev = w, dev
        self.stream = torch.cuda.current_stream(dev)
        hist = [c for c in w.visible_chunks if c != w.q_chunk]
        self.sets = []
        base = torch.cuda.memory_allocated(dev)
        for s in range(n_sets(w)):
            ws_w = synthetic.Workload(**{**w.__dict__, "seed": replica_seed(w.seed, s, rank)})
            layers = []
            for layer in range(w.layers):
                cache = nk.KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, q_tokens_max=w.q_tokens,
                                   device=dev, workspace=ws, smooth_k=recipe, adaptive_v=recipe)
                for slot in hist:
                    k, v = synthetic.device_chunk_kv(ws_w, slot, layer, dev)
                    cache.quantize(slot, k, v)
                k, v = synthetic.device_chunk_kv(ws_w, w.q_chunk, layer, dev)
                q = [synthetic.device_queries(ws_w, layer, step, dev) for step in range(w.attn_calls)]
                out = torch.empty(w.batch, w.q_tokens, w.heads, w.head_dim, dtype=torch.float32, device=dev)
                layers.append(dict(cache=cache, k=k, v=v, q=q, out=out))
            self.sets.append(layers)
        # the multi-layer step quantises all layers' new chunks with one launch
        self.batched = w.layers > 1 and not recipe
        self.qws = None
        if self.batched:
            S = self.sets[0]
            self.qws = nk.quantize_layers([L["cache"] for L in S], w.q_chunk, [L["k"] for L in S],
                                          [L["v"] for L in S])
        torch.cuda.synchronize(dev)
        self.alloc_bytes = torch.cuda.memory_allocated(dev) - base
        self.cache_bytes = sum(L["cache"].nbytes for S in self.sets for L in S) // len(self.sets)

    def step(self, i, ev=None):
        """One step.  ``ev`` (optional): a dict that collects (start, end) CUDA events of the
        quantiser calls ("q") and of each layer's attention calls ("a")."""
        import torch
        import nvfp4_quantised_kv_b200 as nk
        w = self.w
        S = self.sets[i % len(self.sets)]

        def mark():
            e = torch.cuda.Event(enable_timing=True)
            e.record(self.stream)
            return e

        if self.batched:  # every layer's new chunk in one launch
            e0 = mark() if ev is not None else None
            nk.quantize_layers([L["cache"] for L in S], w.q_chunk, [L["k"] for L in S], [L["v"] for L in S],
                               workspace=self.qws)
            if ev is not None:
                ev["q"].append((e0, mark()))
        for L in S:
            if not self.batched:
                e0 = mark() if ev is not None else None
                L["cache"].quantize(w.q_chunk, L["k"], L["v"])
                if ev is not None:
                    ev["q"].append((e0, mark()))
            e0 = mark() if ev is not None else None
            for c in range(w.attn_calls):
                L["cache"].attention(L["q"][c], w.q_chunk, w.n_sink, w.window, out=L["out"])
            if ev is not None:
                ev["a"].append((e0, mark()))

    def check_status(self, what):
        for S in self.sets:
            for L in S:
                assert L["cache"].read_status() == 0, f"device status set during {what}"

    def timed(self, steps, warmup, world, sample_clocks, local):
        import torch
        import torch.distributed as dist
        for i in range(warmup):
            self.step(i)
        torch.cuda.synchronize(self.dev)
        self.check_status("warm-up")
        evs = [{"q": [], "a": []} for _ in range(steps)]
        start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks = ClockSampler(local) if sample_clocks else None
        if world > 1:
            dist.barrier()
        torch.cuda.synchronize(self.dev)
        start.record(self.stream)
        for i in range(steps):
            self.step(i, evs[i])
        end.record(self.stream)
        torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        clk = clocks.stop() if clocks else None
        elapsed = start.elapsed_time(end)
        # quantiser time per step (all layers) and attention time per call
        t_quant = statistics.mean(sum(a.elapsed_time(b) for a, b in e["q"]) for e in evs)
        t_attn = statistics.mean(a.elapsed_time(b) for e in evs for a, b in e["a"]) / self.w.attn_calls
        self.check_status("the timed region")
        return elapsed / steps, t_quant, t_attn, clk

    def graph_replay(self, steps):
        """The same step captured once in a CUDA graph and replayed: every launch of the step (the
        quantiser's memset and kernel, each layer's attention and merge kernels) is one graph; the
        time per replay has no host launch cost in it.  Returns ms per step, or an error string."""
        import torch
        try:
            g = torch.cuda.CUDAGraph()
            side = torch.cuda.Stream(self.dev)
            side.wait_stream(self.stream)
            with torch.cuda.stream(side):
                self.step(0)  # warm the side stream once outside the capture
            torch.cuda.synchronize(self.dev)
            with torch.cuda.graph(g, stream=side, capture_error_mode="thread_local"):
                self.step(0)
            torch.cuda.synchronize(self.dev)
            for _ in range(2):
                g.replay()
            torch.cuda.synchronize(self.dev)
            e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            cur = torch.cuda.current_stream(self.dev)
            e0.record(cur)
            for _ in range(steps):
                g.replay()
            e1.record(cur)
            torch.cuda.synchronize(self.dev)
            self.check_status("the graph replays")
            ms = e0.elapsed_time(e1) / steps
            del g
            return ms
        except Exception as exc:  # reported, not fatal: the stream-timed numbers stand
            return f"{type(exc).__name__}: {exc}"

    def e2e(self, steps, world):
        """The step through the public API with inputs from pinned host memory and outputs back to
        pinned host memory inside the timed region.  An upload stream moves every layer's K and V in
        first (the quantiser needs all of them), then the queries layer by layer; a download stream
        moves each layer's output out as soon as its attention is done; the compute stream runs the
        quantiser and the layers in order.  A buffer is refilled only after the step that read it is
        done with it."""
        import torch
        import torch.distributed as dist
        import nvfp4_quantised_kv_b200 as nk
        w = self.w
        S = self.sets[0]
        L0 = S[0]
        pin = lambda t: t.cpu().pin_memory()
        kh, vh = pin(L0["k"]), pin(L0["v"])
        qh = [pin(x) for x in L0["q"]]
        oh = torch.empty(L0["out"].shape, dtype=torch.float32).pin_memory()
        comp, up, down = self.stream, torch.cuda.Stream(self.dev), torch.cuda.Stream(self.dev)
        n = len(S)
        kv_ready = [torch.cuda.Event() for _ in range(n)]
        q_ready = [torch.cuda.Event() for _ in range(n)]
        kv_consumed = [torch.cuda.Event() for _ in range(n)]
        q_consumed = [torch.cuda.Event() for _ in range(n)]
        out_ready = [[torch.cuda.Event() for _ in range(w.attn_calls)] for _ in range(n)]
        out_read = [[torch.cuda.Event() for _ in range(w.attn_calls)] for _ in range(n)]
        for li in range(n):
            kv_consumed[li].record(comp)
            q_consumed[li].record(comp)
            for c in range(w.attn_calls):
                out_read[li][c].record(down)

        def one_step():
            with torch.cuda.stream(up):
                for li, L in enumerate(S):
                    up.wait_event(kv_consumed[li])
                    L["k"].copy_(kh, non_blocking=True)
                    L["v"].copy_(vh, non_blocking=True)
                    kv_ready[li].record(up)
                for li, L in enumerate(S):
                    up.wait_event(q_consumed[li])
                    for c in range(w.attn_calls):
                        L["q"][c].copy_(qh[c], non_blocking=True)
                    q_ready[li].record(up)
            if self.batched:
                for li in range(n):
                    comp.wait_event(kv_ready[li])
                nk.quantize_layers([L["cache"] for L in S], w.q_chunk, [L["k"] for L in S], [L["v"] for L in S],
                                   workspace=self.qws, stream=comp)
                for li in range(n):
                    kv_consumed[li].record(comp)
            for li, L in enumerate(S):
                if not self.batched:
                    comp.wait_event(kv_ready[li])
                    L["cache"].quantize(w.q_chunk, L["k"], L["v"], stream=comp)
                    kv_consumed[li].record(comp)
                comp.wait_event(q_ready[li])
                for c in range(w.attn_calls):
                    comp.wait_event(out_read[li][c])
                    L["cache"].attention(L["q"][c], w.q_chunk, w.n_sink, w.window, out=L["out"], stream=comp)
                    out_ready[li][c].record(comp)
                    with torch.cuda.stream(down):
                        down.wait_event(out_ready[li][c])
                        oh.copy_(L["out"], non_blocking=True)
                        out_read[li][c].record(down)
                q_consumed[li].record(comp)

        for _ in range(2):
            one_step()
        torch.cuda.synchronize(self.dev)
        if world > 1:
            dist.barrier()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record(comp)
        for _ in range(steps):
            one_step()
        comp.wait_stream(up)
        comp.wait_stream(down)
        e1.record(comp)
        torch.cuda.synchronize(self.dev)
        h2d = n * (kh.numel() * 2 + vh.numel() * 2 + sum(x.numel() * 2 for x in qh))
        d2h = n * oh.numel() * 4 * w.attn_calls
        return e0.elapsed_time(e1) / steps, h2d, d2h


def attention_kernels_per_call(w):
    import ctypes
    import nvfp4_quantised_kv_b200 as nk
    d = nk.CacheDesc(w.batch, w.heads, w.head_dim, w.chunk_tokens, w.capacity, 16, 16, 16, 16, 16, 16, 16)
    tiles = 0
    # tiles per run of consecutive visible chunks
    vis = w.visible_chunks
    i = 0
    while i < len(vis):
        k = i
        while k + 1 < len(vis) and vis[k + 1] == vis[k] + 1:
            k += 1
        tiles += -(-((k - i + 1) * w.chunk_tokens) // 128)
        i = k + 1
    out = nk.attention_plan(d, w.q_tokens, tiles)
    return out[1], out[0]


def measure(w, args, dev, rank, world, local, ws, peaks, src, headline, recipe=False):
    import nvfp4_quantised_kv_b200 as nk  # noqa: F401
    r = Runner(w, dev, rank, ws, recipe)
    steps = args.steps if headline else max(5, args.steps // 2)
    ms, t_quant, t_attn, clk = r.timed(steps, args.warmup, world, headline and rank == 0, local)
    ms, t_quant, t_attn = max_over_ranks([ms, t_quant, t_attn], dev)
    attn_flops, attn_bytes, quant_bytes = work(w)
    step_flops = attn_flops * w.attn_calls * w.layers
    attn_tflops = attn_flops / (t_attn * 1e-3) / 1e12
    quant_gbs = w.layers * quant_bytes / (t_quant * 1e-3) / 1e9  # t_quant: all layers of a step
    q_launches = 1 if r.batched else r.sets[0][0]["cache"].quantize_launches()
    a_kernels, a_ctas = attention_kernels_per_call(w)
    rec = {
        "workload": w.name, "ms_per_step": ms,
        "value": whole_job_rate(step_flops, world, ms) / 1e12, "unit": "TFLOP/s",
        "attention": {"bound": "tensor", "achieved": attn_tflops, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                      "frac": attn_tflops / peaks["bf16_tflops"], "launch_us": t_attn * 1e3,
                      "kernels_per_call": a_kernels, "ctas": a_ctas,
                      "algorithmic_flops_per_call": attn_flops, "algorithmic_bytes_per_call": attn_bytes,
                      "algorithmic_hbm_gbs": attn_bytes / (t_attn * 1e-3) / 1e9},
        "quantize": {"bound": "hbm", "achieved": quant_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": quant_gbs / peaks["hbm_gbs"], "us_per_step": t_quant * 1e3,
                     "layers_per_launch": w.layers if r.batched else 1,
                     "kernels": ("quantize_ticket_kernel (one launch for all layers, after a counter memset)"
                                 if r.batched else
                                 "key_mean_kernel + recipe_amax_kernel + recipe_encode_kernel" if recipe else
                                 "quantize_cluster_kernel" if q_launches == 1 else "amax_kernel + quantize_kernel"),
                     "algorithmic_bytes_per_step": w.layers * quant_bytes},
        "gpu_launches_per_step": (q_launches if r.batched else w.layers * q_launches) + w.layers * w.attn_calls * a_kernels,
    }
    if w.key == "fewstep":
        # memory-bound by the metric's name, tensor-bound by the roofline: both fractions
        t_bytes = attn_bytes / (peaks["hbm_gbs"] * 1e9)
        t_flops = attn_flops / (peaks["bf16_tflops"] * 1e12)
        rec["attention"]["roofline_frac_max_bytes_flops"] = max(t_bytes, t_flops) / (t_attn * 1e-3)
        rec["attention"]["hbm_frac"] = attn_bytes / (t_attn * 1e-3) / (peaks["hbm_gbs"] * 1e9)
    return r, rec, clk, steps


def traffic_for(key, kind="attention"):
    """DRAM bytes from the last ncu capture of this workload: per attention launch, or per layer of
    the multi-layer quantiser launch (``kind="quantize"``); valid only for the source file they were
    taken on (null otherwise)."""
    import hashlib
    prof = os.path.join(ROOT, "profiles", f"traffic_{key}.json")
    if not os.path.exists(prof):
        return None
    with open(prof) as f:
        rec = json.load(f)
    src = "attention.cu" if kind == "attention" else "quantize.cu"
    with open(os.path.join(ROOT, "nvfp4_quantised_kv_b200", "csrc", src), "rb") as f:
        src_sha = hashlib.sha256(f.read()).hexdigest()
    if rec.get(f"{kind}_cu_sha256") != src_sha:
        return None
    return rec.get("attention_dram_bytes_per_launch" if kind == "attention" else "quantize_dram_bytes_per_layer")


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--workload", default="rollout")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget", type=float, default=4.0, help="CPU seconds per reference step")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="CPU seconds for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-sub", action="store_true", help="skip the single-layer sub-records")
    ap.add_argument("--layers", type=int, default=0,
                    help="layers of a multi-layer workload (default: the workload's own count); a "
                         "smaller count runs the same per-layer launches on less device memory")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from nvfp4_quantised_kv_b200 import synthetic
    w = synthetic.WORKLOADS[args.workload]
    if args.layers and args.layers != w.layers:
        if w.layers == 1:
            ap.error("--layers applies to a multi-layer workload")
        w = synthetic.with_layers(w, args.layers)
    if args.impl == "reference":
        return run_reference(args, w)

    import torch
    import torch.distributed as dist
    import nvfp4_quantised_kv_b200 as nk

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        torch.cuda.set_device(local)
        from datetime import timedelta
        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    nk.lib()
    peaks, src = load_peaks()
    # one scratch buffer for every cache of this process (calls run one at a time on one stream)
    ws_bytes = max(nk.workspace_bytes(x.batch, x.heads, x.chunk_tokens, x.capacity, x.q_tokens)
                   for x in synthetic.WORKLOADS.values())
    ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)

    # footprint of the resident caches: NVFP4 as allocated, against a bf16 K/V cache of the same shape
    footprint = None
    if w.layers > 1:
        torch.cuda.synchronize(dev)
        b0 = torch.cuda.memory_allocated(dev)
        bf16 = torch.empty(w.layers, 2, w.batch, w.capacity * w.chunk_tokens, w.heads, w.head_dim,
                           dtype=torch.bfloat16, device=dev)
        bf16_bytes = torch.cuda.memory_allocated(dev) - b0
        del bf16
        torch.cuda.empty_cache()

    runner, rec, clk, steps = measure(w, args, dev, rank, world, local, ws, peaks, src, headline=True)
    if w.layers > 1:
        footprint = {"nvfp4_cache_bytes": runner.cache_bytes, "bf16_cache_bytes": bf16_bytes,
                     "ratio": bf16_bytes / runner.cache_bytes,
                     "scope": f"{w.layers} layers x {w.capacity} chunks x {w.chunk_tokens} tokens x {w.heads} heads,"
                              " K and V, all slots resident; both allocated on the device"}
    e2e_steps = max(3, min(steps, 10))
    e2e_ms, h2d, d2h = runner.e2e(e2e_steps, world)
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)
    graph_ms = runner.graph_replay(e2e_steps)
    if not isinstance(graph_ms, str):
        (graph_ms,) = max_over_ranks([graph_ms], dev)
    del runner
    torch.cuda.empty_cache()

    subs = {}
    if not args.no_sub and args.workload == "rollout":
        for key in SUB_WORKLOADS:
            r2, rec2, _, _ = measure(synthetic.WORKLOADS[key], args, dev, rank, world, local, ws, peaks, src,
                                     headline=False)
            rec2["attention"]["traffic"] = traffic_for(key)
            subs[key] = rec2
            del r2
            torch.cuda.empty_cache()
        # the pages' recipe options (K-smoothing of K, adaptive {4, 6} scales of V) on the 1.3B layer
        r2, rec2, _, _ = measure(synthetic.WORKLOADS["1.3b"], args, dev, rank, world, local, ws, peaks, src,
                                 headline=False, recipe=True)
        rec2["options"] = "K_SMOOTH | V_ADAPTIVE_SCALE"
        subs["1.3b+recipe"] = rec2
        del r2
        torch.cuda.empty_cache()

    if rank == 0:
        attn = rec["attention"]
        step_flops = work(w)[0] * w.attn_calls * w.layers
        line = {
            "metric": METRIC, "value": rec["value"], "unit": "TFLOP/s", "n_gpus": world,
            "steps": steps, "warmup": args.warmup, "ms_per_step": rec["ms_per_step"],
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
            "dtype_detail": "bf16 Q/K/V in; cache NVFP4 (E2M1 + E4M3 + fp32); QK^T and PV fp16 x fp16 "
                            "(exact conversions of the bf16 query and the dequantised K/V) on tcgen05 "
                            "with fp32 accumulate; fp32 output",
            "data": "synthetic (seeded N(0,1) with outlier channels, drawn on the GPU; no dataset or weights)",
            "config": config_of(w),
            "roofline": {"bound": "tensor", "kernel": "attention call (attention_kernel + combine_kernel)",
                         "achieved": attn["achieved"], "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": attn["frac"], "traffic": traffic_for(w.key),
                         "peak_source": f"{src} bf16 burst (cuBLAS 8192^3); fp16 has the same nominal tensor rate",
                         "algorithmic_flops_per_launch": attn["algorithmic_flops_per_call"],
                         "algorithmic_bytes_per_launch": attn["algorithmic_bytes_per_call"],
                         "algorithmic_hbm_gbs": attn["algorithmic_hbm_gbs"], "launch_us": attn["launch_us"],
                         "ctas": attn["ctas"], "kernels_per_call": attn["kernels_per_call"]},
            "quantize": {**rec["quantize"], "peak_source": f"{src} HBM copy",
                         "traffic": (None if traffic_for(w.key, "quantize") is None or rec["quantize"]["layers_per_launch"] == 1
                                     else traffic_for(w.key, "quantize") * w.layers)},
            "footprint": footprint,
            "e2e": {"value": whole_job_rate(step_flops, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms,
                    "how": "public API; an upload stream moves all layers' K/V in, then each layer's queries; a "
                           "download stream moves each layer's output out after its attention; the compute "
                           "stream runs the quantiser and the layers"},
            "graph": ({"ms_per_step": graph_ms, "value": whole_job_rate(step_flops, world, graph_ms) / 1e12,
                       "unit": "TFLOP/s", "steps": e2e_steps,
                       "how": "one step captured in a CUDA graph (inputs resident in HBM), replayed"}
                      if not isinstance(graph_ms, str) else {"error": graph_ms}),
            "gpu_launches": steps * rec["gpu_launches_per_step"],
            "clocks": clk,
            "workloads": subs,
        }
        if world == 1 and not args.no_cpu_baseline:
            o = oracle_sample(w, args.cpu_budget)
            line["cpu_baseline"] = {"value": step_flops / o["step_s_extrapolated"] / 1e12, "unit": "TFLOP/s",
                                    "cores": 1, "kind": "oracle", "sample": o["sample"],
                                    "measured_sample_tflops": o["sample_flops"] / o["sample_attn_s"] / 1e12}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
