"""Benchmark of the NVFP4 KV-cache hot path on B200: one step = quantise the new chunk's K/V
into its cache slot + attention of the query chunk over the sink + window chunks.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload 1.3b] [--impl ours|reference]

Prints one JSON line (rank 0).  ``value`` is attention TFLOP/s over the whole step
(quantise + attention, inputs resident in HBM); ``roofline`` reports the attention kernel
against the measured bf16 tensor peak, ``quantize`` the quantiser against measured HBM
bandwidth, ``e2e`` the same metric through the C ABI with host buffers and the copies in
the timed region, ``cpu_baseline`` the CPU oracle on a bounded sample.  With N > 1 (one
process per GPU under torchrun) every rank runs its own replica of the workload: the path
has no exchange step, so there is no collective in the timed region.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time

import numpy as np

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "NVFP4-KV chunk attention TFLOP/s and KV-quantize GB/s on 1 B200 (% roofline)"
ROTATE = 4  # input / cache / output sets cycled between steps (working set > L2)
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            d = json.load(f)
        return d, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def work(w):
    """Algorithmic FLOPs and bytes of one step (quantise + attn_calls attentions)."""
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
        sm, smax, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in out.splitlines():
            parts = [p.strip() for p in line.split(",")]
            if len(parts) != 7:
                continue
            try:
                sm.append(float(parts[0]))
                smax.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return None
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(smax), "reasons": sorted(reasons),
                "samples": len(sm)}


def oracle_sample(w, budget_s: float):
    """Time the CPU oracle on a bounded sample of the workload; extrapolate to one step."""
    import oracle
    from nvfp4_quantised_kv_b200 import synthetic
    oc = oracle.Cache(1, 1, w.head_dim, w.chunk_tokens, w.capacity)
    # quantise one head of the new chunk (K and V), then extrapolate to every head
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
    step_s = (t_quant_head * w.batch * w.heads
              + t_row * w.batch * w.heads * w.q_tokens * w.attn_calls)
    sample = (f"oracle: quantise 1 head of {len(w.visible_chunks)} chunks x {w.chunk_tokens} tokens, "
              f"attention of {rows_done} query rows x {w.visible_tokens} keys of 1 head; "
              f"extrapolated to {w.batch * w.heads} heads x {w.q_tokens} rows")
    return step_s, sample, t_quant_head + t_rows


def run_reference(args, w):
    """The reference arm: the CPU oracle as it stands, on bounded samples of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    attn_flops, _, _ = work(w)
    flops = attn_flops * w.attn_calls
    for _ in range(args.warmup):
        oracle_sample(w, args.ref_budget)
    times, sample, spent = [], "", 0.0
    for _ in range(args.steps):
        step_s, sample, used = oracle_sample(w, args.ref_budget)
        times.append(step_s)
        spent += used
    step_s = statistics.median(times)
    value = flops / step_s / 1e12
    line = {"impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": config_of(w),
            "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": 1, "kind": "oracle",
                             "sample": sample + " (median over steps; each step extrapolated)"},
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


def config_of(w):
    return {"workload": w.name, "batch": w.batch, "heads": w.heads, "head_dim": w.head_dim,
            "chunk_tokens": w.chunk_tokens, "q_tokens": w.q_tokens, "visible_keys": w.visible_tokens,
            "resident_chunks": w.capacity, "n_sink": w.n_sink, "window": w.window,
            "attention_calls_per_step": w.attn_calls,
            "l2": f"{ROTATE} rotating input/cache/output sets per GPU, each larger than a third of L2; "
                  "consecutive steps touch disjoint memory",
            "parallelism": "replicas"}


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=50)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default="1.3b")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--ref-budget", type=float, default=6.0, help="CPU seconds per reference step")
    ap.add_argument("--cpu-budget", type=float, default=15.0, help="CPU seconds for cpu_baseline")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    args = ap.parse_args()
    args.warmup = max(args.warmup, 3)

    from nvfp4_quantised_kv_b200 import synthetic
    w = synthetic.WORKLOADS[args.workload]
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

    # ---- resident inputs: ROTATE independent sets (cache, new K/V chunk, Q, output)
    def to_dev(bits):
        return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).to(dev).view(torch.bfloat16)

    sets = []
    hist = [c for c in w.visible_chunks if c != w.q_chunk]
    for s in range(ROTATE):
        ws = synthetic.Workload(**{**w.__dict__, "seed": replica_seed(w.seed, s, rank)})
        cache = nk.KVCache(w.batch, w.heads, w.chunk_tokens, w.capacity, q_tokens_max=w.q_tokens, device=dev)
        for slot in hist:
            k, v = synthetic.chunk_kv(ws, slot)
            cache.quantize(slot, to_dev(k), to_dev(v))
        k, v = synthetic.chunk_kv(ws, w.q_chunk)
        q = [to_dev(synthetic.queries(ws, step=i)) for i in range(w.attn_calls)]
        out = torch.empty(w.batch, w.q_tokens, w.heads, w.head_dim, dtype=torch.float32, device=dev)
        sets.append(dict(cache=cache, k=to_dev(k), v=to_dev(v), q=q, out=out, kh=k, vh=v,
                         qh=[synthetic.queries(ws, step=i) for i in range(w.attn_calls)]))
    torch.cuda.synchronize()
    stream = torch.cuda.current_stream()

    def step(i, ev=None):
        S = sets[i % ROTATE]
        if ev is not None:
            ev[0].record(stream)
        S["cache"].quantize(w.q_chunk, S["k"], S["v"])
        if ev is not None:
            ev[1].record(stream)
        for c in range(w.attn_calls):
            S["cache"].attention(S["q"][c], w.q_chunk, w.n_sink, w.window, out=S["out"])
        if ev is not None:
            ev[2].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    for S in sets:
        assert S["cache"].read_status() == 0, "device status set during warm-up"

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    start, end = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    clocks = ClockSampler(local) if rank == 0 else None
    if world > 1:
        dist.barrier()
    torch.cuda.synchronize()
    start.record(stream)
    for i in range(args.steps):
        step(i, evs[i])
    end.record(stream)
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    clk = clocks.stop() if clocks else None
    elapsed_ms = start.elapsed_time(end)
    t_quant = statistics.mean(e[0].elapsed_time(e[1]) for e in evs)
    t_attn = statistics.mean(e[1].elapsed_time(e[2]) for e in evs) / w.attn_calls
    elapsed_ms, t_quant, t_attn = max_over_ranks([elapsed_ms, t_quant, t_attn], dev)
    for S in sets:
        assert S["cache"].read_status() == 0, "device status set during the timed region"

    # ---- end to end through the C ABI with host buffers (pinned), copies inside the region
    S = sets[0]
    kh = torch.from_numpy(S["kh"].view(np.int16)).view(torch.bfloat16).pin_memory()
    vh = torch.from_numpy(S["vh"].view(np.int16)).view(torch.bfloat16).pin_memory()
    qh = [torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).pin_memory() for x in S["qh"]]
    oh = torch.empty(S["out"].shape, dtype=torch.float32).pin_memory()
    e2e_steps = max(3, min(args.steps, 20))

    def e2e_step():
        S["k"].copy_(kh, non_blocking=True)
        S["v"].copy_(vh, non_blocking=True)
        S["cache"].quantize(w.q_chunk, S["k"], S["v"])
        for c in range(w.attn_calls):
            S["q"][c].copy_(qh[c], non_blocking=True)
            S["cache"].attention(S["q"][c], w.q_chunk, w.n_sink, w.window, out=S["out"])
            oh.copy_(S["out"], non_blocking=True)

    for _ in range(2):
        e2e_step()
    torch.cuda.synchronize()
    if world > 1:
        dist.barrier()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    e1.record(stream)
    torch.cuda.synchronize()
    e2e_ms = e0.elapsed_time(e1) / e2e_steps
    (e2e_ms,) = max_over_ranks([e2e_ms], dev)
    if world > 1:
        dist.barrier()

    attn_flops, attn_bytes, quant_bytes = work(w)
    q_launches = sets[0]["cache"].quantize_launches()
    ms_per_step = elapsed_ms / args.steps
    step_flops = attn_flops * w.attn_calls
    value = whole_job_rate(step_flops, world, ms_per_step) / 1e12
    peaks, src = load_peaks()
    attn_tflops = attn_flops / (t_attn * 1e-3) / 1e12
    quant_gbs = quant_bytes / (t_quant * 1e-3) / 1e9
    h2d = kh.numel() * 2 + vh.numel() * 2 + sum(x.numel() * 2 for x in qh)
    d2h = oh.numel() * 4 * w.attn_calls
    traffic = None
    prof = os.path.join(ROOT, "profiles", f"traffic_{w.key}.json")
    if os.path.exists(prof):
        # the DRAM bytes of one ncu capture, valid only for the attention source they were taken on
        import hashlib
        with open(prof) as f:
            rec = json.load(f)
        with open(os.path.join(ROOT, "nvfp4_quantised_kv_b200", "csrc", "attention.cu"), "rb") as f:
            src_sha = hashlib.sha256(f.read()).hexdigest()
        if rec.get("attention_cu_sha256") == src_sha:
            traffic = rec.get("attention_dram_bytes_per_launch")

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": "TFLOP/s", "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms_per_step,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "fp16",
            "dtype_detail": "bf16 Q/K/V in; cache NVFP4 (E2M1 + E4M3 + fp32); QK^T and PV fp16 x fp16 "
                            "(exact conversions of the bf16 query and the dequantised K/V) on tcgen05 "
                            "with fp32 accumulate; fp32 output",
            "data": "synthetic (seeded N(0,1) with outlier channels; no dataset or weights)",
            "config": config_of(w),
            "roofline": {"bound": "tensor", "kernel": "attention_kernel", "achieved": attn_tflops,
                         "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                         "frac": attn_tflops / peaks["bf16_tflops"], "traffic": traffic,
                         "peak_source": f"{src} bf16 burst (cuBLAS 8192^3); fp16 has the same nominal tensor rate",
                         "algorithmic_flops_per_launch": attn_flops,
                         "algorithmic_bytes_per_launch": attn_bytes,
                         "algorithmic_hbm_gbs": attn_bytes / (t_attn * 1e-3) / 1e9,
                         "launch_us": t_attn * 1e3},
            "quantize": {"bound": "hbm",
                         "kernels": ("quantize_cluster_kernel" if q_launches == 1
                                     else "amax_kernel + quantize_kernel"),
                         "achieved": quant_gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                         "frac": quant_gbs / peaks["hbm_gbs"], "algorithmic_bytes_per_call": quant_bytes,
                         "call_us": t_quant * 1e3, "peak_source": f"{src} HBM copy"},
            "e2e": {"value": whole_job_rate(step_flops, world, e2e_ms) / 1e12, "unit": "TFLOP/s",
                    "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms},
            "gpu_launches": args.steps * (q_launches + w.attn_calls),
            "clocks": clk,
        }
        if world == 1 and not args.no_cpu_baseline:
            step_s, sample, _ = oracle_sample(w, args.cpu_budget)
            line["cpu_baseline"] = {"value": step_flops / step_s / 1e12, "unit": "TFLOP/s", "cores": 1,
                                    "kind": "oracle", "sample": sample}
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
