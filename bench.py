#!/usr/bin/env python
"""Benchmark of the LCSA hot path: one streaming chunk of one DiT attention layer.

A step is one pass of the whole hot path over one 8-frame chunk (2 latent
frames): cache append (k/v into the ring + k block means), draft mask (q
block means, fp32 scores over the allowed blocks, top-k) and block-sparse
attention over the kept 128x128 tiles.  Default workload: 768x1408,
12 heads x 128 dims, 66 query blocks, 3 cached block-layers (264 key
blocks), local range 11, topk 20.

Prints one JSON line.  ``value`` is the effective throughput in TFLOP/s
counted over kept tiles only (4 * 128^3 flops per tile); ``ms_per_step`` is
ms per chunk.  ``--impl reference`` times the fp64 CPU oracle on a bounded
sample of the same workload (rank 0 only).

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica of the layer (LCSA rows are independent, there is no exchange step),
so the scaling is weak and the barrier/max reduction is the only collective.
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

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from diffusion_vsr_b200 import workloads as W  # noqa: E402

METRIC = "LCSA ms per 8-frame chunk & effective TFLOP/s at 768×1408; % bf16 tensor peak"
PEAKS_FILE = os.path.join(ROOT, "MEASURED_PEAKS.json")
TRAFFIC_FILE = os.path.join(ROOT, "profiles", "traffic.json")
FALLBACK_BF16_TFLOPS = 1590.0
FALLBACK_HBM_GBS = 6650.0


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lcsa", choices=["lcsa", "reference"])
    ap.add_argument("--workload", default="768x1408", choices=sorted(W.WORKLOADS))
    ap.add_argument("--topk", type=int, default=0, help="override the workload's topk")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args()


def workload(args) -> W.Workload:
    w = W.WORKLOADS[args.workload]
    return w.with_topk(args.topk) if args.topk else w


def peaks():
    if os.path.exists(PEAKS_FILE):
        with open(PEAKS_FILE) as f:
            d = json.load(f)
        return {"bf16_tflops": d["bf16_tflops"], "bf16_tflops_sustained": d.get("bf16_tflops_sustained"),
                "hbm_gbs": d["hbm_gbs"], "source": "measured"}
    return {"bf16_tflops": FALLBACK_BF16_TFLOPS, "bf16_tflops_sustained": None, "hbm_gbs": FALLBACK_HBM_GBS,
            "source": "fallback"}


def source_sha(name: str) -> str:
    with open(os.path.join(ROOT, "diffusion_vsr_b200", "csrc", name), "rb") as f:
        return hashlib.sha256(f.read()).hexdigest()[:16]


def traffic_for(kernel_src: str, workload_name: str):
    """DRAM bytes per launch from a committed ncu capture, if the kernel is unchanged."""
    if not os.path.exists(TRAFFIC_FILE):
        return None
    with open(TRAFFIC_FILE) as f:
        d = json.load(f)
    e = d.get(kernel_src, {}).get(workload_name)
    if not e or e.get("source_sha") != source_sha(kernel_src):
        return None
    return e.get("dram_bytes_per_launch")


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.lines = []

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except OSError:
            self.proc = None
        time.sleep(0.3)
        return self

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.15)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
        return False

    def summary(self):
        sm, mx, reasons = [], None, set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 8:
                continue
            try:
                sm.append(float(parts[0]))
                mx = float(parts[1])
            except ValueError:
                continue
            for n, v in zip(names, parts[4:8]):
                if v.lower() == "active":
                    reasons.add(n)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": mx, "reasons": sorted(reasons), "samples": len(sm)}


def max_over_ranks(x: float, device) -> float:
    """Largest value of ``x`` over all ranks (identity without a process group)."""
    if not (torch.distributed.is_available() and torch.distributed.is_initialized()):
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    torch.distributed.all_reduce(t, op=torch.distributed.ReduceOp.MAX)
    return float(t.item())


def aggregate_tflops(world: int, flops_per_rank_step: float, ms_per_step: float) -> float:
    """Whole-job throughput: every rank's work divided by the slowest rank's time."""
    return world * flops_per_rank_step / (ms_per_step * 1e-3) / 1e12


# ------------------------------------------------------------------ GPU arm

def run_lcsa(args, rank: int, world: int, local_rank: int):
    from diffusion_vsr_b200 import lcsa as L

    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    w = workload(args)
    flop_tile = W.flops_per_tile()
    prefill, steps = W.stream_plan(w)
    # distinct chunk buffers rotated across steps: per-step inputs (q, k, v) plus the
    # 4-layer ring are larger than the 126 MB L2, so no step starts warm
    n_bufs = max(4, min(8, len(steps)))
    positions = [w.kv_len + (i % len(steps)) for i in range(n_bufs)]
    host = [W.gen_layers(w, p, w.q_layers) for p in positions]
    chunks = [[t.to(dev) for t in c] for c in host]
    layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, w.local_range, w.local_mode,
                        device=dev)
    for p in prefill:
        _, k, v = W.gen_layers(w, p, 1, "kv")
        layer.append(k.to(dev), v.to(dev))
    out = torch.empty_like(chunks[0][0])
    stream = torch.cuda.current_stream(dev)

    def step(i):
        # the library's streaming step, chained: the append runs in the SMs the
        # previous step's attention leaves idle, the draft and the attention each
        # start as the kernel before them finishes (programmatic dependent launch)
        q, k, v = chunks[i % n_bufs]
        layer.step(q, k, v, out, overlap_previous=True)

    def step_split(i, ev):
        # the same three calls without programmatic dependence, with events between
        # them: per-kernel times for the roofline
        q, k, v = chunks[i % n_bufs]
        ev[0].record(stream)
        L.lcsa_cache_append(layer.cache, k, v, d_status=layer.status)
        ev[1].record(stream)
        L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status)
        ev[2].record(stream)
        L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, out, d_status=layer.status)
        ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    kept_tiles = int(layer.kept_cnt.sum().item())
    dist = world > 1
    if dist:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        torch.cuda.synchronize()
        t0.record(stream)
        for i in range(args.steps):
            step(args.warmup + i)
        t1.record(stream)
        torch.cuda.synchronize()
    if dist:
        torch.distributed.barrier()
    total_ms = t0.elapsed_time(t1)
    # per-kernel pass (not part of the headline time)
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    for i in range(args.steps):
        step_split(args.warmup + args.steps + i, evs[i])
    torch.cuda.synchronize()
    status = int(layer.status.item())
    if status != 0:
        raise RuntimeError(f"device status {L.status_string(status)}")
    t_append = [e[0].elapsed_time(e[1]) for e in evs]
    t_draft = [e[1].elapsed_time(e[2]) for e in evs]
    t_attn = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = max_over_ranks(total_ms, dev)
    ms_step = total_ms / args.steps
    step_flops = kept_tiles * flop_tile
    value = aggregate_tflops(world, step_flops, ms_step)

    pk = peaks()
    attn_ms = statistics.mean(t_attn)  # the roofline uses the average launch time
    attn_tflops = step_flops / (attn_ms * 1e-3) / 1e12
    H, Nq, nblk = w.heads, w.n_query_blocks, w.blocks_per_layer
    q_bytes = H * Nq * 128 * 128 * 2
    draft_bytes = q_bytes + H * w.n_key_blocks * 128 * 4 + H * Nq * (w.topk + 1) * 4
    append_bytes = 2 * 2 * q_bytes + H * nblk * w.q_layers * 128 * 4
    draft_ms = statistics.mean(t_draft)
    append_ms = statistics.mean(t_append)
    traffic = traffic_for("attention.cu", w.name)
    result = {
        "metric": METRIC,
        "value": round(value, 3),
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "ms_per_chunk": round(ms_step, 5),
        "pct_bf16_peak": round(100 * value / world / pk["bf16_tflops"], 2),
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v with per-head low-rank block bias; random, no weights)",
        "config": {
            "workload": f"{w.name} streaming chunk, one DiT attention layer",
            "heads": H, "head_dim": 128, "query_blocks": Nq, "key_blocks": w.n_key_blocks,
            "kv_len_layers": w.kv_len, "local_range": w.local_range, "topk": w.topk,
            "kept_tiles_per_chunk": kept_tiles, "tflop_per_chunk": round(step_flops / 1e12, 5),
            "l2": f"inputs larger than L2: {n_bufs} distinct chunk buffers rotated, ring "
                  f"{(layer.cache.k.numel() + layer.cache.v.numel()) * 2 / 1e6:.0f} MB "
                  f"({layer.cache.desc.capacity} slots, {w.capacity} resident)",
            "parallelism": f"replicas x{world}" if world > 1 else "single GPU",
            "launch": "append, draft and attention each as a programmatic dependent of the kernel before "
                      "it (LCSA_FLAG_PDL; the append writes a spare ring slot and overlaps the previous "
                      "step's attention); per-kernel times from a separate pass of plain launches",
        },
        "roofline": {
            "kernel": "lcsa_attention (tcgen05 block-sparse attention)",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(attn_tflops / pk["bf16_tflops"], 4),
            "peak_source": f"{pk['source']} dense bf16 (burst)",
            "traffic": traffic,
            "algorithmic_flops_per_launch": step_flops,
            "avg_launch_ms": round(attn_ms, 5),
        },
        "kernels": {
            "attention_ms": round(attn_ms, 5),
            "attention_median_ms": round(statistics.median(t_attn), 5),
            "draft_median_ms": round(statistics.median(t_draft), 5),
            "cache_append_median_ms": round(statistics.median(t_append), 5),
            "draft_ms": round(draft_ms, 5),
            "draft_gbs": round(draft_bytes / (draft_ms * 1e-3) / 1e9, 1),
            "cache_append_ms": round(append_ms, 5),
            "cache_append_gbs": round(append_bytes / (append_ms * 1e-3) / 1e9, 1),
            "hbm_peak_gbs": pk["hbm_gbs"],
        },
        "clocks": clocks.summary(),
        "gpu_launches": 3 * args.steps,
    }
    if not args.no_e2e:
        result["e2e"] = run_e2e(args, L, layer, host, dev, stream, step_flops, world)
    return result


def run_e2e(args, L, layer, host, dev, stream, step_flops, world):
    """Same step through the public API fed from pinned host memory: every step
    copies its q/k/v in and its output out (all inside the timed region),
    overlapped with the previous/next chunk's compute by ``lcsa.HostStream``."""
    pinned = [[t.pin_memory() for t in c] for c in host]
    n = len(pinned)
    outs_host = [torch.empty_like(pinned[0][0]).pin_memory() for _ in range(2)]
    hs = L.HostStream(layer, pinned[0][0].shape, dev)

    def e2e_step(i):
        q, k, v = pinned[i % n]
        hs.submit(q, k, v, outs_host[i % 2])

    steps = max(5, args.steps // 4)
    for i in range(3):
        e2e_step(i)
    hs.drain_into(stream)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    t0.record(stream)
    hs.copy_in.wait_event(t0)  # no copy of the timed chunks starts before t0
    for i in range(steps):
        e2e_step(i)
    hs.drain_into(stream)  # t1 after the last output reached the host
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1) / steps, dev)
    h2d = sum(t.numel() * t.element_size() for t in pinned[0])
    d2h = outs_host[0].numel() * outs_host[0].element_size()
    return {"value": round(aggregate_tflops(world, step_flops, ms), 3), "unit": "TFLOP/s",
            "ms_per_step": round(ms, 4), "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": steps,
            "overlap": "H2D of chunk i+1 and D2H of chunk i-1 overlap chunk i's kernels (two copy streams)"}


# ------------------------------------------------------------ CPU oracle arm

def oracle_prepare(w: W.Workload):
    """Prefill the oracle's cache model, then time the per-chunk part of one
    chunk once: append, the full draft (every row), and the oracle's
    partition of q and gather of the ring."""
    from oracle import lcsa_oracle as O

    oc = O.KVCacheModel(w.capacity)
    prefill, steps = W.stream_plan(w)
    for p in prefill:
        _, k, v = W.gen_layers(w, p, 1, "kv")
        oc.append(k.float().numpy(), v.float().numpy())
    q, k, v = W.gen_layers(w, steps[0], w.q_layers)
    qf = q.float().numpy()
    t0 = time.perf_counter()
    oc.append(k.float().numpy(), v.float().numpy())
    res = O.lcsa_step(qf, oc, w.grid_h, w.grid_w, w.topk, w.local_range,
                      "preserved" if w.local_mode == 0 else "truncated", rows=[])
    qb = O.partition(qf)
    kb, vb = oc.keys()
    t_fixed = time.perf_counter() - t0
    return {"res": res, "qb": qb, "kb": kb, "vb": vb, "t_fixed": t_fixed,
            "kept_tiles": int(res["kept_cnt"].sum())}


def oracle_rows(w: W.Workload, prep, rows_sample: int, seed: int = 0) -> float:
    """Seconds the oracle takes for the attention of ``rows_sample`` rows of the
    prepared chunk (every row when rows_sample >= the chunk's rows)."""
    from oracle import lcsa_oracle as O

    Nq = w.n_query_blocks
    if rows_sample >= w.heads * Nq:
        rows = [(h, i) for h in range(w.heads) for i in range(Nq)]
    else:
        rng = np.random.default_rng(seed)
        rows = [(int(rng.integers(w.heads)), int(rng.integers(Nq))) for _ in range(rows_sample)]
    res, qb, kb, vb = prep["res"], prep["qb"], prep["kb"], prep["vb"]
    scale = 1 / np.sqrt(128.0)
    t0 = time.perf_counter()
    for h, i in rows:
        O.sparse_attention_row(qb[h, i], kb[h], vb[h], res["kept_idx"][h, i, :res["kept_cnt"][h, i]], scale)
    return time.perf_counter() - t0, len(rows)


def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


def cpu_baseline(w: W.Workload, target_s: float = 10.0, max_chunks: int = 4):
    """The oracle on whole chunks (append, draft and attention of every row),
    repeated until about ``target_s`` seconds of CPU work."""
    total_rows = w.heads * w.n_query_blocks
    spent, est, kept, n = 0.0, 0.0, 0, 0
    while n < max_chunks and (n == 0 or spent < target_s):
        prep = oracle_prepare(w)
        t_rows, _ = oracle_rows(w, prep, total_rows)
        spent += prep["t_fixed"] + t_rows
        est += prep["t_fixed"] + t_rows
        kept += prep["kept_tiles"]
        n += 1
    value = kept * W.flops_per_tile() / est / 1e12
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "ms_per_chunk": round(est / n * 1e3, 1),
            "sample": f"{n} x one whole chunk: append + draft + attention of all {total_rows} rows, "
                      f"fp64 NumPy oracle",
            "measured_s": round(spent, 2)}


def run_reference(args):
    """The oracle arm: the per-chunk part (append, full draft, partition) is
    timed once; every step then times the attention of a bounded sample of
    rows, and a step's time is that part plus the sample scaled to the chunk."""
    w = workload(args)
    rows = 16
    total_rows = w.heads * w.n_query_blocks
    prep = oracle_prepare(w)
    ests = []
    for i in range(args.warmup + args.steps):
        t_rows, n = oracle_rows(w, prep, rows, seed=i)
        if i >= args.warmup:
            ests.append(prep["t_fixed"] + t_rows * total_rows / n)
    est = statistics.mean(ests)
    kept = prep["kept_tiles"]
    value = kept * W.flops_per_tile() / est / 1e12
    cores = cpu_cores()
    sample = (f"per-chunk part (append + draft of all {total_rows} rows) timed once "
              f"({prep['t_fixed']:.2f} s); per step the attention of {rows} random rows, scaled to the chunk")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(est * 1e3, 2),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": {"workload": f"{w.name} streaming chunk, one DiT attention layer", "heads": w.heads,
                   "head_dim": 128, "query_blocks": w.n_query_blocks, "key_blocks": w.n_key_blocks,
                   "topk": w.topk, "kept_tiles_per_chunk": kept, "parallelism": "host cores"},
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        if rank == 0:
            print(json.dumps(run_reference(args)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        result = run_lcsa(args, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline:
                result["cpu_baseline"] = cpu_baseline(workload(args))
            print(json.dumps(result), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
