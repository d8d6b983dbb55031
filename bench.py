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
ms per chunk.  ``--sweep`` prints one such line per workload instead, plus one line for the
segment-masked dense attention of the Stage-1 teacher (``--segments``: a
packed sequence of images and videos, each attending only to itself).
``--rope BASE`` runs the streaming step with RoPE applied to q and k.
``--impl reference`` times the fp64 CPU oracle (rank 0 only): each step is
one whole chunk of a slice of the heads (append, draft and attention of every
row of those heads), sized so that the run ends within a few minutes.

Multi-GPU: one process per GPU (torchrun); every rank runs an independent
replica of the layer (LCSA rows are independent, there is no exchange step),
so the scaling is weak and the barrier/max reduction is the only collective.
``--gpus N`` without torchrun starts the N processes itself; under torchrun
WORLD_SIZE must equal N.
"""

from __future__ import annotations

import argparse
import hashlib
import json
import os
import socket
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
SWEEP = (("768x1280", 0), ("768x1408", 0), ("1536x2688", 0), ("4k", 8), ("4k", 16), ("4k", 32))
SWEEP_SEGMENTS = "768x1280"
SEGMENT_METRIC = "segment-masked dense attention (Stage-1 teacher): effective TFLOP/s over the segments' tiles"
REFERENCE_BUDGET_S = 150.0  # wall-clock budget of a whole reference-arm run (warm-up + timed steps)
E2E_MIN_STEPS = 50


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="lcsa", choices=["lcsa", "reference"])
    ap.add_argument("--workload", default="768x1408", choices=sorted(W.WORKLOADS))
    ap.add_argument("--topk", type=int, default=0, help="override the workload's topk")
    ap.add_argument("--bufs", type=int, default=8,
                    help="distinct chunk buffers rotated across steps (fewer: a reduced case for ncu captures)")
    ap.add_argument("--sweep", action="store_true",
                    help="one JSON line per workload (768x1280, 768x1408, 1536x2688, 4K topk 8/16/32)")
    ap.add_argument("--rope", type=float, default=0.0, help="RoPE base for q and k (0: no rotation)")
    ap.add_argument("--segments", default=None, choices=sorted(W.SEGMENT_WORKLOADS),
                    help="time the segment-masked dense attention of this packed sequence of clips instead")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    return ap.parse_args(argv)


def workload_of(name: str, topk: int = 0) -> W.Workload:
    w = W.WORKLOADS[name]
    return w.with_topk(topk) if topk else w


def workload(args) -> W.Workload:
    return workload_of(args.workload, args.topk)


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


def bench_config(w: W.Workload, kept_tiles: int, world: int, rope: float = 0.0) -> dict:
    """The workload a line is measured on; both arms print this same dict."""
    extra = {"rope_base": rope} if rope else {}
    return {**extra,
        "workload": f"{w.name} streaming chunk, one DiT attention layer",
        "heads": w.heads, "head_dim": w.head_dim, "query_blocks": w.n_query_blocks, "key_blocks": w.n_key_blocks,
        "kv_len_layers": w.kv_len, "local_range": w.local_range,
        "local_mode": "preserved" if w.local_mode == 0 else "truncated", "topk": w.topk,
        "kept_tiles_per_chunk": kept_tiles, "tflop_per_chunk": round(kept_tiles * W.flops_per_tile() / 1e12, 5),
        "l2": "inputs larger than L2 (126 MB): distinct chunks' q/k/v rotated across steps, plus the "
              "resident ring of kv_len + 1 block-layers",
        "parallelism": f"replicas x{world}" if world > 1 else "single replica",
    }


# ------------------------------------------------------------- launch helpers

def free_port() -> int:
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def launcher_argv(args_argv, gpus: int, port: int):
    """Command that starts ``gpus`` ranks of this script, one process per GPU."""
    return [sys.executable, "-m", "torch.distributed.run", "--nnodes=1", f"--nproc-per-node={gpus}",
            "--master-addr", "127.0.0.1", "--master-port", str(port), os.path.abspath(__file__), *args_argv]


def check_world(args, env) -> str:
    """'run' when this process is a rank of a job of --gpus ranks, 'launch' when
    it should start them itself; raises SystemExit on a mismatch."""
    if "WORLD_SIZE" not in env:
        return "launch" if args.gpus > 1 and args.impl == "lcsa" else "run"
    world = int(env["WORLD_SIZE"])
    if world != args.gpus:
        raise SystemExit(f"bench.py: --gpus {args.gpus} but WORLD_SIZE={world}: start one rank per GPU "
                         f"(torchrun --nproc-per-node {args.gpus}) or pass --gpus {world}")
    return "run"


# ------------------------------------------------------------------ GPU arm

def unique_kv_bytes(kept_idx: torch.Tensor, kept_cnt: torch.Tensor, n_key_blocks: int) -> int:
    """Bytes of the distinct K and V tiles the kept lists of one step touch."""
    H, Nq, topk = kept_idx.shape
    valid = torch.arange(topk, device=kept_idx.device)[None, None, :] < kept_cnt[:, :, None]
    flat = torch.where(valid, kept_idx + torch.arange(H, device=kept_idx.device)[:, None, None] * n_key_blocks,
                       torch.full_like(kept_idx, -1))
    n = torch.unique(flat[flat >= 0]).numel()
    return int(n) * 2 * 128 * 128 * 2


def measure_lcsa(w: W.Workload, args, world: int, local_rank: int, dev, with_e2e: bool):
    from diffusion_vsr_b200 import lcsa as L

    flop_tile = W.flops_per_tile()
    prefill, steps = W.stream_plan(w)
    # distinct chunk buffers rotated across steps: per-step inputs (q, k, v) plus the
    # 4-layer ring are larger than the 126 MB L2, so no step starts warm
    n_bufs = max(1, args.bufs)
    positions = [w.kv_len + (i % len(steps)) for i in range(n_bufs)]
    host = [W.gen_layers(w, p, w.q_layers) for p in positions]
    chunks = [[t.to(dev) for t in c] for c in host]
    layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, w.local_range, w.local_mode,
                        device=dev, rope_base=args.rope)
    for p in prefill:
        _, k, v = W.gen_layers(w, p, 1, "kv")
        layer.append(k.to(dev), v.to(dev))
    out = torch.empty_like(chunks[0][0])
    stream = torch.cuda.current_stream(dev)
    # with RoPE, the attention of the per-kernel pass reads the draft's rotated q
    # without a rotation of its own, as LcsaLayer.step does
    plain_params = L.make_params(w.heads, w.grid_h, w.grid_w, w.q_layers, w.topk, w.local_range, w.local_mode)
    if args.rope:
        layer.q_rot = torch.empty_like(chunks[0][0])

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
        frame0 = layer.frame
        layer.params.rope.frame0 = frame0
        ev[0].record(stream)
        L.lcsa_cache_append(layer.cache, k, v, d_status=layer.status, rope=layer._rope(frame0))
        layer.frame += k.shape[1]
        ev[1].record(stream)
        if args.rope:
            L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status,
                              q_rot=layer.q_rot)
            attn_params, attn_q = plain_params, layer.q_rot
        else:
            L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status)
            attn_params, attn_q = layer.params, q
        ev[2].record(stream)
        L.lcsa_attention(attn_params, attn_q, layer.cache, layer.kept_idx, layer.kept_cnt, out, d_status=layer.status)
        ev[3].record(stream)

    for i in range(args.warmup):
        step(i)
    torch.cuda.synchronize()
    kept_tiles = int(layer.kept_cnt.sum().item())
    kv_bytes = unique_kv_bytes(layer.kept_idx, layer.kept_cnt, layer.cache.count * w.blocks_per_layer)
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
    # the attention's algorithmic DRAM bytes: Q and O once, every distinct kept K/V tile once
    attn_bytes = 2 * q_bytes + kv_bytes + H * Nq * (w.topk + 1) * 4
    draft_ms = statistics.mean(t_draft)
    append_ms = statistics.mean(t_append)
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    traffic = traffic_for("attention.cu", w.name)
    tensor_frac = attn_tflops / pk["bf16_tflops"]
    hbm_frac = attn_gbs / pk["hbm_gbs"]
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
        "data": "synthetic (seeded N(0,1) bf16 q/k/v" + (" with per-head low-rank block bias" if w.lowrank else "")
                + "; random, no weights)",
        "config": bench_config(w, kept_tiles, world, args.rope),
        "inputs": f"{n_bufs} distinct chunk buffers rotated, ring "
                  f"{(layer.cache.k.numel() + layer.cache.v.numel()) * 2 / 1e6:.0f} MB "
                  f"({layer.cache.desc.capacity} slots, {w.capacity} resident)",
        "launch": "append, draft and attention each as a programmatic dependent of the kernel before it "
                  "(LCSA_FLAG_PDL; the append writes a spare ring slot and overlaps the previous step's "
                  "attention); per-kernel times from a separate pass of plain launches",
        "roofline": {
            "kernel": "lcsa_attention (tcgen05 block-sparse attention)",
            "bound": "tensor",
            "achieved": round(attn_tflops, 2),
            "peak": pk["bf16_tflops"],
            "unit": "TFLOP/s",
            "frac": round(tensor_frac, 4),
            "peak_source": f"{pk['source']} dense bf16 (burst)",
            "traffic": traffic,
            "algorithmic_flops_per_launch": step_flops,
            "avg_launch_ms": round(attn_ms, 5),
            "hbm_bound": {"achieved": round(attn_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": round(hbm_frac, 4), "algorithmic_bytes_per_launch": attn_bytes,
                          "bytes": "Q + O + distinct kept K/V tiles + kept lists"},
            "binding": "tensor" if tensor_frac >= hbm_frac else "hbm",
        },
        "kernels": {
            "attention_ms": round(attn_ms, 5),
            "attention_median_ms": round(statistics.median(t_attn), 5),
            "draft_median_ms": round(statistics.median(t_draft), 5),
            "cache_append_median_ms": round(statistics.median(t_append), 5),
            "draft_ms": round(draft_ms, 5),
            "draft_gbs": round(draft_bytes / (draft_ms * 1e-3) / 1e9, 1),
            "draft_bytes": draft_bytes,
            "cache_append_ms": round(append_ms, 5),
            "cache_append_gbs": round(append_bytes / (append_ms * 1e-3) / 1e9, 1),
            "cache_append_bytes": append_bytes,
            "hbm_peak_gbs": pk["hbm_gbs"],
        },
        "clocks": clocks.summary(),
        "gpu_launches": 3 * args.steps,
    }
    if with_e2e:
        result["e2e"] = run_e2e(args, L, layer, host, dev, stream, step_flops, world)
    del chunks, layer, out
    torch.cuda.empty_cache()
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

    steps = max(E2E_MIN_STEPS, args.steps // 4)
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
            "h2d_gbs": round(h2d / (ms * 1e-3) / 1e9, 1),
            "overlap": "H2D of chunk i+1 and D2H of chunk i-1 overlap chunk i's kernels (two copy streams)"}


def measure_segments(sw: W.SegmentWorkload, args, world: int, local_rank: int, dev):
    """The Stage-1 teacher's segment-masked dense attention of a packed sequence
    of clips: a step appends the pack's k/v (one ring layer per 128-token tile)
    and runs the attention over the segment kept lists (every tile of the own
    segment), both through the C ABI; the kept lists are built once."""
    from diffusion_vsr_b200 import lcsa as L

    seg = L.SegmentAttention(sw.heads, sw.seg_tiles, device=dev)
    q, k, v = [t.to(dev) for t in W.gen_segments(sw)]
    out = torch.empty_like(q)
    stream = torch.cuda.current_stream(dev)
    for _ in range(args.warmup):
        seg.run(q, k, v, out)
    torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    t0 = torch.cuda.Event(enable_timing=True)
    t1 = torch.cuda.Event(enable_timing=True)
    with ClockSampler(local_rank) as clocks:
        torch.cuda.synchronize()
        t0.record(stream)
        for _ in range(args.steps):
            seg.run(q, k, v, out)
        t1.record(stream)
        torch.cuda.synchronize()
    if world > 1:
        torch.distributed.barrier()
    ms_step = max_over_ranks(t0.elapsed_time(t1), dev) / args.steps
    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    for e in evs:
        seg.cache.reset()
        e[0].record(stream)
        L.lcsa_cache_append(seg.cache, k, v, n_layers=seg.tiles, d_status=seg.status)
        e[1].record(stream)
        L.lcsa_attention(seg.params, q, seg.cache, seg.kept_idx, seg.kept_cnt, out, d_status=seg.status)
        e[2].record(stream)
    torch.cuda.synchronize()
    status = int(seg.status.item())
    if status != 0:
        raise RuntimeError(f"device status {L.status_string(status)}")
    t_append = [e[0].elapsed_time(e[1]) for e in evs]
    t_attn = [e[1].elapsed_time(e[2]) for e in evs]
    pk = peaks()
    flops = sw.kept_tiles * W.flops_per_tile()
    tensor_bytes = sw.heads * sw.tokens * 128 * 2  # one of q, k, v, out
    attn_ms = statistics.mean(t_attn)
    append_ms = statistics.mean(t_append)
    attn_tflops = flops / (attn_ms * 1e-3) / 1e12
    # the attention reads q and the whole ring (every key tile is some row's kept tile) and writes out
    attn_bytes = 4 * tensor_bytes + sw.heads * seg.tiles * (seg.topk + 1) * 4
    attn_gbs = attn_bytes / (attn_ms * 1e-3) / 1e9
    append_bytes = 4 * tensor_bytes + sw.heads * seg.tiles * 128 * 4
    tensor_frac = attn_tflops / pk["bf16_tflops"]
    hbm_frac = attn_gbs / pk["hbm_gbs"]
    return {
        "metric": SEGMENT_METRIC,
        "value": round(aggregate_tflops(world, flops, ms_step), 3),
        "unit": "TFLOP/s",
        "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": round(ms_step, 5),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
        "data": "synthetic (seeded N(0,1) bf16 q/k/v; random, no weights)",
        "config": {
            "workload": f"segments {sw.name}: packed clips (latent frames, token rows, token columns) "
                        f"{[list(c) for c in sw.clips]}",
            "heads": sw.heads, "head_dim": sw.head_dim, "tokens": sw.tokens, "segment_tiles": sw.seg_tiles,
            "kept_tiles": sw.kept_tiles, "tflop_per_step": round(flops / 1e12, 5),
            "l2": "inputs larger than L2 (126 MB): q, k, v, out and the ring each "
                  f"{tensor_bytes / 1e6:.0f} MB",
            "parallelism": f"replicas x{world}" if world > 1 else "single replica",
        },
        "launch": "per step: lcsa_cache_append of the whole pack (one ring layer per tile), then lcsa_attention "
                  "over the segment kept lists (built once by lcsa_segment_mask); per-kernel times from a "
                  "separate pass with events between the calls",
        "roofline": {
            "kernel": "lcsa_attention (tcgen05 block-sparse attention)", "bound": "tensor",
            "achieved": round(attn_tflops, 2), "peak": pk["bf16_tflops"], "unit": "TFLOP/s",
            "frac": round(tensor_frac, 4), "peak_source": f"{pk['source']} dense bf16 (burst)", "traffic": None,
            "algorithmic_flops_per_launch": flops, "avg_launch_ms": round(attn_ms, 5),
            "hbm_bound": {"achieved": round(attn_gbs, 1), "peak": pk["hbm_gbs"], "unit": "GB/s",
                          "frac": round(hbm_frac, 4), "algorithmic_bytes_per_launch": attn_bytes,
                          "bytes": "Q + O + the K/V ring + kept lists"},
            "binding": "tensor" if tensor_frac >= hbm_frac else "hbm",
        },
        "kernels": {
            "attention_ms": round(attn_ms, 5), "attention_median_ms": round(statistics.median(t_attn), 5),
            "cache_append_ms": round(append_ms, 5),
            "cache_append_median_ms": round(statistics.median(t_append), 5),
            "cache_append_gbs": round(append_bytes / (append_ms * 1e-3) / 1e9, 1),
            "cache_append_bytes": append_bytes,
        },
        "clocks": clocks.summary(),
        "gpu_launches": 2 * args.steps,
    }


def run_lcsa(args, rank: int, world: int, local_rank: int):
    torch.cuda.set_device(local_rank)
    dev = torch.device("cuda", local_rank)
    if args.segments:
        return [measure_segments(W.SEGMENT_WORKLOADS[args.segments], args, world, local_rank, dev)]
    if args.sweep:
        out = []
        for name, topk in SWEEP:
            out.append(measure_lcsa(workload_of(name, topk), args, world, local_rank, dev, with_e2e=False))
        out.append(measure_segments(W.SEGMENT_WORKLOADS[SWEEP_SEGMENTS], args, world, local_rank, dev))
        return out
    return [measure_lcsa(workload(args), args, world, local_rank, dev, with_e2e=not args.no_e2e)]


# ------------------------------------------------------------ CPU oracle arm

def cpu_cores() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return max(n)
    except Exception:
        pass
    return len(os.sched_getaffinity(0))


class OracleInputs:
    """Host copies (fp32, exact bf16 values) of a workload's prefill layers and
    of a few chunk positions, generated once and sliced by head per step."""

    def __init__(self, w: W.Workload, n_positions: int):
        prefill, steps = W.stream_plan(w)
        self.prefill = []
        for p in prefill:
            _, k, v = W.gen_layers(w, p, 1, "kv")
            self.prefill.append((k.float().numpy(), v.float().numpy()))
        self.chunks = []
        for p in steps[:max(1, n_positions)]:
            q, k, v = W.gen_layers(w, p, w.q_layers)
            self.chunks.append(tuple(t.float().numpy() for t in (q, k, v)))


def oracle_chunk(w: W.Workload, inputs: OracleInputs, chunk: int, heads: slice):
    """Seconds the oracle takes for one whole chunk of the heads ``heads``:
    append of the chunk's k/v into a cache already holding the kv_len prefill
    layers (the prefill itself is not timed), then the draft and the attention
    of every row of those heads.  Returns (seconds, kept tiles)."""
    from oracle import lcsa_oracle as O

    oc = O.KVCacheModel(w.capacity)
    for k, v in inputs.prefill:
        oc.append(k[heads], v[heads])
    q, k, v = (np.ascontiguousarray(t[heads]) for t in inputs.chunks[chunk % len(inputs.chunks)])
    t0 = time.perf_counter()
    oc.append(k, v)
    res = O.lcsa_step(q, oc, w.grid_h, w.grid_w, w.topk, w.local_range,
                      "preserved" if w.local_mode == 0 else "truncated")
    dt = time.perf_counter() - t0
    return dt, int(res["kept_cnt"].sum())


def chunk_kept_tiles(w: W.Workload) -> int:
    """Kept tiles of a steady-state chunk: min(topk, allowed) per row (the
    oracle's allowed mask), every head."""
    from oracle import lcsa_oracle as O

    allowed = O.allowed_mask(w.q_layers, w.capacity, w.grid_h, w.grid_w, w.local_range,
                             "preserved" if w.local_mode == 0 else "truncated")
    return int(w.heads * np.minimum(allowed.sum(axis=1), w.topk).sum())


def cpu_baseline(w: W.Workload, target_s: float = 10.0, max_chunks: int = 4):
    """The oracle on whole chunks (append, draft and attention of every row of
    every head), repeated until about ``target_s`` seconds of CPU work."""
    spent, kept, n = 0.0, 0, 0
    inputs = OracleInputs(w, 2)
    while n < max_chunks and (n == 0 or spent < target_s):
        dt, kt = oracle_chunk(w, inputs, n, slice(0, w.heads))
        spent += dt
        kept += kt
        n += 1
    value = kept * W.flops_per_tile() / spent / 1e12
    total_rows = w.heads * w.n_query_blocks
    return {"value": round(value, 6), "unit": "TFLOP/s", "cores": cpu_cores(), "kind": "oracle",
            "ms_per_chunk": round(spent / n * 1e3, 1),
            "sample": f"{n} x one whole chunk: append + draft + attention of all {total_rows} rows, "
                      f"fp64 NumPy oracle",
            "measured_s": round(spent, 2)}


def reference_heads_per_step(w: W.Workload, steps: int, warmup: int, t_head_s: float,
                             budget_s: float = REFERENCE_BUDGET_S) -> int:
    """Heads per reference step so that (warmup + steps) steps fit ``budget_s``."""
    per_step = budget_s / max(1, steps + warmup)
    return int(max(1, min(w.heads, per_step // max(t_head_s, 1e-6))))


def run_reference(args, world: int):
    """The oracle arm.  Each step is the whole chunk for a slice of the heads
    (every head's cache, draft and attention are independent of the others'):
    the append, the draft and the attention of every row of those heads, all
    actually run and timed; the slice width is sized so that the whole run
    fits a few minutes.  ``value`` = kept-tile flops run / seconds taken."""
    w = workload(args)
    inputs = OracleInputs(w, 2)
    t_head, _ = oracle_chunk(w, inputs, 0, slice(0, 1))  # probe, not counted
    nh = reference_heads_per_step(w, args.steps, args.warmup, t_head)
    times, kept = [], []
    for i in range(args.warmup + args.steps):
        h0 = (i * nh) % w.heads
        heads = slice(h0, min(w.heads, h0 + nh))
        dt, kt = oracle_chunk(w, inputs, i, heads)
        if i >= args.warmup:
            times.append(dt)
            kept.append(kt)
    total_s = sum(times)
    value = sum(kept) * W.flops_per_tile() / total_s / 1e12
    ms_step = total_s / len(times) * 1e3
    kept_chunk = chunk_kept_tiles(w)
    cores = cpu_cores()
    sample = (f"each step: one whole chunk (append + draft + attention of every row) for {nh} of the "
              f"{w.heads} heads, fp64 NumPy oracle; ms_per_chunk extrapolates to all heads")
    return {
        "impl": "reference", "metric": METRIC, "value": round(value, 6), "unit": "TFLOP/s", "n_gpus": world,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(ms_step, 2),
        "ms_per_chunk": round(ms_step * w.heads / nh, 1),
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic (same seeded inputs as the CUDA arm)",
        "config": bench_config(w, kept_chunk, world),
        "cpu_baseline": {"value": round(value, 6), "unit": "TFLOP/s", "cores": cores, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": round(value, 6), "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def main(argv=None):
    args = parse_args(argv)
    mode = check_world(args, os.environ)
    if mode == "launch":
        argv_run = list(sys.argv[1:] if argv is None else argv)
        r = subprocess.run(launcher_argv(argv_run, args.gpus, free_port()))
        sys.exit(r.returncode)
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        # the oracle runs once, on rank 0; the other ranks exit without work
        if rank == 0:
            print(json.dumps(run_reference(args, world)), flush=True)
        return
    if world > 1:
        import datetime
        torch.cuda.set_device(local_rank)
        torch.distributed.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                             device_id=torch.device("cuda", local_rank))
    try:
        results = run_lcsa(args, rank, world, local_rank)
        if rank == 0:
            if not args.no_cpu_baseline and not args.sweep and not args.segments:
                results[0]["cpu_baseline"] = cpu_baseline(workload(args))
            for r in results:
                print(json.dumps(r), flush=True)
    finally:
        if world > 1:
            torch.distributed.destroy_process_group()


if __name__ == "__main__":
    main()
