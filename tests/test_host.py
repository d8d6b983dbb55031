"""CPU-only checks of the host side: the C library loads and exports every
symbol the header declares, host-side argument validation (no GPU call is
made on those paths), and the multi-rank reduction of the benchmark."""

import ctypes
import os
import re

import pytest
import torch
import torch.multiprocessing as mp

from diffusion_vsr_b200 import build as B
from diffusion_vsr_b200 import lcsa as L

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def header_functions():
    with open(os.path.join(ROOT, "include", "lcsa.h")) as f:
        text = f.read()
    return sorted(set(re.findall(r"^\s*(?:const\s+)?\w+\s*\*?\s*(lcsa_\w+)\s*\(", text, re.M)))


@pytest.fixture(scope="module")
def lib():
    B.build()
    return L.load_library()


def test_header_declares_the_three_hot_path_calls():
    fns = header_functions()
    for name in ("lcsa_cache_append", "lcsa_draft_mask", "lcsa_attention"):
        assert name in fns


def test_library_exports_every_declared_symbol(lib):
    for name in header_functions():
        assert hasattr(lib, name), name
    assert set(L.EXPORTED_SYMBOLS) <= set(header_functions())


def test_version_and_status_strings(lib):
    assert lib.lcsa_version() == 102
    assert L.status_string(L.LCSA_OK) == "LCSA_OK"
    assert L.status_string(L.LCSA_ERR_TIMEOUT) == "LCSA_ERR_TIMEOUT"
    assert L.status_string(L.LCSA_ERR_BAD_INDEX | L.LCSA_ERR_TIMEOUT).startswith("LCSA_ERR_TIMEOUT|")


def _fake_cache(**kw):
    c = L.lcsa_kv_cache(0x10000, 0x20000, 0x30000, 4, 0, 4, 2, 4, 4)
    for k, v in kw.items():
        setattr(c, k, v)
    return c


def test_cache_append_rejects_bad_arguments_without_touching_the_gpu(lib):
    c = _fake_cache()
    assert lib.lcsa_cache_append(None, 0x40000, 0x50000, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_cache_append(ctypes.byref(c), None, 0x50000, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_cache_append(ctypes.byref(c), 0x40008, 0x50000, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_cache_append(ctypes.byref(c), 0x40000, 0x50000, 5, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_cache_append(ctypes.byref(c), 0x40000, 0x50000, 0, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    bad = _fake_cache(count=5)
    assert lib.lcsa_cache_append(ctypes.byref(bad), 0x40000, 0x50000, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG


def test_cache_appended_field_is_validated(lib):
    # layers written by the last append: 0..capacity
    z = ctypes.c_void_p(0x60000)
    p = L.make_params(2, 4, 4, 1, 8)
    for bad in (-1, 5):
        c = _fake_cache(appended=bad)
        assert lib.lcsa_draft_mask(ctypes.byref(p), z, ctypes.byref(c), z, z, None, None, None, None, None) == \
            L.LCSA_ERR_INVALID_ARG
        assert lib.lcsa_cache_append(ctypes.byref(c), 0x40000, 0x50000, 1, 0, None, None, None) == \
            L.LCSA_ERR_INVALID_ARG


# A call that passes validation goes on to launch a kernel: with the fake
# pointers of these tests that must only happen where no GPU exists.
no_gpu_only = pytest.mark.skipif(torch.cuda.is_available(),
                                 reason="fake device pointers: runs only where the call cannot reach a GPU")


@no_gpu_only
def test_append_of_more_than_sixteen_layers_passes_validation(lib):
    # the ring slots are computed on the device: any n_layers <= window is accepted
    c = _fake_cache(capacity=40, window=40, count=0, heads=1)
    rc = lib.lcsa_cache_append(ctypes.byref(c), 0x40000, 0x50000, 33, 0, None, None, None)
    assert rc != L.LCSA_ERR_INVALID_ARG
    assert c.count == 0  # nothing enqueued without a GPU: state unchanged


@no_gpu_only
def test_cache_window_and_overlap_rules(lib):
    k, v = 0x40000, 0x50000
    # at most `window` layers resident, window <= capacity
    wide = _fake_cache(capacity=5, window=6, count=4)
    assert lib.lcsa_cache_append(ctypes.byref(wide), k, v, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    over = _fake_cache(capacity=5, window=4, count=5)
    assert lib.lcsa_cache_append(ctypes.byref(over), k, v, 1, 0, None, None, None) == L.LCSA_ERR_INVALID_ARG
    # an append overlapping the previous step must fit the spare slots (5 - 4 = 1 here)
    ok = _fake_cache(capacity=5, window=4, count=4)
    assert lib.lcsa_cache_append(ctypes.byref(ok), k, v, 2, L.LCSA_FLAG_PDL, None, None, None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_cache_append(ctypes.byref(ok), k, v, 1, L.LCSA_FLAG_PDL, None, None, None) != L.LCSA_ERR_INVALID_ARG
    no_spare = _fake_cache(capacity=4, window=0, count=4)
    assert lib.lcsa_cache_append(ctypes.byref(no_spare), k, v, 1, L.LCSA_FLAG_PDL, None, None, None) == \
        L.LCSA_ERR_INVALID_ARG


@pytest.mark.parametrize("field,value", [("head_dim", 64), ("topk", 0), ("local_range", 4), ("local_mode", 2),
                                         ("q_layers", 5), ("heads", 3), ("scale", -1.0), ("grid_w", 5)])
def test_draft_and_attention_reject_bad_params(lib, field, value):
    p = L.make_params(2, 4, 4, 1, 8)
    setattr(p, field, value)
    c = _fake_cache()
    z = ctypes.c_void_p(0x60000)
    assert lib.lcsa_draft_mask(ctypes.byref(p), z, ctypes.byref(c), z, z, None, None, None, None, None) == \
        L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_attention(ctypes.byref(p), z, ctypes.byref(c), z, z, ctypes.c_void_p(0x70000), None, None,
                              None) == L.LCSA_ERR_INVALID_ARG


@no_gpu_only
def test_rope_arguments_are_validated(lib):
    z = ctypes.c_void_p(0x60000)
    c = _fake_cache()
    for base, frame0, ok in [(10000.0, 0, True), (0.0, -5, True), (1.0, 0, False), (-3.0, 0, False),
                             (float("inf"), 0, False), (10000.0, -1, False), (10000.0, (1 << 20) - 2, True),
                             (10000.0, (1 << 20) - 1, False)]:
        p = L.make_params(2, 4, 4, 1, 8, rope_base=base, rope_frame0=frame0)
        rc = lib.lcsa_draft_mask(ctypes.byref(p), z, ctypes.byref(c), z, z, None, None, None, None, None)
        assert (rc != L.LCSA_ERR_INVALID_ARG) == ok, (base, frame0, rc)
        r = L.lcsa_rope(base, frame0)
        rc = lib.lcsa_cache_append(ctypes.byref(c), 0x40000, 0x50000, 1, 0, ctypes.byref(r), None, None)
        if not ok:
            assert rc == L.LCSA_ERR_INVALID_ARG, (base, frame0)


@no_gpu_only
def test_draft_rotated_q_needs_a_rotation_alignment_and_its_own_memory(lib):
    q = 0x4000000  # 2 heads x 2 frames x 32 x 32 tokens x 128 dims bf16 = 1 MiB
    z = ctypes.c_void_p(0x60000)
    c = _fake_cache()
    call = lambda p, q_rot: lib.lcsa_draft_mask(ctypes.byref(p), ctypes.c_void_p(q), ctypes.byref(c), z, z, None,
                                                None, ctypes.c_void_p(q_rot), None, None)
    assert call(L.make_params(2, 4, 4, 1, 8), 0x1000000) == L.LCSA_ERR_INVALID_ARG  # no rotation
    p = L.make_params(2, 4, 4, 1, 8, rope_base=10000.0)
    assert call(p, 0x1000008) == L.LCSA_ERR_INVALID_ARG  # misaligned
    assert call(p, q + (1 << 20) - 16) == L.LCSA_ERR_INVALID_ARG  # overlaps q's last 16 bytes
    assert call(p, q - (1 << 20) + 16) == L.LCSA_ERR_INVALID_ARG  # overlaps q's first 16 bytes
    assert call(p, q + (1 << 20)) != L.LCSA_ERR_INVALID_ARG  # right after q: accepted
    assert call(p, q - (1 << 20)) != L.LCSA_ERR_INVALID_ARG  # right before q: accepted


def test_draft_rejects_too_many_candidates(lib):
    # no window over a 64 x 64 block grid: 4096 per layer x 4 layers > 4096
    p = L.make_params(1, 64, 64, 1, 8, local_range=0)
    c = _fake_cache(heads=1, grid_h=64, grid_w=64)
    z = ctypes.c_void_p(0x60000)
    assert lib.lcsa_draft_mask(ctypes.byref(p), z, ctypes.byref(c), z, z, None, None, None, None, None) == \
        L.LCSA_ERR_INVALID_ARG


def test_attention_rejects_aliased_output(lib):
    p = L.make_params(2, 4, 4, 1, 8)
    c = _fake_cache()
    z = ctypes.c_void_p(0x60000)
    assert lib.lcsa_attention(ctypes.byref(p), z, ctypes.byref(c), z, z, z, None, None, None) == \
        L.LCSA_ERR_INVALID_ARG


def test_segment_mask_rejects_bad_tables(lib):
    z = ctypes.c_void_p(0x60000)

    def call(tiles, heads=2, topk=8, kept=z, cnt=z):
        arr = (ctypes.c_int32 * max(len(tiles), 1))(*tiles)
        return lib.lcsa_segment_mask(arr if tiles is not None else None, len(tiles), heads, topk, kept, cnt, None)

    assert call([]) == L.LCSA_ERR_INVALID_ARG                    # no segment
    assert call([3, 0, 2]) == L.LCSA_ERR_INVALID_ARG             # empty segment
    assert call([3, 9]) == L.LCSA_ERR_INVALID_ARG                # longer than topk
    assert call([3, 2], heads=0) == L.LCSA_ERR_INVALID_ARG
    assert call([3, 2], topk=0) == L.LCSA_ERR_INVALID_ARG
    assert call([1] * (L.LCSA_MAX_SEGMENTS + 1)) == L.LCSA_ERR_INVALID_ARG
    assert call([3, 2], kept=ctypes.c_void_p(0x60002)) == L.LCSA_ERR_INVALID_ARG  # misaligned
    assert call([3, 2], cnt=None) == L.LCSA_ERR_INVALID_ARG
    assert lib.lcsa_segment_mask(None, 2, 2, 8, z, z, None) == L.LCSA_ERR_INVALID_ARG


def test_binding_refuses_cpu_tensors():
    with pytest.raises(ValueError):
        L._ptr(torch.zeros(4))


# ------------------------------------------------ multi-rank bench reduction

def _rank_main(rank, world, port, ms, q):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.distributed.init_process_group("gloo", rank=rank, world_size=world)
    import bench
    got = bench.max_over_ranks(ms[rank], torch.device("cpu"))
    agg = bench.aggregate_tflops(world, 1e12, got)
    q.put((rank, got, agg))
    torch.distributed.destroy_process_group()


def test_bench_takes_max_over_two_gloo_ranks():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    ms = [2.0, 5.0]
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, ms, q)) for r in range(2)]
    for p in procs:
        p.start()
    out = [q.get(timeout=120) for _ in procs]
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    for rank, got, agg in out:
        assert got == 5.0
        assert abs(agg - 2 * 1e12 / 5e-3 / 1e12) < 1e-9


def test_bench_gpus_must_match_world_size():
    import bench
    args = bench.parse_args(["--gpus", "2"])
    with pytest.raises(SystemExit) as e:
        bench.check_world(args, {"WORLD_SIZE": "1"})
    assert "WORLD_SIZE=1" in str(e.value)
    assert bench.check_world(args, {"WORLD_SIZE": "2"}) == "run"
    # without torchrun, --gpus N > 1 starts N ranks itself
    assert bench.check_world(args, {}) == "launch"
    assert bench.check_world(bench.parse_args([]), {}) == "run"
    # the reference arm runs once, on rank 0, whatever N is
    assert bench.check_world(bench.parse_args(["--gpus", "4", "--impl", "reference"]), {}) == "run"
    cmd = bench.launcher_argv(["--gpus", "2", "--steps", "5"], 2, 29500)
    assert cmd[1:4] == ["-m", "torch.distributed.run", "--nnodes=1"]
    assert "--nproc-per-node=2" in cmd and cmd[cmd.index("--master-addr") + 1] == "127.0.0.1"
    assert cmd[-4:] == ["--gpus", "2", "--steps", "5"]


def test_bench_main_exits_nonzero_on_world_mismatch():
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    env = dict(os.environ, WORLD_SIZE="1", RANK="0", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--gpus", "8", "--steps", "1"],
                       capture_output=True, text=True, timeout=300, cwd=root, env=env)
    assert r.returncode != 0 and "WORLD_SIZE=1" in r.stderr


def test_bench_rope_and_segment_options():
    import bench
    from diffusion_vsr_b200 import workloads as W
    a = bench.parse_args(["--rope", "10000", "--segments", "768x1280"])
    assert a.rope == 10000.0 and a.segments == "768x1280"
    assert bench.parse_args([]).rope == 0.0 and bench.parse_args([]).segments is None
    w = W.WORKLOADS["768x1408"]
    # the default line's config carries no RoPE key, so both arms print the same dict
    assert "rope_base" not in bench.bench_config(w, 15840, 1)
    assert bench.bench_config(w, 15840, 1, rope=10000.0)["rope_base"] == 10000.0
    # the segment line's work: every (query tile, key tile) pair of a segment
    sw = W.SEGMENT_WORKLOADS[bench.SWEEP_SEGMENTS]
    assert sw.seg_tiles == [30, 150, 30, 90]
    assert sw.kept_tiles == 12 * (30 ** 2 + 150 ** 2 + 30 ** 2 + 90 ** 2) == 388800


def test_bench_config_is_shared_by_both_arms():
    import bench
    from diffusion_vsr_b200 import workloads as W
    w = W.WORKLOADS["768x1408"]
    kept = bench.chunk_kept_tiles(w)
    assert kept == w.heads * w.n_query_blocks * w.topk == 15840
    a = bench.bench_config(w, kept, 1)
    for key in ("workload", "kv_len_layers", "local_range", "topk", "tflop_per_chunk", "l2", "parallelism"):
        assert key in a
    # ragged: a truncated 5-block window keeps fewer than topk at the edges
    import dataclasses
    wt = dataclasses.replace(W.WORKLOADS["768x1280"], local_mode=1, local_range=5, topk=40)
    assert bench.chunk_kept_tiles(wt) < wt.heads * wt.n_query_blocks * wt.topk
    # a reference step of n heads fits the run's budget
    assert bench.reference_heads_per_step(w, 20, 5, 0.2) == 12
    assert bench.reference_heads_per_step(w, 200, 10, 0.2) == 3
    assert bench.reference_heads_per_step(w, 10000, 10, 5.0) == 1


def test_reference_arm_prints_one_json_line():
    # `bench.py --impl reference` times the oracle (the pages ship no runnable
    # reference) and prints one JSON line with the contract's keys.
    import json
    import subprocess
    import sys
    root = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
    r = subprocess.run([sys.executable, os.path.join(root, "bench.py"), "--impl", "reference", "--workload", "tiny",
                        "--steps", "2", "--warmup", "1"], capture_output=True, text=True, timeout=600, cwd=root)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    assert d["impl"] == "reference" and d["value"] > 0 and d["unit"] == "TFLOP/s"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    import bench
    from diffusion_vsr_b200 import workloads as W
    w = W.WORKLOADS["tiny"]
    assert d["config"] == bench.bench_config(w, bench.chunk_kept_tiles(w), 1)
