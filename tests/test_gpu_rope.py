"""GPU parity of the rotary position embedding (RoPE) folded into the kernels
that read q and k: the cache append rotates k before it is stored and
averaged, the draft mask rotates q before its block means, the attention
rotates the Q tiles before the products.  The oracle rotates q and k itself
(apply_rope, in the kernels' precision: fp32 from fp64 cos/sin, one rounding
per product and sum, then bf16) and runs its unrotated path on them.

Acceptance: the ring (rotated k in block layout) bit-exact against the
oracle's rotated, partitioned k; block means within 1e-6 relative; kept sets
bit-exact except near-tie rows; outputs within max-abs 2e-2 and relative L2
5e-3 of fp64, LSE within 2e-3.
"""

import dataclasses

import numpy as np
import pytest
import torch

from diffusion_vsr_b200 import workloads as W
from tests import harness as Hn
from tests.test_gpu_parity import _check_step

pytestmark = pytest.mark.gpu

BASE = 10000.0


def test_rope_768x1280_every_row():
    w = W.WORKLOADS["768x1280"]
    (res,) = Hn.run_stream(w, check_ring=True, rope_base=BASE)
    assert res.ring_ok and res.kmean_err <= 1e-6
    _check_step(res, w)


def test_rope_768x1408_streaming_with_eviction():
    # three chunks after the prefill: the ring rotates and the time positions advance
    w = W.WORKLOADS["768x1408"]
    seen = []

    def check(res):
        assert res.ring_ok and res.kmean_err <= 1e-6
        _check_step(res, w)
        seen.append(res.position)

    Hn.run_stream(w, n_steps=3, check_ring=True, on_step=check, rope_base=BASE)
    assert len(seen) == 3


def test_rope_cold_start_and_far_stream_positions():
    # a 3-layer cold start then 1-layer chunks; and a stream that starts near the
    # end of the position range (frame 2^20 - 16), where the angles are largest
    w = W.WORKLOADS["768x1280"]
    for res in Hn.run_schedule(dataclasses.replace(w, heads=4), [3, 1, 1], n_rows=32, check_ring=True,
                               rope_base=BASE):
        assert res.ring_ok and res.kmean_err <= 1e-6
        _check_step(res, dataclasses.replace(w, heads=4))
    wt = W.WORKLOADS["tiny"]
    (res,) = Hn.run_stream(wt, check_ring=True, rope_base=BASE, frame_offset=(1 << 20) - 16)
    assert res.ring_ok and res.kmean_err <= 1e-6
    _check_step(res, wt)


def test_rope_1536x2688_sampled_rows_and_chained_launches():
    # the high-resolution workload (token rows and columns up to 95 and 167)
    w = W.WORKLOADS["1536x2688"]
    (res,) = Hn.run_stream(w, n_steps=1, n_rows=48, check_ring=True, rope_base=BASE)
    assert res.ring_ok
    _check_step(res, w)
    # the chained streaming step (programmatic dependent launches) gives the
    # same outputs as plain launches, rotation included
    from diffusion_vsr_b200 import lcsa as L
    w = W.WORKLOADS["768x1408"]
    dev = torch.device("cuda")
    chunks = [[t.to(dev) for t in W.gen_layers(w, w.kv_len + i, w.q_layers)] for i in range(3)]
    prefill = [[t.to(dev) for t in W.gen_layers(w, p, 1, "kv")[1:]] for p in range(w.kv_len)]
    runs = []
    for chained in (True, False):
        layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, device=dev, rope_base=BASE)
        for k, v in prefill:
            layer.append(k, v)
        outs = []
        for q, k, v in chunks:
            out = torch.empty_like(q)
            if chained:
                layer.step(q, k, v, out, overlap_previous=True)
            else:
                frame0 = layer.frame
                L.lcsa_cache_append(layer.cache, k, v, d_status=layer.status, rope=L.lcsa_rope(BASE, frame0))
                layer.frame += k.shape[1]
                layer.params.rope.frame0 = frame0
                L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status)
                L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, out,
                                 d_status=layer.status)
            outs.append((out, layer.kept_idx.clone()))
        torch.cuda.synchronize()
        assert layer.status.item() == 0
        runs.append(outs)
    for (o1, k1), (o2, k2) in zip(*runs):
        assert torch.equal(k1, k2) and torch.equal(o1, o2)


def test_draft_stores_the_rotated_q_the_attention_reads():
    # the draft's rotated copy of q is the oracle's rotation in the kernels'
    # precision bit for bit, and the attention over it (without a rotation of its
    # own) equals the attention that rotates the Q tiles itself, bit for bit
    from diffusion_vsr_b200 import lcsa as L
    from oracle import lcsa_oracle as O
    w = W.WORKLOADS["768x1280"]
    dev = torch.device("cuda")
    layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, device=dev, rope_base=BASE)
    for p in range(w.kv_len):
        _, k, v = W.gen_layers(w, p, 1, "kv")
        layer.append(k.to(dev), v.to(dev))
    q, k, v = [t.to(dev) for t in W.gen_layers(w, w.kv_len, w.q_layers)]
    frame0 = layer.frame
    L.lcsa_cache_append(layer.cache, k, v, d_status=layer.status, rope=L.lcsa_rope(BASE, frame0))
    layer.params.rope.frame0 = frame0
    q_rot = torch.empty_like(q)
    L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status,
                      q_rot=q_rot)
    out_self, out_read = torch.empty_like(q), torch.empty_like(q)
    L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, out_self, d_status=layer.status)
    plain = L.make_params(w.heads, w.grid_h, w.grid_w, w.q_layers, w.topk)
    L.lcsa_attention(plain, q_rot, layer.cache, layer.kept_idx, layer.kept_cnt, out_read, d_status=layer.status)
    torch.cuda.synchronize()
    assert layer.status.item() == 0
    expected = O.apply_rope(q.float().cpu().numpy(), frame0, BASE, "kernel")
    assert np.array_equal(q_rot.float().cpu().numpy(), expected)
    assert torch.equal(out_self, out_read)


def test_rope_changes_the_result():
    # positive control: the rotation is applied (outputs differ from the unrotated path)
    w = W.WORKLOADS["tiny"]
    (plain,) = Hn.run_stream(w)
    (rot,) = Hn.run_stream(w, rope_base=BASE)
    assert not np.array_equal(plain.out_pipeline, rot.out_pipeline)
    assert not np.array_equal(plain.gpu_qmean, rot.gpu_qmean)
