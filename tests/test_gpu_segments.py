"""GPU parity of segment-masked dense attention (the Stage-1 teacher of the
reading notes, 关键设计 1) against the fp64 oracle, through the C ABI.

A packed sequence of clips (images as single-frame videos, and videos) runs
through lcsa_cache_append, lcsa_segment_mask and lcsa_attention; every token
must attend to its own segment only.  Acceptance: kept lists equal to the
segment table exactly; outputs within max-abs 2e-2 and relative L2 5e-3 of the
fp64 oracle, LSE within 2e-3.
"""

import math

import numpy as np
import pytest
import torch

from diffusion_vsr_b200 import workloads as W
from oracle import lcsa_oracle as O
from tests import harness as Hn

pytestmark = pytest.mark.gpu


def _run(spec: W.SegmentWorkload, sample_rows=None, seed_rows=0):
    from diffusion_vsr_b200 import lcsa as L
    dev = torch.device("cuda")
    q, k, v = W.gen_segments(spec)
    sa = L.SegmentAttention(spec.heads, spec.seg_tiles, device=dev)
    out = torch.empty_like(q, device=dev)
    lse = torch.empty(q.shape[:2], dtype=torch.float32, device=dev)
    sa.run(q.to(dev), k.to(dev), v.to(dev), out, lse)
    torch.cuda.synchronize()
    assert sa.status.item() == 0, L.status_string(sa.status.item())
    # kept lists: exactly the segment table (integer work, bit-exact)
    starts = np.concatenate([[0], np.cumsum(spec.seg_tiles)])
    kept = sa.kept_idx.cpu().numpy()
    cnt = sa.kept_cnt.cpu().numpy()
    for s, n in enumerate(spec.seg_tiles):
        rows = slice(starts[s], starts[s + 1])
        assert np.all(cnt[:, rows] == n)
        assert np.all(kept[:, rows, :n] == np.arange(starts[s], starts[s + 1])[None, None, :])
        assert np.all(kept[:, rows, n:] == -1)
    seg = O.segment_ids(spec.clips)
    N = seg.size
    rows = None
    if sample_rows is not None:
        rng = np.random.default_rng(seed_rows)
        # first and last token of every segment, plus random tokens
        ends = np.concatenate([starts[:-1] * 128, starts[1:] * 128 - 1])
        rows = np.unique(np.concatenate([ends, rng.integers(0, N, sample_rows)]))
    ref, ref_lse = O.segment_attention(Hn.f32(q), Hn.f32(k), Hn.f32(v), seg, 1 / math.sqrt(128), query_rows=rows)
    got = Hn.f32(out.cpu())
    got_lse = lse.cpu().numpy()
    if rows is not None:
        got, got_lse = got[:, rows], got_lse[:, rows]
    mx, rl2 = Hn.compare_outputs(got, ref)
    print(f"[segments] {spec.name}: {len(spec.seg_tiles)} segments {spec.seg_tiles} tiles, "
          f"{got.shape[1]} query rows per head against fp64: max-abs {mx:.2e}, rel-L2 {rl2:.2e}")
    assert mx <= Hn.ATOL_OUT and rl2 <= Hn.RTOL_L2_OUT, (mx, rl2)
    assert np.max(np.abs(got_lse - ref_lse)) <= 2e-3


def test_mixed_images_and_videos_every_row():
    # 256x512 px frames (16 x 32 tokens, 4 tiles each): an image, a 3-frame
    # video, an image, a 2-frame video
    _run(W.SEGMENT_WORKLOADS["small"])


def test_single_segment_is_dense_attention_and_single_tile_segments():
    _run(W.SegmentWorkload("one-video", heads=2, clips=((4, 16, 32),), seed=7))
    _run(W.SegmentWorkload("tile-images", heads=3, clips=((1, 8, 16),) * 5 + ((2, 8, 16),), seed=8))


def test_bench_size_sampled_rows():
    # the bench workload (768x1280 frames): first and last token of every
    # segment plus random tokens, every head
    _run(W.SEGMENT_WORKLOADS["768x1280"], sample_rows=64, seed_rows=1)


def test_segment_mask_rejects_a_segment_longer_than_topk():
    from diffusion_vsr_b200 import lcsa as L
    kept = torch.empty((1, 6, 4), dtype=torch.int32, device="cuda")
    cnt = torch.empty((1, 6), dtype=torch.int32, device="cuda")
    with pytest.raises(L.LcsaError):
        L.lcsa_segment_mask([2, 4], 1, kept[:, :6, :3].contiguous(), cnt)  # topk 3 < 4
