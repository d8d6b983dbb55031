"""Workload definitions and seeded synthetic inputs for the LCSA hot path.

This module holds no step of the attention method itself: it only fixes the
shapes of the five workloads and draws their random bf16 inputs, so that the
CUDA path and the CPU oracle are fed the very same bits.

Geometry (FlashVSR code walk-through, "learn.html" page, section 5.3): one
attention token covers 16x16 output pixels (VAE /8, DiT patch [1,2,2] /2), so an
output frame of H x W pixels has (H/16) x (W/16) tokens and one latent frame
covers 4 video frames. A (2,8,8) window block is 2 latent frames x 8 x 8 tokens
= 128 tokens (same page, section 2.2, "WindowPartition3D"). One streaming step
consumes 2 latent frames = 8 video frames (same page, section 2.3) and appends
one block-layer of keys/values.

Value recipe: q, k, v are i.i.d. N(0,1) drawn in fp32 from
``numpy.random.default_rng([seed * 1000 + position, stream])`` (stream 0 = q,
1 = k, 2 = v) and rounded to bf16 with round-to-nearest-even.  The
768x1408 streaming workload adds a per-head low-rank block bias so that the
block-mean scores are not uniform: basis B_h in R^{4x128} ~ N(0,1) (stream 3,
shared by all positions), per-block coefficients c ~ N(0, I_4) (stream 4 for q,
5 for k), and every token of block b gets ``0.15 * (c_b @ B_h)`` added before
rounding.
"""

from __future__ import annotations

import dataclasses
import math
from typing import List, Optional

import numpy as np
import torch

BLOCK_T, BLOCK_Y, BLOCK_X = 2, 8, 8
BLOCK_TOKENS = BLOCK_T * BLOCK_Y * BLOCK_X  # 128
HEAD_DIM = 128

# Stream ids of the per-position generators.
STREAM_Q, STREAM_K, STREAM_V, STREAM_BASIS, STREAM_QCOEF, STREAM_KCOEF = range(6)
LOWRANK_RANK = 4
LOWRANK_AMPLITUDE = 0.15  # 0.3 * (c . B) / 2


def topk_for_resolution(sparse_ratio: float, height_px: int, width_px: int, n_keys: int) -> int:
    """Number of kept key blocks per query block at a given output resolution.

    FlashVSR code walk-through ("learn.html", section 2.2): the kept ratio is
    ``sparse_ratio * 768*1280 / (th*tw)``, i.e. scaled inversely with the
    pixel count so that the absolute amount of attention work stays about the
    one at 768x1280. The ratio applies to the key-block row length.
    ``round`` (not truncation) is used because the float product for
    1536x2688 is 48.000000...01.
    """
    ratio = sparse_ratio * 768 * 1280 / (height_px * width_px)
    return max(1, int(round(ratio * n_keys)))


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    heads: int
    grid_h: int            # blocks per latent frame along y (tokens / 8)
    grid_w: int            # blocks per latent frame along x (tokens / 8)
    q_layers: int          # query block-layers per step (2 latent frames each)
    kv_len: int            # cached block-layers kept besides the current chunk
    topk: int
    chunks: int            # streaming steps of the workload
    seed: int
    local_range: int = 11
    local_mode: int = 0    # 0 boundary-preserved (shifted window), 1 boundary-truncated
    lowrank: bool = False
    height_px: int = 0
    width_px: int = 0
    head_dim: int = HEAD_DIM

    @property
    def tok_h(self) -> int:
        return self.grid_h * BLOCK_Y

    @property
    def tok_w(self) -> int:
        return self.grid_w * BLOCK_X

    @property
    def blocks_per_layer(self) -> int:
        return self.grid_h * self.grid_w

    @property
    def capacity(self) -> int:
        """Ring slots: the kv_len cached layers plus the layers of one step."""
        return self.kv_len + self.q_layers

    @property
    def n_query_blocks(self) -> int:
        return self.q_layers * self.blocks_per_layer

    @property
    def n_key_blocks(self) -> int:
        """Key blocks seen by a step in the steady state (cache full)."""
        return self.capacity * self.blocks_per_layer

    def with_topk(self, topk: int) -> "Workload":
        return dataclasses.replace(self, topk=topk, name=f"{self.name.split('@')[0]}@topk{topk}")

    def with_mode(self, local_mode: int) -> "Workload":
        return dataclasses.replace(self, local_mode=local_mode)


def _c4_topk() -> int:
    return topk_for_resolution(0.20, 1536, 2688, 4 * 12 * 21)


WORKLOADS = {
    "tiny": Workload("tiny", heads=2, grid_h=4, grid_w=4, q_layers=2, kv_len=0, topk=8,
                     chunks=1, seed=0, height_px=512, width_px=512),
    "768x1280": Workload("768x1280", heads=12, grid_h=6, grid_w=10, q_layers=1, kv_len=3,
                         topk=24, chunks=1, seed=1, height_px=768, width_px=1280),
    "768x1408": Workload("768x1408", heads=12, grid_h=6, grid_w=11, q_layers=1, kv_len=3,
                         topk=20, chunks=8, seed=2, lowrank=True, height_px=768, width_px=1408),
    "1536x2688": Workload("1536x2688", heads=12, grid_h=12, grid_w=21, q_layers=1, kv_len=3,
                          topk=_c4_topk(), chunks=4, seed=3, height_px=1536, width_px=2688),
    "4k": Workload("4k", heads=12, grid_h=17, grid_w=30, q_layers=1, kv_len=3, topk=16,
                   chunks=4, seed=4, height_px=2176, width_px=3840),
}
FOURK_TOPK_SWEEP = (8, 16, 32)


def kept_tiles(w: Workload) -> int:
    """Kept 128x128 tiles of one steady-state step when every row keeps topk."""
    return w.heads * w.n_query_blocks * w.topk


def flops_per_tile(head_dim: int = HEAD_DIM) -> int:
    """QK^T plus PV over one 128x128 tile: 2 * (2 * 128 * 128 * d)."""
    return 4 * BLOCK_TOKENS * BLOCK_TOKENS * head_dim


# ---------------------------------------------------------------- generators

def _rng(seed: int, position: int, stream: int) -> np.random.Generator:
    return np.random.default_rng([seed * 1000 + position, stream])


def _normal_f32(rng: np.random.Generator, shape) -> np.ndarray:
    return rng.standard_normal(size=shape, dtype=np.float32)


def _block_bias(w: Workload, position: int, stream: int, n_frames: int) -> np.ndarray:
    """Per-block low-rank bias broadcast to token layout [H, T, Ht, Wt, D] (fp32)."""
    basis = _normal_f32(_rng(w.seed, 0, STREAM_BASIS), (w.heads, LOWRANK_RANK, w.head_dim))
    layers = n_frames // BLOCK_T
    coef = _normal_f32(_rng(w.seed, position, stream),
                       (w.heads, layers, w.grid_h, w.grid_w, LOWRANK_RANK))
    per_block = np.einsum("hlyxr,hrd->hlyxd", coef, basis).astype(np.float32)
    per_block *= np.float32(LOWRANK_AMPLITUDE)
    # Broadcast each block vector over its 2 x 8 x 8 tokens.
    b = per_block[:, :, None, :, None, :, None, :]
    b = np.broadcast_to(b, (w.heads, layers, BLOCK_T, w.grid_h, BLOCK_Y, w.grid_w, BLOCK_X, w.head_dim))
    return b.reshape(w.heads, n_frames, w.tok_h, w.tok_w, w.head_dim)


def _to_bf16(x: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(x)).to(torch.bfloat16)


def gen_layers(w: Workload, position: int, n_layers: int, which: str = "qkv") -> List[Optional[torch.Tensor]]:
    """q, k, v of ``n_layers`` block-layers at stream ``position``, bf16 CPU tensors.

    Shapes: [heads, 2*n_layers, tok_h, tok_w, head_dim] (token layout).
    Entries not requested in ``which`` are None.
    """
    n_frames = BLOCK_T * n_layers
    shape = (w.heads, n_frames, w.tok_h, w.tok_w, w.head_dim)
    out: List[Optional[torch.Tensor]] = []
    for name, stream in (("q", STREAM_Q), ("k", STREAM_K), ("v", STREAM_V)):
        if name not in which:
            out.append(None)
            continue
        x = _normal_f32(_rng(w.seed, position, stream), shape)
        if w.lowrank and name in ("q", "k"):
            x += _block_bias(w, position, STREAM_QCOEF if name == "q" else STREAM_KCOEF, n_frames)
        out.append(_to_bf16(x))
    return out


def stream_plan(w: Workload):
    """Positions of a streaming run: prefill positions, then the timed steps.

    The first ``kv_len`` positions only fill the cache (one block-layer
    each); positions kv_len .. kv_len+chunks-1 are the steps proper, each with
    ``q_layers`` layers of q, k and v.
    """
    prefill = list(range(w.kv_len))
    steps = list(range(w.kv_len, w.kv_len + w.chunks))
    return prefill, steps


# ------------------------------------------- segment-masked attention workloads

@dataclasses.dataclass(frozen=True)
class SegmentWorkload:
    """A packed sequence of clips for the segment-masked attention of the
    Stage-1 teacher (reading notes, 关键设计 1): images are clips of one latent
    frame, videos clips of several; every clip is one segment, its tokens
    contiguous in (t, y, x) row-major order.  Every clip must hold a whole
    number of 128-token tiles."""
    name: str
    heads: int
    clips: tuple            # ((latent frames, token rows, token columns), ...)
    seed: int
    head_dim: int = HEAD_DIM

    @property
    def seg_tokens(self):
        return [f * y * x for f, y, x in self.clips]

    @property
    def seg_tiles(self):
        tiles = []
        for n in self.seg_tokens:
            if n % BLOCK_TOKENS:
                raise ValueError(f"{self.name}: a clip of {n} tokens is not a whole number of 128-token tiles")
            tiles.append(n // BLOCK_TOKENS)
        return tiles

    @property
    def tokens(self) -> int:
        return sum(self.seg_tokens)

    @property
    def kept_tiles(self) -> int:
        """Tiles the masked attention computes: every (query tile, key tile) pair of a segment."""
        return self.heads * sum(t * t for t in self.seg_tiles)


SEGMENT_WORKLOADS = {
    # 256x512 px frames: 16 x 32 tokens = 4 tiles per latent frame
    "small": SegmentWorkload("small", heads=2, clips=((1, 16, 32), (3, 16, 32), (1, 16, 32), (2, 16, 32)), seed=5),
    # 768x1280 px frames (48 x 80 tokens = 30 tiles per latent frame): an image, a
    # 5-latent-frame video, an image, a 3-latent-frame video
    "768x1280": SegmentWorkload("768x1280", heads=12,
                                clips=((1, 48, 80), (5, 48, 80), (1, 48, 80), (3, 48, 80)), seed=6),
}


def gen_segments(w: SegmentWorkload) -> List[torch.Tensor]:
    """q, k, v of a packed segment sequence: bf16 CPU tensors [heads, tokens, head_dim],
    i.i.d. N(0,1) drawn in fp32 from ``default_rng([seed * 1000, stream])`` and rounded RNE."""
    out = []
    for stream in (STREAM_Q, STREAM_K, STREAM_V):
        x = _normal_f32(_rng(w.seed, 0, stream), (w.heads, w.tokens, w.head_dim))
        out.append(_to_bf16(x))
    return out


def bf16_to_f64(t: torch.Tensor) -> np.ndarray:
    """Exact upcast of a bf16 tensor to a float64 numpy array."""
    return t.to(torch.float32).numpy().astype(np.float64)


def describe(w: Workload) -> dict:
    return {
        "workload": w.name,
        "heads": w.heads,
        "head_dim": w.head_dim,
        "tokens_per_chunk": [BLOCK_T * w.q_layers, w.tok_h, w.tok_w],
        "query_blocks": w.n_query_blocks,
        "key_blocks": w.n_key_blocks,
        "kv_len": w.kv_len,
        "local_range": w.local_range,
        "local_mode": "preserved" if w.local_mode == 0 else "truncated",
        "topk": w.topk,
        "resolution": f"{w.height_px}x{w.width_px}",
    }


def sqrt_d(d: int = HEAD_DIM) -> float:
    return math.sqrt(d)
