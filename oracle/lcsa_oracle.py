"""Plain fp64 CPU oracle of locality-constrained sparse attention (LCSA).

TEST INFRASTRUCTURE ONLY.  Nothing on the product path may import, call or
run this module: only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline / reference arm of ``bench.py`` use it.  It shares no code with the
CUDA library; both sides only share the seeded input generators.

What it computes, step by step, in the order of the sources:

* FlashVSR code walk-through, page "FlashVSR 是怎么工作的" (vsr-hover-compare
  learn.html), section 2.2 "局部约束稀疏注意力 (LCSA)": window partition into
  (2,8,8) blocks, the local block mask, block mean pooling, draft scores
  ``einsum(q, k) / sqrt(D)``, masking with -inf, softmax, top-k, and
  block-sparse attention with the original Q, K, V on the kept block pairs.
* Same page, section 2.3 "流式处理 + KV 缓存": the cache keeps the newest
  ``kv_len`` block-layers and drops the oldest.
* Reading notes "FlashVSR: Towards Real-time Diffusion-Based Streaming Video
  Super Resolution" (papernotes.org), 关键设计 1: causal mask (each latent sees
  only the current and past ones); 关键设计 2: (2,8,8) blocks, block-level
  pooled attention map, full 128x128 attention on the top-k block pairs;
  关键设计 3: the mask is computed inside a local window, with the two edge
  rules Boundary-Preserved and Boundary-Truncated.

Readings where the pages are silent or garbled (the same list is kept in the
design notes):

* Boundary-Preserved = the window of ``r`` blocks is shifted to stay inside
  the grid: start = clamp(i - r//2, 0, n - r); every block is visible when
  n <= r.  Boundary-Truncated = |i - j| <= r//2.  ``r <= 0`` means no window.
* The same spatial window applies to every key layer; block-causal means a
  key block in a later block-layer than the query block is masked.
* Top-k keeps exactly min(topk, allowed) blocks per (head, query block), the
  largest scores first, ties to the lower key index (the printed
  threshold-on-the-(k+1)-th-value line is garbled).  Selection uses the raw
  scores; the draft softmax is monotone and only computed for checks.
* The attention scale is 1/sqrt(D), the same as the draft scale.
* Intra-block token order is (t, y, x) row-major.
* Rotary position embedding (RoPE), which the reading notes name (背景,
  关键设计 3) as the relative position code whose periodicity the local
  window contains, with no layout: each adjacent pair of dimensions (2i,
  2i+1) of q and k is rotated by the angle pos * w; the 64 pairs of a 128-dim
  head are split into three axis bands over the token coordinates, time
  (pairs 0-21), rows (22-42) and columns (43-63); inside a band of n pairs
  w_i = base^(-i/n), base 10000; the time position is the absolute latent
  frame index in the stream, the row/column positions the token row/column.
  The rotated q and k are bf16 tensors (the attention's inputs): the rotation
  is taken in the kernel's precision (fp32 cos/sin rounded from fp64, fp32
  products and sum, one rounding each) and rounded to bf16 (nearest even),
  because that rounding decides the bf16 values everything after is computed
  from.
* Segment-masked attention (the Stage-1 teacher of the reading notes'
  关键设计 1): a packed sequence of segments, each one clip (a video, or an
  image as a single-frame video), its tokens contiguous and in the clip's
  (t, y, x) row-major order; the attention is dense within a segment and
  there is none across segments (the block-diagonal mask of the alpha_ij
  equation).  No causal rule applies in that stage.

Parity: every function below is pinned by ``tests/test_oracle.py`` against
closed forms, brute force and library routines; none is "parity unpinned".
"""

from __future__ import annotations

import math
from collections import deque
from typing import Dict, Iterable, List, Optional, Sequence, Tuple

import numpy as np

BLOCK = (2, 8, 8)
BLOCK_TOKENS = 128


# ----------------------------------------------------------------- partition

def partition(x: np.ndarray) -> np.ndarray:
    """WindowPartition3D.partition(x, (2,8,8)) of the code walk-through, 2.2.

    x: [H, T, Y, X, D] token layout  ->  [H, n_blocks, 128, D].
    Block id = layer * (Y/8 * X/8) + by * (X/8) + bx; token id inside the
    block = (t % 2) * 64 + (y % 8) * 8 + (x % 8).
    """
    H, T, Y, X, D = x.shape
    bt, by, bx = BLOCK
    if T % bt or Y % by or X % bx:
        raise ValueError("token grid must be a multiple of the (2,8,8) block")
    v = x.reshape(H, T // bt, bt, Y // by, by, X // bx, bx, D)
    v = v.transpose(0, 1, 3, 5, 2, 4, 6, 7)
    return np.ascontiguousarray(v.reshape(H, (T // bt) * (Y // by) * (X // bx), BLOCK_TOKENS, D))


def reverse_partition(b: np.ndarray, T: int, Y: int, X: int) -> np.ndarray:
    """Inverse of ``partition``: [H, n_blocks, 128, D] -> [H, T, Y, X, D]."""
    H, nb, n, D = b.shape
    bt, by, bx = BLOCK
    v = b.reshape(H, T // bt, Y // by, X // bx, bt, by, bx, D)
    v = v.transpose(0, 1, 4, 2, 5, 3, 6, 7)
    return np.ascontiguousarray(v.reshape(H, T, Y, X, D))


# ---------------------------------------------------------------- draft mask

def block_means(blocks: np.ndarray) -> np.ndarray:
    """avgpool over the 128 tokens of each block (code walk-through 2.2)."""
    return blocks.astype(np.float64).mean(axis=2)


def window_1d(n: int, r: int, mode: str) -> np.ndarray:
    """Bool [n, n]: may block i see block j along one axis of the block grid.

    Local block mask of the code walk-through 2.2 (default local_range 11,
    include_self) under the two edge rules named in the reading notes'
    关键设计 3 (see the module docstring for the reading).
    """
    i = np.arange(n)[:, None]
    j = np.arange(n)[None, :]
    if r <= 0:
        return np.ones((n, n), dtype=bool)
    h = r // 2
    if mode == "preserved":
        if n <= r:
            return np.ones((n, n), dtype=bool)
        start = np.clip(i - h, 0, n - r)
        return (j >= start) & (j < start + r)
    if mode == "truncated":
        return np.abs(i - j) <= h
    raise ValueError(mode)


def allowed_mask(q_layers: int, k_layers: int, grid_h: int, grid_w: int,
                 local_range: int, mode: str) -> np.ndarray:
    """Bool [Nq, Nk]: local window AND block-causal (reading notes 关键设计 1, 3).

    The queries are the newest ``q_layers`` of the ``k_layers`` key layers;
    query layer qi sits at key layer (k_layers - q_layers + qi) and sees key
    layers up to and including that one.
    """
    wy = window_1d(grid_h, local_range, mode)
    wx = window_1d(grid_w, local_range, mode)
    spatial = (wy[:, None, :, None] & wx[None, :, None, :]).reshape(grid_h * grid_w, grid_h * grid_w)
    q_abs = (k_layers - q_layers) + np.arange(q_layers)
    layer_ok = np.arange(k_layers)[None, :] <= q_abs[:, None]
    m = layer_ok[:, None, :, None] & spatial[None, :, None, :]
    return m.reshape(q_layers * grid_h * grid_w, k_layers * grid_h * grid_w)


def draft_scores(mq: np.ndarray, mk: np.ndarray) -> np.ndarray:
    """einsum("hld,hmd->hlm", q, k) / sqrt(D) on the pooled vectors (2.2)."""
    d = mq.shape[-1]
    return np.einsum("hld,hmd->hlm", mq, mk) / math.sqrt(d)


def masked_scores(scores: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """scores + local mask: -inf outside the allowed set (2.2)."""
    return np.where(allowed[None], scores, -np.inf)


def draft_softmax(scores: np.ndarray, allowed: np.ndarray) -> np.ndarray:
    """attn_map = softmax(scores + mask, dim=-1) (2.2); checks only."""
    s = masked_scores(scores, allowed)
    m = s.max(axis=-1, keepdims=True)
    e = np.exp(s - m)
    return e / e.sum(axis=-1, keepdims=True)


def select_topk(scores: np.ndarray, allowed: np.ndarray, topk: int) -> Tuple[np.ndarray, np.ndarray]:
    """Keep min(topk, allowed) key blocks per (head, query block).

    Order: larger score first, ties to the lower key index.  Returns
    kept_idx [H, Nq, topk] int32 (ascending, padded with -1) and
    kept_cnt [H, Nq] int32.
    """
    H, Nq, Nk = scores.shape
    kept = np.full((H, Nq, max(topk, 0)), -1, dtype=np.int32)
    cnt = np.zeros((H, Nq), dtype=np.int32)
    for h in range(H):
        for i in range(Nq):
            cand = np.nonzero(allowed[i])[0]
            order = np.lexsort((cand, -scores[h, i, cand]))  # primary: -score, secondary: index
            take = np.sort(cand[order[:min(topk, cand.size)]])
            kept[h, i, :take.size] = take
            cnt[h, i] = take.size
    return kept, cnt


# ------------------------------------------------------------ sparse attention

def sparse_attention_row(q_blk: np.ndarray, k_blocks: np.ndarray, v_blocks: np.ndarray,
                         kept: Sequence[int], scale: float, return_probs: bool = False):
    """Exact softmax(q k^T * scale) V over the tokens of the kept key blocks.

    block_sparse_attn_func of the code walk-through 2.2: full 128x128
    attention with the original Q, K, V, only for the kept block pairs
    (reading notes 关键设计 2).  q_blk [128, D]; k_blocks/v_blocks
    [Nk, 128, D] of one head.  Returns (out [128, D], lse [128]) and the
    probability matrix when asked.  An empty kept list gives zeros and -inf.
    """
    kept = list(kept)
    q_blk = np.asarray(q_blk, dtype=np.float64)
    if not kept:
        out = np.zeros_like(q_blk, dtype=np.float64)
        lse = np.full(q_blk.shape[0], -np.inf)
        return (out, lse, None) if return_probs else (out, lse)
    keys = k_blocks[kept].reshape(-1, k_blocks.shape[-1]).astype(np.float64)
    vals = v_blocks[kept].reshape(-1, v_blocks.shape[-1]).astype(np.float64)
    logits = (q_blk @ keys.T) * scale
    m = logits.max(axis=1, keepdims=True)
    p = np.exp(logits - m)
    l = p.sum(axis=1, keepdims=True)
    out = (p @ vals) / l
    lse = (m + np.log(l))[:, 0]
    if return_probs:
        return out, lse, p / l
    return out, lse


def sparse_attention(qb: np.ndarray, kb: np.ndarray, vb: np.ndarray, kept_idx: np.ndarray,
                     kept_cnt: np.ndarray, scale: float,
                     rows: Optional[Iterable[Tuple[int, int]]] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Block-sparse attention over all (or the listed) (head, query block) rows.

    qb [H, Nq, 128, D], kb/vb [H, Nk, 128, D] fp64.  Returns out
    [H, Nq, 128, D] and lse [H, Nq, 128]; rows not computed stay NaN.
    """
    H, Nq = qb.shape[:2]
    out = np.full(qb.shape, np.nan)
    lse = np.full(qb.shape[:3], np.nan)
    if rows is None:
        rows = [(h, i) for h in range(H) for i in range(Nq)]
    for h, i in rows:
        o, s = sparse_attention_row(qb[h, i], kb[h], vb[h], kept_idx[h, i, :kept_cnt[h, i]], scale)
        out[h, i] = o
        lse[h, i] = s
    return out, lse


def dense_block_causal_attention(q_tok: np.ndarray, k_tok: np.ndarray, v_tok: np.ndarray,
                                 scale: float) -> np.ndarray:
    """Brute-force dense attention with the block-causal rule, in token layout.

    q_tok [H, Tq, Y, X, D] are the newest Tq frames of k_tok/v_tok
    [H, Tk, Y, X, D].  A query token of frame t sees every key token whose
    block-layer (frame // 2) is not later than its own.  No partition is used.
    """
    H, Tq, Y, X, D = q_tok.shape
    Tk = k_tok.shape[1]
    q = q_tok.reshape(H, Tq, Y * X, D)
    k = k_tok.reshape(H, Tk * Y * X, D)
    v = v_tok.reshape(H, Tk * Y * X, D)
    key_layer = np.repeat(np.arange(Tk) // 2, Y * X)
    out = np.empty((H, Tq, Y * X, D))
    for h in range(H):
        for t in range(Tq):
            q_layer = (Tk - Tq + t) // 2
            vis = key_layer <= q_layer
            logits = (q[h, t] @ k[h, vis].T) * scale
            p = np.exp(logits - logits.max(axis=1, keepdims=True))
            out[h, t] = (p @ v[h, vis]) / p.sum(axis=1, keepdims=True)
    return out.reshape(H, Tq, Y, X, D)


# ------------------------------------------------------------------- RoPE

ROPE_BANDS = (("t", 0, 22), ("y", 22, 21), ("x", 43, 21))  # (axis, first pair, pairs) of a 128-dim head


def rope_angles(positions: np.ndarray, n_pairs: int, base: float) -> np.ndarray:
    """Angles pos * w_i, w_i = base^(-i / n_pairs), i < n_pairs, in fp64: [len(positions), n_pairs]."""
    w = np.power(float(base), -np.arange(n_pairs, dtype=np.float64) / n_pairs)
    return np.asarray(positions, dtype=np.float64)[:, None] * w[None, :]


def apply_rope(x_tok: np.ndarray, frame0: int, base: float, precision: str = "exact") -> np.ndarray:
    """Rotate every dimension pair of a token-layout tensor [H, T, Y, X, 128].

    Pair (2i, 2i+1) of the token at (frame t, row y, column x) turns by the
    angle of its band's coordinate: (frame0 + t), y or x times w_i.
    precision "exact": fp64 arithmetic, no rounding.  "kernel": cos and sin
    rounded to fp32, a' = fl(fl(a cos) - fl(b sin)), b' = fl(fl(a sin) + fl(b cos))
    in fp32, then rounded to bf16 (round to nearest even); returned as fp32
    holding the bf16 values.
    """
    if precision not in ("exact", "kernel"):
        raise ValueError(precision)
    H, T, Y, X, D = x_tok.shape
    if D != 128:
        raise ValueError("the band layout is that of a 128-dim head")
    pos = {"t": np.arange(T) + frame0, "y": np.arange(Y), "x": np.arange(X)}
    shape = {"t": (1, T, 1, 1), "y": (1, 1, Y, 1), "x": (1, 1, 1, X)}
    if precision == "exact":
        out = np.array(x_tok, dtype=np.float64)
    else:
        out = np.array(x_tok, dtype=np.float32)
    for axis, p0, n in ROPE_BANDS:
        ang = rope_angles(pos[axis], n, base)  # [len, n]
        c, s = np.cos(ang), np.sin(ang)
        if precision == "kernel":
            c, s = c.astype(np.float32), s.astype(np.float32)
        for i in range(n):
            d = 2 * (p0 + i)
            ci = c[:, i].reshape(shape[axis])
            si = s[:, i].reshape(shape[axis])
            a = out[..., d].copy()
            b = out[..., d + 1].copy()
            out[..., d] = a * ci - b * si
            out[..., d + 1] = a * si + b * ci
    if precision == "kernel":
        import torch
        out = torch.from_numpy(out).to(torch.bfloat16).to(torch.float32).numpy()
    return out


# ------------------------------------------------------ segment-masked attention

def segment_ids(clips: Sequence[Tuple[int, int, int]]) -> np.ndarray:
    """Segment id of every token of a packed sequence of clips.

    clips: (latent frames, token rows, token columns) per clip, in sequence
    order; an image is a clip of one frame (reading notes, 关键设计 1: images
    are single-frame videos).  Clip s contributes f*Y*X consecutive tokens of
    id s.
    """
    return np.concatenate([np.full(f * y * x, s, dtype=np.int64) for s, (f, y, x) in enumerate(clips)])


def segment_attention(q: np.ndarray, k: np.ndarray, v: np.ndarray, seg: np.ndarray, scale: float,
                      row_chunk: int = 128, query_rows: Optional[np.ndarray] = None) -> Tuple[np.ndarray, np.ndarray]:
    """Dense attention under the block-diagonal segment mask (关键设计 1):

        alpha_ij = exp(q_i k_j^T * scale) 1[seg(i) = seg(j)]
                   / sum_l exp(q_i k_l^T * scale) 1[seg(i) = seg(l)],
        out_i = sum_j alpha_ij v_j.

    q, k, v: [H, N, D] (any float dtype holding exact values; arithmetic in
    fp64); seg: [N] segment id per token.  The query rows are taken
    ``row_chunk`` at a time, each row's softmax over all N keys with the mask.
    Returns out [H, N, D] and the natural-log denominator lse [H, N]; with
    ``query_rows`` (token indices) only those rows: out [H, len, D], lse [H, len].
    """
    H, N, D = q.shape
    seg = np.asarray(seg)
    rows = np.arange(N) if query_rows is None else np.asarray(query_rows)
    out = np.empty((H, rows.size, D))
    lse = np.empty((H, rows.size))
    for h in range(H):
        kh = k[h].astype(np.float64)
        vh = v[h].astype(np.float64)
        for r0 in range(0, rows.size, row_chunk):
            sel = rows[r0:r0 + row_chunk]
            qr = q[h, sel].astype(np.float64)
            logits = (qr @ kh.T) * scale
            same = seg[sel, None] == seg[None, :]
            logits = np.where(same, logits, -np.inf)
            m = logits.max(axis=1, keepdims=True)
            p = np.exp(logits - m)
            l = p.sum(axis=1, keepdims=True)
            out[h, r0:r0 + row_chunk] = (p @ vh) / l
            lse[h, r0:r0 + row_chunk] = (m + np.log(l))[:, 0]
    return out, lse


# -------------------------------------------------------------- KV cache model

class KVCacheModel:
    """Streaming KV cache of the code walk-through, section 2.3.

    Holds partitioned k/v block-layers ([H, blocks_per_layer, 128, D] each),
    oldest first.  ``capacity`` = kv_len cached layers + the layers of one
    step; appending beyond it drops the oldest layer.
    """

    def __init__(self, capacity: int):
        self.layers: deque = deque(maxlen=capacity)
        self.capacity = capacity

    def append(self, k_tok: np.ndarray, v_tok: np.ndarray) -> None:
        """Append every block-layer of a token-layout chunk [H, 2L, Y, X, D]."""
        kb = partition(k_tok)
        vb = partition(v_tok)
        n_layers = k_tok.shape[1] // 2
        per = kb.shape[1] // n_layers
        for l in range(n_layers):
            self.layers.append((kb[:, l * per:(l + 1) * per], vb[:, l * per:(l + 1) * per]))

    @property
    def count(self) -> int:
        return len(self.layers)

    def keys(self) -> Tuple[np.ndarray, np.ndarray]:
        """Resident k and v blocks, oldest layer first: [H, count*per, 128, D]."""
        return (np.concatenate([k for k, _ in self.layers], axis=1),
                np.concatenate([v for _, v in self.layers], axis=1))


# --------------------------------------------------------------- whole step

def lcsa_step(q_tok: np.ndarray, cache: KVCacheModel, grid_h: int, grid_w: int, topk: int,
              local_range: int = 11, mode: str = "preserved", scale: Optional[float] = None,
              rows: Optional[Iterable[Tuple[int, int]]] = None,
              kept_override: Optional[Tuple[np.ndarray, np.ndarray]] = None) -> Dict[str, np.ndarray]:
    """One LCSA step after the chunk's k/v were appended to ``cache``.

    q_tok [H, 2*q_layers, 8*grid_h, 8*grid_w, D].  Returns the draft scores,
    the allowed mask, the kept lists and (for ``rows`` or every row) the
    output in token layout plus lse.  ``kept_override`` replaces the draft
    selection (used to feed a given mask to the attention step).
    """
    H, Tq, Y, X, D = q_tok.shape
    q_layers = Tq // 2
    if scale is None:
        scale = 1.0 / math.sqrt(D)
    qb = partition(q_tok)
    kb, vb = cache.keys()  # any float dtype holding exact values; arithmetic below is fp64
    k_layers = cache.count
    mq = block_means(qb)
    mk = block_means(kb)
    scores = draft_scores(mq, mk)
    allowed = allowed_mask(q_layers, k_layers, grid_h, grid_w, local_range, mode)
    if kept_override is None:
        kept_idx, kept_cnt = select_topk(scores, allowed, topk)
    else:
        kept_idx, kept_cnt = kept_override
    out_b, lse_b = sparse_attention(qb, kb, vb, kept_idx, kept_cnt, scale, rows)
    return {
        "mq": mq, "mk": mk, "scores": scores, "allowed": allowed,
        "kept_idx": kept_idx, "kept_cnt": kept_cnt,
        "out_blocks": out_b, "lse_blocks": lse_b,
        "out_tok": reverse_partition(out_b, Tq, Y, X),
        "lse_tok": reverse_partition(lse_b[..., None], Tq, Y, X)[..., 0],
    }


def near_tie_rows(scores: np.ndarray, allowed: np.ndarray, mq: np.ndarray, mk: np.ndarray,
                  topk: int, rel: float = 1e-5, scale: str = "dot") -> np.ndarray:
    """Bool [H, Nq]: rows whose top-k boundary is within fp32 noise.

    A row is exempt from the bit-exact mask comparison when its k-th and
    (k+1)-th largest allowed scores differ by at most ``rel`` times a
    magnitude scale of those two scores.  ``scale="dot"`` (used for the
    acceptance test) takes the scale that bounds the rounding error of a dot
    product, sum_d |mq_d * mk_d| / sqrt(D), the larger of the two blocks (and
    at least the scores' magnitudes); ``scale="score"`` takes the plain
    max(|s_k|, |s_k+1|), reported beside it.  Rows with allowed <= topk are
    never exempt.
    """
    if scale not in ("dot", "score"):
        raise ValueError(scale)
    H, Nq, Nk = scores.shape
    d = mq.shape[-1]
    out = np.zeros((H, Nq), dtype=bool)
    for h in range(H):
        for i in range(Nq):
            cand = np.nonzero(allowed[i])[0]
            if cand.size <= topk:
                continue
            order = np.lexsort((cand, -scores[h, i, cand]))
            a, b = cand[order[topk - 1]], cand[order[topk]]
            sa, sb = scores[h, i, a], scores[h, i, b]
            mag = max(abs(sa), abs(sb))
            if scale == "dot":
                mag = max(mag, np.abs(mq[h, i] * mk[h, a]).sum() / math.sqrt(d),
                          np.abs(mq[h, i] * mk[h, b]).sum() / math.sqrt(d))
            out[h, i] = abs(sa - sb) <= rel * mag
    return out


def valid_topk(kept: Sequence[int], scores_row: np.ndarray, allowed_row: np.ndarray, topk: int,
               tol: float) -> bool:
    """Is ``kept`` a top-k of the allowed scores up to an absolute tolerance?

    Used for near-tie rows, where several sets are correct: the count must be
    min(topk, allowed), every kept block allowed, and no dropped allowed
    block may beat a kept one by more than ``tol``.
    """
    kept = np.asarray(kept)
    cand = np.nonzero(allowed_row)[0]
    if kept.size != min(topk, cand.size) or np.unique(kept).size != kept.size:
        return False
    if not np.all(allowed_row[kept]):
        return False
    dropped = np.setdiff1d(cand, kept)
    if dropped.size == 0:
        return True
    return scores_row[dropped].max() <= scores_row[kept].min() + tol
