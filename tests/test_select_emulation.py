"""CPU check of the selection algorithm the draft-mask kernel uses for its top-k.

The kernel maps each fp32 score to a 32-bit key whose unsigned ascending order
is the descending score order (-0 folded onto +0), finds the k-th smallest key
T with an 8-bit radix select of up to four passes that stops after the pass
whose bin holding the k-th key is kept whole, and keeps every key < T plus the
first keys equal to T in ascending candidate index.  This file restates those
steps in Python, bit for bit, and checks them against a plain sort on
(-score, index) — the selection rule of the draft mask (ties to the lower
index) — on random, tie-heavy and signed-zero inputs.  It exercises the method,
not the CUDA code (the GPU parity tests do that).
"""

import numpy as np
import pytest

INT_MAX = 2**31 - 1


def desc_key(score: np.float32) -> int:
    u = int(np.float32(score).view(np.uint32))
    if u == 0x80000000:
        u = 0
    ordered = (~u & 0xFFFFFFFF) if (u & 0x80000000) else (u | 0x80000000)
    return ~ordered & 0xFFFFFFFF


def radix_select(keys, k):
    """(T, keys equal to T to keep, passes) as the kernel computes them."""
    prefix, mask, k_rem, passes = 0, 0, k, 0
    for p in range(4):
        passes += 1
        shift = 24 - 8 * p
        hist = [0] * 256
        for key in keys:
            if (key & mask) == prefix:
                hist[(key >> shift) & 255] += 1
        run = 0
        for d in range(256):
            if run + hist[d] >= k_rem:
                below, digit, whole = run, d, run + hist[d] == k_rem
                break
            run += hist[d]
        k_rem -= below
        prefix |= digit << shift
        mask |= 255 << shift
        if whole:
            return prefix | ((1 << shift) - 1), INT_MAX, passes
    return prefix, k_rem, passes


def select(scores, k):
    keys = [desc_key(s) for s in scores]
    T, k_eq, passes = radix_select(keys, k)
    kept, eq_seen = [], 0
    for c, key in enumerate(keys):
        if key < T:
            kept.append(c)
        elif key == T:
            if eq_seen < k_eq:
                kept.append(c)
            eq_seen += 1
    return kept, passes


def reference(scores, k):
    order = np.lexsort((np.arange(len(scores)), -scores.astype(np.float64)))
    return sorted(order[:k].tolist())


def test_key_order_is_descending_score_order():
    vals = np.array([np.inf, 3.5, 1.0, 1e-30, 0.0, -0.0, -1e-30, -1.0, -7.25, -np.inf], dtype=np.float32)
    keys = [desc_key(v) for v in vals]
    assert keys[4] == keys[5]  # -0 ties with +0
    rest = keys[:5] + keys[6:]
    assert all(a < b for a, b in zip(rest, rest[1:]))


@pytest.mark.parametrize("mode", ["normal", "ties", "zeros", "draft_like"])
def test_radix_select_keeps_the_top_k_with_ties_to_the_lower_index(mode):
    rng = np.random.default_rng({"normal": 0, "ties": 1, "zeros": 2, "draft_like": 3}[mode])
    for _ in range(300):
        n = int(rng.integers(1, 600))
        k = int(rng.integers(1, n + 1))
        if mode == "normal":
            s = rng.standard_normal(n).astype(np.float32)
        elif mode == "ties":
            s = rng.integers(-3, 3, n).astype(np.float32)
        elif mode == "zeros":
            s = (rng.standard_normal(n) * 1e-3).astype(np.float32)
            s[rng.random(n) < 0.3] = -0.0
            s[rng.random(n) < 0.2] = 0.0
        else:
            s = (0.3 + 0.05 * rng.standard_normal(n)).astype(np.float32)
            k = min(k, 20)
        kept, _ = select(s, k)
        assert kept == reference(s, k)


def test_all_scores_equal_keep_the_lowest_indices():
    s = np.zeros(264, dtype=np.float32)
    kept, passes = select(s, 20)
    assert kept == list(range(20))
    assert passes == 4  # one bin holds every key at every digit: no early stop


def test_early_stop_on_draft_like_scores():
    rng = np.random.default_rng(7)
    passes = [select((0.3 + 0.05 * rng.standard_normal(264)).astype(np.float32), 20)[1] for _ in range(200)]
    assert max(passes) <= 4 and np.mean(passes) < 3.5
