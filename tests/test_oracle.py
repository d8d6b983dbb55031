"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Every function of ``oracle.lcsa_oracle`` is checked here against closed
forms, brute force, library routines or invariants, so that a dropped term,
a wrong sign or index, or a transposed operand fails at least one test.
CPU only.
"""

import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import lcsa_oracle as O
from diffusion_vsr_b200 import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def rnd(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


# ------------------------------------------------------------------ partition

def test_partition_groups_each_window_in_row_major_order():
    H, T, Y, X = 2, 4, 16, 24
    coords = np.zeros((H, T, Y, X, 4))
    for h, t, y, x in itertools.product(range(H), range(T), range(Y), range(X)):
        coords[h, t, y, x] = (h, t, y, x)
    b = O.partition(coords)
    gh, gw = Y // 8, X // 8
    assert b.shape == (H, (T // 2) * gh * gw, 128, 4)
    for h in range(H):
        for blk in range(b.shape[1]):
            layer, rem = divmod(blk, gh * gw)
            by, bx = divmod(rem, gw)
            toks = b[h, blk]
            assert np.all(toks[:, 0] == h)
            assert np.all(toks[:, 1] // 2 == layer)
            assert np.all(toks[:, 2] // 8 == by)
            assert np.all(toks[:, 3] // 8 == bx)
            # the 128 tokens are distinct and in (t, y, x) row-major order
            keys = [tuple(r) for r in toks[:, 1:].astype(int)]
            assert len(set(keys)) == 128
            assert keys == sorted(keys)


def test_partition_round_trip_is_identity():
    x = rnd((3, 6, 16, 32, 8), 1)
    b = O.partition(x)
    assert np.array_equal(O.reverse_partition(b, 6, 16, 32), x)


def test_partition_rejects_ragged_grid():
    with pytest.raises(ValueError):
        O.partition(np.zeros((1, 2, 12, 16, 4)))


# ---------------------------------------------------------------- local mask

@pytest.mark.parametrize("n", [1, 3, 6, 11, 12, 17, 30])
@pytest.mark.parametrize("r", [3, 5, 11])
def test_window_preserved_closed_form(n, r):
    m = O.window_1d(n, r, "preserved")
    h = r // 2
    for i in range(n):
        row = np.nonzero(m[i])[0]
        # exactly min(r, n) contiguous blocks that include the block itself
        assert row.size == min(r, n)
        assert m[i, i]
        assert row[-1] - row[0] + 1 == row.size
        # centred whenever the centred window fits in the grid
        if n > r and h <= i <= n - 1 - h:
            assert row[0] == i - h and row[-1] == i + h
        # otherwise pushed against the nearer edge
        if n > r and i < h:
            assert row[0] == 0
        if n > r and i > n - 1 - h:
            assert row[-1] == n - 1


@pytest.mark.parametrize("n", [1, 4, 11, 21])
@pytest.mark.parametrize("r", [3, 11])
def test_window_truncated_closed_form(n, r):
    m = O.window_1d(n, r, "truncated")
    h = r // 2
    for i in range(n):
        assert m[i].sum() == min(i, h) + min(n - 1 - i, h) + 1
        assert m[i, i]


def test_window_global_when_range_not_positive():
    assert O.window_1d(7, 0, "preserved").all()


@pytest.mark.parametrize("mode", ["preserved", "truncated"])
def test_allowed_mask_counts(mode):
    gh, gw, r = 12, 21, 11
    k_layers, q_layers = 4, 2
    m = O.allowed_mask(q_layers, k_layers, gh, gw, r, mode)
    nb = gh * gw
    assert m.shape == (q_layers * nb, k_layers * nb)
    wy = O.window_1d(gh, r, mode).sum(1)
    wx = O.window_1d(gw, r, mode).sum(1)
    for qi in range(q_layers):
        visible_layers = k_layers - q_layers + qi + 1
        for by in range(gh):
            for bx in range(gw):
                row = m[qi * nb + by * gw + bx]
                assert row.sum() == visible_layers * wy[by] * wx[bx]
                # nothing in a later layer than the query's own
                assert not row[visible_layers * nb:].any()
    if mode == "preserved":
        # closed form: min(r,gh)*min(r,gw) per visible layer
        assert m[0].sum() == (k_layers - q_layers + 1) * min(r, gh) * min(r, gw)


def test_allowed_mask_is_block_causal_across_query_layers():
    m = O.allowed_mask(2, 2, 2, 2, 11, "preserved")
    # first query layer sees only layer 0, second sees both
    assert m[:4, :4].all() and not m[:4, 4:].any()
    assert m[4:].all()


# --------------------------------------------------------------- draft scores

def test_block_means_and_scores_closed_form():
    H, nb, D = 2, 3, 16
    u = rnd((H, nb, D), 2)
    w = rnd((H, nb + 1, D), 3)
    qb = np.repeat(u[:, :, None, :], 128, axis=2)
    kb = np.repeat(w[:, :, None, :], 128, axis=2)
    # zero-mean perturbation per block leaves the mean unchanged
    pert = rnd((H, nb, 128, D), 4)
    pert -= pert.mean(axis=2, keepdims=True)
    mq = O.block_means(qb + pert)
    mk = O.block_means(kb)
    np.testing.assert_allclose(mq, u, rtol=0, atol=1e-13)
    s = O.draft_scores(mq, mk)
    assert s.shape == (H, nb, nb + 1)
    for h in range(H):
        for i in range(nb):
            for j in range(nb + 1):
                expect = sum(u[h, i, d] * w[h, j, d] for d in range(D)) / math.sqrt(D)
                assert abs(s[h, i, j] - expect) < 1e-12


def test_draft_softmax_rows_sum_to_one_and_mask_is_zero():
    s = rnd((2, 8, 16), 5)
    allowed = O.allowed_mask(1, 2, 2, 4, 3, "truncated")
    p = O.draft_softmax(s, allowed)
    np.testing.assert_allclose(p.sum(-1), 1.0, atol=1e-12)
    assert np.all(p[:, ~allowed] == 0)


# ---------------------------------------------------------------------- top-k

def test_topk_ties_go_to_lower_index():
    H, Nq, Nk = 2, 8, 16
    allowed = O.allowed_mask(1, 2, 2, 4, 3, "truncated")
    scores = np.zeros((H, Nq, Nk))  # q == 0 gives all-zero scores
    kept, cnt = O.select_topk(scores, allowed, 3)
    for h in range(H):
        for i in range(Nq):
            cand = np.nonzero(allowed[i])[0]
            assert list(kept[h, i, :cnt[h, i]]) == list(cand[:3])


def test_topk_matches_brute_force_subset_search():
    rng = np.random.default_rng(6)
    for trial in range(30):
        nk = int(rng.integers(3, 10))
        k = int(rng.integers(1, nk + 1))
        scores = rng.standard_normal((1, 1, nk))
        allowed = rng.random((1, nk)) < 0.8
        allowed[0, 0] = True
        kept, cnt = O.select_topk(scores, allowed, k)
        cand = list(np.nonzero(allowed[0])[0])
        kk = min(k, len(cand))
        best = max(itertools.combinations(cand, kk), key=lambda c: sum(scores[0, 0, list(c)]))
        assert sorted(best) == list(kept[0, 0, :cnt[0, 0]])
        assert cnt[0, 0] == kk
        assert np.all(kept[0, 0, cnt[0, 0]:] == -1)


def test_topk_partial_ties_prefer_lower_index():
    scores = np.array([[[1.0, 2.0, 2.0, 0.5, 2.0]]])
    allowed = np.ones((1, 5), dtype=bool)
    kept, cnt = O.select_topk(scores, allowed, 2)
    assert list(kept[0, 0]) == [1, 2]


def test_kept_count_is_min_of_topk_and_allowed():
    allowed = O.allowed_mask(1, 3, 5, 6, 3, "truncated")
    scores = rnd((3, 30, 90), 7)
    for topk in (1, 4, 9, 13, 40):
        _, cnt = O.select_topk(scores, allowed, topk)
        assert np.array_equal(cnt, np.minimum(topk, allowed.sum(1))[None].repeat(3, 0))


def test_near_tie_exemption():
    mq = np.ones((1, 1, 4))
    mk = np.ones((1, 3, 4))
    allowed = np.ones((1, 3), dtype=bool)
    tie = np.array([[[1.0, 0.5, 0.5]]])
    gap = np.array([[[1.0, 0.5, 0.3]]])
    assert O.near_tie_rows(tie, allowed, mq, mk, 2)[0, 0]
    assert not O.near_tie_rows(gap, allowed, mq, mk, 2)[0, 0]
    # allowed <= topk is never exempt
    assert not O.near_tie_rows(tie, allowed, mq, mk, 3)[0, 0]


def test_near_tie_scales_dot_product_bound_versus_plain_scores():
    # k-th and (k+1)-th scores 0.5 and 0.4999 (gap 1e-4).  Plain score scale:
    # 1e-5 * 0.5 = 5e-6 < gap, not exempt.  Dot-product scale: the products
    # mq_d * mk_d are +-100 (they cancel in the score), sum |.| / sqrt(2) = 141.4,
    # 1e-5 * 141.4 = 1.4e-3 > gap, exempt.
    mq = np.ones((1, 1, 2))
    mk = np.array([[[100.0, -100.0], [100.0, -99.0], [100.0, -99.5]]])
    allowed = np.ones((1, 3), dtype=bool)
    s = np.array([[[1.0, 0.5, 0.4999]]])
    assert O.near_tie_rows(s, allowed, mq, mk, 2, scale="dot")[0, 0]
    assert not O.near_tie_rows(s, allowed, mq, mk, 2, scale="score")[0, 0]
    # a gap below 1e-5 of the scores themselves is exempt under both
    s2 = np.array([[[1.0, 0.5, 0.5 - 1e-6]]])
    assert O.near_tie_rows(s2, allowed, mq, mk, 2, scale="score")[0, 0]
    with pytest.raises(ValueError):
        O.near_tie_rows(s, allowed, mq, mk, 2, scale="bogus")


def test_valid_topk_accepts_either_side_of_a_tie_only():
    s = np.array([3.0, 1.0, 1.0, 0.0])
    a = np.ones(4, dtype=bool)
    assert O.valid_topk([0, 1], s, a, 2, 1e-9)
    assert O.valid_topk([0, 2], s, a, 2, 1e-9)
    assert not O.valid_topk([0, 3], s, a, 2, 1e-9)
    assert not O.valid_topk([0], s, a, 2, 1e-9)


# ------------------------------------------------------------------ attention

def _small_stream(H=2, layers=3, gh=2, gw=3, D=16, seed=8):
    Y, X = gh * 8, gw * 8
    k = rnd((H, 2 * layers, Y, X, D), seed)
    v = rnd((H, 2 * layers, Y, X, D), seed + 1)
    q = rnd((H, 2, Y, X, D), seed + 2)
    return q, k, v


def _cache_from(k, v, capacity):
    c = O.KVCacheModel(capacity)
    c.append(k, v)
    return c


def test_sparse_equals_dense_block_causal_when_everything_is_kept():
    q, k, v = _small_stream()
    H, _, Y, X, D = q.shape
    cache = _cache_from(k, v, 3)
    res = O.lcsa_step(q, cache, Y // 8, X // 8, topk=10 ** 6, local_range=0)
    dense = O.dense_block_causal_attention(q, k, v, 1 / math.sqrt(D))
    np.testing.assert_allclose(res["out_tok"], dense, rtol=0, atol=1e-12)
    # window covering the grid gives the same as no window
    res11 = O.lcsa_step(q, cache, Y // 8, X // 8, topk=10 ** 6, local_range=11)
    np.testing.assert_allclose(res11["out_tok"], dense, rtol=0, atol=1e-12)


def test_sparse_equals_library_sdpa_with_block_causal_mask():
    q, k, v = _small_stream(layers=2, gh=2, gw=2, seed=11)
    H, Tq, Y, X, D = q.shape
    # two query layers: the whole chunk attends with the block-causal rule
    q2 = rnd((H, 4, Y, X, D), 12)
    cache = _cache_from(k, v, 2)
    res = O.lcsa_step(q2, cache, Y // 8, X // 8, topk=10 ** 6, local_range=0)
    n = Y * X
    key_layer = np.repeat(np.arange(4) // 2, n)
    q_layer = np.repeat(np.arange(4) // 2, n)
    mask = torch.from_numpy(key_layer[None, :] <= q_layer[:, None])
    qt = torch.from_numpy(q2.reshape(H, 4 * n, D))
    kt = torch.from_numpy(k.reshape(H, 4 * n, D))
    vt = torch.from_numpy(v.reshape(H, 4 * n, D))
    ref = torch.nn.functional.scaled_dot_product_attention(qt, kt, vt, attn_mask=mask).numpy()
    np.testing.assert_allclose(res["out_tok"].reshape(H, 4 * n, D), ref, rtol=0, atol=1e-12)


def test_attention_rows_sum_to_one_and_lse_matches_library():
    from scipy.special import logsumexp
    rng = np.random.default_rng(13)
    qb = rng.standard_normal((128, 32))
    kb = rng.standard_normal((6, 128, 32))
    vb = rng.standard_normal((6, 128, 32))
    kept = [0, 2, 5]
    out, lse, p = O.sparse_attention_row(qb, kb, vb, kept, 0.3, return_probs=True)
    np.testing.assert_allclose(p.sum(1), 1.0, atol=1e-12)
    logits = qb @ kb[kept].reshape(-1, 32).T * 0.3
    np.testing.assert_allclose(lse, logsumexp(logits, axis=1), rtol=1e-13)
    # out is the probability-weighted mean of the kept values, row by row
    vals = vb[kept].reshape(-1, 32)
    for r in (0, 77, 127):
        w = np.exp(logits[r] - logsumexp(logits[r]))
        np.testing.assert_allclose(out[r], (w[:, None] * vals).sum(0), atol=1e-12)


def test_constant_values_give_constant_output():
    rng = np.random.default_rng(14)
    qb = rng.standard_normal((128, 16))
    kb = rng.standard_normal((4, 128, 16))
    vb = np.full((4, 128, 16), 0.375)
    out, _ = O.sparse_attention_row(qb, kb, vb, [1, 3], 0.25)
    np.testing.assert_allclose(out, 0.375, atol=1e-14)


def test_intra_block_permutations():
    rng = np.random.default_rng(15)
    qb = rng.standard_normal((128, 16))
    kb = rng.standard_normal((4, 128, 16))
    vb = rng.standard_normal((4, 128, 16))
    kept = [0, 1, 3]
    out, lse = O.sparse_attention_row(qb, kb, vb, kept, 0.25)
    perm = rng.permutation(128)
    # keys: attention over a set, invariant to their order inside a block
    out_k, _ = O.sparse_attention_row(qb, kb[:, perm], vb[:, perm], kept, 0.25)
    np.testing.assert_allclose(out_k, out, atol=1e-12)
    # queries: output rows follow the permutation
    out_q, lse_q = O.sparse_attention_row(qb[perm], kb, vb, kept, 0.25)
    np.testing.assert_allclose(out_q, out[perm], atol=1e-12)
    np.testing.assert_allclose(lse_q, lse[perm], atol=1e-12)


def test_empty_kept_list_gives_zero_output():
    out, lse = O.sparse_attention_row(np.ones((128, 4)), np.ones((2, 128, 4)), np.ones((2, 128, 4)), [], 1.0)
    assert np.all(out == 0) and np.all(np.isneginf(lse))


def test_sparse_attention_matches_masked_dense_softmax():
    # the kept tiles of a row, written as a dense token mask over all keys
    rng = np.random.default_rng(16)
    q, k, v = _small_stream(H=1, layers=3, gh=3, gw=3, D=16, seed=17)
    cache = _cache_from(k, v, 3)
    res = O.lcsa_step(q, cache, 3, 3, topk=4, local_range=3, mode="truncated")
    qb = O.partition(q)
    kb, vb = cache.keys()
    for i in rng.choice(qb.shape[1], 4, replace=False):
        kept = res["kept_idx"][0, i, :res["kept_cnt"][0, i]]
        tokmask = np.zeros(kb.shape[1] * 128, dtype=bool)
        for j in kept:
            tokmask[j * 128:(j + 1) * 128] = True
        logits = qb[0, i] @ kb[0].reshape(-1, 16).T / 4.0
        logits[:, ~tokmask] = -np.inf
        p = np.exp(logits - logits.max(1, keepdims=True))
        ref = p @ vb[0].reshape(-1, 16) / p.sum(1, keepdims=True)
        np.testing.assert_allclose(res["out_blocks"][0, i], ref, atol=1e-12)


# ------------------------------------------------------------------- RoPE

def _placed(vec, T, Y, X, t, y, x):
    z = np.zeros((1, T, Y, X, vec.size))
    z[0, t, y, x] = vec
    return z


def test_rope_dot_products_depend_only_on_relative_position():
    # q at (t1, y1, x1), k at (t2, y2, x2): moving both by the same offset along
    # every axis (time through frame0, space inside a bigger grid) keeps q.k
    rng = np.random.default_rng(41)
    qv, kv = rng.standard_normal(128), rng.standard_normal(128)
    T, Y, X = 4, 24, 24
    for (t1, y1, x1), (t2, y2, x2), (dt, dy, dx) in [((0, 1, 2), (3, 5, 0), (7, 4, 9)),
                                                    ((2, 0, 0), (0, 7, 7), (1000, 10, 3))]:
        def dot(f0, oy, ox, q_only_y=0):
            qy = y1 + oy + q_only_y
            q = O.apply_rope(_placed(qv, T, Y, X, t1, qy, x1 + ox), f0, 10000.0)
            k = O.apply_rope(_placed(kv, T, Y, X, t2, y2 + oy, x2 + ox), f0, 10000.0)
            return float(q[0, t1, qy, x1 + ox] @ k[0, t2, y2 + oy, x2 + ox])
        base = dot(5, 0, 0)
        assert abs(dot(5 + dt, dy, dx) - base) < 1e-9 * (np.abs(qv).sum() * np.abs(kv).sum())
        # moving the query alone changes it
        assert abs(dot(5, 0, 0, q_only_y=1) - base) > 1e-6


def test_rope_preserves_pair_norms_and_is_identity_at_the_origin():
    rng = np.random.default_rng(42)
    x = rng.standard_normal((2, 2, 8, 16, 128))
    r = O.apply_rope(x, 11, 10000.0)
    np.testing.assert_allclose(np.hypot(r[..., 0::2], r[..., 1::2]), np.hypot(x[..., 0::2], x[..., 1::2]),
                               rtol=1e-12)
    assert not np.allclose(r, x)
    # frame 0, row 0, column 0: every angle is 0
    np.testing.assert_array_equal(O.apply_rope(x, 0, 10000.0)[:, 0, 0, 0], x[:, 0, 0, 0])
    xb = torch.from_numpy(x.astype(np.float32)).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(O.apply_rope(xb, 0, 10000.0, "kernel")[:, 0, 0, 0], xb[:, 0, 0, 0])


def test_rope_pair_is_a_complex_multiplication_with_the_band_frequencies():
    # closed forms of the band layout: 22 + 21 + 21 pairs; inside a band the
    # first pair turns by the position itself and the frequencies fall
    # geometrically by base^(-1/n) down to base^(-(n-1)/n)
    assert [n for _, _, n in O.ROPE_BANDS] == [22, 21, 21]
    assert [p0 for _, p0, _ in O.ROPE_BANDS] == [0, 22, 43]
    rng = np.random.default_rng(43)
    x = rng.standard_normal((1, 3, 8, 8, 128))
    f0, base = 4, 10000.0
    r = O.apply_rope(x, f0, base)
    t, y, xx = 2, 5, 3
    pos = {"t": f0 + t, "y": y, "x": xx}
    for axis, p0, n in O.ROPE_BANDS:
        for i in (0, 1, n - 1):
            w = 1.0 if i == 0 else (base ** (-1.0 / n)) ** i
            z = complex(x[0, t, y, xx, 2 * (p0 + i)], x[0, t, y, xx, 2 * (p0 + i) + 1]) * np.exp(1j * pos[axis] * w)
            assert abs(r[0, t, y, xx, 2 * (p0 + i)] - z.real) < 1e-9
            assert abs(r[0, t, y, xx, 2 * (p0 + i) + 1] - z.imag) < 1e-9


def test_rope_kernel_precision_is_the_exact_rotation_rounded_to_bf16():
    rng = np.random.default_rng(44)
    x = torch.from_numpy(rng.standard_normal((1, 2, 8, 16, 128)).astype(np.float32)).to(torch.bfloat16)
    xf = x.to(torch.float32).numpy()
    exact = O.apply_rope(xf, 9, 10000.0)
    kern = O.apply_rope(xf, 9, 10000.0, "kernel")
    # bf16 values (8 significant bits): within half a bf16 ulp of the exact
    # rotation, plus the fp32 arithmetic before the rounding
    assert np.array_equal(torch.from_numpy(kern).to(torch.bfloat16).to(torch.float32).numpy(), kern)
    tol = np.abs(exact) * 2.0 ** -8 + 1e-6
    assert np.all(np.abs(kern - exact) <= tol)
    with pytest.raises(ValueError):
        O.apply_rope(xf, 0, 10000.0, "bogus")


# -------------------------------------------------- segment-masked attention

def test_segment_ids_follow_the_clips():
    seg = O.segment_ids([(1, 2, 4), (3, 2, 4), (1, 4, 4)])
    assert seg.size == 8 + 24 + 16
    assert np.array_equal(np.bincount(seg), [8, 24, 16])
    assert np.all(np.diff(seg) >= 0)


def test_segment_attention_equals_library_sdpa_with_block_diagonal_mask():
    rng = np.random.default_rng(31)
    seg = O.segment_ids([(1, 4, 8), (2, 4, 8), (1, 2, 8)])
    H, N, D = 2, seg.size, 16
    q, k, v = (rng.standard_normal((H, N, D)) for _ in range(3))
    out, lse = O.segment_attention(q, k, v, seg, 0.25, row_chunk=40)
    mask = torch.from_numpy(seg[:, None] == seg[None, :])
    ref = torch.nn.functional.scaled_dot_product_attention(
        torch.from_numpy(q)[None], torch.from_numpy(k)[None], torch.from_numpy(v)[None], attn_mask=mask,
        scale=0.25)[0].numpy()
    np.testing.assert_allclose(out, ref, atol=1e-12)
    # a subset of query rows gives those rows of the full result
    rows = np.array([0, 5, 47, 63, 64, 100, N - 1])
    o_sub, l_sub = O.segment_attention(q, k, v, seg, 0.25, row_chunk=3, query_rows=rows)
    np.testing.assert_allclose(o_sub, out[:, rows], atol=1e-12)
    np.testing.assert_allclose(l_sub, lse[:, rows], atol=1e-12)
    # lse: log-sum-exp of the row's logits over its own segment only
    from scipy.special import logsumexp
    for h, i in [(0, 0), (1, N - 1), (0, 40), (1, 100)]:
        own = seg == seg[i]
        np.testing.assert_allclose(lse[h, i], logsumexp(q[h, i] @ k[h, own].T * 0.25), atol=1e-12)


def test_segment_attention_is_each_segment_alone():
    # brute force: every segment attended on its own, without any mask
    rng = np.random.default_rng(32)
    clips = [(1, 4, 4), (3, 4, 4), (2, 2, 4)]
    seg = O.segment_ids(clips)
    H, N, D = 1, seg.size, 8
    q, k, v = (rng.standard_normal((H, N, D)) for _ in range(3))
    out, _ = O.segment_attention(q, k, v, seg, 0.5)
    for s in range(len(clips)):
        idx = np.nonzero(seg == s)[0]
        logits = q[0, idx] @ k[0, idx].T * 0.5
        p = np.exp(logits - logits.max(1, keepdims=True))
        np.testing.assert_allclose(out[0, idx], p @ v[0, idx] / p.sum(1, keepdims=True), atol=1e-12)
    # a token changing only another segment's keys/values does not move this segment's output
    k2, v2 = k.copy(), v.copy()
    other = seg == 1
    k2[:, other] += 3.0
    v2[:, other] -= 7.0
    out2, _ = O.segment_attention(q, k2, v2, seg, 0.5)
    np.testing.assert_allclose(out2[:, ~other], out[:, ~other], atol=1e-12)


def test_one_segment_is_plain_dense_attention_and_constant_values_pass_through():
    rng = np.random.default_rng(33)
    H, N, D = 2, 64, 8
    q, k = rng.standard_normal((H, N, D)), rng.standard_normal((H, N, D))
    v = np.full((H, N, D), 2.5)
    out, _ = O.segment_attention(q, k, v, np.zeros(N, dtype=int), 0.3)
    np.testing.assert_allclose(out, 2.5, atol=1e-12)
    v = rng.standard_normal((H, N, D))
    out, _ = O.segment_attention(q, k, v, np.zeros(N, dtype=int), 0.3)
    ref = torch.nn.functional.scaled_dot_product_attention(torch.from_numpy(q), torch.from_numpy(k),
                                                           torch.from_numpy(v), scale=0.3).numpy()
    np.testing.assert_allclose(out, ref, atol=1e-12)


# ------------------------------------------------------------------ KV cache

def test_cache_keeps_newest_layers_and_drops_oldest():
    H, Y, X, D = 1, 8, 8, 2
    cache = O.KVCacheModel(3)
    chunks = []
    for n in range(6):
        k = np.full((H, 2, Y, X, D), float(n))
        cache.append(k, -k)
        chunks.append(n)
        kb, vb = cache.keys()
        expect = chunks[max(0, len(chunks) - 3):]
        assert cache.count == len(expect)
        assert [kb[0, l, 0, 0] for l in range(cache.count)] == expect
        assert np.array_equal(vb, -kb)


def test_cache_multi_layer_append_splits_layers():
    cache = O.KVCacheModel(4)
    k = np.concatenate([np.full((1, 2, 8, 16, 2), 1.0), np.full((1, 2, 8, 16, 2), 2.0)], axis=1)
    cache.append(k, k)
    assert cache.count == 2
    kb, _ = cache.keys()
    assert np.all(kb[0, :2] == 1.0) and np.all(kb[0, 2:] == 2.0)


# ----------------------------------------------------------- page facts / configs

def test_page_facts_golden():
    with open(os.path.join(GOLDEN, "page_facts.json")) as f:
        facts = json.load(f)
    g = facts["geometry"]
    assert int(np.prod(g["block"])) == g["tokens_per_block"] == W.BLOCK_TOKENS
    assert g["px_per_block_side"] == 8 * g["px_per_token"]
    assert (g["local_range_blocks"] // 2) * g["px_per_block_side"] == g["local_half_extent_px"]
    for res in facts["resolutions"]:
        w = W.WORKLOADS[res["workload"]]
        assert w.tok_h == res["height_px"] // g["px_per_token"]
        assert w.tok_w == res["width_px"] // g["px_per_token"]
        assert w.blocks_per_layer == res["blocks_per_layer"]
    t = facts["topk_scaling"]
    assert W.topk_for_resolution(t["sparse_ratio"], *t["resolution"], t["n_keys"]) == t["topk"]
    assert W.WORKLOADS["1536x2688"].topk == t["topk"]
    # the formula leaves the 768x1280 base at the base ratio: 20% of 240
    assert W.topk_for_resolution(0.2, 768, 1280, 240) == 48
