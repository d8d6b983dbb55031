"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Acceptance: the kept block set is bit-exact except on near-tie rows (which
must still be a valid top-k); outputs fed the oracle's own mask are within
max-abs 2e-2 and relative L2 5e-3 of the fp64 oracle; the ring holds exactly
the partitioned layers; block means within 1e-6 relative.
"""

import math

import numpy as np
import pytest
import torch

from diffusion_vsr_b200 import workloads as W
from oracle import lcsa_oracle as O
from tests import harness as Hn

pytestmark = pytest.mark.gpu


def _lib():
    from diffusion_vsr_b200 import lcsa
    return lcsa


def _check_step(res, w):
    ref = res.oracle
    assert res.status == 0, _lib().status_string(res.status)
    # q block means and fp32 draft scores against fp64
    np.testing.assert_allclose(res.gpu_qmean, ref["mq"], rtol=1e-6, atol=1e-7)
    allowed = ref["allowed"]
    gs = res.gpu_scores
    assert np.all(np.isneginf(gs[:, ~allowed]))
    mag = (np.linalg.norm(ref["mq"], axis=-1)[:, :, None] * np.linalg.norm(ref["mk"], axis=-1)[:, None, :]
           / math.sqrt(128))
    err = np.abs(gs - ref["scores"])[:, allowed]
    assert np.all(err <= 1e-5 * mag[:, allowed] + 1e-9)
    # kept sets
    exact, exempt, bad = Hn.check_mask(res, w)
    print(f"[parity] {w.name} position {res.position}: {exact + exempt} rows, {exact} compared bit-exactly, "
          f"{exempt} near-tie exempt (dot-product scale; {res.exempt_score_scale} under the plain score scale), "
          f"{len(res.rows)} attention rows against fp64")
    assert bad == 0, f"{bad} rows differ ({exact} exact, {exempt} near-tie)"
    assert exempt <= Hn.MAX_EXEMPT_FRAC * (exact + exempt), (exempt, exact)
    # attention with the oracle's mask
    hs, iis = zip(*res.rows)
    g = res.out_oracle_mask[list(hs), list(iis)]
    o = ref["out_blocks"][list(hs), list(iis)]
    mx, rl2 = Hn.compare_outputs(g, o)
    assert mx <= Hn.ATOL_OUT and rl2 <= Hn.RTOL_L2_OUT, (mx, rl2)
    lse_g = res.lse_oracle_mask[list(hs), list(iis)]
    lse_o = ref["lse_blocks"][list(hs), list(iis)]
    assert np.max(np.abs(lse_g - lse_o)) <= 2e-3
    # the full pipeline equals the oracle-mask run bit for bit where the masks agree
    same = np.all(res.gpu_kept == ref["kept_idx"], axis=-1) & (res.gpu_cnt == ref["kept_cnt"])
    assert np.array_equal(res.out_pipeline[same], res.out_oracle_mask[same])
    return mx, rl2


def test_tiny_full_parity_with_ring():
    w = W.WORKLOADS["tiny"]
    (res,) = Hn.run_stream(w, check_ring=True)
    assert res.ring_ok and res.kmean_err <= 1e-6
    _check_step(res, w)


def test_tiny_dense_equivalence_when_everything_is_kept():
    # topk >= allowed and the window covers the grid: the CUDA path must equal
    # dense block-causal attention.
    w = W.WORKLOADS["tiny"].with_topk(32)
    (res,) = Hn.run_stream(w)
    assert np.all(res.gpu_cnt[:, :16] == 16) and np.all(res.gpu_cnt[:, 16:] == 32)
    _check_step(res, w)
    q, k, v = W.gen_layers(w, 0, w.q_layers)
    dense = O.dense_block_causal_attention(Hn.f32(q), Hn.f32(k), Hn.f32(v), 1 / math.sqrt(128))
    mx, rl2 = Hn.compare_outputs(res.out_pipeline, O.partition(dense))
    assert mx <= Hn.ATOL_OUT and rl2 <= Hn.RTOL_L2_OUT


def test_768x1280_full_parity():
    w = W.WORKLOADS["768x1280"]
    (res,) = Hn.run_stream(w, check_ring=True)
    assert res.ring_ok and res.kmean_err <= 1e-6
    _check_step(res, w)


def test_768x1408_streaming_eight_chunks():
    # every row of all 8 chunks; from the second chunk on the oldest layer is dropped
    w = W.WORKLOADS["768x1408"]
    seen = []

    def check(res):
        assert res.ring_ok and res.kmean_err <= 1e-6
        assert len(res.rows) == w.heads * w.n_query_blocks
        _check_step(res, w)
        seen.append(res.position)

    Hn.run_stream(w, check_ring=True, on_step=check)
    assert len(seen) == 8


def test_1536x2688_all_rows_with_eviction():
    # two chunks, every row; the second chunk's append drops the oldest layer
    w = W.WORKLOADS["1536x2688"]
    seen = []

    def check(res):
        assert res.ring_ok
        assert len(res.rows) == w.heads * w.n_query_blocks
        _check_step(res, w)
        seen.append(res.position)

    Hn.run_stream(w, n_steps=2, check_ring=True, on_step=check)
    assert len(seen) == 2


@pytest.mark.parametrize("topk", W.FOURK_TOPK_SWEEP)
def test_4k_all_rows(topk):
    # every row; at topk 16 a second, evicting chunk as well
    w = W.WORKLOADS["4k"].with_topk(topk)
    seen = []

    def check(res):
        assert len(res.rows) == w.heads * w.n_query_blocks
        _check_step(res, w)
        seen.append(res.position)

    n_steps = 2 if topk == 16 else 1
    Hn.run_stream(w, n_steps=n_steps, check_ring=(topk == 16), on_step=check)
    assert len(seen) == n_steps


def test_truncated_window_ragged_counts():
    # Boundary-Truncated with a 5-block window: edge rows allow fewer blocks
    # than topk, so kept counts are ragged.
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["768x1280"], local_mode=1, local_range=5, topk=40, heads=4)
    (res,) = Hn.run_stream(w)
    assert len(np.unique(res.gpu_cnt)) > 1 and res.gpu_cnt.min() < 40
    _check_step(res, w)


def test_cold_start_three_layers_then_streaming():
    # The first chunk of a stream carries 3 block-layers (6 latent frames) into
    # an empty cache; the next chunks carry 1 layer each and see the cached
    # ones, the oldest dropped once kv_len + 1 slots are full.
    w = W.WORKLOADS["768x1280"]
    results = Hn.run_schedule(w, [3, 1, 1], n_rows=24, check_ring=True)
    nb = w.blocks_per_layer
    first = results[0]
    # block-causal inside the chunk: query layer L allows the keys of layers 0..L
    allowed = first.oracle["allowed"].sum(axis=1)
    assert np.array_equal(allowed, np.repeat([nb, 2 * nb, 3 * nb], nb))
    assert [r.oracle["allowed"].shape[1] for r in results] == [3 * nb, 4 * nb, 4 * nb]
    for res in results:
        assert res.ring_ok and res.kmean_err <= 1e-6
        _check_step(res, w)


def test_global_window_1536x2688():
    # local_range <= 0: no local window (every key block of the visible layers
    # is a candidate), the per-layer alternative a hybrid local/global stack uses
    import dataclasses
    w = dataclasses.replace(W.WORKLOADS["1536x2688"], local_range=0)
    (res,) = Hn.run_stream(w, n_steps=1, n_rows=12)
    assert res.oracle["allowed"].sum(axis=1).min() == w.capacity * w.blocks_per_layer
    _check_step(res, w)


def test_deterministic_byte_identical():
    w = W.WORKLOADS["768x1280"]
    a = Hn.run_stream(w, n_rows=4)[0]
    b = Hn.run_stream(w, n_rows=4)[0]
    assert np.array_equal(a.gpu_kept, b.gpu_kept)
    assert np.array_equal(a.gpu_scores, b.gpu_scores)
    assert np.array_equal(a.out_pipeline, b.out_pipeline)


def test_programmatic_dependent_launch_matches_plain_launches():
    # LcsaLayer.step(overlap_previous=True) launches all three kernels as
    # programmatic dependents (each starts before the previous kernel completes
    # and waits for its results in-kernel; the append writes a spare ring slot
    # while the previous step's attention still runs); over a stream with
    # eviction the outputs and kept lists equal those of plain launches bit for bit.
    L = _lib()
    w = W.WORKLOADS["768x1408"]
    dev = torch.device("cuda")
    chunks = [[t.to(dev) for t in W.gen_layers(w, w.kv_len + i, w.q_layers)] for i in range(6)]
    prefill = [[t.to(dev) for t in W.gen_layers(w, p, 1, "kv")[1:]] for p in range(w.kv_len)]
    runs = []
    for chained in (True, False):
        layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, device=dev)
        for k, v in prefill:
            layer.append(k, v)
        outs = []
        for q, k, v in chunks:
            out = torch.empty_like(q)
            if chained:
                layer.step(q, k, v, out, overlap_previous=True)
            else:
                L.lcsa_cache_append(layer.cache, k, v, d_status=layer.status)
                L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, d_status=layer.status)
                L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, out,
                                 d_status=layer.status)
            outs.append((out, layer.kept_idx.clone(), layer.kept_cnt.clone()))
        torch.cuda.synchronize()
        assert layer.status.item() == 0
        runs.append(outs)
    for (o1, k1, c1), (o2, k2, c2) in zip(*runs):
        assert torch.equal(k1, k2) and torch.equal(c1, c2) and torch.equal(o1, o2)


def test_chained_draft_after_multi_layer_append_matches_plain_launches():
    # A cold-start append of 3 block-layers, then a draft of only the newest
    # layer launched as a programmatic dependent of that append: the draft must
    # not read the key means of any of the 3 layers before the append completed
    # (the cache records how many layers the append wrote).  Kept lists and
    # scores equal those of plain launches bit for bit.
    import dataclasses
    L = _lib()
    w = W.WORKLOADS["768x1280"]
    dev = torch.device("cuda")
    q3, k3, v3 = [t.to(dev) for t in W.gen_layers(w, 0, 3)]
    q_new = q3[:, 4:6].contiguous()  # the newest layer's queries
    runs = []
    for chained in (True, False):
        cache = L.KVCache.allocate(4, w.heads, w.grid_h, w.grid_w, dev)
        st = torch.zeros((1,), dtype=torch.int32, device=dev)
        p = L.make_params(w.heads, w.grid_h, w.grid_w, 1, w.topk, flags=L.LCSA_FLAG_PDL if chained else 0)
        kept = torch.empty((w.heads, w.blocks_per_layer, w.topk), dtype=torch.int32, device=dev)
        cnt = torch.empty((w.heads, w.blocks_per_layer), dtype=torch.int32, device=dev)
        scores = torch.empty((w.heads, w.blocks_per_layer, 3 * w.blocks_per_layer), dtype=torch.float32,
                             device=dev)
        for _ in range(3):  # the same append and draft, repeated
            cache.reset()
            L.lcsa_cache_append(cache, k3, v3, d_status=st)
            assert cache.desc.appended == 3 and cache.count == 3
            L.lcsa_draft_mask(p, q_new, cache, kept, cnt, scores, d_status=st)
        torch.cuda.synchronize()
        assert st.item() == 0
        runs.append((kept.clone(), cnt.clone(), scores.clone()))
    for a, b in zip(*runs):
        assert torch.equal(a, b)


def test_host_stream_matches_direct_steps():
    # Overlapped host streaming (copy in / compute / copy out on three streams)
    # gives, chunk by chunk, exactly the outputs of the same steps run directly.
    L = _lib()
    w = W.WORKLOADS["768x1408"]
    dev = torch.device("cuda")
    chunks = [W.gen_layers(w, w.kv_len + i, w.q_layers) for i in range(5)]
    prefill = [W.gen_layers(w, p, 1, "kv") for p in range(w.kv_len)]

    def fresh_layer():
        layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, w.topk, device=dev)
        for _, k, v in prefill:
            layer.append(k.to(dev), v.to(dev))
        return layer

    direct = fresh_layer()
    ref = []
    for q, k, v in chunks:
        out = torch.empty_like(q, device=dev)
        direct.step(q.to(dev), k.to(dev), v.to(dev), out)
        ref.append(out.cpu())
    streamed = fresh_layer()
    hs = L.HostStream(streamed, chunks[0][0].shape, dev)
    pinned = [[t.pin_memory() for t in c] for c in chunks]
    outs = [torch.empty_like(chunks[0][0]).pin_memory() for _ in chunks]
    for (q, k, v), o in zip(pinned, outs):
        hs.submit(q, k, v, o)
    hs.drain_into(torch.cuda.current_stream())
    torch.cuda.synchronize()
    assert direct.status.item() == 0 and streamed.status.item() == 0
    for o, r in zip(outs, ref):
        assert torch.equal(o, r)


# ------------------------------------------------------------------ edge cases

def _tiny_setup(topk=8, heads=None):
    import dataclasses
    L = _lib()
    w = W.WORKLOADS["tiny"]
    if heads is not None:
        w = dataclasses.replace(w, heads=heads)
    q, k, v = [t.cuda() for t in W.gen_layers(w, 0, w.q_layers)]
    layer = L.LcsaLayer(w.heads, w.grid_h, w.grid_w, w.q_layers, w.kv_len, topk, device="cuda")
    layer.append(k, v)
    return L, w, q, k, v, layer


def _check_ragged_rows(heads, counts, seed):
    """Attention over hand-made kept lists with `counts` tiles per row."""
    topk = 4
    L, w, q, k, v, layer = _tiny_setup(topk=topk, heads=heads)
    Nq = w.n_query_blocks
    kept = torch.full((w.heads, Nq, topk), -1, dtype=torch.int32)
    cnt = torch.zeros((w.heads, Nq), dtype=torch.int32)
    rng = np.random.default_rng(seed)
    for h in range(w.heads):
        for i in range(Nq):
            c = int(rng.choice(counts))
            sel = np.sort(rng.choice(32, size=c, replace=False))
            kept[h, i, :c] = torch.from_numpy(sel.astype(np.int32))
            cnt[h, i] = c
    out = torch.empty_like(q)
    lse = torch.empty(q.shape[:4], dtype=torch.float32, device="cuda")
    L.lcsa_attention(layer.params, q, layer.cache, kept.cuda(), cnt.cuda(), out, lse, d_status=layer.status)
    torch.cuda.synchronize()
    assert layer.status.item() == 0, L.status_string(layer.status.item())
    qb = O.partition(Hn.f32(q))
    kb = O.partition(Hn.f32(k))
    vb = O.partition(Hn.f32(v))
    ob = O.partition(Hn.f32(out))
    lb = O.partition(lse.cpu().numpy()[..., None])[..., 0]
    for h in range(w.heads):
        for i in range(Nq):
            ro, rl = O.sparse_attention_row(qb[h, i], kb[h], vb[h], kept[h, i, :cnt[h, i]].numpy(), 1 / math.sqrt(128))
            if cnt[h, i] == 0:
                assert np.all(ob[h, i] == 0) and np.all(np.isneginf(lb[h, i]))
            else:
                assert np.max(np.abs(ob[h, i] - ro)) <= Hn.ATOL_OUT
                assert np.max(np.abs(lb[h, i] - rl)) <= 2e-3


def test_zero_and_single_tile_rows():
    # 64 rows: one row per CTA, 0..4 tiles each
    _check_ragged_rows(heads=None, counts=[0, 1, 2, 3, 4], seed=3)


def test_consecutive_single_tile_rows_in_one_cta():
    # 12 heads x 32 query blocks = 384 rows over at most 148 persistent CTAs:
    # every CTA walks two or three rows, mostly with a single kept tile, so the
    # second MMA issuer often has no tile in two rows in a row.
    _check_ragged_rows(heads=12, counts=[0, 1, 1, 1, 1, 2], seed=5)


def test_bad_kept_index_is_reported_and_row_zeroed():
    L, w, q, k, v, layer = _tiny_setup(topk=8)
    L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt)
    good = torch.empty_like(q)
    L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, good)
    kept = layer.kept_idx.clone()
    cnt = layer.kept_cnt.clone()
    kept[1, 5, 0] = 32          # one past the last key block
    cnt[0, 7] = 9               # more than topk
    out = torch.empty_like(q)
    layer.status.zero_()
    L.lcsa_attention(layer.params, q, layer.cache, kept, cnt, out, d_status=layer.status)
    torch.cuda.synchronize()
    assert layer.status.item() & L.LCSA_ERR_BAD_INDEX
    ob, gb = O.partition(Hn.f32(out)), O.partition(Hn.f32(good))
    assert np.all(ob[1, 5] == 0) and np.all(ob[0, 7] == 0)
    mask = np.ones(ob.shape[:2], dtype=bool)
    mask[1, 5] = mask[0, 7] = False
    assert np.array_equal(ob[mask], gb[mask])


def test_forced_watchdog_expiry_reports_timeout_and_context_survives():
    L, w, q, k, v, layer = _tiny_setup(topk=8)
    L.lcsa_draft_mask(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt)
    ref = torch.empty_like(q)
    L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, ref)
    p = L.make_params(w.heads, w.grid_h, w.grid_w, w.q_layers, 8, flags=L.LCSA_FLAG_FORCE_TIMEOUT)
    out = torch.empty_like(q)
    layer.status.zero_()
    L.lcsa_attention(p, q, layer.cache, layer.kept_idx, layer.kept_cnt, out, d_status=layer.status)
    torch.cuda.synchronize()
    assert layer.status.item() & L.LCSA_ERR_TIMEOUT
    # the context is still usable and gives the same result as before
    again = torch.empty_like(q)
    L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, again)
    torch.cuda.synchronize()
    assert torch.equal(again, ref)


def test_cache_append_forced_timeout_reports_status_and_context_survives():
    """The append's bounded copy waits: a forced expiry is reported, nothing hangs or faults."""
    L, w, q, k, v, layer = _tiny_setup(topk=8)
    n = w.q_layers
    ref = L.KVCache.allocate(n, w.heads, w.grid_h, w.grid_w, device="cuda")
    L.lcsa_cache_append(ref, k, v)
    cache = L.KVCache.allocate(n, w.heads, w.grid_h, w.grid_w, device="cuda")
    st = torch.zeros(1, dtype=torch.int32, device="cuda")
    L.lcsa_cache_append(cache, k, v, d_status=st, flags=L.LCSA_FLAG_FORCE_TIMEOUT)
    torch.cuda.synchronize()
    assert st.item() & L.LCSA_ERR_TIMEOUT
    # the context is still usable: a normal append gives the reference ring bit for bit
    cache.reset()
    st.zero_()
    L.lcsa_cache_append(cache, k, v, d_status=st)
    torch.cuda.synchronize()
    assert st.item() == 0
    assert torch.equal(cache.k, ref.k) and torch.equal(cache.v, ref.v) and torch.equal(cache.kmean, ref.kmean)


def test_invalid_arguments_are_rejected():
    L, w, q, k, v, layer = _tiny_setup()
    out = torch.empty_like(q)
    bad = L.make_params(w.heads, w.grid_h, w.grid_w, w.q_layers, 8, local_range=4)  # even range
    with pytest.raises(L.LcsaError) as e:
        L.lcsa_attention(bad, q, layer.cache, layer.kept_idx, layer.kept_cnt, out)
    assert e.value.code == L.LCSA_ERR_INVALID_ARG
    too_many = L.make_params(w.heads, w.grid_h, w.grid_w, 3, 8)  # more query layers than cached
    with pytest.raises(L.LcsaError):
        L.lcsa_draft_mask(too_many, q, layer.cache, layer.kept_idx, layer.kept_cnt)
    with pytest.raises(L.LcsaError):
        L.lcsa_attention(layer.params, q, layer.cache, layer.kept_idx, layer.kept_cnt, q)  # aliasing
