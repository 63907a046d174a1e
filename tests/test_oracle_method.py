"""Pins of the oracle's CSA2 steps: the pages' figures, closed forms, invariants, brute force.

CPU only.  Brute-force references here are written with plain Python loops so
that a dropped term, a wrong sign or index, or a transposed operand in the
oracle's vectorised code fails one of them.
"""
import json
import math
import os

import numpy as np
import pytest

from oracle import csa2 as C
from oracle import formats as F

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")
RNG = np.random.default_rng(11)


def golden():
    return json.load(open(os.path.join(GOLDEN, "byte_accounting.json")))


# ----------------------------------------------------------------- the pages' figures
def test_layer_schedule_matches_pages():
    g = golden()["layer_schedule"]
    modes = [C.layer_mode(i) for i in range(C.NUM_LAYERS)]
    assert len(modes) == g["num_layers"]
    assert [i for i, m in enumerate(modes) if m == "swa"] == g["swa_only"]
    assert [i for i, m in enumerate(modes) if m == "full"] == g["full"]
    assert [i for i, m in enumerate(modes) if m == "reindex"] == g["reindex"]
    assert modes.count("reuse") == g["reuse_count"]


def test_entries_and_bytes_per_token():
    g = golden()
    enc = sum(1.0 / r for l, r in C.FULL_LAYERS.items() if l < 20)
    dec = sum(1.0 / r for l, r in C.FULL_LAYERS.items() if l >= 20)
    assert enc == g["entries_per_token"]["encoder"]
    assert dec == g["entries_per_token"]["decoder"]
    assert C.entries_per_token() == g["entries_per_token"]["total"]
    assert C.global_kv_bytes_per_token() == g["global_kv_bytes_per_token"]["v4_1_flash"]


def test_global_kv_at_one_million_tokens():
    g = golden()["global_kv_at_1m_context_gib"]
    gib = C.global_kv_bytes_per_token() * 2 ** 20 / 2 ** 30
    assert round(gib, g["printed_digits"]) == g["value"]
    # "1M" must be 2^20 here: 10^6 tokens would print 0.83
    assert round(C.global_kv_bytes_per_token() * 1e6 / 2 ** 30, 2) != g["value"]


def test_about_a_quarter_of_v4():
    g = golden()["global_kv_bytes_per_token"]
    assert 3.9 < g["v4_flash"] / C.global_kv_bytes_per_token() < 4.0


# ----------------------------------------------------------------- compressor
def test_compressor_ratio_one_is_identity():
    x = RNG.normal(size=(13, 8)).astype(np.float32)
    np.testing.assert_array_equal(C.compress(x, 1), x)


@pytest.mark.parametrize("r", [2, 4])
def test_compressor_mean_of_identical_rows(r):
    row = RNG.normal(size=(1, 16)).astype(np.float32)
    x = np.repeat(row, 3 * r + 1, axis=0)           # ragged tail of one token
    out = C.compress(x, r)
    assert out.shape[0] == 3                         # incomplete group makes no entry
    np.testing.assert_array_equal(out, np.repeat(row, 3, axis=0))


def test_compressor_weighted_sum_brute_force():
    x = RNG.normal(size=(9, 5)).astype(np.float32)
    w = RNG.uniform(size=9).astype(np.float32)
    out = C.compress(x, 3, w)
    for j in range(3):
        for d in range(5):
            acc = np.float32(w[3 * j] * x[3 * j, d])
            for t in (3 * j + 1, 3 * j + 2):
                acc = np.float32(acc + np.float32(w[t] * x[t, d]))
            assert out[j, d] == acc


def test_fixed_exp_against_the_exponential():
    """exp_fp32 is exp within its rounding bound (argument reduction in fp32: about 2^-23 (1 + |x|)),
    exactly 1 at 0, 0 below the fp32 normal range."""
    rng = np.random.default_rng(3)
    x = np.concatenate([-np.abs(rng.normal(size=50000)) * 30, -rng.uniform(0, 1, 50000), [0.0, -1e-30]])
    x = x.astype(np.float32)
    e = C.exp_fp32(x)
    ref = np.exp(x.astype(np.float64))
    ok = ref > 2.0 ** -126
    assert np.all(np.abs(e[ok] - ref[ok]) <= 1.5e-7 * (1 + np.abs(x[ok])) * ref[ok])
    assert C.exp_fp32(np.float32(0)) == 1.0 and C.exp_fp32(np.float32(-200)) == 0.0
    assert C.exp_fp32(np.float32(-1e-30)) == 1.0


def test_gated_compressor_reductions():
    """Equal logits give the plain mean (compress, bit for bit); one dominant logit per channel picks
    that token's latent exactly; weights of a group sum to one."""
    rng = np.random.default_rng(4)
    for r in (1, 2, 4):
        x = rng.normal(size=(5 * r + r - 1, 24)).astype(np.float32)   # a ragged tail makes no entry
        g = np.full_like(x, 0.7)
        np.testing.assert_array_equal(C.compress_gated(x, g, r), C.compress(x, r))
        pick = rng.integers(0, r, size=24)
        g = np.zeros_like(x)
        for j in range(5):
            g[j * r + pick, np.arange(24)] = 200.0
        want = np.stack([x[j * r + pick, np.arange(24)] for j in range(5)])
        np.testing.assert_array_equal(C.compress_gated(x, g, r), want)
    # general logits: a convex combination, per channel, of the group's tokens
    x = rng.normal(size=(12, 8)).astype(np.float32)
    g = rng.normal(size=(12, 8)).astype(np.float32) * 3
    out = C.compress_gated(x, g, 3)
    for j in range(4):
        w = np.exp(g[3 * j:3 * j + 3].astype(np.float64))
        w /= w.sum(axis=0)
        np.testing.assert_allclose(out[j], (w * x[3 * j:3 * j + 3]).sum(axis=0), rtol=1e-5, atol=1e-6)


def test_prefill_entry_count():
    # a 262144-token prefix plus an 8192-token chunk at ratio 2
    assert 262144 // 2 == 131072 and 8192 // 2 == 4096


# ----------------------------------------------------------------- indexer
def brute_scores(q_ix, w, keys):
    qh = C.quantised_query(q_ix)
    out = []
    for k in keys.tolist():
        s = 0.0
        for h in range(len(w)):
            dot = 0.0
            for i in range(len(k)):
                dot += float(qh[h][i]) * k[i]
            s += float(w[h]) * (dot if dot > 0 else 0.0)
        out.append(s)
    return np.array(out)


def test_indexer_score_brute_force():
    H, n = 5, 11
    q = RNG.normal(size=(H, 128)).astype(np.float32)
    w = RNG.uniform(-0.5, 1, size=H).astype(np.float32)
    c, s = F.pack_indexer(RNG.normal(size=(n, 128)).astype(np.float32))
    keys = F.unpack_indexer(c, s)
    np.testing.assert_allclose(C.indexer_scores(q, w, keys), brute_scores(q, w, keys), rtol=1e-12, atol=1e-12)


def test_indexer_query_is_mxfp4_quantised():
    q = RNG.normal(size=(3, 128)).astype(np.float32)
    qh = C.quantised_query(q)
    assert not np.array_equal(qh, q.astype(np.float64))
    # every per-32 block of q^ is an e2m1 multiple of one power of two
    for h in range(3):
        for b in range(4):
            blk = qh[h, 32 * b:32 * b + 32]
            e = int(np.ceil(np.log2(np.float32(np.max(np.abs(q[h, 32 * b:32 * b + 32]))) / np.float32(6))))
            np.testing.assert_array_equal(np.isin(np.abs(blk) / 2.0 ** e, F.E2M1_MAGNITUDES), True)


def test_topk_invariant_under_positive_weight_rescale():
    H, n = 8, 300
    q = RNG.normal(size=(H, 128)).astype(np.float32)
    w = RNG.uniform(size=H).astype(np.float32)
    c, s = F.pack_indexer(RNG.normal(size=(n, 128)).astype(np.float32))
    keys = F.unpack_indexer(c, s)
    a = C.topk(C.indexer_scores(q, w, keys), 17)
    b = C.topk(C.indexer_scores(q, w * np.float32(4), keys), 17)
    np.testing.assert_array_equal(a, b)


# ----------------------------------------------------------------- top-k
def brute_topk(scores, k, n_valid=None):
    n = len(scores) if n_valid is None else n_valid
    cand = [j for j in range(n) if scores[j] != -math.inf]
    sel = []
    for i in cand:
        rank = sum(1 for j in cand if scores[j] > scores[i] or (scores[j] == scores[i] and j < i))
        if rank < k:
            sel.append(i)
    return sorted(sel) + [-1] * (k - len(sel))


@pytest.mark.parametrize("case", range(6))
def test_topk_against_rank_definition(case):
    rng = np.random.default_rng(100 + case)
    n = int(rng.integers(1, 60))
    s = rng.integers(-3, 4, size=n).astype(np.float64)     # many ties
    s[rng.uniform(size=n) < 0.1] = -math.inf
    k = int(rng.integers(1, 70))
    nv = int(rng.integers(0, n + 1))
    np.testing.assert_array_equal(C.topk(s, k, nv), brute_topk(s, k, nv))
    np.testing.assert_array_equal(C.topk(s, k), brute_topk(s, k))


def test_topk_equals_full_sort():
    s = RNG.normal(size=5000)
    want = np.sort(np.argsort(-s, kind="stable")[:512])
    np.testing.assert_array_equal(C.topk(s, 512), want)


# ----------------------------------------------------------------- attention
def brute_attend(q, keys, tau):
    H = len(q)
    o, lse = [], []
    for h in range(H):
        logits = [tau * sum(a * b for a, b in zip(q[h], k)) for k in keys]
        m = max(logits)
        e = [math.exp(x - m) for x in logits]
        z = sum(e)
        o.append([sum(e[j] * keys[j][d] for j in range(len(keys))) / z for d in range(len(q[h]))])
        lse.append(m + math.log(z))
    return np.array(o), np.array(lse)


def test_attend_brute_force():
    q = RNG.normal(size=(3, 6))
    keys = RNG.normal(size=(7, 6))
    o, lse = C.attend(q, keys, 0.7)
    bo, bl = brute_attend(q.tolist(), keys.tolist(), 0.7)
    np.testing.assert_allclose(o, bo, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=1e-12, atol=1e-12)


def test_attend_empty_set():
    o, lse = C.attend(np.ones((2, 4)), np.zeros((0, 4)), 1.0)
    assert not o.any() and np.all(lse == -math.inf)


def _tiny_cache(n_tokens, ratio, B=1, seed=5):
    rng = np.random.default_rng(seed)
    cache = C.Cache(B, n_tokens // ratio + 4, ratio)
    for b in range(B):
        kv = rng.normal(size=(n_tokens, 512)).astype(np.float32)
        ix = rng.normal(size=(n_tokens, 128)).astype(np.float32)
        cache.num_entries[b] = cache.pack(b, 0, kv, ix)
    return cache, rng


def test_sparse_equals_dense_when_k_covers_everything():
    cache, rng = _tiny_cache(80, 2)
    q = rng.normal(size=(4, 512))
    q_ix = rng.normal(size=(4, 128)).astype(np.float32)
    w = rng.uniform(size=4).astype(np.float32)
    pos = 79
    idx, _, _ = C.full_select(cache, 0, pos, q_ix, w, k=64)
    assert (idx[:40] == np.arange(40)).all() and (idx[40:] == -1).all()
    o, lse = C.sparse_attention(cache, 0, q, idx, 0.05)
    od, ld = C.attend(q, cache.main_values(0, np.arange(40)), 0.05)
    np.testing.assert_allclose(o, od, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, ld, rtol=1e-12)


def test_full_respects_causality():
    cache, rng = _tiny_cache(100, 2)
    q_ix = rng.normal(size=(4, 128)).astype(np.float32)
    w = rng.uniform(size=4).astype(np.float32)
    for pos in (0, 1, 2, 17, 60):
        idx, _, _ = C.full_select(cache, 0, pos, q_ix, w, k=8)
        sel = idx[idx >= 0]
        assert len(sel) == min(8, (pos + 1) // 2)
        assert (sel < (pos + 1) // 2).all()


def test_reuse_equals_full_and_reindex_invariants():
    cache, rng = _tiny_cache(600, 1)
    q = rng.normal(size=(4, 512))
    q_ix = rng.normal(size=(4, 128)).astype(np.float32)
    w = rng.uniform(size=4).astype(np.float32)
    swa_c, swa_s = F.pack_swa(rng.normal(size=(128, 512)).astype(np.float32))
    pos = 599
    full = C.decode_layer("full", cache, 0, pos, q, 0.04, (swa_c, swa_s), q_ix=q_ix, w=w, k=32, pool_k=128)
    reuse = C.decode_layer("reuse", cache, 0, pos, q, 0.04, (swa_c, swa_s), idx=full["idx"])
    np.testing.assert_array_equal(full["o"], reuse["o"])
    np.testing.assert_array_equal(full["lse"], reuse["lse"])
    pool = full["pool"]
    assert set(full["idx"].tolist()) <= set(pool.tolist())
    # Reindex with the Full layer's own query re-finds the Full layer's top-k
    ri, _ = C.reindex_select(cache, 0, pos, q_ix, w, 32, pool)
    np.testing.assert_array_equal(ri, full["idx"])
    # Reindex with a fresh query stays inside the pool
    q2 = rng.normal(size=(4, 128)).astype(np.float32)
    ri2, _ = C.reindex_select(cache, 0, pos, q2, w, 32, pool)
    assert set(ri2.tolist()) <= set(pool.tolist())
    # with the pool = every visible entry, Reindex == Full
    allpool = np.arange(600)
    ri3, _ = C.reindex_select(cache, 0, pos, q2, w, 32, allpool)
    f3, _, _ = C.full_select(cache, 0, pos, q2, w, 32)
    np.testing.assert_array_equal(ri3, f3)


def test_merge_equals_one_softmax_over_union():
    q = RNG.normal(size=(3, 16))
    k1 = RNG.normal(size=(5, 16))
    k2 = RNG.normal(size=(9, 16))
    o1, l1 = C.attend(q, k1, 0.3)
    o2, l2 = C.attend(q, k2, 0.3)
    o, lse = C.merge(o1, l1, o2, l2)
    ou, lu = C.attend(q, np.concatenate([k1, k2]), 0.3)
    np.testing.assert_allclose(o, ou, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(lse, lu, rtol=1e-12)
    ob, lb = C.merge(o2, l2, o1, l1)
    np.testing.assert_allclose(o, ob, rtol=1e-13, atol=1e-14)
    np.testing.assert_allclose(lse, np.log(np.exp(l1) + np.exp(l2)), rtol=1e-12)


def test_merge_with_an_empty_side():
    q = RNG.normal(size=(2, 8))
    k = RNG.normal(size=(4, 8))
    o1, l1 = C.attend(q, k, 1.0)
    oe, le = C.attend(q, np.zeros((0, 8)), 1.0)
    o, lse = C.merge(o1, l1, oe, le)
    np.testing.assert_array_equal(o, o1)
    np.testing.assert_array_equal(lse, l1)
    o, lse = C.merge(oe, le, oe, le)
    assert not o.any() and np.all(lse == -math.inf)


def test_swa_equals_dense_over_last_window():
    rng = np.random.default_rng(9)
    R, W = 160, 128
    x = rng.normal(size=(400, 512)).astype(np.float32)
    codes = np.zeros((R, 512), np.uint8)
    scale = np.zeros(R, np.float32)
    pos = 377
    for t in range(pos - R + 1, pos + 1):                # ring holds the last R tokens
        codes[t % R], scale[t % R] = F.pack_swa(x[t])
    q = rng.normal(size=(2, 512))
    o, lse = C.swa_attention(q, pos, codes, scale, W, 0.05)
    keys = []
    for t in range(pos - W + 1, pos + 1):
        c, s = F.pack_swa(x[t])
        keys.append([float(F.e4m3_decode(np.uint8(v))) * float(s) for v in c.tolist()])
    bo, bl = brute_attend(q.tolist(), keys, 0.05)
    np.testing.assert_allclose(o, bo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(lse, bl, rtol=1e-12)
    # at the start of a sequence the window is shorter
    o0, _ = C.swa_attention(q, 0, codes[[0] * R], scale[[0] * R], W, 0.05)
    np.testing.assert_allclose(o0, np.repeat(F.unpack_swa(codes[:1], scale[:1]), 2, 0), rtol=1e-12)


# ----------------------------------------------------------------- one whole layer
def _brute_window_keys(codes, scale, pos, window):
    """Dequantised SWA tokens of positions max(0, pos - window + 1) .. pos, element by element."""
    R = codes.shape[0]
    keys = []
    for t in range(max(0, pos - window + 1), pos + 1):
        s = float(scale[t % R])
        keys.append([float(F.e4m3_decode(np.uint8(c))) * s for c in codes[t % R].tolist()])
    return keys


@pytest.mark.parametrize("mode", ["full", "reindex", "reuse"])
def test_decode_layer_is_one_softmax_over_entries_and_window(mode):
    """A layer's output is one softmax over its listed entries and its window tokens together.

    The listed entries are re-derived by brute force (scores by loops, rank definition), the
    window by position arithmetic, and the attention by plain loops, so that a layer that drops
    a branch, passes a wrong window or merges with wrong weights fails here.
    """
    rng = np.random.default_rng(21)
    cache, _ = _tiny_cache(40, 1, seed=23)
    n = int(cache.num_entries[0])
    H, W, R, pos, k, tau = 3, 5, 8, 37, 6, 0.05
    q = rng.normal(size=(H, 512))
    q_ix = rng.normal(size=(4, 128)).astype(np.float32)
    w = rng.uniform(size=4).astype(np.float32)
    x = rng.normal(size=(R, 512)).astype(np.float32)
    codes = np.zeros((R, 512), np.uint8)
    scale = np.zeros(R, np.float32)
    for t in range(pos - R + 1, pos + 1):
        codes[t % R], scale[t % R] = F.pack_swa(x[t % R])
    vis = min(n, pos + 1)
    keys_ix = F.unpack_indexer(cache.ix_codes[0, :vis], cache.ix_scales[0, :vis])
    s_all = brute_scores(q_ix, w, keys_ix)
    if mode == "full":
        out = C.decode_layer("full", cache, 0, pos, q, tau, (codes, scale), window=W, q_ix=q_ix, w=w, k=k)
        want = brute_topk(list(s_all), k)
    elif mode == "reindex":
        pool = np.array([3, 7, 11, 12, 19, 25, 30, 31, 36, -1], np.int64)
        out = C.decode_layer("reindex", cache, 0, pos, q, tau, (codes, scale), window=W, q_ix=q_ix, w=w,
                             k=k, pool=pool)
        ps = [s_all[p] if p >= 0 else -math.inf for p in pool.tolist()]
        want = [int(pool[j]) if j >= 0 else -1 for j in brute_topk(ps, k)]
    else:
        idx = np.array([2, 9, -1, 33, 14], np.int64)
        out = C.decode_layer("reuse", cache, 0, pos, q, tau, (codes, scale), window=W, idx=idx)
        want = idx.tolist()
    np.testing.assert_array_equal(np.asarray(out["idx"]), want)
    listed = [j for j in want if j >= 0]
    main = F.unpack_main(cache.kv_codes[0, listed], cache.kv_scales[0, listed]).tolist()
    keys = main + _brute_window_keys(codes, scale, pos, W)
    assert len(keys) == len(listed) + W
    bo, bl = brute_attend(q.tolist(), keys, tau)
    np.testing.assert_allclose(out["o"], bo, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(out["lse"], bl, rtol=1e-12)


# ----------------------------------------------------------------- the 40-layer stack
def _tiny_model(seed=31, T=120, H=2, HI=3, R=8):
    """Four small caches (one per Full layer, at its ratio) and per-layer inputs at position T - 1."""
    rng = np.random.default_rng(seed)
    caches = {}
    for layer, r in C.FULL_LAYERS.items():
        cache = C.Cache(1, T // r + 2, r)
        kv = rng.normal(size=(T, 512)).astype(np.float32)
        ix = rng.normal(size=(T, 128)).astype(np.float32)
        cache.num_entries[0] = cache.pack(0, 0, kv, ix)
        caches[layer] = cache
    pos = T - 1
    layers = []
    for _ in range(C.NUM_LAYERS):
        codes, scale = np.zeros((R, 512), np.uint8), np.zeros(R, np.float32)
        for t in range(pos - R + 1, pos + 1):
            codes[t % R], scale[t % R] = F.pack_swa(rng.normal(size=512).astype(np.float32))
        layers.append({"q": rng.normal(size=(H, 512)), "q_ix": rng.normal(size=(HI, 128)).astype(np.float32),
                       "w": rng.uniform(size=HI).astype(np.float32), "swa": (codes, scale)})
    return caches, pos, layers


def test_decode_model_follows_the_layer_schedule():
    """Every layer of the stack against brute force: the window-only layers, each Full layer's
    own selection over its own cache, the pool of the decoder's Full layer, each Reindex layer's
    selection inside that pool, and every layer's output as one softmax over the entries of the
    nearest earlier selecting layer (from that layer's cache) plus its window."""
    caches, pos, layers = _tiny_model()
    k, pool_k, W, tau = 6, 20, 5, 0.05
    out = C.decode_model(caches, 0, pos, layers, tau, k=k, pool_k=pool_k, window=W)
    assert len(out) == C.NUM_LAYERS == 40
    brute_s = {}
    head = None
    for layer in range(C.NUM_LAYERS):
        L, m = layers[layer], C.layer_mode(layer)
        win = _brute_window_keys(L["swa"][0], L["swa"][1], pos, W)
        if m == "swa":
            bo, bl = brute_attend(L["q"].tolist(), win, tau)
            np.testing.assert_allclose(out[layer]["o"], bo, rtol=1e-11, atol=1e-12)
            continue
        if m == "full":
            cache = caches[layer]
            vis = cache.visible(0, pos)
            keys = F.unpack_indexer(cache.ix_codes[0, :vis], cache.ix_scales[0, :vis])
            s = list(brute_scores(L["q_ix"], L["w"], keys))
            np.testing.assert_array_equal(out[layer]["idx"], brute_topk(s, k))
            if layer == 20:
                np.testing.assert_array_equal(out[layer]["pool"], brute_topk(s, pool_k))
            head, head_cache = layer, cache
        elif m == "reindex":
            cache = caches[20]
            pool = out[20]["pool"]
            keys = F.unpack_indexer(cache.ix_codes[0, pool], cache.ix_scales[0, pool])
            s = list(brute_scores(L["q_ix"], L["w"], keys))
            want = [int(pool[j]) if j >= 0 else -1 for j in brute_topk(s, k)]
            np.testing.assert_array_equal(out[layer]["idx"], want)
            head, head_cache = layer, cache
        assert out[layer]["head"] == head
        listed = [j for j in out[head]["idx"].tolist() if j >= 0]
        main = F.unpack_main(head_cache.kv_codes[0, listed], head_cache.kv_scales[0, listed]).tolist()
        bo, bl = brute_attend(L["q"].tolist(), main + win, tau)
        np.testing.assert_allclose(out[layer]["o"], bo, rtol=1e-11, atol=1e-12)
        np.testing.assert_allclose(out[layer]["lse"], bl, rtol=1e-12)
        brute_s[layer] = True
    assert len(brute_s) == 38                       # every CSA2 layer checked


def test_library_plan_is_the_pages_schedule():
    """csa2_plan_v41 (host code of the library, no GPU) against the oracle's schedule."""
    from compressed_sparse_attention_score_b200 import build
    build.build()
    import compressed_sparse_attention_score_b200 as K
    plan, ratios = K.csa2_plan_v41()
    names = {0: "full", 1: "reindex", 2: "reuse", K.LAYER_SWA: "swa"}
    assert [names[m] for m, _, _ in plan] == [C.layer_mode(i) for i in range(C.NUM_LAYERS)]
    full = sorted(C.FULL_LAYERS)
    assert [plan[f][2] for f in full] == [0, 1, 2, 3]
    assert ratios == [C.FULL_LAYERS[f] for f in full]
    for i, (m, src, cache) in enumerate(plan):
        if names[m] == "reuse":          # the nearest earlier Full or Reindex layer
            want = max(j for j in range(i) if C.layer_mode(j) in ("full", "reindex"))
            assert src == want and cache == plan[want][2]
        if names[m] == "reindex":
            assert src == C.pool_layer() and cache == plan[C.pool_layer()][2]
