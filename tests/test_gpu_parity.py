"""GPU parity: every CSA2 step through the C ABI against the CPU oracle, element by element.

Sizes here span several tiles and a ragged tail and still let the oracle finish
in seconds; test_gpu_full_size.py covers the full configurations by sampling.
"""
import math

import numpy as np
import pytest
import torch

from oracle import csa2 as OC
from oracle import formats as OF
from workloads import configs as W
from workloads import normal, uniform

from tests.helpers import (K, check_attention, check_topk, fill_main, gpu_attend_given, gpu_cache, oracle_seq,
                           oracle_swa, to_np)

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _err():
    return torch.zeros(1, dtype=torch.int32, device=DEV)


# ------------------------------------------------------------------ packers
def _planted_latents(B, T, d, seed, dtype):
    x = normal((B, T, d), seed, "pack", d, device=DEV)
    t = lambda i: (T - 1 - i) if T > 6 else T - 1  # noqa: E731  (plant near the end: kept by a ring)
    x[0, t(0), :32] = 0.0                    # zero blocks
    x[0, t(1), :16] *= 1e-5                  # subnormal E4M3 scales
    x[0, t(2), :] *= 1e3                     # saturating E4M3 scales
    x[B - 1, t(3), 5] = 1e-40                # a subnormal input
    x[0, t(4), :] = 0.25
    x[0, t(5), :] = torch.tensor([0.75, -1.25, 1.75, 2.5, 3.5, 5.0, 6.0, 0.5] * (d // 8))  # e2m1 ties
    return x.to(dtype)


@pytest.mark.parametrize("ratio", [1, 2, 4])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
@pytest.mark.parametrize("weighted", [False, True])
def test_pack_kv_bit_exact(ratio, dtype, weighted):
    k = K()
    B, T = 3, 1001
    kv = _planted_latents(B, T, 512, 1, dtype)
    ix = _planted_latents(B, T, 128, 2, dtype)
    pw = uniform((B, T), 0, "pack_w", device=DEV) if weighted else None
    n = T // ratio
    cache = k.GlobalKVCache(B, ratio, seq_stride=n + 5)
    first = torch.tensor([0, 3, 5], dtype=torch.int32, device=DEV)
    err = _err()
    k.csa2_pack_kv(kv, ix, first, cache, pool_w=pw, err=err)
    assert k.csa2_check(err) == 0
    for b in range(B):
        w_np = None if pw is None else to_np(pw[b])
        ekv = OC.compress(to_np(kv[b]), ratio, w_np)
        eix = OC.compress(to_np(ix[b]), ratio, w_np)
        mc, ms = OF.pack_main(ekv)
        ic, isc = OF.pack_indexer(eix)
        f = int(first[b])
        sl = slice(b * (n + 5) + f, b * (n + 5) + f + n)
        np.testing.assert_array_equal(to_np(cache.kv_codes[sl]), mc)
        np.testing.assert_array_equal(to_np(cache.kv_scales[sl]), ms)
        np.testing.assert_array_equal(to_np(cache.ix_codes[sl]), ic)
        np.testing.assert_array_equal(to_np(cache.ix_scales[sl]), isc)


def test_pack_kv_paged_and_out_of_range():
    k = K()
    spec = W.scaled(W.mixed64(), [700, 1300, 260], B=3)
    spec.page_size = 256
    spec.paged = True
    table, pages = W.page_layout(spec, DEV)
    cache = k.GlobalKVCache(3, 1, num_slots=pages * 256, page_table=table, page_size=256)
    err = _err()
    for b in range(3):
        kv, ix = W.token_latents(spec, b, DEV)
        v = cache.seq_view(b)
        v.ratio = spec.seq_ratio(b)
        k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), torch.zeros(1, dtype=torch.int32, device=DEV),
                       v, err=err)
        c = oracle_seq(spec, b, gen_device=DEV)
        n = spec.entries(b)
        tb = table[b].cpu().numpy()
        slots = np.array([tb[e // 256] * 256 + e % 256 for e in range(n)])
        np.testing.assert_array_equal(to_np(cache.kv_codes)[slots], c.kv_codes[0, :n])
        np.testing.assert_array_equal(to_np(cache.kv_scales)[slots], c.kv_scales[0, :n])
        np.testing.assert_array_equal(to_np(cache.ix_codes)[slots], c.ix_codes[0, :n])
        np.testing.assert_array_equal(to_np(cache.ix_scales)[slots], c.ix_scales[0, :n])
    assert k.csa2_check(err) == 0
    # writing past the last page is refused on the device, not faulted
    kv, ix = W.token_latents(spec, 2, DEV)
    v = cache.seq_view(2)
    k.csa2_pack_kv(kv[None, :300].contiguous(), ix[None, :300].contiguous(),
                   torch.full((1,), 200, dtype=torch.int32, device=DEV), v, err=err)
    assert k.csa2_check(err) == 5


@pytest.mark.parametrize("R,T", [(128, 300), (512, 300), (128, 1)])
def test_pack_swa_bit_exact(R, T):
    k = K()
    B = 2
    x = _planted_latents(B, T, 512, 3, torch.bfloat16)
    pos = (torch.arange(T, dtype=torch.int32, device=DEV) + 1000)[None].repeat(B, 1).contiguous()
    codes = torch.zeros((B, R, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((B, R), dtype=torch.float32, device=DEV)
    err = _err()
    k.csa2_pack_swa(x, pos, codes, scale, err=err)
    assert k.csa2_check(err) == 0
    for b in range(B):
        keep = slice(max(0, T - R), T)
        oc, osc = oracle_swa(to_np(x[b])[keep], to_np(pos[b])[keep], R)
        np.testing.assert_array_equal(to_np(codes[b]), oc)
        np.testing.assert_array_equal(to_np(scale[b]), osc)


# ------------------------------------------------------------------ indexer + top-k
def test_index_score_full_and_candidates():
    k = K()
    spec = W.scaled(W.tiny_full(), [3001, 5000], B=2)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    q_pos[0, 0] = 1999                      # an earlier query sees fewer entries
    err = _err()
    s = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, err=err)
    assert k.csa2_check(err) == 0
    for b in range(2):
        c = oracle_seq(spec, b, main_rows=[], gen_device=DEV)
        nvis = c.visible(0, int(q_pos[b, 0]))
        ref = OC.indexer_scores(to_np(q_ix[b, 0]), to_np(w[b, 0]), c.indexer_values(0, np.arange(nvis)))
        got = to_np(s[b, 0])
        assert np.all(np.isneginf(got[nvis:]))
        np.testing.assert_allclose(got[:nvis], ref, rtol=2e-6, atol=2e-6 * np.abs(ref).max())
    # candidate lists with pads
    cand = torch.full((2, 1, 700), -1, dtype=torch.int32, device=DEV)
    cand[:, :, :650] = torch.randint(0, 999, (2, 1, 650), dtype=torch.int32, device=DEV)
    sc = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, cand=cand, err=err)
    assert k.csa2_check(err) == 0
    full = to_np(s)
    got = to_np(sc)
    cn = to_np(cand)
    for b in range(2):
        assert np.all(np.isneginf(got[b, 0, 650:]))
        np.testing.assert_array_equal(got[b, 0, :650], full[b, 0, cn[b, 0, :650]])


def test_index_score_full_ragged_rows():
    """A Full scan of rows of very different lengths deals its CTAs to the rows by their visible
    tiles and splits the -inf tails over all CTAs: every row's scores must still equal the
    oracle's, with -inf from its visible entries to the end of a row longer than any sequence
    (a row that sees nothing is all -inf)."""
    k = K()
    lengths = [257, 3001, 20000, 700, 129, 5000, 64]
    spec = W.scaled(W.tiny_full(), lengths, B=len(lengths), q_len=3)   # 21 query rows
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    q_pos = q_pos.clone()
    q_pos[3, :] = -1                        # sees no entry
    q_pos[1, 0] = 999                       # earlier queries of a longer sequence
    q_pos[2, 1] = 4321
    n_out = spec.max_entries + 777
    err = _err()
    s = k.csa2_index_score(q_ix, w, q_pos, cache, n_out, err=err)
    assert k.csa2_check(err) == 0
    assert s.shape[-1] == n_out
    for b in range(len(lengths)):
        c = oracle_seq(spec, b, main_rows=[], gen_device=DEV)
        for qi in range(3):
            nvis = c.visible(0, int(q_pos[b, qi])) if int(q_pos[b, qi]) >= 0 else 0
            got = to_np(s[b, qi])
            assert np.all(np.isneginf(got[nvis:])), (b, qi)
            if nvis:
                ref = OC.indexer_scores(to_np(q_ix[b, qi]), to_np(w[b, qi]), c.indexer_values(0, np.arange(nvis)))
                np.testing.assert_allclose(got[:nvis], ref, rtol=2e-6, atol=2e-6 * np.abs(ref).max())


def test_index_score_rejects_bad_candidates():
    k = K()
    spec = W.scaled(W.tiny_full(), [600], B=1)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    cand = torch.tensor([[[3, 299, 300, -1]]], dtype=torch.int32, device=DEV)
    err = _err()
    sc = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, cand=cand, err=err)
    assert k.csa2_check(err) == 5
    got = to_np(sc)[0, 0]
    assert np.isfinite(got[:2]).all() and np.isneginf(got[2:]).all()


@pytest.mark.parametrize("case", ["random", "ties", "short", "neg_inf", "pool", "long", "zeros", "odd", "unaligned",
                                  "long_odd", "long8", "const", "narrow", "mid"])
def test_topk_rows(case):
    k_ = K()
    g = torch.Generator(device="cpu").manual_seed(7)
    R, N, k, k2 = 5, 9000, 512, 0
    if case == "random":
        s = torch.randn((R, N), generator=g)
    elif case == "ties":
        s = torch.randint(-4, 5, (R, N), generator=g).float()
    elif case == "short":
        N = 300
        s = torch.randn((R, N), generator=g)
    elif case == "neg_inf":
        s = torch.randn((R, N), generator=g)
        s[torch.rand((R, N), generator=g) < 0.97] = -math.inf
    elif case == "pool":
        N, k2 = 70000, 16384
        s = torch.randn((R, N), generator=g) * 100
    elif case == "long":                        # the 2^20-entry rows of a Full scan (16-CTA clusters)
        R, N, k2 = 3, 1 << 20, 16384
        s = torch.randn((R, N), generator=g).abs() * 50
        s[:, ::1000] = s[:, ::1000].round()      # some exact ties
    elif case in ("odd", "unaligned"):          # rows the kernel must read one score at a time
        N, k2 = (9003, 1024) if case == "odd" else (9000, 1024)
        s = torch.randn((R, N), generator=g) * 10
    elif case == "mid":                         # 8-CTA clusters whose chunks exceed shared memory
        N, k2 = 200000, 16384
        s = torch.randn((R, N), generator=g) * 20
    elif case == "const":                       # every finite score equal: one key, ties by index
        s = torch.full((R, N), 1.5)
        s[:, 1::7] = -math.inf
    elif case == "narrow":                      # scores within 1 % of each other (most key bits shared)
        s = 1000.0 + torch.rand((R, N), generator=g) * 10.0
    elif case == "long8":                       # more 2^20-entry rows than 16-CTA clusters fit at once
        R, N, k2 = 8, 1 << 20, 16384
        s = torch.randn((R, N), generator=g) * 30
    elif case == "long_odd":
        R, N, k2 = 2, (1 << 20) - 3, 16384
        s = torch.randn((R, N), generator=g) * 50
    else:                                       # most scores equal (a fully-ReLU-zeroed row)
        N, k2 = 300000, 16384
        s = torch.zeros((R, N))
        s[:, 5::97] = torch.randn((R, len(range(5, N, 97))), generator=g)
    n_valid = torch.tensor(([N, N - 1, N // 2, 511, 0] + [N - 7 * i for i in range(1, 4)])[:R], dtype=torch.int32)
    if case == "unaligned":                     # row base 4 bytes past a 16-byte boundary
        buf = torch.empty(R * N + 1, dtype=torch.float32, device=DEV)
        sd = buf[1:].view(R, N)
        sd.copy_(s)
        assert sd.data_ptr() % 16 == 4
    else:
        sd = s.to(DEV)
    val = torch.empty((R, k), dtype=torch.float32, device=DEV)
    out = k_.csa2_topk(sd, k, n_valid=n_valid.to(DEV), val=val, k2=k2)
    idx = to_np(out[0])
    val = to_np(val)
    for r in range(R):
        srow = s[r].double().numpy()
        ref = OC.topk(srow, k, int(n_valid[r]))
        np.testing.assert_array_equal(idx[r], ref)      # same fp32 inputs: exact
        sel = idx[r][idx[r] >= 0]
        np.testing.assert_array_equal(val[r][: len(sel)], s[r].numpy()[sel])
        assert np.all(np.isneginf(val[r][len(sel):]))
        if k2:
            np.testing.assert_array_equal(to_np(out[2])[r], OC.topk(srow, k2, int(n_valid[r])))


# ------------------------------------------------------------------ attention
def _swa_state(spec, layer, R=128):
    """Device SWA ring for one layer plus the oracle's rings (one per sequence)."""
    k = K()
    x, pos = W.swa_tokens(spec, layer, DEV)
    codes = torch.zeros((spec.B, R, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((spec.B, R), dtype=torch.float32, device=DEV)
    err = _err()
    k.csa2_pack_swa(x, pos, codes, scale, err=err)
    assert k.csa2_check(err) == 0
    rings = [oracle_swa(to_np(x[b]), to_np(pos[b]), R) for b in range(spec.B)]
    return codes, scale, rings


def test_swa_attention_and_sequence_start():
    k = K()
    spec = W.scaled(W.tiny_full(), [4096, 60, 1], B=3)
    q, _, _, q_pos = W.query_tensors(spec, 0, DEV)
    codes, scale, rings = _swa_state(spec, 0)
    o, lse = k.csa2_swa_attn(q, q_pos, codes, scale, spec.tau)
    for b in range(3):
        oo, ol = OC.swa_attention(to_np(q[b, 0]), int(q_pos[b, 0]), rings[b][0], rings[b][1], 128, spec.tau)
        check_attention(to_np(o[b, 0]), to_np(lse[b, 0]), oo, ol, f"swa b={b}")


def test_empty_batches_are_no_ops():
    """Zero sequences, tokens or rows: every entry point returns without touching anything."""
    k = K()
    spec = W.scaled(W.tiny_full(), [600], B=1)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    x, pos = W.swa_tokens(spec, 0, DEV)
    codes = torch.zeros((1, 128, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((1, 128), dtype=torch.float32, device=DEV)
    err = _err()
    kv, ix = W.token_latents(spec, 0, DEV)
    k.csa2_pack_kv(kv[None, :0].contiguous(), ix[None, :0].contiguous(), torch.zeros(1, dtype=torch.int32, device=DEV),
                   cache.seq_view(0), err=err)
    k.csa2_pack_swa(x[:, :0], pos[:, :0], codes, scale, err=err)
    assert int(codes.count_nonzero()) == 0 and int(scale.count_nonzero()) == 0
    sc = k.csa2_index_score(q_ix[:0], w[:0], q_pos[:0], cache, spec.max_entries, err=err)
    assert sc.numel() == 0
    idx = k.csa2_topk(torch.empty((0, 1000), device=DEV), 16)[0]
    assert idx.numel() == 0
    o, lse = k.csa2_sparse_attn("full", q[:0], q_pos[:0], cache, spec.tau, spec.max_entries, q_ix=q_ix[:0], w=w[:0],
                                err=err)
    assert o.numel() == 0 and lse.numel() == 0
    o2, l2 = k.csa2_swa_attn(q[:0], q_pos[:0], codes, scale, spec.tau, err=err)
    om, lm = k.csa2_merge(o2, l2, o2, l2)
    assert om.numel() == 0 and lm.numel() == 0
    assert k.csa2_check(err) == 0


def test_merge_matches_oracle_and_aliases():
    k = K()
    rows = 3 * 64
    o1 = normal((rows, 512), 1, "m1", device=DEV)
    o2 = normal((rows, 512), 1, "m2", device=DEV)
    l1 = normal((rows,), 1, "l1", device=DEV) * 3
    l2 = normal((rows,), 1, "l2", device=DEV) * 3
    l1[:5] = -math.inf
    l2[3:7] = -math.inf
    ref_o, ref_l = OC.merge(to_np(o1), to_np(l1), to_np(o2), to_np(l2))
    o, lse = k.csa2_merge(o1, l1, o2, l2)
    check_attention(to_np(o), to_np(lse), ref_o, ref_l, "merge")
    k.csa2_merge(o1, l1, o2, l2, o=o1, lse=l1)                 # in place
    check_attention(to_np(o1), to_np(l1), ref_o, ref_l, "merge in place")


def _run_layer(k, mode, spec, cache, q, q_ix, w, q_pos, codes, scale, fused, pool_k=0, pool_io=None, idx_in=None,
               idx_out=None, err=None):
    """One layer on the GPU: fused (the SWA ring joins csa2_sparse_attn's softmax) or three calls."""
    if fused:
        o, lse = k.csa2_sparse_attn(mode, q, q_pos, cache, spec.tau, spec.max_entries, k=spec.k, q_ix=q_ix, w=w,
                                    pool_k=pool_k, pool_io=pool_io, idx_in=idx_in, idx_out=idx_out, err=err,
                                    swa_codes=codes, swa_scale=scale)
        return o, lse, None, None
    o1, l1 = k.csa2_sparse_attn(mode, q, q_pos, cache, spec.tau, spec.max_entries, k=spec.k, q_ix=q_ix, w=w,
                                pool_k=pool_k, pool_io=pool_io, idx_in=idx_in, idx_out=idx_out, err=err)
    o2, l2 = k.csa2_swa_attn(q, q_pos, codes, scale, spec.tau, err=err)
    o, lse = k.csa2_merge(o1, l1, o2, l2)
    return o, lse, o1, l1


def _decode_layer_parity(spec, cache, mode, layer, rings, codes, scale, pool=None, pool_k=0, idx_in=None,
                         oracle_caches=None, fused=False):
    """Run one layer on the GPU (sparse + SWA + merge) and compare with the oracle per sequence.

    fused=True passes the SWA ring to csa2_sparse_attn (one softmax over both key sets);
    otherwise the branches run separately and csa2_merge combines them.  Every sequence's
    attention is compared: where the GPU's selection legitimately differs from the oracle's at
    a near-tie (check_topk), the GPU layer is run again in Reuse mode on the oracle's indices
    and that output is compared instead.
    """
    k = K()
    q, q_ix, w, q_pos = W.query_tensors(spec, layer, DEV)
    err = _err()
    idx_out = torch.empty((spec.B, 1, spec.k), dtype=torch.int32, device=DEV)
    pool_io = pool
    if mode == "full" and pool_k:
        pool_io = torch.empty((spec.B, 1, pool_k), dtype=torch.int32, device=DEV)
    o, lse, o1, l1 = _run_layer(k, mode, spec, cache, q, q_ix, w, q_pos, codes, scale, fused, pool_k=pool_k,
                                pool_io=pool_io, idx_in=idx_in, idx_out=idx_out, err=err)
    assert k.csa2_check(err) == 0
    ref_pools = np.full((spec.B, 1, max(pool_k, 1)), -1, np.int64)
    ref_idxs = np.full((spec.B, 1, spec.k), -1, np.int64)
    same = []
    for b in range(spec.B):
        c = oracle_caches[b]
        pos = int(q_pos[b, 0])
        qib, wb = to_np(q_ix[b, 0]), to_np(w[b, 0])
        if mode == "full":
            ref_idx, ref_pool, scores = OC.full_select(c, 0, pos, qib, wb, spec.k, pool_k)
            same.append(check_topk(to_np(idx_out[b, 0]), scores, ref_idx, spec.k, f"full idx b={b}"))
            if pool_k:
                check_topk(to_np(pool_io[b, 0]), scores, ref_pool, pool_k, f"pool b={b}")
                ref_pools[b, 0] = ref_pool
        elif mode == "reindex":
            ref_idx, pscores = OC.reindex_select(c, 0, pos, qib, wb, spec.k, to_np(pool[b, 0]))
            pl = to_np(pool[b, 0])
            gi = to_np(idx_out[b, 0])
            gpos = np.array([np.searchsorted(pl, v) if v >= 0 else -1 for v in gi])
            rpos = np.array([np.searchsorted(pl, v) if v >= 0 else -1 for v in ref_idx])
            same.append(check_topk(gpos, pscores, rpos, spec.k, f"reindex idx b={b}"))
        else:
            ref_idx = to_np(idx_in[b, 0])
            same.append(True)
        ref_idxs[b, 0] = ref_idx
    ref_idx_t = torch.from_numpy(ref_idxs).to(torch.int32).to(DEV)
    if not all(same):   # near-tie selections: the GPU attends the oracle's entries instead
        o_r, lse_r, o1_r, l1_r = _run_layer(k, "reuse", spec, cache, q, q_ix, w, q_pos, codes, scale, fused,
                                            idx_in=ref_idx_t, err=err)
        assert k.csa2_check(err) == 0
    compared = 0
    for b in range(spec.B):
        src = (o, lse, o1, l1) if same[b] else (o_r, lse_r, o1_r, l1_r)
        c = oracle_caches[b]
        fill_main(c, spec, b, ref_idxs[b, 0], gen_device=DEV)
        ref = OC.decode_layer("reuse", c, 0, int(q_pos[b, 0]), to_np(q[b, 0]), spec.tau, rings[b],
                              idx=ref_idxs[b, 0])
        if src[2] is not None:
            check_attention(to_np(src[2][b, 0]), to_np(src[3][b, 0]), *ref["sparse"], f"{mode} sparse b={b}")
        check_attention(to_np(src[0][b, 0]), to_np(src[1][b, 0]), ref["o"], ref["lse"], f"{mode} merged b={b}")
        compared += 1
    assert compared == spec.B
    # the oracle's own selections, for the layers that consume them
    return ref_idx_t, torch.from_numpy(ref_pools).to(torch.int32).to(DEV)


@pytest.mark.parametrize("fused", [False, True])
def test_full_decode_tiny_config(fused):
    spec = W.tiny_full()
    cache = gpu_cache(spec)
    codes, scale, rings = _swa_state(spec, 0)
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    _decode_layer_parity(spec, cache, "full", 0, rings, codes, scale, oracle_caches=oc, fused=fused)


@pytest.mark.parametrize("fused", [False, True])
def test_reuse_decode_scaled_fused_variant(fused):
    spec = W.scaled(W.reuse64k(), [3000, 600, 9000], B=3)
    cache = gpu_cache(spec)
    codes, scale, rings = _swa_state(spec, 1)
    idx = W.reuse_indices(spec, DEV)
    idx[1, 0, 100:] = -1
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    _decode_layer_parity(spec, cache, "reuse", 1, rings, codes, scale, idx_in=idx, oracle_caches=oc, fused=fused)


def test_reuse_decode_scaled():
    spec = W.scaled(W.reuse64k(), [5000, 4097, 513, 700], B=4)
    cache = gpu_cache(spec)
    codes, scale, rings = _swa_state(spec, 0)
    idx = W.reuse_indices(spec, DEV)
    idx[2, 0, 500:] = -1                                      # ragged: fewer than k given
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    _decode_layer_parity(spec, cache, "reuse", 0, rings, codes, scale, idx_in=idx, oracle_caches=oc)


@pytest.mark.parametrize("kk,fused", [(128, True), (256, True), (300, True), (384, False), (300, False),
                                      (512, False)])
def test_reuse_decode_key_counts(kk, fused):
    """2 to 5 key tiles per row (one CTA each), tiles that mix listed entries with window tokens."""
    spec = W.scaled(W.reuse64k(), [6000, 2500, 4096, 777], B=4, k=kk)
    cache = gpu_cache(spec)
    codes, scale, rings = _swa_state(spec, 2)
    idx = W.reuse_indices(spec, DEV)
    idx[3, 0, kk // 2:] = -1
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    _decode_layer_parity(spec, cache, "reuse", 2, rings, codes, scale, idx_in=idx, oracle_caches=oc, fused=fused)


def test_reuse_rejects_out_of_range_indices():
    k = K()
    spec = W.scaled(W.reuse64k(), [1000], B=1)
    cache = gpu_cache(spec)
    q, _, _, q_pos = W.query_tensors(spec, 0, DEV)
    idx = W.reuse_indices(spec, DEV)
    idx[0, 0, 7] = 1000                      # == num_entries
    idx[0, 0, 9] = -7
    err = _err()
    o, lse = k.csa2_sparse_attn("reuse", q, q_pos, cache, spec.tau, spec.max_entries, idx_in=idx, err=err)
    assert k.csa2_check(err) == 5
    c = oracle_seq(spec, 0, gen_device=DEV)
    good = to_np(idx[0, 0]).copy()
    good[[7, 9]] = -1
    oo, ol = OC.sparse_attention(c, 0, to_np(q[0, 0]), good, spec.tau)
    check_attention(to_np(o[0, 0]), to_np(lse[0, 0]), oo, ol, "reuse with rejected indices")


def test_hierarchical_full_then_reindex_scaled():
    spec = W.scaled(W.hier1m(), 40000, B=2, pool_k=2048, n_reindex=2)
    cache = gpu_cache(spec)
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    codes, scale, rings = _swa_state(spec, 0)
    # Reindex and Reuse layers consume the oracle's pool and indices on both sides
    idx_full, pool = _decode_layer_parity(spec, cache, "full", 0, rings, codes, scale, pool_k=spec.pool_k,
                                          oracle_caches=oc)
    for layer in (1, 2):
        codes, scale, rings = _swa_state(spec, layer)
        _decode_layer_parity(spec, cache, "reindex", layer, rings, codes, scale, pool=pool, pool_k=spec.pool_k,
                             oracle_caches=oc, fused=layer == 2)
    # the Reuse layers after it consume the Full layer's indices
    codes, scale, rings = _swa_state(spec, 5)
    _decode_layer_parity(spec, cache, "reuse", 5, rings, codes, scale, idx_in=idx_full, oracle_caches=oc)


def test_prefill_chunk_scaled():
    k = K()
    spec = W.scaled(W.prefill8k(), [2000 + 300], B=1, q_len=300)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    x, pos = W.swa_tokens(spec, 0, DEV)
    R = 512
    codes = torch.zeros((1, R, 512), dtype=torch.uint8, device=DEV)
    scale = torch.zeros((1, R), dtype=torch.float32, device=DEV)
    err = _err()
    k.csa2_pack_swa(x, pos, codes, scale, err=err)
    idx_out = torch.empty((1, spec.q_len, spec.k), dtype=torch.int32, device=DEV)
    o1, l1 = k.csa2_sparse_attn("full", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w,
                                idx_out=idx_out, err=err)
    o2, l2 = k.csa2_swa_attn(q, q_pos, codes, scale, spec.tau, err=err)
    o, lse = k.csa2_merge(o1, l1, o2, l2)
    assert k.csa2_check(err) == 0
    c = oracle_seq(spec, 0, main_rows=[], gen_device=DEV)
    ring = oracle_swa(to_np(x[0]), to_np(pos[0]), R)
    rows = [0, 1, 2, 57, 150, 298, 299]
    compared = 0
    for qi in rows:
        p = int(q_pos[0, qi])
        ref_idx, _, scores = OC.full_select(c, 0, p, to_np(q_ix[0, qi]), to_np(w[0, qi]), spec.k)
        assert (ref_idx[ref_idx >= 0] < (p + 1) // 2).all()
        go, gl = o[0, qi], lse[0, qi]
        if not check_topk(to_np(idx_out[0, qi]), scores, ref_idx, spec.k, f"prefill q={qi}"):
            go, gl = gpu_attend_given(q[:, qi:qi + 1].contiguous(), q_pos[:, qi:qi + 1].contiguous(), cache,
                                      spec.tau, spec.max_entries, ref_idx[None, None], swa=(codes, scale))
            go, gl = go[0, 0], gl[0, 0]
        fill_main(c, spec, 0, ref_idx, gen_device=DEV)
        ref = OC.decode_layer("reuse", c, 0, p, to_np(q[0, qi]), spec.tau, ring, idx=ref_idx)
        check_attention(to_np(go), to_np(gl), ref["o"], ref["lse"], f"prefill q={qi}")
        compared += 1
    assert compared == len(rows)


def test_mixed_paged_batch_scaled():
    k = K()
    spec = W.scaled(W.mixed64(), [5000, 3000, 1200, 4097, 900, 2600], B=6)
    table, pages = W.page_layout(spec, DEV)
    base = k.GlobalKVCache(6, 1, num_slots=pages * 256, page_table=table, page_size=256)
    err = _err()
    for b in range(6):
        kv, ix = W.token_latents(spec, b, DEV)
        v = base.seq_view(b)
        v.ratio = spec.seq_ratio(b)
        k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), torch.zeros(1, dtype=torch.int32, device=DEV),
                       v, err=err)
        base.num_entries[b] = spec.entries(b)
    full_ids = [b for b in range(6) if spec.seq_mode(b) == "full"]
    reuse_ids = [b for b in range(6) if spec.seq_mode(b) == "reuse"]
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    idx_all = W.reuse_indices(spec, DEV)
    for ids, mode, ratio in ((full_ids, "full", 2), (reuse_ids, "reuse", 1)):
        sel = torch.tensor(ids, device=DEV)
        view = k.GlobalKVCache(len(ids), ratio, num_slots=base.num_slots, page_table=table[sel].contiguous(),
                               page_size=256, planes=base.planes, num_entries=base.num_entries[sel].contiguous())
        maxe = max(spec.entries(b) for b in ids)
        idx_out = torch.empty((len(ids), 1, 512), dtype=torch.int32, device=DEV)
        o, lse = k.csa2_sparse_attn(mode, q[sel].contiguous(), q_pos[sel].contiguous(), view, spec.tau, maxe,
                                    q_ix=q_ix[sel].contiguous(), w=w[sel].contiguous(),
                                    idx_in=idx_all[sel].contiguous() if mode == "reuse" else None,
                                    idx_out=idx_out if mode == "full" else None, err=err)
        assert k.csa2_check(err) == 0
        compared = 0
        for j, b in enumerate(ids):
            c = oracle_seq(spec, b, main_rows=[], gen_device=DEV)
            p = int(q_pos[b, 0])
            go, gl = o[j, 0], lse[j, 0]
            if mode == "full":
                ref_idx, _, scores = OC.full_select(c, 0, p, to_np(q_ix[b, 0]), to_np(w[b, 0]), 512)
                if not check_topk(to_np(idx_out[j, 0]), scores, ref_idx, 512, f"mixed full b={b}"):
                    one = k.GlobalKVCache(1, ratio, num_slots=base.num_slots, page_table=table[b:b + 1].contiguous(),
                                          page_size=256, planes=base.planes,
                                          num_entries=base.num_entries[b:b + 1].contiguous())
                    go, gl = gpu_attend_given(q[b:b + 1].contiguous(), q_pos[b:b + 1].contiguous(), one, spec.tau,
                                              maxe, ref_idx[None, None])
                    go, gl = go[0, 0], gl[0, 0]
            else:
                ref_idx = to_np(idx_all[b, 0])
            fill_main(c, spec, b, ref_idx, gen_device=DEV)
            oo, ol = OC.sparse_attention(c, 0, to_np(q[b, 0]), ref_idx, spec.tau)
            check_attention(to_np(go), to_np(gl), oo, ol, f"mixed {mode} b={b}")
            compared += 1
        assert compared == len(ids)


# ------------------------------------------------------------------ predecessor variants and dense attention
def test_full_decode_ratio4():
    """The predecessor's CSA: 4 tokens per entry, lightning indexer, top-512 (Full mode at r = 4)."""
    spec = W.scaled(W.tiny_full(), [8192, 6001], B=2, ratio=4)
    cache = gpu_cache(spec)
    codes, scale, rings = _swa_state(spec, 0)
    oc = [oracle_seq(spec, b, main_rows=[], gen_device=DEV) for b in range(spec.B)]
    assert [int(c.num_entries[0]) for c in oc] == [2048, 1500]
    _decode_layer_parity(spec, cache, "full", 0, rings, codes, scale, oracle_caches=oc, fused=True)


def _dense_parity(spec, cache, fused, tau=None):
    k = K()
    tau = spec.tau if tau is None else tau
    q, _, _, q_pos = W.query_tensors(spec, 0, DEV)
    codes, scale, rings = _swa_state(spec, 0)
    err = _err()
    if fused:
        o, lse = k.csa2_sparse_attn("dense", q, q_pos, cache, tau, spec.max_entries, err=err, swa_codes=codes,
                                    swa_scale=scale)
    else:
        o, lse = k.csa2_sparse_attn("dense", q, q_pos, cache, tau, spec.max_entries, err=err)
    assert k.csa2_check(err) == 0
    for b in range(spec.B):
        c = oracle_seq(spec, b, gen_device=DEV)
        pos = int(q_pos[b, 0])
        every = np.arange(c.visible(0, pos))
        if fused:
            ref = OC.decode_layer("reuse", c, 0, pos, to_np(q[b, 0]), tau, rings[b], idx=every)
            check_attention(to_np(o[b, 0]), to_np(lse[b, 0]), ref["o"], ref["lse"], f"dense+swa b={b}")
        else:
            oo, ol = OC.sparse_attention(c, 0, to_np(q[b, 0]), every, tau)
            check_attention(to_np(o[b, 0]), to_np(lse[b, 0]), oo, ol, f"dense b={b}")


@pytest.mark.parametrize("fused", [False, True])
def test_dense_attention_hca_ratio128(fused):
    """The predecessor's HCA: 128 tokens per entry, then attention over every entry."""
    spec = W.scaled(W.tiny_full(), [128 * 700, 128 * 333 + 77, 128 * 3], B=3, ratio=128)
    cache = gpu_cache(spec)
    _dense_parity(spec, cache, fused)


def test_dense_attention_over_many_entries():
    """9000 and 5000 entries: more keys than one cluster holds at 4096 per segment, and (at 8192
    per segment) a second segment merged through the workspace."""
    spec = W.scaled(W.reuse64k(), [9000, 5000], B=2)
    cache = gpu_cache(spec)
    _dense_parity(spec, cache, fused=True)


def test_dense_attention_many_rows():
    """Enough rows that each row runs on one CTA (no key-split cluster) when its keys fit."""
    spec = W.scaled(W.reuse64k(), [300 + 7 * i for i in range(40)], B=40)
    cache = gpu_cache(spec)
    _dense_parity(spec, cache, fused=True)


def test_dense_and_full_report_a_short_max_entries():
    """A query that sees more entries than max_entries sets CSA2_ERR_SHAPE instead of silently
    leaving the tail out."""
    k = K()
    spec = W.scaled(W.tiny_full(), [3000], B=1)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    for mode in ("full", "dense"):
        err = _err()
        k.csa2_sparse_attn(mode, q, q_pos, cache, spec.tau, 1000, q_ix=q_ix, w=w, err=err)
        assert k.csa2_check(err) == 2, mode


# ------------------------------------------------------------------ query magnitudes
@pytest.mark.parametrize("B", [3, 40])
@pytest.mark.parametrize("case", ["large", "small", "mixed"])
def test_query_magnitudes_are_exact(case, B):
    """bf16 queries far outside fp16 range (1e5) or deep in its subnormals (1e-6) attend as exactly
    as N(0,1) ones: the per-head power-of-two prescale keeps every value.  B = 3 runs the one-tile
    cluster kernel, B = 40 the several-tile kernel."""
    k = K()
    spec = W.scaled(W.reuse64k(), [4000 + 37 * b for b in range(B)], B=B)
    cache = gpu_cache(spec)
    q, _, _, q_pos = W.query_tensors(spec, 0, DEV)
    g = q.float()
    if case == "large":
        g, tau = g * 1e5, 1e-5
    elif case == "small":
        g, tau = g * 1e-6, 1e6
    else:  # one head mixes both magnitudes; others stay N(0,1)/sqrt(512)
        g[:, :, 5, :256] *= 1e5
        g[:, :, 5, 256:] *= 1e-6
        g[:, :, 9] *= 1e5
        tau = 1e-5
    q = g.to(torch.bfloat16).contiguous()
    idx = W.reuse_indices(spec, DEV)
    codes, scale, rings = _swa_state(spec, 0)
    err = _err()
    o, lse = k.csa2_sparse_attn("reuse", q, q_pos, cache, tau, spec.max_entries, idx_in=idx, err=err,
                                swa_codes=codes, swa_scale=scale)
    assert k.csa2_check(err) == 0
    assert torch.isfinite(o).all()
    for b in range(0, B, max(1, B // 5)):
        c = oracle_seq(spec, b, main_rows=to_np(idx[b, 0]), gen_device=DEV)
        ref = OC.decode_layer("reuse", c, 0, int(q_pos[b, 0]), to_np(q[b, 0]), tau, rings[b], idx=to_np(idx[b, 0]))
        check_attention(to_np(o[b, 0]), to_np(lse[b, 0]), ref["o"], ref["lse"], f"{case} b={b}")


# ------------------------------------------------------------------ fused prefill indexer
@pytest.mark.parametrize("tma", [False, True])
def test_prefill_fused_selection(tma):
    """A prefill chunk of 1100 query tokens (Full mode, no pool) selects with the fused indexer:
    every row's top-512 must equal the unfused path's (materialised scores + csa2_topk) bit for
    bit, the same fp32 score arithmetic feeding the same exact selection; sampled rows against
    the oracle too.  tma: a cache layout the tensor map can describe, or the gathering path."""
    k = K()
    spec = W.scaled(W.prefill8k(), [6000 + 1100], B=1, q_len=1100)
    if tma:
        cache = k.GlobalKVCache(1, spec.ratio, seq_stride=(spec.max_entries + 127) // 128 * 128)
        kv, ix = W.token_latents(spec, 0, DEV)
        k.csa2_pack_kv(kv[None].contiguous(), ix[None].contiguous(), torch.zeros(1, dtype=torch.int32, device=DEV),
                       cache, err=_err())
        cache.num_entries[0] = spec.entries(0)
    else:
        cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    err = _err()
    assert k.csa2_workspace_size("full", 1, spec.q_len, spec.max_entries, spec.k) == spec.q_len * spec.k * 4
    idx = torch.empty((1, spec.q_len, spec.k), dtype=torch.int32, device=DEV)
    k.csa2_sparse_attn("full", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w, idx_out=idx, err=err)
    scores = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, err=err)
    ref = k.csa2_topk(scores, spec.k)[0]
    assert k.csa2_check(err) == 0
    assert torch.equal(idx, ref), f"{int((idx != ref).any(-1).sum())} rows differ"
    c = oracle_seq(spec, 0, main_rows=[], gen_device=DEV)
    for qi in (0, 1, 2, 511, 512, 1097, 1098, 1099):
        p = int(q_pos[0, qi])
        ref_idx, _, s = OC.full_select(c, 0, p, to_np(q_ix[0, qi]), to_np(w[0, qi]), spec.k)
        check_topk(to_np(idx[0, qi]), s, ref_idx, spec.k, f"fused prefill q={qi}")


def test_prefill_fused_ties_and_short_rows():
    """Rows of one repeated score (every key ties: the lowest entries win), rows that see fewer
    entries than k (all of them, -1 padded) and a chunk whose length is not a multiple of the
    CTA's three query tokens."""
    k = K()
    spec = W.scaled(W.prefill8k(), [2 * 700 + 1025], B=1, q_len=1025)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    q_ix = q_ix.clone()
    q_ix[0, :400] = 0.0            # every score 0: ties everywhere
    q_pos = q_pos.clone()
    q_pos[0, 400:420] = torch.arange(20, device=DEV, dtype=torch.int32) * 50   # early positions: few entries
    err = _err()
    idx = torch.empty((1, spec.q_len, spec.k), dtype=torch.int32, device=DEV)
    k.csa2_sparse_attn("full", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w, idx_out=idx, err=err)
    scores = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, err=err)
    ref = k.csa2_topk(scores, spec.k)[0]
    assert k.csa2_check(err) == 0
    assert torch.equal(idx, ref), f"{int((idx != ref).any(-1).sum())} rows differ"
    assert torch.equal(idx[0, 0], torch.arange(512, dtype=torch.int32, device=DEV))   # ties: lowest entries
    for qi in range(400, 420):
        nvis = min(spec.entries(0), (int(q_pos[0, qi]) + 1) // 2)
        want = list(range(min(nvis, 512))) if nvis <= 512 else None
        if want is not None:
            got = to_np(idx[0, qi])
            assert got[:nvis].tolist() == want and (got[nvis:] == -1).all()


# ------------------------------------------------------------------ this step's window token in the attention launch
@pytest.mark.parametrize("case", ["reuse4", "reuse32", "full1", "short4"])
def test_swa_new_token_in_the_attention_launch(case):
    """csa2_sparse_attn with swa_new (the step's window token quantised inside the launch) must equal
    csa2_pack_swa of that token followed by csa2_sparse_attn, bit for bit: the ring's codes and scale
    and the layer's o and lse.  reuse4: one-tile clusters; reuse32: two-CTA clusters of the general
    kernel; full1: the Full path (scan, top-k, attention); short4: one-tile clusters of sequences
    whose window is not yet full, so that the token is the key of a thread in each of the four
    warp pairs of the window tile (positions 5, 40, 77 and 1000)."""
    k = K()
    if case == "full1":
        spec = W.scaled(W.tiny_full(), [3001], B=1)
    elif case == "short4":
        spec = W.scaled(W.reuse64k(), [6, 41, 78, 1001], B=4)
    else:
        B = 4 if case == "reuse4" else 32
        spec = W.scaled(W.reuse64k(), [3000 + 37 * b for b in range(B)], B=B)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    x, pos = W.swa_tokens(spec, 0, DEV)
    err = _err()
    ring = [torch.zeros((spec.B, 128, 512), dtype=torch.uint8, device=DEV),
            torch.zeros((spec.B, 128), dtype=torch.float32, device=DEV)]
    k.csa2_pack_swa(x[:, :-1].contiguous(), pos[:, :-1].contiguous(), ring[0], ring[1], err=err)
    ring2 = [t.clone() for t in ring]
    mode = "full" if case == "full1" else "reuse"
    kw = dict(q_ix=q_ix, w=w) if mode == "full" else dict(idx_in=W.reuse_indices(spec, DEV))
    k.csa2_pack_swa(x[:, -1:].contiguous(), pos[:, -1:].contiguous(), ring[0], ring[1], err=err)
    o1, l1 = k.csa2_sparse_attn(mode, q, q_pos, cache, spec.tau, spec.max_entries, err=err, swa_codes=ring[0],
                                swa_scale=ring[1], **kw)
    o2, l2 = k.csa2_sparse_attn(mode, q, q_pos, cache, spec.tau, spec.max_entries, err=err, swa_codes=ring2[0],
                                swa_scale=ring2[1], swa_new=x[:, -1:].contiguous(), **kw)
    assert k.csa2_check(err) == 0
    assert torch.equal(ring[0], ring2[0]) and torch.equal(ring[1], ring2[1])
    assert torch.equal(o1, o2) and torch.equal(l1, l2)


# ------------------------------------------------------------------ fused Reindex selection
@pytest.mark.parametrize("B,P,tokens", [(8, 16384, 2 * 20000), (3, 5000, 2 * 9000), (4, 3000, 2 * 4000),
                                        (300, 700, 2 * 1500), (2, 400, 2 * 1000)])
def test_reindex_fused_selection(B, P, tokens):
    """Reindex over a pool of at most 16384 candidates scores and selects in one launch (each
    row's keys spread over its cluster's shared memory).  Its choice must equal the unfused path's bit for
    bit: csa2_index_score over the pool, csa2_topk of those scores, mapped through the pool.
    Pools are ascending with -1 pads and entries the query cannot see; some rows score every
    candidate 0 (all tied: the earliest candidates win); P = 400 < k pads the selection; B = 300
    rows run one CTA per row."""
    k = K()
    spec = W.scaled(W.tiny_full(), [tokens] * B, B=B)
    cache = gpu_cache(spec)
    q, q_ix, w, q_pos = W.query_tensors(spec, 0, DEV)
    q_ix = q_ix.clone()
    q_ix[0] = 0.0                                   # every score of row 0 ties
    n = spec.entries(0)
    g = torch.Generator(device="cpu").manual_seed(1234 + P)
    pool = torch.full((B, 1, P), -1, dtype=torch.int32)
    for b in range(B):
        m = P - (b % 3) * 7                          # a few -1 pads at the end of some rows
        pool[b, 0, :m] = torch.randperm(n, generator=g)[:m].sort().values.to(torch.int32)
    pool = pool.to(DEV)
    q_pos = q_pos.clone()
    q_pos[1, 0] = tokens - 700                      # an earlier query: candidates it cannot see
    err = _err()
    assert k.csa2_workspace_size("reindex", B, 1, spec.max_entries, spec.k, P) == (B * spec.k * 4 + 255) // 256 * 256
    idx = torch.empty((B, 1, spec.k), dtype=torch.int32, device=DEV)
    k.csa2_sparse_attn("reindex", q, q_pos, cache, spec.tau, spec.max_entries, q_ix=q_ix, w=w, pool_k=P,
                       pool_io=pool, idx_out=idx, err=err)
    scores = k.csa2_index_score(q_ix, w, q_pos, cache, spec.max_entries, cand=pool, err=err)
    pos = k.csa2_topk(scores, spec.k)[0]
    ref = torch.where(pos >= 0, pool.gather(-1, pos.clamp(min=0).long()), torch.full_like(pos, -1))
    assert k.csa2_check(err) == 0
    assert torch.equal(idx, ref), f"{int((idx != ref).any(-1).sum())} of {B} rows differ"
    assert torch.equal(idx[0, 0, :min(P, spec.k)], pool[0, 0, :min(P, spec.k)])   # all tied: earliest win
    if P < spec.k:
        assert (idx[:, :, P:] == -1).all()


# ------------------------------------------------------------------ gated compressor and decode-time append
@pytest.mark.parametrize("ratio", [1, 2, 4, 128])
@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_pack_kv_gated_bit_exact(ratio, dtype):
    k = K()
    B, T = 2, 128 * 3 + 5 if ratio == 128 else 601
    kv = _planted_latents(B, T, 512, 5, dtype)
    ix = _planted_latents(B, T, 128, 6, dtype)
    gkv = normal((B, T, 512), 0, "gate_kv", device=DEV) * 4
    gix = normal((B, T, 128), 0, "gate_ix", device=DEV) * 4
    gkv[0, : 2 * ratio] = 0.5                      # equal logits: the plain mean
    gix[1, :ratio, :7] = 90.0                      # one dominant logit per channel
    n = T // ratio
    cache = k.GlobalKVCache(B, ratio, seq_stride=n + 3)
    first = torch.tensor([0, 3], dtype=torch.int32, device=DEV)
    err = _err()
    k.csa2_pack_kv_gated(kv, ix, gkv, gix, first, cache, err=err)
    assert k.csa2_check(err) == 0
    for b in range(B):
        mc, ms = OF.pack_main(OC.compress_gated(to_np(kv[b]), to_np(gkv[b]), ratio))
        ic, isc = OF.pack_indexer(OC.compress_gated(to_np(ix[b]), to_np(gix[b]), ratio))
        f = int(first[b])
        sl = slice(b * (n + 3) + f, b * (n + 3) + f + n)
        np.testing.assert_array_equal(to_np(cache.kv_codes[sl]), mc)
        np.testing.assert_array_equal(to_np(cache.kv_scales[sl]), ms)
        np.testing.assert_array_equal(to_np(cache.ix_codes[sl]), ic)
        np.testing.assert_array_equal(to_np(cache.ix_scales[sl]), isc)


@pytest.mark.parametrize("ratio", [1, 2, 4])
def test_append_kv_token_by_token_equals_pack_kv(ratio):
    """Appending tokens one decode step at a time (staging the incomplete group) writes the same
    bytes and entry counts as packing the whole run at once, and as the oracle."""
    k = K()
    B, T = 2, 4 * 7 + 3
    kv = _planted_latents(B, T, 512, 7, torch.bfloat16)
    ix = _planted_latents(B, T, 128, 8, torch.bfloat16)
    n = T // ratio
    cache = k.GlobalKVCache(B, ratio, seq_stride=n + 1)
    stage = torch.zeros((B, ratio, 640), dtype=torch.float32, device=DEV)
    err = _err()
    for t in range(T):
        pos = torch.full((B,), t, dtype=torch.int32, device=DEV)
        k.csa2_append_kv(kv[:, t].contiguous(), ix[:, t].contiguous(), pos, cache, stage=stage, err=err)
        if t == T // 2:   # padding rows (negative positions) leave every sequence alone
            k.csa2_append_kv(kv[:, 0].contiguous() * 7, ix[:, 0].contiguous() * 7,
                             torch.full((B,), -1, dtype=torch.int32, device=DEV), cache, stage=stage, err=err)
    assert k.csa2_check(err) == 0
    assert to_np(cache.num_entries).tolist() == [n, n]
    for b in range(B):
        ekv, eix = OC.compress(to_np(kv[b]), ratio), OC.compress(to_np(ix[b]), ratio)
        mc, ms = OF.pack_main(ekv)
        ic, isc = OF.pack_indexer(eix)
        sl = slice(b * (n + 1), b * (n + 1) + n)
        np.testing.assert_array_equal(to_np(cache.kv_codes[sl]), mc)
        np.testing.assert_array_equal(to_np(cache.kv_scales[sl]), ms)
        np.testing.assert_array_equal(to_np(cache.ix_codes[sl]), ic)
        np.testing.assert_array_equal(to_np(cache.ix_scales[sl]), isc)
